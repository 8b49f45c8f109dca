"""The bounded-wait failure path on the GPU: a wait that nothing satisfies
must end after its limit with MOE_ERR_TIMEOUT in the device status word, the
status must clear on read, and the context must stay usable."""
import time

import pytest
import torch

from routed_grouped_gemm_router_b200 import binding as B
from routed_grouped_gemm_router_b200.inputs import small_inputs

import gpu_util as U

pytestmark = pytest.mark.gpu


def test_wait_that_runs_out_reports_timeout_and_context_survives():
    assert B.last_device_status() == 0
    t0 = time.time()
    assert B.lib().moe_selftest_wait_timeout(50, None) == 0
    st = B.last_device_status()
    elapsed = time.time() - t0
    assert st == 5, B.status_str(st)           # MOE_ERR_TIMEOUT
    assert elapsed < 5.0
    assert B.last_device_status() == 0          # cleared by the read
    # the device is still usable: a full layer afterwards matches the oracle
    inp = small_inputs(128, 64, 4, 2, 64, seed=1)
    st_, grads = U.run_layer(inp, 2)
    fwd, bwd = U.oracle_full(inp, 2)
    U.assert_rel(U.to_np(st_.Y), fwd["Y"], "Y")
    for name in ("dX", "dW_gu", "dW_d", "dlogits"):
        U.assert_rel(U.to_np(grads[name]), bwd[name], name)


def test_selftest_rejects_bad_limits():
    assert B.lib().moe_selftest_wait_timeout(0, None) == 1
    assert B.lib().moe_selftest_wait_timeout(10000, None) == 1
