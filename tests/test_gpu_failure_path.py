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


def test_gemms_refuse_segment_bounds_out_of_order():
    """Segment bounds that are not monotone (two neighbouring bounds swapped)
    make the expert GEMMs run no tile: the forward leaves h, g|u and O as
    they were, the backward writes zero weight gradients, the status reads
    MOE_ERR_DEVICE_CHECK, and a correct call afterwards still matches. Every
    bound used here lies inside [0, T*k], so even a GEMM that skipped the
    check would stay inside its buffers."""
    T, H, E, k, I = 300, 128, 8, 2, 128
    inp = small_inputs(T, H, E, k, I, seed=11)
    st, grads = U.run_layer(inp, k)
    d = U.to_dev(inp)
    p = st.perm
    off = p["offsets"].clone()
    assert int(off[1]) < int(off[2]) <= T * k        # expert 1 holds rows
    off[1], off[2] = p["offsets"][2], p["offsets"][1]  # now off[1] > off[2]
    h, gu, O = (torch.full_like(t, 7.0) for t in (st.h, st.gu, st.O))
    B.moe_experts_fwd(p["Xp"], off, p["sorted_pair"], st.topk_w, T, E, k, d["W_gu"], d["W_d"], h=h, gu_save=gu, O=O)
    assert B.last_device_status() == 6               # MOE_ERR_DEVICE_CHECK
    assert bool((h == 7).all()) and bool((gu == 7).all()) and bool((O == 7).all())
    g = B.moe_layer_bwd(d["dY"], p["Xp"], st.gu, st.h, st.probs, st.topk_idx, st.topk_w, off, p["sorted_pair"],
                        p["pair_pos"], T, E, k, d["W_gu"], d["W_d"])
    assert B.last_device_status() == 6
    assert not bool(g["dW_gu"].any()) and not bool(g["dW_d"].any())
    assert B.last_device_status() == 0               # cleared by the read
    st2, grads2 = U.run_layer(inp, k)
    for name in ("Y", "h", "O"):
        assert torch.equal(getattr(st2, name), getattr(st, name)), name
    for name in ("dX", "dW_gu", "dW_d", "dlogits"):
        assert torch.equal(grads2[name], grads[name]), name
