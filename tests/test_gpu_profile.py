"""Profiling hooks on the GPU: per-kernel event times and the GEMMs'
effective SM clock from their own cycle and nanosecond counters. Measurement
only: the layer's results are the same with profiling on."""
import pytest
import torch

from routed_grouped_gemm_router_b200 import binding as B
from routed_grouped_gemm_router_b200.inputs import small_inputs

import gpu_util as U

pytestmark = pytest.mark.gpu


def test_profile_times_clock_and_results():
    inp = small_inputs(1500, 512, 16, 4, 384, seed=3)
    st0, g0 = U.run_layer(inp, 4)
    B.profile_enable(True)
    st1, g1 = U.run_layer(inp, 4)
    prof = B.profile_read()
    clocks = {n: B.profile_read_clock(n) for n in prof}
    B.profile_enable(False)
    assert torch.equal(st0.Y, st1.Y) and all(torch.equal(g0[n], g1[n]) for n in g0)
    for n in ("route_hist", "permute_scan_scatter", "gemm_fwd_gate_up", "gemm_bwd_wgrad_down", "combine_dx",
              "router_bwd"):
        assert n in prof and prof[n][0] > 0 and prof[n][1] >= 1, n
    for n, mhz in clocks.items():
        if n.startswith("gemm_"):
            assert 300 < mhz < 2500, (n, mhz)  # a real SM clock
        else:
            assert mhz == 0, n  # only the GEMMs count cycles
    # restricted to one kernel: only that one is recorded, and still its clock
    B.profile_enable(True)
    B.profile_only("gemm_fwd_down")
    U.run_layer(inp, 4)
    prof = B.profile_read()
    assert set(prof) == {"gemm_fwd_down"}
    assert 300 < B.profile_read_clock("gemm_fwd_down") < 2500
    assert B.profile_read_clock("gemm_fwd_gate_up") == 0
    B.profile_enable(False)
