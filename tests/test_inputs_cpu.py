"""The seeded input recipe (CPU): shapes, storage dtypes, distributions,
determinism, the draw order's independence of the backward flag, and the
stress workloads' popularity bias (dead experts, Zipf masses), including the
realised routing of the stress batches."""
import math

import numpy as np
import pytest
import torch

from oracle import moe_oracle as orc
from routed_grouped_gemm_router_b200.inputs import WORKLOADS, Workload, make_inputs, small_inputs, zipf_bias


def test_shapes_and_dtypes():
    inp = small_inputs(96, 64, 6, 2, 48, seed=3)
    assert inp.X.shape == (96, 64) and inp.X.dtype == torch.bfloat16
    assert inp.W_r.shape == (6, 64) and inp.W_r.dtype == torch.float32
    assert inp.W_gu.shape == (6, 96, 64) and inp.W_gu.dtype == torch.bfloat16
    assert inp.W_d.shape == (6, 64, 48) and inp.W_d.dtype == torch.bfloat16
    assert inp.logits.shape == (96, 6) and inp.logits.dtype == torch.float32
    assert inp.dY.shape == (96, 64) and inp.dY.dtype == torch.bfloat16
    assert inp.bias is None


def test_same_seed_same_inputs_other_seed_other_inputs():
    a, b, c = (small_inputs(64, 32, 4, 2, 32, seed=s) for s in (5, 5, 6))
    for name in ("X", "W_r", "W_gu", "W_d", "logits", "dY"):
        assert torch.equal(getattr(a, name), getattr(b, name)), name
        assert not torch.equal(getattr(a, name), getattr(c, name)), name


def test_forward_only_draws_the_same_forward_inputs():
    """dY is drawn after every forward input, so leaving it out changes nothing else."""
    a = small_inputs(64, 32, 4, 2, 32, seed=2, with_dy=True)
    b = small_inputs(64, 32, 4, 2, 32, seed=2, with_dy=False)
    assert b.dY is None
    for name in ("X", "W_r", "W_gu", "W_d", "logits"):
        assert torch.equal(getattr(a, name), getattr(b, name)), name


def test_distributions():
    inp = small_inputs(512, 256, 8, 2, 128, seed=0)
    for name, std in (("X", 1.0), ("dY", 1.0), ("W_gu", 0.02), ("W_d", 0.02), ("W_r", 0.02)):
        t = getattr(inp, name).float()
        n = t.numel()
        # four standard errors of the sample mean and of the sample standard deviation
        assert abs(t.mean().item()) < 4 * std / math.sqrt(n), name
        assert abs(t.std().item() / std - 1.0) < 4 / math.sqrt(2 * n), name
    # bf16 storage: every value is exactly representable in bf16
    for name in ("X", "W_gu", "W_d", "dY"):
        t = getattr(inp, name)
        assert torch.equal(t.float().to(torch.bfloat16), t), name


def test_logits_are_the_fp32_router_linear():
    inp = small_inputs(40, 24, 5, 2, 16, seed=9)
    want = inp.X.double() @ inp.W_r.double().t()
    np.testing.assert_allclose(inp.logits.numpy(), want.numpy(), rtol=1e-5, atol=1e-5)


def test_zipf_bias_masses_and_dead_experts():
    """exp(bias) over the live experts is the Zipf(s) distribution: it sums to
    1, its largest mass is 1 / H(live, s) (about 27.5 % for 108 experts at
    s = 1.2), successive ranks fall as r^-s; the dead experts sit at -1e4."""
    E, s, dead = 128, 1.2, 20
    b = zipf_bias(E, s, dead, torch.Generator().manual_seed(0)).double()
    assert int((b == -1.0e4).sum()) == dead
    live = b[b > -1.0e4]
    assert live.numel() == E - dead
    p = torch.exp(live).sort(descending=True).values
    assert abs(p.sum().item() - 1.0) < 1e-6
    harmonic = sum(r ** -s for r in range(1, E - dead + 1))
    assert abs(p[0].item() - 1.0 / harmonic) < 1e-7
    assert abs(p[0].item() - 0.275) < 0.005
    ratios = (p[1:] / p[:-1]).numpy()
    want = np.array([((r + 1) / r) ** -s for r in range(1, E - dead)])
    np.testing.assert_allclose(ratios, want, rtol=1e-5)


@pytest.mark.parametrize("name", ["zipf-t64", "zipf-t32768"])
def test_stress_batches_route_as_described(name):
    """Routed by the oracle: the 20 dead experts get no pair, the top expert
    is in nearly every token's top k, and the expert counts sum to T k."""
    wl = WORKLOADS[name]
    if wl.T > 4096:  # the popularity pattern does not depend on T: check on a cut of the batch
        wl = Workload(wl.name, 4096, wl.H, wl.E, wl.k, wl.I, wl.zipf_s, wl.dead_experts)
    inp = make_inputs(wl, seed=0, with_dy=False)
    idx, _, _ = orc.route(inp.logits.numpy(), wl.k)
    counts = np.bincount(np.asarray(idx).reshape(-1), minlength=wl.E)
    assert counts.sum() == wl.T * wl.k
    dead = (inp.bias == -1.0e4).numpy()
    assert dead.sum() == 20 and counts[dead].sum() == 0
    assert counts.max() >= 0.95 * wl.T
