"""Helpers shared by the GPU parity tests (not a test module)."""
from __future__ import annotations

import numpy as np
import torch

from oracle import moe_oracle as orc
from routed_grouped_gemm_router_b200 import binding as B
from routed_grouped_gemm_router_b200 import layer

# Output/gradient tolerance: bf16 operands with fp32 accumulation; the CUDA
# path also rounds h (and g, u, dGU, dXp, hw) to bf16 between its GEMMs.
REL_TOL = 2e-2
# Routing weights: fp32 softmax/renormalisation against float64 (a few ulp of
# expf plus one division): far below 1e-5 for weights in [0, 1].
W_ABS_TOL = 1e-5


def max_rel_err(gpu, ref) -> float:
    g = np.asarray(gpu, dtype=np.float64)
    r = np.asarray(ref, dtype=np.float64)
    scale = np.abs(r).max()
    err = np.abs(g - r).max() if r.size else 0.0
    return float(err / scale) if scale > 0 else float(err)


def assert_rel(gpu, ref, name, tol=REL_TOL):
    e = max_rel_err(gpu, ref)
    assert e <= tol, f"{name}: max|err| / max|ref| = {e:.3e} > {tol}"
    return e


def to_np(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy() if t.dtype != torch.int32 else t.cpu().numpy()


def to_dev(inp, dev="cuda"):
    return dict(X=inp.X.to(dev), W_gu=inp.W_gu.to(dev), W_d=inp.W_d.to(dev), logits=inp.logits.to(dev),
                dY=None if inp.dY is None else inp.dY.to(dev))


def run_layer(inp, k, backward=True, save_gu=True, stream=None, gather=False):
    d = to_dev(inp)
    st = layer.forward(d["logits"], d["X"], d["W_gu"], d["W_d"], k, save_gu=save_gu, stream=stream, gather=gather)
    grads = layer.backward(st, d["dY"], d["W_gu"], d["W_d"], stream=stream) if backward else None
    status = B.last_device_status(stream)
    assert status == 0, f"device status {B.status_str(status)}"
    return st, grads


def check_routing_exact(st, ref):
    assert (to_np(st.topk_idx) == ref["idx"]).all(), "top-k ids differ from the oracle"
    assert (to_np(st.perm["counts"]) == ref["counts"]).all()
    assert (to_np(st.perm["offsets"]) == ref["offsets"]).all()
    assert (to_np(st.perm["sorted_pair"]) == ref["sorted_pair"]).all()
    assert (to_np(st.perm["pair_pos"]) == ref["pair_pos"]).all()
    np.testing.assert_allclose(to_np(st.topk_w), ref["w"], atol=W_ABS_TOL, rtol=0)
    np.testing.assert_allclose(to_np(st.probs), ref["probs"], atol=1e-6, rtol=1e-4)


def oracle_full(inp, k):
    fwd = orc.layer_forward(inp.logits, inp.X, inp.W_gu, inp.W_d, k)
    bwd = orc.layer_backward(fwd, inp.dY, inp.X, inp.W_gu, inp.W_d, k) if inp.dY is not None else None
    return fwd, bwd


def assert_same_results(a, ga, b, gb):
    """Two runs of the layer (gathered and permuted operand loads) agree bit
    for bit: the GEMMs see the same operand tiles in the same order."""
    for name in ("Y", "h", "O"):
        assert torch.equal(getattr(a, name), getattr(b, name)), name
    if a.gu is not None:
        assert torch.equal(a.gu, b.gu), "gu"
    if ga is not None:
        for name in ("dX", "dW_gu", "dW_d", "dlogits"):
            assert torch.equal(ga[name], gb[name]), name
