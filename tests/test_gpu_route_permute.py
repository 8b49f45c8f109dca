"""moe_route_permute (routing fused with the expert histogram, then one
scan-and-scatter kernel) against moe_route followed by moe_permute: every
output bit for bit, on shapes that cover one and many 32-token chunks,
ragged chunk tails, E from 1 to 1024 (both selection paths of the routing
kernel), k from 1 to E, exact ties and the empty batch. The two-call path is
itself pinned to the oracle by the other parity tests; the layer (which now
routes through moe_route_permute) is checked against the oracle there too."""
import numpy as np
import pytest
import torch

from oracle import moe_oracle as orc
from routed_grouped_gemm_router_b200 import binding as B

pytestmark = pytest.mark.gpu

CASES = [  # (T, E, k, H)
    (1, 4, 2, 64), (31, 8, 2, 0), (32, 8, 2, 64), (33, 8, 8, 0), (1000, 37, 5, 64), (1023, 33, 1, 0),
    (1025, 128, 8, 256), (8192, 128, 8, 0), (16384, 128, 8, 0), (4097, 256, 16, 0), (3000, 257, 7, 0),
    (2000, 1000, 8, 0), (777, 1024, 40, 0), (64, 1, 1, 0), (300, 64, 64, 64), (65536, 32, 4, 0),
]


def _both(logits, k, X):
    idx, w, probs = B.moe_route(logits, k)
    ref = B.moe_permute(idx, logits.shape[1], X)
    idx2, w2, probs2, got = B.moe_route_permute(logits, k, X)
    torch.cuda.synchronize()
    assert B.last_device_status() == 0
    return (idx, w, probs, ref), (idx2, w2, probs2, got)


@pytest.mark.parametrize("T,E,k,H", CASES, ids=["T%d_E%d_k%d_H%d" % c for c in CASES])
def test_route_permute_equals_route_then_permute(T, E, k, H):
    g = torch.Generator().manual_seed(T * 7 + E * 3 + k)
    logits = (torch.randn(T, E, generator=g) * 2).cuda()
    X = torch.randn(T, H, generator=g).to(torch.bfloat16).cuda() if H else None
    (idx, w, probs, ref), (idx2, w2, probs2, got) = _both(logits, k, X)
    assert torch.equal(idx, idx2) and torch.equal(w, w2) and torch.equal(probs, probs2)
    for name in ("counts", "offsets", "sorted_pair", "pair_pos") + (("Xp",) if H else ()):
        assert torch.equal(ref[name], got[name]), name
    if T * E <= 2_000_000:  # and the oracle's routing / permutation, exactly
        ridx, _, _ = orc.route(logits.cpu().numpy(), k)
        counts, offsets, sorted_pair, pair_pos = orc.permute(ridx, E)
        assert (idx2.cpu().numpy() == ridx).all()
        assert (got["counts"].cpu().numpy() == counts).all() and (got["offsets"].cpu().numpy() == offsets).all()
        assert (got["sorted_pair"].cpu().numpy() == sorted_pair).all()
        assert (got["pair_pos"].cpu().numpy() == pair_pos).all()


def test_route_permute_ties_and_stress_bias():
    """Exact ties and signed zeros (both selection paths), and a Zipf-like
    bias with dead experts and one expert in nearly every token."""
    g = torch.Generator().manual_seed(5)
    vals = torch.tensor([-1.0, -0.0, 0.0, 0.5, 2.0, -1e4])
    for E, k in ((37, 5), (128, 8), (300, 9), (1024, 8)):
        logits = vals[torch.randint(0, len(vals), (700, E), generator=g)].contiguous().cuda()
        (idx, w, probs, ref), (idx2, w2, probs2, got) = _both(logits, k, None)
        assert torch.equal(idx, idx2) and torch.equal(w, w2) and torch.equal(probs, probs2)
        for name in ("counts", "offsets", "sorted_pair", "pair_pos"):
            assert torch.equal(ref[name], got[name]), name
        ridx, _, _ = orc.route(logits.cpu().numpy(), k)
        assert (idx2.cpu().numpy() == ridx).all()
    T, E, k = 5000, 128, 8
    bias = torch.log(torch.arange(1, E + 1, dtype=torch.float32) ** -1.2)
    bias[100:] = -1e4
    logits = (torch.randn(T, E, generator=g) * 0.9 + bias).cuda()
    (idx, w, probs, ref), (idx2, w2, probs2, got) = _both(logits, k, None)
    assert int(got["counts"][100:].sum()) == 0 and int(got["counts"][0]) > 0.9 * T
    for name in ("counts", "offsets", "sorted_pair", "pair_pos"):
        assert torch.equal(ref[name], got[name]), name


def test_route_permute_empty_batch_and_bad_workspace():
    logits = torch.empty(0, 16, device="cuda")
    idx, w, probs, perm = B.moe_route_permute(logits, 4)
    assert int(perm["counts"].abs().sum()) == 0 and int(perm["offsets"].abs().sum()) == 0
    logits = torch.randn(100, 16, device="cuda")
    with pytest.raises(B.MoeError) as err:
        B.moe_route_permute(logits, 4, ws=torch.empty(1, dtype=torch.uint8, device="cuda"))
    assert err.value.status == 3  # MOE_ERR_WORKSPACE
    assert B.last_device_status() == 0
