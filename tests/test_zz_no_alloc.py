"""moe_permute_noalloc, the permute entry point for callers that cannot
allocate device memory (it uses a fixed scratch array inside the library
instead of a caller workspace), must give exactly the results of moe_permute.

Collected last on purpose; it also passes when run alone in a fresh process.
"""
import ctypes

import pytest
import torch

from routed_grouped_gemm_router_b200 import binding as B

pytestmark = pytest.mark.gpu


SCRATCH_INTS = 262144  # the library's fixed scratch: 1 MiB of int32
CHUNK = 2048           # pairs per histogram chunk


def _noalloc_call(idx, E, X, expect=0):
    """One moe_permute_noalloc call with fresh outputs (X may be None: no
    row gather). Returns the outputs; asserts the status is `expect`."""
    T, k = idx.shape
    H = 0 if X is None else X.shape[1]
    dev = idx.device
    out = dict(counts=torch.full((E,), -7, dtype=torch.int32, device=dev),
               offsets=torch.full((E + 1,), -7, dtype=torch.int32, device=dev),
               sorted_pair=torch.full((T * k,), -7, dtype=torch.int32, device=dev),
               pair_pos=torch.full((T * k,), -7, dtype=torch.int32, device=dev))
    if X is not None:
        out["Xp"] = torch.zeros(T * k, H, dtype=torch.bfloat16, device=dev)
    p = lambda t: ctypes.c_void_p(t.data_ptr()) if t is not None else None
    st = B.lib().moe_permute_noalloc(p(idx), T, E, k, p(out["counts"]), p(out["offsets"]), p(out["sorted_pair"]),
                                     p(out["pair_pos"]), p(X), H, p(out.get("Xp")),
                                     ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == expect, B.status_str(st)
    return out


def _noalloc(idx, E, X):
    return _noalloc_call(idx, E, X)


@pytest.mark.parametrize("T,E,k,H", [(8192, 128, 8, 256), (1000, 37, 5, 64)])
def test_noalloc_permute_matches_permute_twice(T, E, k, H):
    g = torch.Generator().manual_seed(T + E)
    logits = torch.randn(T, E, generator=g).cuda()
    X = torch.randn(T, H, generator=g).to(torch.bfloat16).cuda()
    idx, _, _ = B.moe_route(logits, k)
    ref = B.moe_permute(idx, E, X)
    for _ in range(2):  # the second call reuses the scratch the first call left behind
        got = _noalloc(idx, E, X)
        torch.cuda.synchronize()
        for name in ("counts", "offsets", "sorted_pair", "pair_pos", "Xp"):
            assert torch.equal(got[name], ref[name]), name
    assert B.last_device_status() == 0


@pytest.mark.parametrize("E,k", [(128, 8), (1000, 1)])
def test_noalloc_scratch_limit_exactly(E, k):
    """A problem whose histogram fills the scratch exactly is accepted and
    gives moe_permute's results; one more pair (one more chunk of E counters)
    is refused with MOE_ERR_WORKSPACE and writes nothing."""
    chunks = SCRATCH_INTS // E
    P = chunks * CHUNK
    assert P % k == 0
    T = P // k
    assert -(-(T * k) // CHUNK) * E <= SCRATCH_INTS
    g = torch.Generator().manual_seed(E + k)
    # distinct experts per token, as routing produces: a random first expert,
    # then the next k - 1 in cyclic order
    first = torch.randint(0, E, (T, 1), generator=g)
    idx = ((first + torch.arange(k)) % E).to(torch.int32).contiguous().cuda()
    ref = B.moe_permute(idx, E)
    for _ in range(2):
        got = _noalloc_call(idx, E, None)
        torch.cuda.synchronize()
        for name in ("counts", "offsets", "sorted_pair", "pair_pos"):
            assert torch.equal(got[name], ref[name]), name
    # one pair more: T*k = P + 1 (k = 1) or T + 1 tokens (k > 1) -> one more chunk
    T2 = T + 1
    assert -(-(T2 * k) // CHUNK) * E > SCRATCH_INTS
    idx2 = torch.zeros(T2, k, dtype=torch.int32, device="cuda")
    idx2[:, :] = torch.arange(k, dtype=torch.int32, device="cuda")
    out = _noalloc_call(idx2, E, None, expect=3)
    torch.cuda.synchronize()
    for name in ("counts", "offsets", "sorted_pair", "pair_pos"):
        assert (out[name] == -7).all(), f"{name} written by a refused call"
    assert B.last_device_status() == 0


def test_noalloc_rejects_problems_beyond_its_scratch():
    # ceil(T*k/2048) * E > 262144 ints: refused before anything is launched
    p = ctypes.c_void_p(256)
    st = B.lib().moe_permute_noalloc(p, 1 << 20, 1024, 8, p, p, p, p, None, 0, None, None)
    assert st == 3, B.status_str(st)
