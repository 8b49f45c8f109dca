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


def _noalloc(idx, E, X):
    T, k = idx.shape
    H = X.shape[1]
    dev = idx.device
    out = dict(counts=torch.full((E,), -7, dtype=torch.int32, device=dev),
               offsets=torch.full((E + 1,), -7, dtype=torch.int32, device=dev),
               sorted_pair=torch.full((T * k,), -7, dtype=torch.int32, device=dev),
               pair_pos=torch.full((T * k,), -7, dtype=torch.int32, device=dev),
               Xp=torch.zeros(T * k, H, dtype=torch.bfloat16, device=dev))
    p = lambda t: ctypes.c_void_p(t.data_ptr())
    st = B.lib().moe_permute_noalloc(p(idx), T, E, k, p(out["counts"]), p(out["offsets"]), p(out["sorted_pair"]),
                                     p(out["pair_pos"]), p(X), H, p(out["Xp"]),
                                     ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == 0, B.status_str(st)
    return out


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


def test_noalloc_rejects_problems_beyond_its_scratch():
    # ceil(T*k/2048) * E > 262144 ints: refused before anything is launched
    p = ctypes.c_void_p(256)
    st = B.lib().moe_permute_noalloc(p, 1 << 20, 1024, 8, p, p, p, p, None, 0, None, None)
    assert st == 3, B.status_str(st)
