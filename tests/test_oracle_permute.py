"""Pins of the oracle's expert indexing (counts, offsets, stable permutation)
against brute-force loops and invariants. CPU only."""
import numpy as np
import pytest

from oracle import moe_oracle as orc


def _bruteforce(idx, E):
    flat = [int(x) for x in np.asarray(idx).reshape(-1)]
    counts = [0] * E
    buckets = [[] for _ in range(E)]
    for q, e in enumerate(flat):        # pairs visited in ascending pair id
        counts[e] += 1
        buckets[e].append(q)
    sorted_pair = [q for b in buckets for q in b]
    return counts, sorted_pair


@pytest.mark.parametrize("T,E,k,seed", [(1, 1, 1, 0), (7, 5, 3, 1), (64, 8, 2, 2),
                                        (33, 17, 4, 3), (100, 128, 8, 4)])
def test_permute_matches_bruteforce(T, E, k, seed):
    rng = np.random.default_rng(seed)
    idx = np.stack([rng.permutation(E)[:k] for _ in range(T)]).astype(np.int32)
    counts, offsets, sorted_pair, pair_pos = orc.permute(idx, E)
    c_ref, sp_ref = _bruteforce(idx, E)
    assert counts.shape == (E,), "counts are one value per expert"
    assert counts.tolist() == c_ref
    assert sorted_pair.tolist() == sp_ref
    assert offsets[0] == 0 and offsets[-1] == T * k
    assert (np.diff(offsets) == counts).all()
    P = T * k
    assert sorted(sorted_pair.tolist()) == list(range(P)), "bijection on [0, P)"
    assert (pair_pos[sorted_pair] == np.arange(P)).all()
    assert (sorted_pair[pair_pos] == np.arange(P)).all()
    flat = idx.reshape(-1)
    for e in range(E):
        seg = sorted_pair[offsets[e]:offsets[e + 1]]
        assert (flat[seg] == e).all()
        assert (np.diff(seg) > 0).all(), "stable: ascending pair id inside a segment"


def test_unpermute_inverts_permute():
    rng = np.random.default_rng(5)
    T, E, k, H = 50, 6, 3, 4
    idx = np.stack([rng.permutation(E)[:k] for _ in range(T)]).astype(np.int32)
    _, _, sorted_pair, pair_pos = orc.permute(idx, E)
    X = rng.normal(size=(T * k, H))
    Xp = X[sorted_pair]
    assert (Xp[pair_pos] == X).all()


def test_empty_experts_have_empty_segments():
    idx = np.array([[3, 0], [0, 3], [3, 0]], dtype=np.int32)
    counts, offsets, sorted_pair, pair_pos = orc.permute(idx, 5)
    assert counts.tolist() == [3, 0, 0, 3, 0]
    assert offsets.tolist() == [0, 3, 3, 3, 6, 6]
    assert sorted_pair.tolist() == [1, 2, 5, 0, 3, 4]
