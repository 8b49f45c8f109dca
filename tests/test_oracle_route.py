"""Pins of the oracle's routing (softmax -> top-k -> renormalise) against
closed forms, a brute-force rank count and invariants. CPU only."""
import math
import os

import numpy as np
import pytest

from oracle import moe_oracle as orc

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "route_closed_form.txt")


def _eval(expr: str) -> float:
    return float(eval(expr, {"__builtins__": {}}, {"log": math.log, "exp": math.exp}))


def _golden_cases():
    cases = []
    with open(GOLDEN) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            name, logits, k, idx, w = [s.strip() for s in line.split("|")]
            cases.append((name, [_eval(x) for x in logits.split(",")], int(k),
                          [int(x) for x in idx.split(",")], [_eval(x) for x in w.split(",")]))
    return cases


@pytest.mark.parametrize("case", _golden_cases(), ids=lambda c: c[0])
def test_route_closed_form(case):
    _, logits, k, idx_ref, w_ref = case
    l = np.array([logits], dtype=np.float32)
    idx, w, probs = orc.route(l, k)
    assert idx[0].tolist() == idx_ref
    # the logits are fp32-rounded ln values: allow fp32 input rounding only
    np.testing.assert_allclose(w[0], w_ref, rtol=1e-6, atol=1e-7)


def _bruteforce_select(row, k):
    """Expert e takes slot r iff exactly r experts beat it, where e' beats e when
    its logit is larger, or equal with a smaller index."""
    E = len(row)
    slots = {}
    for e in range(E):
        beaten_by = sum(1 for f in range(E)
                        if row[f] > row[e] or (row[f] == row[e] and f < e))
        if beaten_by < k:
            slots[beaten_by] = e
    return [slots[r] for r in range(k)]


@pytest.mark.parametrize("seed", range(6))
def test_selection_matches_rank_count(seed):
    rng = np.random.default_rng(seed)
    E = int(rng.integers(2, 13))
    T = 40
    # few distinct values -> many exact ties, plus signed zeros
    vals = np.array([-1.5, -0.0, 0.0, 0.25, 2.0, -1e4], dtype=np.float32)
    l = vals[rng.integers(0, len(vals), size=(T, E))]
    for k in range(1, E + 1):
        idx = orc.select_topk(l, k)
        for t in range(T):
            assert idx[t].tolist() == _bruteforce_select(l[t].tolist(), k)


def test_k_equals_E_gives_softmax():
    rng = np.random.default_rng(1)
    l = rng.normal(size=(16, 7)).astype(np.float32)
    idx, w, _ = orc.route(l, 7)
    for t in range(16):
        z = [math.exp(float(x)) for x in l[t]]
        Z = sum(z)
        ref = [z[e] / Z for e in idx[t]]
        np.testing.assert_allclose(w[t], ref, rtol=1e-12)


def test_k1_weight_is_one_and_weights_sum_to_one():
    rng = np.random.default_rng(2)
    l = (rng.normal(size=(64, 9)) * 3).astype(np.float32)
    _, w1, _ = orc.route(l, 1)
    np.testing.assert_allclose(w1, 1.0, rtol=1e-15)
    for k in (2, 3, 5, 9):
        _, w, _ = orc.route(l, k)
        np.testing.assert_allclose(w.sum(axis=1), 1.0, rtol=1e-12)
        assert (np.diff(w, axis=1) <= 1e-15).all(), "weights follow the descending logit order"


def test_dead_experts_never_selected():
    rng = np.random.default_rng(3)
    l = rng.normal(size=(128, 12)).astype(np.float32)
    l[:, [1, 5, 7]] -= 1e4
    idx, w, probs = orc.route(l, 8)
    assert not np.isin(idx, [1, 5, 7]).any()
    assert (probs[:, [1, 5, 7]] == 0).all()


def test_probs_are_row_softmax():
    rng = np.random.default_rng(4)
    l = rng.normal(size=(5, 6)).astype(np.float32)
    _, _, p = orc.route(l, 2)
    for t in range(5):
        z = [math.exp(float(x)) for x in l[t]]
        np.testing.assert_allclose(p[t], np.array(z) / sum(z), rtol=1e-13)
