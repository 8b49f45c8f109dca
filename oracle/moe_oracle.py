"""CPU oracle of the fused MoE expert layer -- TEST INFRASTRUCTURE ONLY.

Plain, slow, obviously-correct float64 numpy restatement of what the layer
computes. Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU
baseline leg may import it; the product path never does, and it shares no code
with the CUDA library (the two only share the seeded input generator).

Sources (page title, then the part of the page):
  * "Integration of fused moe kernel (e.g., megablocks) for efficient moe
    training" (axolotl issue #3155), *Feature description*: the reference
    semantics are Hugging Face's for-loop over experts -- each expert takes the
    tokens routed to it, runs its MLP and adds the result back. The experts here
    are SwiGLU without bias (the same thread: "changed to silu"). The router is
    a Linear(H -> E) whose weight is [E, H] (the same thread, discussion of the
    router's weight shape).
  * fused-MoE Triton project summary (sourcepulse), *How It Works* and
    *Highlighted Details*: softmax -> top-k routing, expert indexing by sorting
    inputs by expert, grouped GEMM over the sorted rows.
  * "[WIP] Qwen3 MoE support" (torchtune PR #2820), review comment on routing:
    top-k scores are renormalised by their sum plus 1e-20.
  * "[MoE] Improve moe kernels for unsloth fine tuning #3812", review of the
    token-routing logic: per-expert counts are ``bincount(flat experts,
    minlength=E)`` (a length-E vector) and the gather indices are the stable
    ``argsort`` of the flattened expert ids; stacked weights are
    ``[E, 2I, H]`` (gate/up) and ``[E, H, I]`` (down).
  * modelopt ``moe`` helpers, ``a2a_moe`` *Flow*: expand (token, expert) pairs,
    run the experts, then weight each result by its routing weight and sum each
    token's top-k results.
  * fused-MoE Triton project summary (sourcepulse), *Highlighted Details*:
    LoRA on the fused expert weights (``lora_*`` functions; the update itself
    is the published LoRA form W + scale B A).

Readings where the pages are silent (each is also listed in the design notes):
  1. top-k is taken on the fp32 logits (softmax is strictly increasing, so the
     set is the same as on the probabilities), order: logit descending, expert
     index ascending (lower index wins a tie).
  2. rows [0, I) of ``W_gu[e]`` are the gate projection, rows [I, 2I) the up.
  3. SwiGLU: h = silu(g) * u with silu(x) = x / (1 + exp(-x)); no bias/clamp.
  4. the routing weight multiplies the expert output before the per-token sum.
  5. backward: the top-k selection is a constant; gradients flow through
     softmax -> gather -> renormalisation (what autograd of that chain gives).
  6. LoRA: one adapter per expert on each stacked weight (gate|up fused), one
     scale; the base weights are frozen (their gradient is still returned).

Notation: T tokens, H hidden, E experts, k top-k, I expert intermediate size,
P = T*k pairs, pair id q = t*k + j (j = rank of the expert in token t's top-k).
"""
from __future__ import annotations

import numpy as np

RENORM_EPS = 1e-20  # torchtune PR #2820: denominator = sum of top scores + 1e-20


def _f64(a) -> np.ndarray:
    """Widen an input (numpy, or a CPU torch tensor of any float dtype) to float64."""
    if hasattr(a, "detach"):
        a = a.detach().float().numpy()
    return np.asarray(a, dtype=np.float64)


# --------------------------------------------------------------------------- route
def softmax(logits) -> np.ndarray:
    """Row softmax in float64 (fused-MoE summary, *Highlighted Details*: fused
    softmax-topk)."""
    l = _f64(logits)
    z = np.exp(l - l.max(axis=1, keepdims=True))
    return z / z.sum(axis=1, keepdims=True)


def select_topk(logits, k: int) -> np.ndarray:
    """Indices [T, k] of each row's k largest logits, ordered by logit
    descending then expert index ascending (reading 1)."""
    l = np.asarray(logits.numpy() if hasattr(logits, "numpy") else logits, dtype=np.float32)
    T, E = l.shape
    expert_ids = np.broadcast_to(np.arange(E), (T, E))
    # lexsort: last key is primary -> primary -logit (descending), secondary index
    order = np.lexsort((expert_ids, -l), axis=1)
    return order[:, :k].astype(np.int32)


def route(logits, k: int):
    """softmax -> top-k -> renormalise (torchtune PR #2820 review comment).

    Returns (idx [T,k] int32, w [T,k] float64, probs [T,E] float64)."""
    probs = softmax(logits)
    idx = select_topk(logits, k)
    top = np.take_along_axis(probs, idx.astype(np.int64), axis=1)
    w = top / (top.sum(axis=1, keepdims=True) + RENORM_EPS)
    return idx, w, probs


# ------------------------------------------------------------------------- permute
def permute(idx, E: int):
    """Expert indexing (unsloth PR #3812, review of the routing logic):
    counts = bincount(flat ids, minlength=E); sorted_pair = stable argsort of
    the flat ids; offsets = exclusive prefix sum of counts; pair_pos = inverse
    permutation (row of pair q in the expert-sorted order)."""
    flat = np.asarray(idx).reshape(-1).astype(np.int64)
    counts = np.bincount(flat, minlength=E).astype(np.int32)
    offsets = np.zeros(E + 1, dtype=np.int32)
    offsets[1:] = np.cumsum(counts)
    sorted_pair = np.argsort(flat, kind="stable").astype(np.int32)
    pair_pos = np.empty_like(sorted_pair)
    pair_pos[sorted_pair] = np.arange(flat.size, dtype=np.int32)
    return counts, offsets, sorted_pair, pair_pos


# ------------------------------------------------------------------------- experts
def silu(x: np.ndarray) -> np.ndarray:
    with np.errstate(over="ignore"):
        return x / (1.0 + np.exp(-x))


def sigmoid(x: np.ndarray) -> np.ndarray:
    with np.errstate(over="ignore"):
        return 1.0 / (1.0 + np.exp(-x))


def expert_mlp(x: np.ndarray, W_gu_e: np.ndarray, W_d_e: np.ndarray):
    """SwiGLU expert on rows x [m, H] (float64). Returns g, u, h [m, I] and the
    unweighted output o [m, H]."""
    I = W_d_e.shape[1]
    g = x @ W_gu_e[:I].T
    u = x @ W_gu_e[I:].T
    h = silu(g) * u
    o = h @ W_d_e.T
    return g, u, h, o


def layer_forward(logits, X, W_gu, W_d, k: int) -> dict:
    """Whole forward: route, permute, loop over experts, weight, combine.

    The loop over experts is the for-loop of axolotl issue #3155; the weighting
    and per-token sum are the last two steps of the ``a2a_moe`` flow."""
    X = _f64(X)
    W_gu = _f64(W_gu)
    W_d = _f64(W_d)
    T, H = X.shape
    E = W_gu.shape[0]
    I = W_d.shape[2]
    idx, w, probs = route(logits, k)
    counts, offsets, sorted_pair, pair_pos = permute(idx, E)
    P = T * k
    w_flat = w.reshape(-1)
    g = np.zeros((P, I))
    u = np.zeros((P, I))
    h = np.zeros((P, I))
    o = np.zeros((P, H))
    O = np.zeros((P, H))
    for e in range(E):
        lo, hi = int(offsets[e]), int(offsets[e + 1])
        if lo == hi:
            continue
        q = sorted_pair[lo:hi]
        tok = q // k
        g[lo:hi], u[lo:hi], h[lo:hi], o[lo:hi] = expert_mlp(X[tok], W_gu[e], W_d[e])
        O[lo:hi] = w_flat[q, None] * o[lo:hi]
    Y = combine(O, pair_pos, T, k)
    return dict(idx=idx, w=w, probs=probs, counts=counts, offsets=offsets,
                sorted_pair=sorted_pair, pair_pos=pair_pos, g=g, u=u, h=h, o=o, O=O, Y=Y)


def combine(O: np.ndarray, pair_pos, T: int, k: int) -> np.ndarray:
    """Y[t] = sum over j of O[pair_pos[t*k + j]] (``a2a_moe`` flow, last step)."""
    pos = np.asarray(pair_pos).reshape(T, k)
    Y = np.zeros((T, O.shape[1]))
    for j in range(k):
        Y += O[pos[:, j]]
    return Y


# ------------------------------------------------------------------------ backward
def router_backward(dw: np.ndarray, w: np.ndarray, probs: np.ndarray, idx) -> np.ndarray:
    """d logits from d(renormalised weights), the top-k set held constant.

    With S = sum_j p[idx_j] + 1e-20 and w_j = p[idx_j] / S:
      dp[idx_j] = (dw_j - sum_i dw_i w_i) / S, dp = 0 off the selected set;
      dlogits = p * (dp - sum_e p_e dp_e)   (softmax Jacobian)."""
    idx = np.asarray(idx).astype(np.int64)
    top = np.take_along_axis(probs, idx, axis=1)
    S = top.sum(axis=1, keepdims=True) + RENORM_EPS
    dtop = (dw - (dw * w).sum(axis=1, keepdims=True)) / S
    dp = np.zeros_like(probs)
    np.put_along_axis(dp, idx, dtop, axis=1)
    return probs * (dp - (probs * dp).sum(axis=1, keepdims=True))


def layer_backward(fwd: dict, dY, X, W_gu, W_d, k: int) -> dict:
    """Backward of ``layer_forward`` for upstream gradient dY [T, H].

    Per pair q = (t, j) on expert e in row r:
      dw_q = <dY_t, o_r>, do_r = w_q dY_t, dW_d[e] += do_r^T h_r,
      dh_r = do_r W_d[e], du = dh * silu(g), dg = dh * u * s * (1 + g (1 - s))
      with s = sigmoid(g), dW_gate[e] += dg^T X_t, dW_up[e] += du^T X_t,
      dX_t += dg W_gate[e] + du W_up[e]; then d logits via ``router_backward``."""
    dY = _f64(dY)
    X = _f64(X)
    W_gu = _f64(W_gu)
    W_d = _f64(W_d)
    T, H = X.shape
    E = W_gu.shape[0]
    I = W_d.shape[2]
    offsets, sorted_pair = fwd["offsets"], fwd["sorted_pair"]
    w_flat = fwd["w"].reshape(-1)
    dw_flat = np.zeros(T * k)
    dX = np.zeros((T, H))
    dW_gu = np.zeros((E, 2 * I, H))
    dW_d = np.zeros((E, H, I))
    for e in range(E):
        lo, hi = int(offsets[e]), int(offsets[e + 1])
        if lo == hi:
            continue
        q = sorted_pair[lo:hi]
        tok = q // k
        g, u, h, o = fwd["g"][lo:hi], fwd["u"][lo:hi], fwd["h"][lo:hi], fwd["o"][lo:hi]
        dYr = dY[tok]
        dw_flat[q] = (dYr * o).sum(axis=1)
        do = w_flat[q, None] * dYr
        dW_d[e] = do.T @ h
        dh = do @ W_d[e]
        s = sigmoid(g)
        du = dh * g * s
        dg = dh * u * s * (1.0 + g * (1.0 - s))
        dW_gu[e, :I] = dg.T @ X[tok]
        dW_gu[e, I:] = du.T @ X[tok]
        dX[tok] += dg @ W_gu[e, :I] + du @ W_gu[e, I:]   # tokens are distinct within e
    dw = dw_flat.reshape(T, k)
    dlogits = router_backward(dw, fwd["w"], fwd["probs"], fwd["idx"])
    return dict(dX=dX, dW_gu=dW_gu, dW_d=dW_d, dlogits=dlogits, dw=dw)


# ------------------------------------------------------------------ router Linear
def router_logits(X, W_r) -> np.ndarray:
    """logits = X W_r^T in float64. W_r [E, H] is the router's Linear(H -> E)
    weight ("Integration of fused moe kernel (e.g., megablocks) for efficient
    moe training", axolotl issue #3155, discussion of the router's weight
    shape: [num_experts, hidden_size], or nn.Linear(hidden_size, num_experts))."""
    return _f64(X) @ _f64(W_r).T


def router_logits_backward(dlogits, X, W_r):
    """Gradients of ``router_logits`` for upstream d logits [T, E]:
    dW_r = dlogits^T X  [E, H], and the router's share of dX, dlogits W_r  [T, H]
    (the layer's dX is the experts' dX plus this)."""
    dl = _f64(dlogits)
    return dl.T @ _f64(X), dl @ _f64(W_r)


# ------------------------------------------------------------------ LoRA adapters
# Source: fused-MoE Triton project summary (sourcepulse), *Highlighted
# Details*: LoRA (and QLoRA) on the fused expert weights, with conversion
# between the fused and the unfused adapter formats. The pages give no
# formulas; the adapter is the published LoRA update (Hu et al., "LoRA:
# Low-Rank Adaptation of Large Language Models", 2021): a frozen weight W
# [out, in] is used as W + scale * B A with A [r, in], B [out, r] trainable.
# Reading: one adapter per expert on each stacked weight -- A_gu [E, r, H] and
# B_gu [E, 2I, r] on W_gu (the fused gate|up format), A_d [E, r, I] and B_d
# [E, H, r] on W_d -- and one scale for all of them.
def lora_effective_weights(W_gu, W_d, A_gu, B_gu, A_d, B_d, scale: float):
    """The weights the layer uses: W_gu[e] + scale B_gu[e] A_gu[e] and
    W_d[e] + scale B_d[e] A_d[e], in float64."""
    W_gu_eff = _f64(W_gu) + scale * np.einsum("eor,eri->eoi", _f64(B_gu), _f64(A_gu))
    W_d_eff = _f64(W_d) + scale * np.einsum("eor,eri->eoi", _f64(B_d), _f64(A_d))
    return W_gu_eff, W_d_eff


def lora_layer_forward(logits, X, W_gu, W_d, k: int, A_gu, B_gu, A_d, B_d, scale: float) -> dict:
    """``layer_forward`` with the adapted weights (route, permute, SwiGLU
    experts, weighted combine are unchanged)."""
    W_gu_eff, W_d_eff = lora_effective_weights(W_gu, W_d, A_gu, B_gu, A_d, B_d, scale)
    fwd = layer_forward(logits, X, W_gu_eff, W_d_eff, k)
    fwd["W_gu_eff"], fwd["W_d_eff"] = W_gu_eff, W_d_eff
    return fwd


def lora_layer_backward(fwd: dict, dY, X, k: int, A_gu, B_gu, A_d, B_d, scale: float) -> dict:
    """Backward of ``lora_layer_forward``. dX and dlogits are those of the
    layer with the adapted weights; the gradient reaching a weight, G = dL/dW
    (the same for the frozen W and for W + scale B A), gives by the chain rule
    of W + scale B A: dA = scale B^T G and dB = scale G A^T, per expert."""
    g = layer_backward(fwd, dY, X, fwd["W_gu_eff"], fwd["W_d_eff"], k)
    sc = float(scale)
    G_gu, G_d = g["dW_gu"], g["dW_d"]
    g["dA_gu"] = sc * np.einsum("eor,eoi->eri", _f64(B_gu), G_gu)
    g["dB_gu"] = sc * np.einsum("eoi,eri->eor", G_gu, _f64(A_gu))
    g["dA_d"] = sc * np.einsum("eor,eoi->eri", _f64(B_d), G_d)
    g["dB_d"] = sc * np.einsum("eoi,eri->eor", G_d, _f64(A_d))
    return g


# ----------------------------------------------------------- sampled (large sizes)
def _pairs_by_expert(tokens, idx):
    """(row in the sample, slot j) pairs of the sampled tokens, grouped by expert."""
    groups = {}
    for n, t in enumerate(tokens):
        for j in range(idx.shape[1]):
            groups.setdefault(int(idx[t, j]), []).append((n, j))
    return groups


def token_forward(tokens, idx, w, X, W_gu, W_d) -> np.ndarray:
    """Y rows for a subset of tokens given the routing (idx, w) of the whole
    batch. Every output row depends only on its own token's pairs, so this is
    exact for the sampled rows; the pairs are visited expert by expert."""
    tokens = [int(t) for t in tokens]
    Xs = _f64(X[tokens])
    out = np.zeros((len(tokens), Xs.shape[1]))
    for e, pairs in sorted(_pairs_by_expert(tokens, idx).items()):
        n = np.array([a for a, _ in pairs])
        j = np.array([b for _, b in pairs])
        _, _, _, o = expert_mlp(Xs[n], _f64(W_gu[e]), _f64(W_d[e]))
        wt = np.asarray(w)[np.asarray(tokens)[n], j]
        np.add.at(out, n, wt[:, None] * o)
    return out


def token_backward(tokens, idx, w, probs, dY, X, W_gu, W_d) -> dict:
    """dX and d logits rows for a subset of tokens (each depends only on the
    token's own pairs), with the same formulas as ``layer_backward``."""
    tokens = [int(t) for t in tokens]
    tk = np.asarray(tokens)
    Xs = _f64(X[tokens])
    dYs = _f64(dY[tokens])
    k = idx.shape[1]
    dX = np.zeros_like(Xs)
    dw = np.zeros((len(tokens), k))
    for e, pairs in sorted(_pairs_by_expert(tokens, idx).items()):
        n = np.array([a for a, _ in pairs])
        j = np.array([b for _, b in pairs])
        Wgu = _f64(W_gu[e])
        Wd = _f64(W_d[e])
        I = Wd.shape[1]
        g, u, h, o = expert_mlp(Xs[n], Wgu, Wd)
        dw[n, j] = (dYs[n] * o).sum(axis=1)
        dh = (np.asarray(w)[tk[n], j][:, None] * dYs[n]) @ Wd
        s = sigmoid(g)
        du = dh * g * s
        dg = dh * u * s * (1.0 + g * (1.0 - s))
        np.add.at(dX, n, dg @ Wgu[:I] + du @ Wgu[I:])
    dlogits = router_backward(dw, np.asarray(w)[tk], np.asarray(probs)[tk], np.asarray(idx)[tk])
    return dict(dX=dX, dlogits=dlogits, dw=dw)


def expert_weight_grads(e: int, offsets, sorted_pair, w, dY, X, W_gu, W_d, k: int):
    """dW_gu[e] [2I, H] and dW_d[e] [H, I] for one expert (all its rows)."""
    lo, hi = int(offsets[e]), int(offsets[e + 1])
    Wgu = _f64(W_gu[e])
    Wd = _f64(W_d[e])
    I = Wd.shape[1]
    H = Wd.shape[0]
    if lo == hi:
        return np.zeros((2 * I, H)), np.zeros((H, I))
    q = np.asarray(sorted_pair[lo:hi]).astype(np.int64)
    tok = q // k
    x = _f64(X[tok])
    dYr = _f64(dY[tok])
    g, u, h, o = expert_mlp(x, Wgu, Wd)
    do = np.asarray(w).reshape(-1)[q, None] * dYr
    dW_d = do.T @ h
    dh = do @ Wd
    s = sigmoid(g)
    du = dh * g * s
    dg = dh * u * s * (1.0 + g * (1.0 - s))
    dW_gu = np.concatenate([dg.T @ x, du.T @ x], axis=0)
    return dW_gu, dW_d
