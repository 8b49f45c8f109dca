"""The layer's steps written with the CPU oracle, in the form the
expert-parallel plumbing calls them (the interface of ep.CudaOps), so that
the plumbing can be run on CPU ranks (test helper, not a test module).

Each step reuses the oracle's own functions: routing and permutation
(route, permute), the experts on explicitly given rows and weights
(token_forward with one pair per row), their backward (token_backward and
expert_weight_grads with one pair per row), combine and router_backward.
Tensors are float64 / int32 torch CPU tensors."""
from __future__ import annotations

import numpy as np
import torch

from oracle import moe_oracle as orc


def _t(a, dtype=torch.float64):
    return torch.from_numpy(np.ascontiguousarray(a)).to(dtype)


class OracleOps:
    def route_permute(self, logits, k, X):
        idx, w, probs = orc.route(logits.numpy(), k)
        E = logits.shape[1]
        counts, offsets, sorted_pair, pair_pos = orc.permute(idx, E)
        perm = dict(counts=_t(counts, torch.int32), offsets=_t(offsets, torch.int32),
                    sorted_pair=_t(sorted_pair, torch.int32), pair_pos=_t(pair_pos, torch.int32),
                    Xp=X[torch.from_numpy(np.asarray(sorted_pair) // k)])
        return _t(idx, torch.int32), _t(w), _t(probs), perm

    def pack_rows(self, offsets, sorted_pair, topk_w, T, E, k, E_l):
        off = offsets.numpy()
        le = np.zeros(T * k, dtype=np.int32)
        for e in range(E):
            le[off[e]:off[e + 1]] = e % E_l
        rw = topk_w.reshape(-1)[sorted_pair.long()]
        return _t(le, torch.int32), rw.clone()

    def permute(self, ids, E, X):
        k = ids.shape[1]
        counts, offsets, sorted_pair, pair_pos = orc.permute(ids.numpy(), E)
        return dict(counts=_t(counts, torch.int32), offsets=_t(offsets, torch.int32),
                    sorted_pair=_t(sorted_pair, torch.int32), pair_pos=_t(pair_pos, torch.int32),
                    Xp=X[torch.from_numpy(np.asarray(sorted_pair) // k)])

    def experts_fwd(self, Xp, offsets, sorted_pair, w, T, E, k, W_gu, W_d):
        # one pair per row (k = 1): row q's output is w_q times its expert's MLP
        assert k == 1
        if T == 0:
            return None, None, torch.zeros(0, Xp.shape[1], dtype=torch.float64)
        sp = sorted_pair.long()
        X_arr = torch.empty_like(Xp)
        X_arr[sp] = Xp
        ids = np.zeros((T, 1), dtype=np.int64)
        off = offsets.numpy()
        for e in range(E):
            ids[sp[off[e]:off[e + 1]].numpy(), 0] = e
        O_arr = orc.token_forward(range(T), ids, w.numpy().reshape(T, 1), X_arr.numpy(), W_gu, W_d)
        return None, None, _t(O_arr)[sp]

    def combine(self, O, pair_pos, T, k):
        return _t(orc.combine(O.numpy(), pair_pos.numpy(), T, k))

    def gather(self, idx, E, rows):
        k = idx.shape[1]
        _, _, sorted_pair, _ = orc.permute(idx.numpy(), E)
        return rows[torch.from_numpy(np.asarray(sorted_pair) // k)]

    def layer_bwd_pair_dw(self, dY, Xp, gu, h, w, offsets, sorted_pair, pair_pos, T, E, k, W_gu, W_d):
        assert k == 1
        if T == 0:  # no rows: no dX rows, no routing-weight gradients, zero weight gradients
            H, I = W_d.shape[1], W_d.shape[2]
            return dict(dX=torch.zeros(0, H, dtype=torch.float64), dw=torch.zeros(0, dtype=torch.float64),
                        dW_gu=torch.zeros(E, 2 * I, H, dtype=torch.float64),
                        dW_d=torch.zeros(E, H, I, dtype=torch.float64))
        sp = sorted_pair.long()
        X_arr = Xp[pair_pos.long()]
        ids = np.zeros((T, 1), dtype=np.int64)
        off = offsets.numpy()
        for e in range(E):
            ids[sp[off[e]:off[e + 1]].numpy(), 0] = e
        wa = w.numpy().reshape(T, 1)
        probs = np.zeros((T, E))
        probs[np.arange(T), ids[:, 0]] = 1.0  # only the router part reads it; its output is unused here
        b = orc.token_backward(range(T), ids, wa, probs, dY.numpy(), X_arr.numpy(), W_gu, W_d)
        dW_gu, dW_d = zip(*[orc.expert_weight_grads(e, off, sorted_pair.numpy(), wa, dY.numpy(), X_arr.numpy(),
                                                    W_gu, W_d, 1) for e in range(E)])
        return dict(dX=_t(b["dX"]), dw=_t(b["dw"].reshape(-1)), dW_gu=_t(np.stack(dW_gu)), dW_d=_t(np.stack(dW_d)))

    def router_bwd_from_dw(self, dw_rows, pair_pos, probs, idx, w):
        T, k = idx.shape
        dw = dw_rows.numpy()[pair_pos.numpy()].reshape(T, k)
        return _t(orc.router_backward(dw, w.numpy(), probs.numpy(), idx.numpy()))
