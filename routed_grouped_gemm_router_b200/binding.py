"""Thin ctypes binding of the C ABI in include/moe.h.

Each function has the C call's name and only marshals arguments: it checks
dtypes/shapes/devices of the torch tensors, allocates missing outputs with
torch (the library itself never allocates) and passes raw pointers and the
current CUDA stream. Every step of the layer runs in the CUDA library; when
the library is missing this module raises instead of computing anything.
"""
from __future__ import annotations

import ctypes
import os
import re

import torch

from . import build as _build

_LIB = None
_c_void = ctypes.c_void_p
_c_int = ctypes.c_int
_c_size = ctypes.c_size_t

_SIGNATURES = {
    "moe_status_str": (ctypes.c_char_p, [_c_int]),
    "moe_launch_count": (ctypes.c_ulonglong, []),
    "moe_last_device_status": (_c_int, [_c_void]),
    "moe_route": (_c_int, [_c_void, _c_int, _c_int, _c_int, _c_void, _c_void, _c_void, _c_void]),
    "moe_permute_workspace_bytes": (_c_size, [_c_int, _c_int, _c_int]),
    "moe_permute": (_c_int, [_c_void, _c_int, _c_int, _c_int, _c_void, _c_void, _c_void, _c_void, _c_void,
                             _c_int, _c_void, _c_void, _c_size, _c_void]),
    "moe_route_permute_workspace_bytes": (_c_size, [_c_int, _c_int, _c_int]),
    "moe_route_permute": (_c_int, [_c_void, _c_int, _c_int, _c_int] + [_c_void] * 7 + [_c_void, _c_int, _c_void,
                                                                                     _c_void, _c_size, _c_void]),
    "moe_ep_pack_rows": (_c_int, [_c_void, _c_void, _c_void, _c_int, _c_int, _c_int, _c_int, _c_void, _c_void,
                                  _c_void]),
    "moe_layer_bwd_pair_dw": (_c_int, [_c_void] * 8 + [_c_int] * 5 + [_c_void] * 6 + [_c_void, _c_size, _c_void]),
    "moe_router_bwd_from_dw": (_c_int, [_c_void] * 5 + [_c_int] * 3 + [_c_void, _c_void]),
    "moe_permute_noalloc": (_c_int, [_c_void, _c_int, _c_int, _c_int, _c_void, _c_void, _c_void, _c_void,
                                     _c_void, _c_int, _c_void, _c_void]),
    "moe_experts_fwd": (_c_int, [_c_void, _c_void, _c_void, _c_void, _c_int, _c_int, _c_int, _c_int, _c_int,
                                 _c_void, _c_void, _c_void, _c_void, _c_void, _c_void]),
    "moe_experts_fwd_x": (_c_int, [_c_void, _c_void, _c_void, _c_void, _c_int, _c_int, _c_int, _c_int, _c_int,
                                   _c_void, _c_void, _c_void, _c_void, _c_void, _c_void]),
    "moe_combine": (_c_int, [_c_void, _c_void, _c_int, _c_int, _c_int, _c_void, _c_void]),
    "moe_layer_bwd_workspace_bytes": (_c_size, [_c_int, _c_int, _c_int, _c_int, _c_int, _c_int]),
    "moe_layer_bwd": (_c_int, [_c_void] * 10 + [_c_int] * 5 + [_c_void] * 6 + [_c_void, _c_size, _c_void]),
    "moe_layer_bwd_x_workspace_bytes": (_c_size, [_c_int, _c_int, _c_int, _c_int, _c_int, _c_int]),
    "moe_layer_bwd_x": (_c_int, [_c_void] * 10 + [_c_int] * 5 + [_c_void] * 6 + [_c_void, _c_size, _c_void]),
    "moe_layer_bwd_dw_f32": (_c_int, [_c_void] * 10 + [_c_int] * 5 + [_c_void] * 5 + [_c_int, _c_void, _c_void,
                                                                                     _c_size, _c_void]),
    "moe_layer_bwd_x_dw_f32": (_c_int, [_c_void] * 10 + [_c_int] * 5 + [_c_void] * 5 + [_c_int, _c_void, _c_void,
                                                                                       _c_size, _c_void]),
    "moe_experts_fwd_lora": (_c_int, [_c_void] * 4 + [_c_int] * 5 + [_c_void] * 2 + [_c_int, ctypes.c_float]
                             + [_c_void] * 9 + [_c_void]),
    "moe_layer_bwd_lora_workspace_bytes": (_c_size, [_c_int] * 7),
    "moe_layer_bwd_lora": (_c_int, [_c_void] * 10 + [_c_int] * 5 + [_c_void] * 2 + [_c_int, ctypes.c_float]
                           + [_c_void] * 11 + [_c_int] + [_c_void] * 4 + [_c_size, _c_void]),
    "moe_router_workspace_bytes": (_c_size, [_c_int, _c_int, _c_int]),
    "moe_router_fwd": (_c_int, [_c_void, _c_void, _c_int, _c_int, _c_int, _c_int, _c_void, _c_void, _c_void,
                                _c_void, _c_void, _c_size, _c_void]),
    "moe_router_bwd": (_c_int, [_c_void, _c_void, _c_void, _c_int, _c_int, _c_int, _c_void, _c_void, _c_void,
                                _c_size, _c_void]),
    "moe_selftest_wait_timeout": (_c_int, [_c_int, _c_void]),
    "moe_profile_enable": (_c_int, [_c_int]),
    "moe_profile_only": (_c_int, [ctypes.c_char_p]),
    "moe_profile_read": (_c_int, [ctypes.c_char_p, ctypes.POINTER(ctypes.c_double), ctypes.POINTER(_c_int)]),
    "moe_profile_kernel_name": (ctypes.c_char_p, [_c_int]),
    "moe_profile_read_clock": (_c_int, [ctypes.c_char_p, ctypes.POINTER(ctypes.c_double)]),
}


class MoeError(RuntimeError):
    def __init__(self, call: str, status: int):
        super().__init__(f"{call} failed: {status_str(status)} ({status})")
        self.status = status


def lib() -> ctypes.CDLL:
    """Loads libmoe.so (building it first when nvcc is available)."""
    global _LIB
    if _LIB is None:
        path = _build.LIB_PATH
        if not _build.up_to_date():
            _build.build()
        if not os.path.exists(path):
            raise RuntimeError("libmoe.so is not built; the MoE layer has no other implementation")
        l = ctypes.CDLL(path)
        for name, (res, args) in _SIGNATURES.items():
            f = getattr(l, name)
            f.restype = res
            f.argtypes = args
        _LIB = l
    return _LIB


def header_symbols() -> list[str]:
    """Function names declared in include/*.h."""
    names = []
    for f in sorted(os.listdir(_build.INCLUDE)):
        if f.endswith(".h"):
            text = open(os.path.join(_build.INCLUDE, f)).read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            names += re.findall(r"\b(moe_[a-z_0-9]+)\s*\(", text)
    return sorted(set(names))


def status_str(status: int) -> str:
    return lib().moe_status_str(status).decode()


def _check(call: str, status: int):
    if status != 0:
        raise MoeError(call, status)


def _ptr(t: torch.Tensor | None):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _need(t: torch.Tensor, dtype, shape, name):
    if t.dtype != dtype or tuple(t.shape) != tuple(shape) or not t.is_contiguous() or not t.is_cuda:
        raise ValueError(f"{name}: expected contiguous CUDA {dtype} {tuple(shape)}, got "
                         f"{t.dtype} {tuple(t.shape)} on {t.device}")


def launch_count() -> int:
    """Kernels the library has launched in this process so far."""
    return int(lib().moe_launch_count())


def last_device_status(stream=None) -> int:
    return lib().moe_last_device_status(_stream(stream))


# ------------------------------------------------------------------- calls
def moe_route(logits: torch.Tensor, k: int, topk_idx=None, topk_w=None, probs=None, want_probs=True, stream=None):
    T, E = logits.shape
    dev = logits.device
    _need(logits, torch.float32, (T, E), "logits")
    topk_idx = torch.empty(T, k, dtype=torch.int32, device=dev) if topk_idx is None else topk_idx
    topk_w = torch.empty(T, k, dtype=torch.float32, device=dev) if topk_w is None else topk_w
    if probs is None and want_probs:
        probs = torch.empty(T, E, dtype=torch.float32, device=dev)
    _check("moe_route", lib().moe_route(_ptr(logits), T, E, k, _ptr(topk_idx), _ptr(topk_w), _ptr(probs),
                                        _stream(stream)))
    return topk_idx, topk_w, probs


def moe_permute(topk_idx: torch.Tensor, E: int, X: torch.Tensor | None = None, out=None, ws=None, stream=None):
    T, k = topk_idx.shape
    dev = topk_idx.device
    _need(topk_idx, torch.int32, (T, k), "topk_idx")
    P = T * k
    o = dict(out or {})
    o.setdefault("counts", torch.empty(E, dtype=torch.int32, device=dev))
    o.setdefault("offsets", torch.empty(E + 1, dtype=torch.int32, device=dev))
    o.setdefault("sorted_pair", torch.empty(P, dtype=torch.int32, device=dev))
    o.setdefault("pair_pos", torch.empty(P, dtype=torch.int32, device=dev))
    H = 0
    if X is not None:
        H = X.shape[1]
        _need(X, torch.bfloat16, (T, H), "X")
        o.setdefault("Xp", torch.empty(P, H, dtype=torch.bfloat16, device=dev))
    need = lib().moe_permute_workspace_bytes(T, E, k)
    if ws is None:
        ws = torch.empty(max(need, 1), dtype=torch.uint8, device=dev)
    _check("moe_permute", lib().moe_permute(
        _ptr(topk_idx), T, E, k, _ptr(o["counts"]), _ptr(o["offsets"]), _ptr(o["sorted_pair"]),
        _ptr(o["pair_pos"]), _ptr(X), H, _ptr(o.get("Xp")), _ptr(ws), ws.numel(), _stream(stream)))
    return o


def moe_route_permute(logits: torch.Tensor, k: int, X: torch.Tensor | None = None, topk_idx=None, topk_w=None,
                      probs=None, want_probs=True, out=None, ws=None, stream=None):
    """moe_route then moe_permute in one call (two kernels plus the gather);
    returns (topk_idx, topk_w, probs, perm) with perm as moe_permute's."""
    T, E = logits.shape
    dev = logits.device
    _need(logits, torch.float32, (T, E), "logits")
    P = T * k
    topk_idx = torch.empty(T, k, dtype=torch.int32, device=dev) if topk_idx is None else topk_idx
    topk_w = torch.empty(T, k, dtype=torch.float32, device=dev) if topk_w is None else topk_w
    if probs is None and want_probs:
        probs = torch.empty(T, E, dtype=torch.float32, device=dev)
    _need(topk_idx, torch.int32, (T, k), "topk_idx")
    _need(topk_w, torch.float32, (T, k), "topk_w")
    o = dict(out or {})
    o.setdefault("counts", torch.empty(E, dtype=torch.int32, device=dev))
    o.setdefault("offsets", torch.empty(E + 1, dtype=torch.int32, device=dev))
    o.setdefault("sorted_pair", torch.empty(P, dtype=torch.int32, device=dev))
    o.setdefault("pair_pos", torch.empty(P, dtype=torch.int32, device=dev))
    H = 0
    if X is not None:
        H = X.shape[1]
        _need(X, torch.bfloat16, (T, H), "X")
        o.setdefault("Xp", torch.empty(P, H, dtype=torch.bfloat16, device=dev))
    need = lib().moe_route_permute_workspace_bytes(T, E, k)
    if ws is None:
        ws = torch.empty(max(need, 1), dtype=torch.uint8, device=dev)
    _check("moe_route_permute", lib().moe_route_permute(
        _ptr(logits), T, E, k, _ptr(topk_idx), _ptr(topk_w), _ptr(probs), _ptr(o["counts"]), _ptr(o["offsets"]),
        _ptr(o["sorted_pair"]), _ptr(o["pair_pos"]), _ptr(X), H, _ptr(o.get("Xp")), _ptr(ws), ws.numel(),
        _stream(stream)))
    return topk_idx, topk_w, probs, o


def moe_experts_fwd(Xp, offsets, sorted_pair, topk_w, T, E, k, W_gu, W_d, h=None, gu_save=None, O=None,
                    save_gu=True, stream=None, gather=False):
    """gather=True: `Xp` is X [T, H] in token order (moe_experts_fwd_x)."""
    P = T * k
    H = W_gu.shape[2]
    I = W_d.shape[2]
    dev = Xp.device
    _need(Xp, torch.bfloat16, (T if gather else P, H), "X" if gather else "Xp")
    _need(W_gu, torch.bfloat16, (E, 2 * I, H), "W_gu")
    _need(W_d, torch.bfloat16, (E, H, I), "W_d")
    h = torch.empty(P, I, dtype=torch.bfloat16, device=dev) if h is None else h
    if gu_save is None and save_gu:
        gu_save = torch.empty(P, 2 * I, dtype=torch.bfloat16, device=dev)
    O = torch.empty(P, H, dtype=torch.bfloat16, device=dev) if O is None else O
    name = "moe_experts_fwd_x" if gather else "moe_experts_fwd"
    _check(name, getattr(lib(), name)(
        _ptr(Xp), _ptr(offsets), _ptr(sorted_pair), _ptr(topk_w), T, E, k, H, I, _ptr(W_gu), _ptr(W_d),
        _ptr(h), _ptr(gu_save), _ptr(O), _stream(stream)))
    return h, gu_save, O


def _lora_check(lora, E, H, I):
    r = lora["A_gu"].shape[1]
    _need(lora["A_gu"], torch.bfloat16, (E, r, H), "A_gu")
    _need(lora["B_gu"], torch.bfloat16, (E, 2 * I, r), "B_gu")
    _need(lora["A_d"], torch.bfloat16, (E, r, I), "A_d")
    _need(lora["B_d"], torch.bfloat16, (E, H, r), "B_d")
    return r


def moe_experts_fwd_lora(Xp, offsets, sorted_pair, topk_w, T, E, k, W_gu, W_d, lora: dict, h=None, gu_save=None,
                         O=None, Z_gu=None, Z_d=None, save_gu=True, stream=None):
    """moe_experts_fwd with LoRA adapters: lora = {A_gu, B_gu, A_d, B_d
    (bf16), scale}. Returns h, gu_save, O, Z_gu, Z_d (the adapter
    activations the backward takes)."""
    P = T * k
    H = W_gu.shape[2]
    I = W_d.shape[2]
    dev = Xp.device
    _need(Xp, torch.bfloat16, (P, H), "Xp")
    r = _lora_check(lora, E, H, I)
    h = torch.empty(P, I, dtype=torch.bfloat16, device=dev) if h is None else h
    if gu_save is None and save_gu:
        gu_save = torch.empty(P, 2 * I, dtype=torch.bfloat16, device=dev)
    O = torch.empty(P, H, dtype=torch.bfloat16, device=dev) if O is None else O
    Z_gu = torch.empty(P, r, dtype=torch.bfloat16, device=dev) if Z_gu is None else Z_gu
    Z_d = torch.empty(P, r, dtype=torch.bfloat16, device=dev) if Z_d is None else Z_d
    _check("moe_experts_fwd_lora", lib().moe_experts_fwd_lora(
        _ptr(Xp), _ptr(offsets), _ptr(sorted_pair), _ptr(topk_w), T, E, k, H, I, _ptr(W_gu), _ptr(W_d), r,
        float(lora["scale"]), _ptr(lora["A_gu"]), _ptr(lora["B_gu"]), _ptr(lora["A_d"]), _ptr(lora["B_d"]),
        _ptr(h), _ptr(gu_save), _ptr(O), _ptr(Z_gu), _ptr(Z_d), _stream(stream)))
    return h, gu_save, O, Z_gu, Z_d


def moe_layer_bwd_lora(dY, Xp, gu_save, h, probs, topk_idx, topk_w, offsets, sorted_pair, pair_pos, T, E, k,
                       W_gu, W_d, lora: dict, Z_gu, Z_d, out=None, ws=None, stream=None, accumulate=False,
                       base_grads=False):
    """Backward of the adapted layer: dX, dlogits and the fp32 adapter
    gradients dA_gu, dB_gu, dA_d, dB_d (added to out's when accumulate);
    base_grads=True also gives the bf16 dW_gu, dW_d (else the base weights
    are frozen and their GEMMs skipped)."""
    H = W_gu.shape[2]
    I = W_d.shape[2]
    dev = dY.device
    r = _lora_check(lora, E, H, I)
    if accumulate and not (out and all(n in out for n in ("dA_gu", "dB_gu", "dA_d", "dB_d"))):
        raise ValueError("accumulate needs dA_gu, dB_gu, dA_d and dB_d given in `out`")
    o = dict(out or {})
    f32 = torch.float32
    o.setdefault("dX", torch.empty(T, H, dtype=torch.bfloat16, device=dev))
    o.setdefault("dlogits", torch.empty(T, E, dtype=f32, device=dev))
    o.setdefault("dA_gu", torch.empty(E, r, H, dtype=f32, device=dev))
    o.setdefault("dB_gu", torch.empty(E, 2 * I, r, dtype=f32, device=dev))
    o.setdefault("dA_d", torch.empty(E, r, I, dtype=f32, device=dev))
    o.setdefault("dB_d", torch.empty(E, H, r, dtype=f32, device=dev))
    for n, shape in (("dA_gu", (E, r, H)), ("dB_gu", (E, 2 * I, r)), ("dA_d", (E, r, I)), ("dB_d", (E, H, r))):
        _need(o[n], f32, shape, n)
    if base_grads:
        o.setdefault("dW_gu", torch.empty(E, 2 * I, H, dtype=torch.bfloat16, device=dev))
        o.setdefault("dW_d", torch.empty(E, H, I, dtype=torch.bfloat16, device=dev))
    need = lib().moe_layer_bwd_lora_workspace_bytes(T, E, k, H, I, r, 1 if gu_save is None else 0)
    if ws is None:
        ws = torch.empty(max(need, 1), dtype=torch.uint8, device=dev)
    _check("moe_layer_bwd_lora", lib().moe_layer_bwd_lora(
        _ptr(dY), _ptr(Xp), _ptr(gu_save), _ptr(h), _ptr(probs), _ptr(topk_idx), _ptr(topk_w), _ptr(offsets),
        _ptr(sorted_pair), _ptr(pair_pos), T, E, k, H, I, _ptr(W_gu), _ptr(W_d), r, float(lora["scale"]),
        _ptr(lora["A_gu"]), _ptr(lora["B_gu"]), _ptr(lora["A_d"]), _ptr(lora["B_d"]), _ptr(Z_gu), _ptr(Z_d),
        _ptr(o["dX"]), _ptr(o["dA_gu"]), _ptr(o["dB_gu"]), _ptr(o["dA_d"]), _ptr(o["dB_d"]),
        1 if accumulate else 0, _ptr(o.get("dW_gu") if base_grads else None),
        _ptr(o.get("dW_d") if base_grads else None), _ptr(o["dlogits"]), _ptr(ws), ws.numel(), _stream(stream)))
    return o


def moe_combine(O, pair_pos, T, k, Y=None, stream=None):
    H = O.shape[1]
    Y = torch.empty(T, H, dtype=torch.bfloat16, device=O.device) if Y is None else Y
    _check("moe_combine", lib().moe_combine(_ptr(O), _ptr(pair_pos), T, k, H, _ptr(Y), _stream(stream)))
    return Y


def moe_layer_bwd(dY, Xp, gu_save, h, probs, topk_idx, topk_w, offsets, sorted_pair, pair_pos, T, E, k,
                  W_gu, W_d, out=None, ws=None, stream=None, gather=False, dw_dtype=torch.bfloat16,
                  accumulate=False):
    """gather=True: `Xp` is X [T, H] in token order (moe_layer_bwd_x).
    dw_dtype=torch.float32: fp32 weight gradients (moe_layer_bwd_dw_f32);
    accumulate=True then adds them to out["dW_gu"] / out["dW_d"]."""
    H = W_gu.shape[2]
    I = W_d.shape[2]
    dev = dY.device
    f32 = dw_dtype == torch.float32
    if not f32 and dw_dtype != torch.bfloat16:
        raise ValueError(f"dw_dtype must be bfloat16 or float32, not {dw_dtype}")
    if accumulate and not (f32 and out and "dW_gu" in out and "dW_d" in out):
        raise ValueError("accumulate needs float32 dW_gu and dW_d given in `out`")
    o = dict(out or {})
    o.setdefault("dX", torch.empty(T, H, dtype=torch.bfloat16, device=dev))
    o.setdefault("dW_gu", torch.empty(E, 2 * I, H, dtype=dw_dtype, device=dev))
    o.setdefault("dW_d", torch.empty(E, H, I, dtype=dw_dtype, device=dev))
    o.setdefault("dlogits", torch.empty(T, E, dtype=torch.float32, device=dev))
    _need(o["dW_gu"], dw_dtype, (E, 2 * I, H), "dW_gu")
    _need(o["dW_d"], dw_dtype, (E, H, I), "dW_d")
    query = lib().moe_layer_bwd_x_workspace_bytes if gather else lib().moe_layer_bwd_workspace_bytes
    need = query(T, E, k, H, I, 1 if gu_save is None else 0)
    if ws is None:
        ws = torch.empty(max(need, 1), dtype=torch.uint8, device=dev)
    name = "moe_layer_bwd_x" if gather else "moe_layer_bwd"
    head = (_ptr(dY), _ptr(Xp), _ptr(gu_save), _ptr(h), _ptr(probs), _ptr(topk_idx), _ptr(topk_w), _ptr(offsets),
            _ptr(sorted_pair), _ptr(pair_pos), T, E, k, H, I, _ptr(W_gu), _ptr(W_d), _ptr(o["dX"]),
            _ptr(o["dW_gu"]), _ptr(o["dW_d"]))
    tail = (_ptr(o["dlogits"]), _ptr(ws), ws.numel(), _stream(stream))
    if f32:
        name += "_dw_f32"
        _check(name, getattr(lib(), name)(*head, 1 if accumulate else 0, *tail))
    else:
        _check(name, getattr(lib(), name)(*head, *tail))
    return o


def moe_ep_pack_rows(offsets, sorted_pair, topk_w, T, E, k, experts_per_rank, out=None, stream=None):
    """Per expert-sorted row: its expert's index on the owner rank and its
    routing weight; returns (local_expert [T*k] int32, row_w [T*k] fp32)."""
    P = T * k
    dev = offsets.device
    o = dict(out or {})
    le = o.get("local_expert", torch.empty(P, dtype=torch.int32, device=dev))
    rw = o.get("row_w", torch.empty(P, dtype=torch.float32, device=dev))
    _check("moe_ep_pack_rows", lib().moe_ep_pack_rows(_ptr(offsets), _ptr(sorted_pair), _ptr(topk_w), T, E, k,
                                                      experts_per_rank, _ptr(le), _ptr(rw), _stream(stream)))
    return le, rw


def moe_layer_bwd_pair_dw(dY, Xp, gu_save, h, topk_w, offsets, sorted_pair, pair_pos, T, E, k, W_gu, W_d,
                          out=None, ws=None, stream=None):
    """moe_layer_bwd returning each pair's routing-weight gradient (out["dw"]
    [T*k] fp32) in place of d logits; returns the dict of dX, dW_gu, dW_d, dw."""
    H = W_gu.shape[2]
    I = W_d.shape[2]
    dev = dY.device
    o = dict(out or {})
    o.setdefault("dX", torch.empty(T, H, dtype=torch.bfloat16, device=dev))
    o.setdefault("dW_gu", torch.empty(E, 2 * I, H, dtype=torch.bfloat16, device=dev))
    o.setdefault("dW_d", torch.empty(E, H, I, dtype=torch.bfloat16, device=dev))
    o.setdefault("dw", torch.empty(T * k, dtype=torch.float32, device=dev))
    need = lib().moe_layer_bwd_workspace_bytes(T, E, k, H, I, 1 if gu_save is None else 0)
    if ws is None or ws.numel() < need:
        ws = torch.empty(max(need, 1), dtype=torch.uint8, device=dev)
    _check("moe_layer_bwd_pair_dw", lib().moe_layer_bwd_pair_dw(
        _ptr(dY), _ptr(Xp), _ptr(gu_save), _ptr(h), _ptr(topk_w), _ptr(offsets), _ptr(sorted_pair), _ptr(pair_pos),
        T, E, k, H, I, _ptr(W_gu), _ptr(W_d), _ptr(o["dX"]), _ptr(o["dW_gu"]), _ptr(o["dW_d"]), _ptr(o["dw"]),
        _ptr(ws), ws.numel(), _stream(stream)))
    return o


def moe_router_bwd_from_dw(dw_rows, pair_pos, probs, topk_idx, topk_w, dlogits=None, stream=None):
    """d logits from routing-weight gradients given per expert-sorted row."""
    T, E = probs.shape
    k = topk_idx.shape[1]
    if dlogits is None:
        dlogits = torch.empty(T, E, dtype=torch.float32, device=probs.device)
    _check("moe_router_bwd_from_dw", lib().moe_router_bwd_from_dw(
        _ptr(dw_rows), _ptr(pair_pos), _ptr(probs), _ptr(topk_idx), _ptr(topk_w), T, E, k, _ptr(dlogits),
        _stream(stream)))
    return dlogits


def _router_ws(T, H, E, dev, ws):
    need = lib().moe_router_workspace_bytes(T, H, E)
    if ws is None:
        ws = torch.empty(max(need, 1), dtype=torch.uint8, device=dev)
    return ws


def moe_router_fwd(X, W_r, k, out=None, want_logits=True, want_probs=True, ws=None, stream=None):
    """logits = X W_r^T on the GPU, then routing; returns a dict with
    logits, topk_idx, topk_w, probs (logits/probs None when not wanted)."""
    T, H = X.shape
    E = W_r.shape[0]
    dev = X.device
    _need(X, torch.bfloat16, (T, H), "X")
    _need(W_r, torch.float32, (E, H), "W_r")
    o = dict(out or {})
    if want_logits:
        o.setdefault("logits", torch.empty(T, E, dtype=torch.float32, device=dev))
    if want_probs:
        o.setdefault("probs", torch.empty(T, E, dtype=torch.float32, device=dev))
    o.setdefault("topk_idx", torch.empty(T, k, dtype=torch.int32, device=dev))
    o.setdefault("topk_w", torch.empty(T, k, dtype=torch.float32, device=dev))
    ws = _router_ws(T, H, E, dev, ws)
    _check("moe_router_fwd", lib().moe_router_fwd(
        _ptr(X), _ptr(W_r), T, H, E, k, _ptr(o.get("logits")), _ptr(o["topk_idx"]), _ptr(o["topk_w"]),
        _ptr(o.get("probs")), _ptr(ws), ws.numel(), _stream(stream)))
    return o


def moe_router_bwd(dlogits, X, W_r, dX=None, dW_r=None, want_dW_r=True, ws=None, stream=None):
    """dW_r = dlogits^T X (fp32, allocated when not given and wanted) and, when
    dX is given, dX += dlogits W_r in place. Returns (dW_r, dX)."""
    T, E = dlogits.shape
    H = W_r.shape[1]
    dev = dlogits.device
    _need(dlogits, torch.float32, (T, E), "dlogits")
    _need(W_r, torch.float32, (E, H), "W_r")
    _need(X, torch.bfloat16, (T, H), "X")
    if dX is not None:
        _need(dX, torch.bfloat16, (T, H), "dX")
    if dW_r is None and want_dW_r:
        dW_r = torch.empty(E, H, dtype=torch.float32, device=dev)
    ws = _router_ws(T, H, E, dev, ws)
    _check("moe_router_bwd", lib().moe_router_bwd(
        _ptr(dlogits), _ptr(X), _ptr(W_r), T, H, E, _ptr(dW_r), _ptr(dX), _ptr(ws), ws.numel(),
        _stream(stream)))
    return dW_r, dX


# --------------------------------------------------------------- profiling
def profile_enable(on: bool = True):
    _check("moe_profile_enable", lib().moe_profile_enable(1 if on else 0))


def profile_only(name: str | None):
    """Record only kernel `name` (None: all) until the next profile_enable."""
    _check("moe_profile_only", lib().moe_profile_only(None if name is None else name.encode()))


def profile_kernel_names() -> list[str]:
    names, i = [], 0
    while True:
        n = lib().moe_profile_kernel_name(i)
        if n is None:
            return names
        names.append(n.decode())
        i += 1


def profile_read() -> dict:
    """{kernel name: (total device ms, launches)} of the recorded launches."""
    out = {}
    for n in profile_kernel_names():
        ms = ctypes.c_double()
        cnt = ctypes.c_int()
        _check("moe_profile_read", lib().moe_profile_read(n.encode(), ctypes.byref(ms), ctypes.byref(cnt)))
        if cnt.value:
            out[n] = (ms.value, cnt.value)
    return out


def profile_read_clock(name: str) -> float:
    """Effective SM clock (MHz) of GEMM kernel `name` over its recorded
    launches, from the kernel's own cycle and nanosecond counters (0: none)."""
    mhz = ctypes.c_double()
    _check("moe_profile_read_clock", lib().moe_profile_read_clock(name.encode(), ctypes.byref(mhz)))
    return mhz.value
