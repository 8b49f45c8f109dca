"""The C-ABI library builds, loads without a GPU, exports every function the
header declares, and rejects bad arguments before touching a device."""
import ctypes
import os

import pytest

from routed_grouped_gemm_router_b200 import binding as B


def test_library_exports_every_declared_symbol():
    lib = B.lib()
    names = B.header_symbols()
    assert {"moe_route", "moe_permute", "moe_experts_fwd", "moe_combine", "moe_layer_bwd"} <= set(names)
    for n in names:
        assert hasattr(lib, n), f"libmoe.so does not export {n}"


def test_status_strings():
    assert B.status_str(0) == "MOE_OK"
    assert B.status_str(1) == "MOE_ERR_INVALID_ARG"
    assert B.status_str(5) == "MOE_ERR_TIMEOUT"
    assert B.status_str(99) == "MOE_ERR_UNKNOWN"


def test_workspace_queries():
    lib = B.lib()
    assert lib.moe_permute_workspace_bytes(0, 8, 2) == 0
    assert lib.moe_permute_workspace_bytes(8192, 128, 8) >= 32 * 128 * 4
    assert lib.moe_permute_workspace_bytes(4, 2, 3) == 0, "k > E is invalid"
    P, H, I = 8192 * 8, 2048, 768
    need = lib.moe_layer_bwd_workspace_bytes(8192, 128, 8, H, I, 0)
    assert need >= P * (2 * H + 3 * I) * 2
    assert lib.moe_layer_bwd_workspace_bytes(8192, 128, 8, H, I, 1) >= need + P * 2 * I * 2
    assert lib.moe_layer_bwd_workspace_bytes(8192, 128, 8, 2047, I, 0) == 0, "H must be a multiple of 8"


NULL = None


def test_invalid_arguments_rejected_without_device():
    lib = B.lib()
    p = ctypes.c_void_p(256)  # aligned dummy address; never dereferenced
    odd = ctypes.c_void_p(257)
    # shapes
    assert lib.moe_route(p, 4, 3, 4, p, p, p, NULL) == 1          # k > E
    assert lib.moe_route(p, 4, 2000, 4, p, p, p, NULL) == 1       # E > 1024
    assert lib.moe_route(p, -1, 8, 2, p, p, p, NULL) == 1         # T < 0
    assert lib.moe_route(p, 1 << 28, 16, 16, p, p, p, NULL) == 1  # T*k >= 2^31
    # pointers
    assert lib.moe_route(NULL, 4, 8, 2, p, p, p, NULL) == 1
    assert lib.moe_route(odd, 4, 8, 2, p, p, p, NULL) == 1
    assert lib.moe_combine(p, p, 4, 2, 12, p, NULL) == 1          # H not a multiple of 8
    assert lib.moe_permute(p, 4, 8, 2, NULL, p, p, p, NULL, 0, NULL, p, 4096, NULL) == 1
    assert lib.moe_permute(p, 4, 8, 2, p, p, p, p, p, 16, NULL, p, 4096, NULL) == 1  # X without Xp
    # workspace
    assert lib.moe_permute(p, 4, 8, 2, p, p, p, p, NULL, 0, NULL, p, 0, NULL) == 3
    need = lib.moe_layer_bwd_workspace_bytes(4, 8, 2, 16, 16, 0)
    args = [p] * 10 + [4, 8, 2, 16, 16] + [p] * 6
    assert lib.moe_layer_bwd(*args, p, need - 1, NULL) == 3
    assert lib.moe_layer_bwd(*([p, p, NULL] + [p] * 7 + [4, 8, 2, 16, 16] + [p] * 6), p, need - 1, NULL) == 3
    # fp32 weight gradients: the same checks; dW pointers must be 16-byte aligned
    f32_args = [p] * 10 + [4, 8, 2, 16, 16] + [p] * 5
    for name in ("moe_layer_bwd_dw_f32", "moe_layer_bwd_x_dw_f32"):
        fn = getattr(lib, name)
        q = (lib.moe_layer_bwd_x_workspace_bytes if "_x_" in name else lib.moe_layer_bwd_workspace_bytes)(
            4, 8, 2, 16, 16, 0)
        assert fn(*f32_args, 0, p, p, q - 1, NULL) == 3
        assert fn(*f32_args, 1, p, p, q - 1, NULL) == 3
        assert fn(*([p] * 10 + [4, 8, 2, 16, 16] + [p] * 4 + [odd]), 0, p, p, q, NULL) == 1
        assert fn(*([p] * 10 + [4, 8, 2, 16, 16] + [p] * 3 + [NULL, p]), 1, p, p, q, NULL) == 1
        assert fn(*([p] * 10 + [4, 8, 2, 16, 12] + [p] * 5), 0, p, p, q, NULL) == 1  # I not a multiple of 8


def test_empty_batch_needs_no_device():
    lib = B.lib()
    p = ctypes.c_void_p(256)
    assert lib.moe_route(p, 0, 8, 2, p, p, p, NULL) == 0
    assert lib.moe_experts_fwd(p, p, p, p, 0, 8, 2, 16, 16, p, p, p, p, p, NULL) == 0
    assert lib.moe_combine(p, p, 0, 2, 16, p, NULL) == 0


def test_profile_names():
    names = B.profile_kernel_names()
    assert "gemm_fwd_gate_up" in names and "router_bwd" in names
    assert len(names) == len(set(names))
    d = ctypes.c_double()
    assert B.lib().moe_profile_read_clock(b"no_such_kernel", ctypes.byref(d)) == 1
    assert B.lib().moe_profile_read_clock(None, ctypes.byref(d)) == 1


def test_router_linear_arguments_rejected_without_device():
    lib = B.lib()
    p = ctypes.c_void_p(256)
    odd = ctypes.c_void_p(264 + 2)
    assert lib.moe_router_workspace_bytes(8192, 2048, 128) >= 3 * 128 * 2048 * 2 + 3 * 8192 * 128 * 2
    assert lib.moe_router_workspace_bytes(8, 12, 4) == 0, "H must be a multiple of 8"
    assert lib.moe_router_workspace_bytes(8, 16, 2000) == 0, "E > 1024"
    need = lib.moe_router_workspace_bytes(16, 16, 4)
    # forward: shapes, pointers, workspace
    assert lib.moe_router_fwd(p, p, 16, 12, 4, 2, p, p, p, p, p, need, NULL) == 1   # H % 8
    assert lib.moe_router_fwd(p, p, 16, 16, 4, 5, p, p, p, p, p, need, NULL) == 1   # k > E
    assert lib.moe_router_fwd(NULL, p, 16, 16, 4, 2, p, p, p, p, p, need, NULL) == 1
    assert lib.moe_router_fwd(p, odd, 16, 16, 4, 2, p, p, p, p, p, need, NULL) == 1
    assert lib.moe_router_fwd(p, p, 16, 16, 4, 2, NULL, p, p, NULL, p, need - 1, NULL) == 3
    assert lib.moe_router_fwd(p, p, 0, 16, 4, 2, NULL, NULL, NULL, NULL, NULL, 0, NULL) == 0  # empty batch
    # backward
    assert lib.moe_router_bwd(p, p, p, 16, 16, 4, NULL, NULL, NULL, 0, NULL) == 0      # nothing asked
    assert lib.moe_router_bwd(NULL, p, p, 16, 16, 4, p, NULL, p, need, NULL) == 1      # no dlogits
    assert lib.moe_router_bwd(p, NULL, p, 16, 16, 4, p, NULL, p, need, NULL) == 1      # dW_r needs X
    assert lib.moe_router_bwd(p, p, NULL, 16, 16, 4, NULL, p, p, need, NULL) == 1      # dX needs W_r
    assert lib.moe_router_bwd(p, p, p, 16, 16, 4, p, p, p, need - 1, NULL) == 3
    assert "gemm_router_logits" in B.profile_kernel_names()


def test_lora_arguments_rejected_without_device():
    lib = B.lib()
    p = ctypes.c_void_p(256)
    odd = ctypes.c_void_p(264 + 2)
    T, E, k, H, I = 4, 8, 2, 16, 16
    assert lib.moe_layer_bwd_lora_workspace_bytes(T, E, k, H, I, 16, 0) > lib.moe_layer_bwd_workspace_bytes(
        T, E, k, H, I, 0), "room for the adapter terms"
    for r in (0, 7, 12, 520):
        assert lib.moe_layer_bwd_lora_workspace_bytes(T, E, k, H, I, r, 0) == 0, f"rank {r}"
    assert lib.moe_layer_bwd_lora_workspace_bytes(T, E, k, H, I, 512, 0) > 0

    def fwd(r=16, a_gu=p, z_gu=p, scale=2.0):
        # Xp, offsets, sorted_pair, topk_w, T, E, k, H, I, W_gu, W_d, r, scale, A_gu, B_gu, A_d, B_d, h, gu, O, Z_gu, Z_d
        return lib.moe_experts_fwd_lora(p, p, p, p, T, E, k, H, I, p, p, r, scale, a_gu, p, p, p, p, p, p, z_gu, p,
                                        NULL)

    assert fwd(r=12) == 1
    assert fwd(r=520) == 1
    assert fwd(a_gu=NULL) == 1
    assert fwd(a_gu=odd) == 1
    assert fwd(z_gu=NULL) == 1
    need = lib.moe_layer_bwd_lora_workspace_bytes(T, E, k, H, I, 16, 0)

    def bwd(r=16, da=p, ws_bytes=need, dW_gu=NULL):
        head = [p] * 10 + [T, E, k, H, I] + [p, p, r, 2.0] + [p] * 4 + [p, p] + [p, da, p, p, p]
        return lib.moe_layer_bwd_lora(*head, 0, dW_gu, NULL, p, p, ws_bytes, NULL)

    assert bwd(r=9) == 1
    assert bwd(da=NULL) == 1                 # adapter gradients are required
    assert bwd(dW_gu=odd) == 1               # an optional base gradient must still be aligned
    assert bwd(ws_bytes=need - 1) == 3
    names = B.profile_kernel_names()
    assert {"gemm_lora_z_gate_up", "gemm_lora_da_down", "lora_weight_rows"} <= set(names)


C_CONSUMER = r"""
#include <stdio.h>
#include <string.h>
#include "moe.h"
int main(void) {
  /* calls that need no device: status strings, workspace sizes, argument checks */
  if (strcmp(moe_status_str(MOE_OK), moe_status_str(MOE_ERR_INVALID_ARG)) == 0) return 10;
  if (moe_permute_workspace_bytes(8192, 128, 8) == 0) return 11;
  if (moe_layer_bwd_workspace_bytes(8192, 128, 8, 2048, 768, 0) == 0) return 12;
  if (moe_layer_bwd_workspace_bytes(8192, 128, 8, 2047, 768, 0) != 0) return 13;
  if (moe_layer_bwd_lora_workspace_bytes(8192, 128, 8, 2048, 768, 12, 0) != 0) return 14;
  if (moe_router_workspace_bytes(8192, 2048, 128) == 0) return 15;
  void* p = (void*)(size_t)256;
  if (moe_route((const float*)p, 4, 3, 4, (int32_t*)p, (float*)p, (float*)p, NULL) != MOE_ERR_INVALID_ARG) return 16;
  if (moe_combine((const moe_bf16*)p, (const int32_t*)p, 4, 2, 12, (moe_bf16*)p, NULL) != MOE_ERR_INVALID_ARG) return 17;
  if (moe_profile_kernel_name(0) == NULL) return 18;
  printf("ok\n");
  return 0;
}
"""


def test_header_is_c_and_matches_the_library(tmp_path):
    """A plain C99 program compiled against include/moe.h and linked to the
    built library: the header is valid C, and its declarations resolve to the
    library's exports and behave as documented without a device."""
    import shutil
    import subprocess
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("no C compiler")
    lib = B.lib()._name
    src = tmp_path / "consumer.c"
    src.write_text(C_CONSUMER)
    exe = tmp_path / "consumer"
    inc = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include")
    r = subprocess.run([gcc, "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror", "-I", inc, str(src), lib,
                        f"-Wl,-rpath,{os.path.dirname(lib)}", "-o", str(exe)], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0 and r.stdout.strip() == "ok", (r.returncode, r.stdout, r.stderr)
