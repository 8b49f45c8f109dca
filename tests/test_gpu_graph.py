"""The whole layer step (the C-ABI calls of forward and backward, and of the
router Linear) captured once into a CUDA graph and replayed: the replay gives
bit-identical results to eager execution, also on new inputs copied into the
captured buffers."""
import pytest
import torch

from routed_grouped_gemm_router_b200 import binding as B
from routed_grouped_gemm_router_b200 import layer
from routed_grouped_gemm_router_b200.inputs import small_inputs

import gpu_util as U

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("router", [False, True])
def test_layer_step_replays_in_a_cuda_graph(router):
    T, H, E, k, I = 700, 256, 12, 3, 192
    dev = torch.device("cuda")
    a = small_inputs(T, H, E, k, I, seed=41)
    b = small_inputs(T, H, E, k, I, seed=42)
    d = U.to_dev(a)
    W_r = a.W_r.to(dev)
    bufs = layer.allocate(T, E, k, H, I, dev, router=router)
    X = d["X"].clone()
    logits = d["logits"].clone()
    dY = d["dY"].clone()

    def step():
        if router:
            st = layer.forward_from_x(X, W_r, d["W_gu"], d["W_d"], k, bufs=bufs)
            return st, layer.backward_to_x(st, dY, X, W_r, d["W_gu"], d["W_d"], bufs=bufs)
        st = layer.forward(logits, X, d["W_gu"], d["W_d"], k, bufs=bufs)
        return st, layer.backward(st, dY, d["W_gu"], d["W_d"], bufs=bufs)

    def snapshot(st, g):
        out = {"Y": st.Y.clone(), "dX": g["dX"].clone(), "dW_gu": g["dW_gu"].clone(), "dW_d": g["dW_d"].clone(),
               "dlogits": g["dlogits"].clone(), "idx": st.topk_idx.clone()}
        if router:
            out["dW_r"] = g["dW_r"].clone()
        return out

    # eager reference on both input sets (the buffers are reused by the graph)
    ref = []
    for inp in (a, b):
        X.copy_(inp.X.to(dev)); logits.copy_(inp.logits.to(dev)); dY.copy_(inp.dY.to(dev))
        ref.append(snapshot(*step()))
    torch.cuda.synchronize()

    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):  # warm the library's lazy set-up outside the capture
        step()
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        st, grads = step()
    for i, inp in enumerate((a, b)):
        X.copy_(inp.X.to(dev)); logits.copy_(inp.logits.to(dev)); dY.copy_(inp.dY.to(dev))
        g.replay()
        torch.cuda.synchronize()
        got = snapshot(st, grads)
        for name, t in ref[i].items():
            assert torch.equal(got[name], t), f"input set {i}: {name} differs after graph replay"
    assert B.last_device_status() == 0


def test_lora_step_replays_in_a_cuda_graph():
    """forward_lora + backward_lora (base weights frozen) captured once and
    replayed on two input sets: bit-identical to eager execution."""
    from routed_grouped_gemm_router_b200.inputs import make_lora
    T, H, E, k, I, r = 600, 256, 10, 3, 160, 16
    dev = torch.device("cuda")
    a = small_inputs(T, H, E, k, I, seed=51)
    b = small_inputs(T, H, E, k, I, seed=52)
    d = U.to_dev(a)
    lora = {n: t.to(dev) for n, t in make_lora(E, H, I, r, seed=3).items()}
    lora["scale"] = 2.0
    bufs = layer.allocate(T, E, k, H, I, dev, lora_r=r)
    X = d["X"].clone()
    logits = d["logits"].clone()
    dY = d["dY"].clone()

    def step():
        st = layer.forward_lora(logits, X, d["W_gu"], d["W_d"], k, lora, bufs=bufs)
        return st, layer.backward_lora(st, dY, d["W_gu"], d["W_d"], bufs=bufs)

    def snapshot(st, g):
        out = {n: g[n].clone() for n in ("dX", "dlogits", "dA_gu", "dB_gu", "dA_d", "dB_d")}
        out["Y"] = st.Y.clone()
        return out

    ref = []
    for inp in (a, b):
        X.copy_(inp.X.to(dev)); logits.copy_(inp.logits.to(dev)); dY.copy_(inp.dY.to(dev))
        ref.append(snapshot(*step()))
    torch.cuda.synchronize()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        step()
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        st, grads = step()
    for i, inp in enumerate((a, b)):
        X.copy_(inp.X.to(dev)); logits.copy_(inp.logits.to(dev)); dY.copy_(inp.dY.to(dev))
        g.replay()
        torch.cuda.synchronize()
        got = snapshot(st, grads)
        for name, t in ref[i].items():
            assert torch.equal(got[name], t), f"input set {i}: {name} differs after graph replay"
    assert B.last_device_status() == 0
