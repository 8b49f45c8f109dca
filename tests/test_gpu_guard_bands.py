"""Out-of-bounds writes (compute-sanitizer is closed here, so canaries stand
in for it): every output buffer and workspace of the layer is surrounded by
64 KiB guard bands filled with a canary byte. After a whole forward and
backward through the C ABI on ragged shapes, every band must be intact and
the results equal to those of the same step on plain buffers, bit for bit."""
import pytest
import torch

from routed_grouped_gemm_router_b200 import binding as B
from routed_grouped_gemm_router_b200 import layer
from routed_grouped_gemm_router_b200.inputs import small_inputs

import gpu_util as U

pytestmark = pytest.mark.gpu

GUARD = 64 * 1024  # bytes on each side
CANARY = 0x5B


class Guarded:
    """Buffers carved out of byte arrays with canary bands on both sides."""

    def __init__(self, dev):
        self.dev = dev
        self.raw = []

    def empty(self, shape, dtype):
        n = 1
        for s in shape:
            n *= s
        nbytes = n * torch.empty(0, dtype=dtype).element_size()
        raw = torch.full((GUARD + nbytes + GUARD,), CANARY, dtype=torch.uint8, device=self.dev)
        self.raw.append((raw, nbytes))
        return raw[GUARD:GUARD + nbytes].view(dtype).view(*shape)

    def like(self, t):
        return self.empty(tuple(t.shape), t.dtype)

    def intact(self):
        bad = []
        for i, (raw, nbytes) in enumerate(self.raw):
            head, tail = raw[:GUARD], raw[GUARD + nbytes:]
            if not (bool((head == CANARY).all()) and bool((tail == CANARY).all())):
                bad.append(i)
        return bad


def _guarded_bufs(T, E, k, H, I, dev, g):
    plain = layer.allocate(T, E, k, H, I, dev)
    out = {}
    for name, v in plain.items():
        if isinstance(v, dict):
            out[name] = {n: g.like(t) for n, t in v.items()}
        elif v is None:
            out[name] = None
        else:
            out[name] = g.like(v)
    return out


SHAPES = [
    (300, 200, 6, 2, 136),     # ragged H and I (partial TMA boxes everywhere)
    (1200, 512, 32, 4, 384),
    (2148, 256, 4, 2, 320),    # one expert across eight pair tiles plus a tail
    (97, 64, 1000, 8, 64),     # many empty experts
    (1, 64, 4, 2, 64),
]


@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "T%d_H%d_E%d_k%d_I%d" % s)
def test_no_write_outside_the_buffers(shape):
    T, H, E, k, I = shape
    inp = small_inputs(T, H, E, k, I, seed=sum(shape) + 5)
    if shape == (2148, 256, 4, 2, 320):
        inp.logits = (inp.logits + torch.tensor([30.0, 0, 0, 0])).contiguous()
    d = U.to_dev(inp)
    g = Guarded("cuda")
    bufs = _guarded_bufs(T, E, k, H, I, "cuda", g)
    st = layer.forward(d["logits"], d["X"], d["W_gu"], d["W_d"], k, bufs=bufs)
    grads = layer.backward(st, d["dY"], d["W_gu"], d["W_d"], bufs=bufs)
    assert B.last_device_status() == 0
    torch.cuda.synchronize()
    assert g.intact() == [], "a kernel wrote outside its buffer"
    ref_st, ref_g = U.run_layer(inp, k)
    for name in ("Y", "h", "O"):
        assert torch.equal(getattr(st, name), getattr(ref_st, name)), name
    for name in ("dX", "dW_gu", "dW_d", "dlogits"):
        assert torch.equal(grads[name], ref_g[name]), name
