"""Failure detection on the GPU without a GPU fault: every wait inside the tensor-core kernels is
bounded. With the bound set to 1 ns a wait runs out at once, the kernel records status flag 2,
drains its own loads and MMAs and returns; the host reads the flag, and the same process then
runs the layer correctly. Nothing here traps, faults or hangs a GPU."""
import pytest
import torch

import oracle as O

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import sparse_hierarchical_attention_b200 as lh
    from sparse_hierarchical_attention_b200 import LighthouseLayer, Shape, _lib

from gpu_util import assert_close, np64

LH_ERR_DEVICE = 5


def _inputs(shape, seed):
    g = torch.Generator(device="cuda").manual_seed(seed)
    return [torch.randn(shape.B, shape.H, shape.N, shape.d, generator=g, device="cuda").to(shape.dtype)
            for _ in range(4)]


@pytest.mark.parametrize("d", [128, 64])
@pytest.mark.parametrize("det", [False, True])
@pytest.mark.parametrize("S", [128, 512])
def test_wait_timeout_is_reported_and_the_next_call_is_correct(S, det, d):
    """One CTA per attention kernel at S = 128 (several at 512): the forward, and the one-pass
    (det=False) or two-pass (det=True) backward, all run out of their waits. At d = 64 the
    one-pass kernel's compute warps still meet at the barriers around the dQ staging."""
    shape = Shape(1, 1, S, d, 4, 1, S, torch.bfloat16, det)  # L = 1: dense causal attention
    q, k, v, d_o = _inputs(shape, S)
    layer = LighthouseLayer(shape)
    prev = lh.lh_set_wait_limit_ns(1)
    try:
        o, saved = layer.forward(q, k, v)
        layer.backward(saved, d_o)
        torch.cuda.synchronize()
    finally:
        lh.lh_set_wait_limit_ns(prev)
    rc, flags = lh.lh_check(layer.ws)
    assert rc == LH_ERR_DEVICE and flags & 2, (rc, flags)
    assert not flags & 4, "an abort-path drain ran out"
    assert lh.lh_check(layer.ws) == (0, 0)  # the read cleared the word
    # the same process, the default bound: the layer matches the oracle
    o, saved = layer.forward(q, k, v)
    dq, dk, dv = layer.backward(saved, d_o)
    layer.check()
    geo = O.Geometry(S, 4, 1, S).check()
    wo, sv = O.layer_fwd(np64(q), np64(k), np64(v), geo, 8, store="bf16")
    wq, wk, wv = O.layer_bwd(sv, np64(d_o))
    assert_close(np64(o), wo, torch.bfloat16, "O", mode="literal")
    for got, want, n in ((dq, wq, "dQ"), (dk, wk, "dK"), (dv, wv, "dV")):
        assert_close(np64(got), want, torch.bfloat16, n)


def test_wait_timeout_reaches_the_no_alloc_caller():
    """lh_attn_bwd_static keeps its status word in its static array: lh_check_static reads the
    timeout there and clears it."""
    S = 256
    shape = Shape(1, 2, S, 128, 4, 1, S, torch.bfloat16)
    qs, ks, vs, dos = _inputs(shape, 3)
    ws = torch.zeros(lh.lh_workspace_bytes(shape), dtype=torch.uint8, device="cuda")
    os_ = torch.empty(1, 2, S, 128, dtype=torch.float32, device="cuda")
    lse = torch.empty(1, 2, S, dtype=torch.float32, device="cuda")
    lh.lh_attn_fwd(shape, qs, ks, vs, os_, lse, ws)
    grads = [torch.empty_like(os_) for _ in range(3)]
    assert _lib.lh_check_static() == (0, 0)
    prev = lh.lh_set_wait_limit_ns(1)
    try:
        _lib.lh_attn_bwd_static(shape, qs, ks, vs, os_, lse, dos, *grads)
        torch.cuda.synchronize()
    finally:
        lh.lh_set_wait_limit_ns(prev)
    rc, flags = _lib.lh_check_static()
    assert rc == LH_ERR_DEVICE and flags & 2 and not flags & 4, (rc, flags)
    assert _lib.lh_check_static() == (0, 0)
    _lib.lh_attn_bwd_static(shape, qs, ks, vs, os_, lse, dos, *grads)
    assert _lib.lh_check_static() == (0, 0)
    assert lh.lh_check(ws) == (0, 0)
    want_o, want_lse = O.attn_fwd(np64(qs), np64(ks), np64(vs))  # each side on its own forward
    wq, wk, wv = O.attn_bwd(np64(qs), np64(ks), np64(vs), want_o, want_lse, np64(dos))
    for got, want, n in zip(grads, (wq, wk, wv), ("dq", "dk", "dv")):
        assert_close(np64(got), want, torch.bfloat16, n, mode="literal")
