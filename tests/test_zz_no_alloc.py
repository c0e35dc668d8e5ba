"""lh_attn_bwd_static, the attention backward for callers that cannot allocate device memory
(a plugin whose host framework owns all allocations, or code that must not call the allocator):
its scratch is a static device array inside the library. Collected last on purpose."""
import ctypes

import pytest
import torch

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import sparse_hierarchical_attention_b200 as lh
    from sparse_hierarchical_attention_b200 import Shape, _lib


def _inputs(shape, seed):
    B, H, S, d = shape.B, shape.H, shape.S, shape.d
    g = torch.Generator(device="cuda").manual_seed(seed)
    qs, ks, vs, dos = (torch.randn(B, H, S, d, generator=g, device="cuda").to(shape.dtype)
                       for _ in range(4))
    os_ = torch.empty(B, H, S, d, dtype=torch.float32, device="cuda")
    lse = torch.empty(B, H, S, dtype=torch.float32, device="cuda")
    ws = torch.zeros(lh.lh_workspace_bytes(shape), dtype=torch.uint8, device="cuda")
    lh.lh_attn_fwd(shape, qs, ks, vs, os_, lse, ws)
    return qs, ks, vs, os_, lse, dos, ws


def _grads(shape):
    return [torch.empty(shape.B, shape.H, shape.S, shape.d, dtype=torch.float32, device="cuda")
            for _ in range(3)]


def _both(shape, seed):
    """(static grads, workspace grads) of the same inputs, each from its own output buffers."""
    qs, ks, vs, os_, lse, dos, ws = _inputs(shape, seed)
    got, want = _grads(shape), _grads(shape)
    _lib.lh_attn_bwd_static(shape, qs, ks, vs, os_, lse, dos, *got)
    lh.lh_attn_bwd(shape, qs, ks, vs, os_, lse, dos, *want, ws)
    torch.cuda.synchronize()
    assert lh.lh_check(ws) == (0, 0)
    return got, want


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_static_scratch_matches_workspace_version_twice(dtype):
    """Two calls in a row (the second on other inputs and sizes) give lh_attn_bwd's gradients
    bit for bit: the same deterministic kernels run on the same inputs; only D's address
    differs."""
    for seed, (H, S, d) in enumerate([(4, 1024, 128), (2, 333, 64)]):
        shape = Shape(1, H, S, d, 4, 1, S, dtype, deterministic=True)
        got, want = _both(shape, seed)
        for a, b, n in zip(got, want, ("dq", "dk", "dv")):
            assert torch.equal(a, b), f"static {n} differs (call {seed})"
    assert _lib.lh_check_static() == (0, 0)  # no fault latched in the static status word


def test_static_scratch_on_the_one_pass_backward():
    """Without LH_DETERMINISTIC both entry points run the one-pass backward: dK and dV agree bit
    for bit, dQ (atomic fp32 adds in a varying order) to fp32 rounding."""
    shape = Shape(1, 4, 1024, 128, 4, 1, 1024, torch.bfloat16)
    for seed in (11, 12):
        (gq, gk, gv), (wq, wk, wv) = _both(shape, seed)
        assert torch.equal(gk, wk) and torch.equal(gv, wv)
        rms = wq.pow(2).mean().sqrt()
        assert ((gq - wq).abs() / torch.maximum(wq.abs(), rms)).max().item() <= 1e-4
    assert _lib.lh_check_static() == (0, 0)


def test_static_scratch_at_its_row_limit():
    """B*H*S equal to LH_STATIC_SCRATCH_ROWS is accepted and fills D to its last row."""
    shape = Shape(1, 256, 4096, 64, 4, 1, 4096, deterministic=True)
    assert shape.B * shape.H * shape.S == _lib.LH_STATIC_SCRATCH_ROWS
    got, want = _both(shape, 7)
    for a, b, n in zip(got, want, ("dq", "dk", "dv")):
        assert torch.equal(a, b), f"static {n} differs at the row limit"
    assert _lib.lh_check_static() == (0, 0)


def test_static_scratch_rejects_oversized_shapes():
    S = 1 << 15
    shape = Shape(1, 64, S, 128, 4, 1, S)  # B*H*S = 2^21 rows > the 2^20 limit
    assert shape.B * shape.H * shape.S > _lib.LH_STATIC_SCRATCH_ROWS
    rc = _lib._lib.lh_attn_bwd_static(ctypes.byref(shape.c()), *([None] * 9), None)
    assert rc == 3  # LH_ERR_WORKSPACE, before any launch
