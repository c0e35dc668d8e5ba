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

from gpu_util import assert_close, np64


def _run(shape, seed, static):
    B, H, S, d = shape.B, shape.H, shape.S, shape.d
    g = torch.Generator(device="cuda").manual_seed(seed)
    qs, ks, vs, dos = (torch.randn(B, H, S, d, generator=g, device="cuda").to(shape.dtype)
                       for _ in range(4))
    os_ = torch.empty(B, H, S, d, dtype=torch.float32, device="cuda")
    lse = torch.empty(B, H, S, dtype=torch.float32, device="cuda")
    ws = torch.zeros(lh.lh_workspace_bytes(shape), dtype=torch.uint8, device="cuda")
    lh.lh_attn_fwd(shape, qs, ks, vs, os_, lse, ws)
    grads = [torch.empty(B, H, S, d, dtype=torch.float32, device="cuda") for _ in range(3)]
    if static:
        _lib.lh_attn_bwd_static(shape, qs, ks, vs, os_, lse, dos, *grads)
    else:
        lh.lh_attn_bwd(shape, qs, ks, vs, os_, lse, dos, *grads, ws)
    torch.cuda.synchronize()
    return grads


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_static_scratch_matches_workspace_version_twice(dtype):
    """Two calls in a row (the second on other inputs and sizes) match lh_attn_bwd."""
    for seed, (H, S, d) in enumerate([(4, 1024, 128), (2, 333, 64)]):
        shape = Shape(1, H, S, d, 4, 1, S, dtype)
        got = _run(shape, seed, static=True)
        want = _run(shape, seed, static=False)
        for a, b, n in zip(got, want, ("dq", "dk", "dv")):
            assert_close(np64(a), np64(b), dtype, f"static {n}", mode="scaled")


def test_static_scratch_rejects_oversized_shapes():
    S = 1 << 15
    shape = Shape(1, 64, S, 128, 4, 1, S)  # B*H*S = 2^21 rows > the 2^20 limit
    assert shape.B * shape.H * shape.S > _lib.LH_STATIC_SCRATCH_ROWS
    rc = _lib._lib.lh_attn_bwd_static(ctypes.byref(shape.c()), *([None] * 9), None)
    assert rc == 3  # LH_ERR_WORKSPACE, before any launch
