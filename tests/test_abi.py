"""The C ABI without a GPU: the library loads, exports every declared symbol, validates shapes
and sizes its buffers; invalid calls return errors before any launch."""
import ctypes

import pytest
import torch

import sparse_hierarchical_attention_b200 as lh
from sparse_hierarchical_attention_b200 import Shape, _lib


def test_every_declared_symbol_is_exported():
    names = _lib.header_functions()
    assert len(names) >= 20
    for n in names:
        assert hasattr(_lib._lib, n), n


def test_version():
    assert "sm_100a" in lh.lh_version()


@pytest.mark.parametrize("N,p,L,S,want", [
    (131072, 4, 6, 8192, dict(R=43648, C=128, T=1024, m=64, k=63, M=1364, G=1)),
    (1048576, 4, 7, 16384, dict(R=349440, C=256, T=4096, m=64, k=63, M=5460, G=1)),
    (98304, 4, 6, 6144, dict(R=32736, C=96, T=1024, m=64, k=63, M=1364, G=1)),
    (2048, 4, 3, 512, dict(R=640, C=128, T=16, m=4, k=3, M=20, G=1)),
    (640, 4, 1, 640, dict(R=0, C=640, T=1, m=1, k=0, M=0, G=1)),
    # the pages' ablation p = 2, L = 3, k = 1536 at 98K: S = C + k, strata of 16 chunks
    (98304, 2, 3, 24576 + 1536, dict(R=73728, C=24576, T=4, m=17, k=1, M=6, G=16)),
    (4096, 4, 3, 256 + 96, dict(R=1280, C=256, T=16, m=11, k=3, M=20, G=8)),
])
def test_sizes(N, p, L, S, want):
    assert lh.lh_validate(Shape(1, 2, N, 128, p, L, S)) == want


@pytest.mark.parametrize("bad", [
    Shape(1, 2, 1000, 128, 4, 6, 64),      # N not a multiple of p^(L-1)
    Shape(1, 2, 4096, 128, 4, 6, 3),       # S < C = 4: not every coarsest cell fits
    Shape(1, 2, 4096, 128, 4, 3, 256 * 22),  # m = 22 > M + 1 = 21
    Shape(0, 2, 4096, 128, 4, 3, 256),     # empty batch
    Shape(1, 2, 4096, 128, 1, 3, 256),     # p < 2
    Shape(1, 6, 4096, 128, 4, 3, 256, Hkv=4),  # 6 query heads do not split over 4 key heads
    Shape(1, 2, 4096, 128, 4, 3, 256, Hkv=4),  # more key/value heads than query heads
    Shape(1, 2, 4096, 128, 4, 3, 256, Hkv=-1),
])
def test_invalid_shapes(bad):
    assert _lib.lh_validate_status(bad) == 1
    assert lh.lh_workspace_bytes(bad) == 0


def test_unsupported_head_dim():
    assert _lib.lh_validate_status(Shape(1, 2, 4096, 96, 4, 3, 256 * 4)) == 2


@pytest.mark.parametrize("shape,status", [
    (Shape(1, 1, 32768, 128, 4, 8, 2 * 64), 0),      # M + k = 21907 keys: inside the limit
    (Shape(1, 1, 131072, 128, 4, 9, 2 * 64), 2),     # M + k = 87443 keys: over 200 KiB
    (Shape(1, 1, 2 * 17 * 17, 64, 17, 3, 2), 2),     # p = 17
    (Shape(1, 1, 2 * 2 ** 12, 64, 2, 13, 2), 2),     # L = 13
    (Shape(1, 1, 2 * 16 ** 2, 64, 16, 3, 2 * 17), 0),  # p = 16, L = 3
    (Shape(1, 1, 2 * 2 ** 11, 64, 2, 12, 2 * 64), 0),  # p = 2, L = 12
    (Shape(1, 1, 98304, 64, 2, 3, 24576 + 1), 2),    # one stratum of all 24576 chunks: too many keys
])
def test_gpu_path_limits(shape, status):
    assert _lib.lh_validate_status(shape) == status


def test_null_pointers_rejected_before_launch():
    s = Shape(1, 2, 4096, 128, 4, 3, 1024).c()
    rc = _lib._lib.lh_layer_fwd(ctypes.byref(s), None, None, None, None, None, None, None)
    assert rc == 1
    rc = _lib._lib.lh_select_topk(ctypes.byref(s), None, None, None)
    assert rc == 1


def test_misaligned_pointer_rejected_before_launch():
    s = Shape(1, 2, 4096, 128, 4, 3, 1024).c()
    p = ctypes.c_void_p(0x1000 + 4)
    rc = _lib._lib.lh_select_topk(ctypes.byref(s), p, ctypes.c_void_p(0x2000), None)
    assert rc == 1


def test_workspace_and_saved_sizes_grow_with_shape():
    a, b = Shape(1, 2, 4096, 128, 4, 3, 1024), Shape(1, 4, 4096, 128, 4, 3, 1024)
    assert 0 < lh.lh_workspace_bytes(a) < lh.lh_workspace_bytes(b)
    assert 0 < lh.lh_saved_bytes(a) < lh.lh_saved_bytes(b)
    offs = lh.lh_saved_offsets(a)
    assert offs == sorted(offs) and all(o % 256 == 0 for o in offs)


def test_grouped_heads_workspace_and_launches():
    """Hkv = 0 is Hkv = H; with fewer key/value heads the key and value pyramids shrink and the
    key-score scratch appears; the saved context (per query head) is unchanged."""
    plain = Shape(1, 8, 4096, 128, 4, 3, 1024)
    assert lh.lh_workspace_bytes(plain) == lh.lh_workspace_bytes(Shape(1, 8, 4096, 128, 4, 3, 1024, Hkv=8))
    grouped = Shape(1, 8, 4096, 128, 4, 3, 1024, Hkv=2)
    assert lh.lh_validate(grouped)["C"] == 256
    assert lh.lh_saved_bytes(grouped) == lh.lh_saved_bytes(plain)
    assert lh.lh_workspace_bytes(grouped) <= lh.lh_workspace_bytes(plain)  # the larger region wins
    f1, b1 = lh.lh_launches(plain)
    f2, b2 = lh.lh_launches(grouped)
    assert f2 > f1 and b2 == b1 + 1  # a key/value pooling pass; a second spread


def test_launch_plan():
    f, b = lh.lh_launches(Shape(1, 32, 131072, 128, 4, 6, 8192))
    assert f >= 5 and b >= 3


def test_binding_refuses_host_tensors():
    s = Shape(1, 1, 256, 64, 4, 3, 64)
    x = torch.zeros(1, 1, 256 + 80, dtype=torch.float32)
    with pytest.raises(lh.LighthouseError):
        lh.lh_select_topk(s, x, torch.zeros(1, 1, 64, dtype=torch.int32))


def test_wait_limit_setter_returns_the_previous_bound_and_restores_the_default():
    prev = lh.lh_set_wait_limit_ns(12345)
    assert lh.lh_set_wait_limit_ns(0) == 12345
    assert lh.lh_set_wait_limit_ns(prev) == 2_000_000_000


def test_flags_other_than_deterministic_are_rejected():
    s = Shape(1, 2, 4096, 128, 4, 3, 256)
    c = s.c()
    c.flags = 2
    assert _lib._lib.lh_validate(ctypes.byref(c), None) == 1  # LH_ERR_INVALID_ARG
    assert lh.lh_validate(Shape(1, 2, 4096, 128, 4, 3, 256, deterministic=True))["C"] == 256


@pytest.mark.parametrize("shape,row0,status", [
    (Shape(1, 2, 4096, 128, 4, 3, 256 * 4, torch.float32), 0, 2),  # fp32: unsupported
    (Shape(1, 2, 4096, 64, 4, 3, 256 * 4), 0, 2),                 # d = 64: unsupported
    (Shape(1, 2, 4096, 128, 4, 3, 256 * 4), 64, 2),               # row0 not a multiple of 128
    (Shape(1, 2, 4096, 128, 4, 3, 256 * 4), -128, 1),             # negative row0
    (Shape(1, 2, 4096, 128, 4, 3, 256 * 5 + 4), 0, 2),            # S not a multiple of 128
])
def test_context_parallel_attention_rejects_before_any_launch(shape, row0, status):
    c = shape.c()
    assert _lib._lib.lh_attn_fwd_cp(ctypes.byref(c), row0, *([None] * 7)) == status
    assert _lib._lib.lh_attn_bwd_cp(ctypes.byref(c), row0, *([None] * 11)) == status
