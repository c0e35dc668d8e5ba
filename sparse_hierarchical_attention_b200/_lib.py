"""ctypes binding of liblh.so (include/lh.h): argument marshalling only.

Every function here has the name of the C entry point it calls and takes torch tensors where
the C function takes device pointers. It converts them to pointers, passes the current CUDA
stream, and raises LighthouseError on a non-zero status. No arithmetic of the layer happens
here: every step runs in the CUDA kernels of liblh.so. There is no fallback: if the library
is missing, importing this module raises.
"""
from __future__ import annotations

import ctypes
import os
import re
from dataclasses import dataclass

import torch

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "liblh.so")
HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "lh.h")

LH_F32, LH_BF16 = 0, 1
_DTYPES = {torch.float32: LH_F32, torch.bfloat16: LH_BF16}


class LighthouseError(RuntimeError):
    pass


LH_DETERMINISTIC = 1


class lh_shape(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int) for n in ("B", "H", "N", "d", "p", "L", "S", "dtype", "flags", "Hkv")]


class lh_sizes(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int64) for n in ("R", "C", "T", "m", "k", "M", "G")]


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is not built: run `python -m "
                          "sparse_hierarchical_attention_b200.build` (needs nvcc)")
    lib = ctypes.CDLL(LIB_PATH)
    P, I, Z = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
    SP = ctypes.POINTER(lh_shape)
    sig = {
        "lh_status_string": ([I], ctypes.c_char_p),
        "lh_version": ([], ctypes.c_char_p),
        "lh_validate": ([SP, ctypes.POINTER(lh_sizes)], I),
        "lh_workspace_bytes": ([SP], Z),
        "lh_saved_bytes": ([SP], Z),
        "lh_saved_offsets": ([SP, ctypes.POINTER(ctypes.c_size_t)], I),
        "lh_launches": ([SP, ctypes.POINTER(I), ctypes.POINTER(I)], I),
        "lh_workspace_init": ([P, P], I),
        "lh_check": ([P, P, ctypes.POINTER(ctypes.c_uint32)], I),
        "lh_set_wait_limit_ns": ([ctypes.c_uint64], ctypes.c_uint64),
        "lh_build_pyramid": ([SP, P, P, P, P, P, P, P, P, P], I),
        "lh_score": ([SP, P, P, P, P, P], I),
        "lh_select_topk": ([SP, P, P, P], I),
        "lh_gather": ([SP, P, P, P, P, P, P, P, P, P, P, P, P], I),
        "lh_attn_fwd": ([SP, P, P, P, P, P, P, P], I),
        "lh_attn_bwd": ([SP, P, P, P, P, P, P, P, P, P, P, P], I),
        "lh_attn_fwd_cp": ([SP, ctypes.c_int64, P, P, P, P, P, P, P], I),
        "lh_attn_bwd_cp": ([SP, ctypes.c_int64, P, P, P, P, P, P, P, P, P, P, P], I),
        "lh_scatter": ([SP, P, P, P, P], I),
        "lh_scatter_bwd": ([SP, P, P, P, P, P], I),
        "lh_gather_bwd": ([SP, P, P, P, P, P, P, P, P], I),
        "lh_layer_fwd": ([SP, P, P, P, P, P, P, P], I),
        "lh_layer_bwd": ([SP, P, P, P, P, P, P, P], I),
        "lh_attn_bwd_static": ([SP, P, P, P, P, P, P, P, P, P, P], I),
        "lh_check_static": ([P, ctypes.POINTER(ctypes.c_uint32)], I),
    }
    for name, (args, res) in sig.items():
        fn = getattr(lib, name)
        fn.argtypes, fn.restype = args, res
    return lib


_lib = _load()


def header_functions():
    """Names of the functions include/lh.h declares."""
    text = open(HEADER).read()
    return sorted(set(re.findall(r"^\s*(?:const\s+)?\w+\*?\s+\*?(lh_\w+)\(", text, re.M)))


@dataclass(frozen=True)
class Shape:
    """One layer call: N tokens, H heads, d = d_head, pooling p, L levels, S rows kept.

    deterministic: run the attention backward without atomics (LH_DETERMINISTIC), so that
    dQ is bit-identical from run to run; slower at d = 128.
    Hkv: key/value heads when they are fewer than H (grouped-query heads; 0 = H). Query head h
    then uses key/value head h // (H // Hkv); K, V and their gradients have Hkv heads."""

    B: int
    H: int
    N: int
    d: int
    p: int
    L: int
    S: int
    dtype: torch.dtype = torch.bfloat16
    deterministic: bool = False
    Hkv: int = 0

    @property
    def kv_heads(self):
        return self.Hkv or self.H

    def c(self):
        return lh_shape(self.B, self.H, self.N, self.d, self.p, self.L, self.S, _DTYPES[self.dtype],
                        LH_DETERMINISTIC if self.deterministic else 0, self.Hkv)


def _ptr(t):
    if t is None:
        return None
    if not t.is_cuda:
        raise LighthouseError("tensor is not on a CUDA device")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _check(rc):
    if rc != 0:
        raise LighthouseError(f"liblh: {_lib.lh_status_string(rc).decode()} (status {rc})")


def lh_version():
    return _lib.lh_version().decode()


def lh_validate(shape: Shape):
    sz = lh_sizes()
    _check(_lib.lh_validate(ctypes.byref(shape.c()), ctypes.byref(sz)))
    return {n: getattr(sz, n) for n, _ in lh_sizes._fields_}


def lh_validate_status(shape: Shape) -> int:
    return _lib.lh_validate(ctypes.byref(shape.c()), None)


def lh_workspace_bytes(shape: Shape) -> int:
    return _lib.lh_workspace_bytes(ctypes.byref(shape.c()))


def lh_saved_bytes(shape: Shape) -> int:
    return _lib.lh_saved_bytes(ctypes.byref(shape.c()))


def lh_saved_offsets(shape: Shape):
    offs = (ctypes.c_size_t * 6)()
    _check(_lib.lh_saved_offsets(ctypes.byref(shape.c()), offs))
    return list(offs)


def lh_launches(shape: Shape):
    """(kernel launches of one lh_layer_fwd, of one lh_layer_bwd) for this shape."""
    f, b = ctypes.c_int(0), ctypes.c_int(0)
    _check(_lib.lh_launches(ctypes.byref(shape.c()), ctypes.byref(f), ctypes.byref(b)))
    return f.value, b.value


def lh_set_wait_limit_ns(ns: int) -> int:
    """Bound of every wait inside the tensor-core kernels (0 = the default 2 s); returns the
    previous bound."""
    return int(_lib.lh_set_wait_limit_ns(ctypes.c_uint64(ns)))


def lh_workspace_init(ws, stream=None):
    _check(_lib.lh_workspace_init(_ptr(ws), _stream(stream)))


def lh_check(ws, stream=None):
    flags = ctypes.c_uint32(0)
    rc = _lib.lh_check(_ptr(ws), _stream(stream), ctypes.byref(flags))
    return rc, flags.value


def lh_build_pyramid(shape, q, k, v, pq, pk, pv, score, ws, stream=None):
    _check(_lib.lh_build_pyramid(ctypes.byref(shape.c()), _ptr(q), _ptr(k), _ptr(v), _ptr(pq),
                                 _ptr(pk), _ptr(pv), _ptr(score), _ptr(ws), _stream(stream)))


def lh_score(shape, q, k, score, ws, stream=None):
    _check(_lib.lh_score(ctypes.byref(shape.c()), _ptr(q), _ptr(k), _ptr(score), _ptr(ws),
                         _stream(stream)))


def lh_select_topk(shape, score, idx, stream=None):
    _check(_lib.lh_select_topk(ctypes.byref(shape.c()), _ptr(score), _ptr(idx), _stream(stream)))


def lh_gather(shape, q, k, v, pq, pk, pv, idx, q_sub, k_sub, v_sub, ws, stream=None):
    _check(_lib.lh_gather(ctypes.byref(shape.c()), _ptr(q), _ptr(k), _ptr(v), _ptr(pq), _ptr(pk),
                          _ptr(pv), _ptr(idx), _ptr(q_sub), _ptr(k_sub), _ptr(v_sub), _ptr(ws),
                          _stream(stream)))


def lh_attn_fwd(shape, q_sub, k_sub, v_sub, o_sub, lse, ws, stream=None):
    _check(_lib.lh_attn_fwd(ctypes.byref(shape.c()), _ptr(q_sub), _ptr(k_sub), _ptr(v_sub),
                            _ptr(o_sub), _ptr(lse), _ptr(ws), _stream(stream)))


def lh_attn_bwd(shape, q_sub, k_sub, v_sub, o_sub, lse, do_sub, dq_sub, dk_sub, dv_sub, ws,
                stream=None):
    _check(_lib.lh_attn_bwd(ctypes.byref(shape.c()), _ptr(q_sub), _ptr(k_sub), _ptr(v_sub),
                            _ptr(o_sub), _ptr(lse), _ptr(do_sub), _ptr(dq_sub), _ptr(dk_sub),
                            _ptr(dv_sub), _ptr(ws), _stream(stream)))


def lh_attn_fwd_cp(shape, row0, q_sub, k_seen, v_seen, o_sub, lse, ws, stream=None):
    _check(_lib.lh_attn_fwd_cp(ctypes.byref(shape.c()), row0, _ptr(q_sub), _ptr(k_seen), _ptr(v_seen),
                               _ptr(o_sub), _ptr(lse), _ptr(ws), _stream(stream)))


def lh_attn_bwd_cp(shape, row0, q_sub, k_seen, v_seen, o_sub, lse, do_sub, dq_sub, dk_seen, dv_seen,
                   ws, stream=None):
    _check(_lib.lh_attn_bwd_cp(ctypes.byref(shape.c()), row0, _ptr(q_sub), _ptr(k_seen), _ptr(v_seen),
                               _ptr(o_sub), _ptr(lse), _ptr(do_sub), _ptr(dq_sub), _ptr(dk_seen),
                               _ptr(dv_seen), _ptr(ws), _stream(stream)))


def lh_scatter(shape, idx, o_sub, o, stream=None):
    _check(_lib.lh_scatter(ctypes.byref(shape.c()), _ptr(idx), _ptr(o_sub), _ptr(o),
                           _stream(stream)))


def lh_scatter_bwd(shape, idx, d_o, do_sub, ws, stream=None):
    _check(_lib.lh_scatter_bwd(ctypes.byref(shape.c()), _ptr(idx), _ptr(d_o), _ptr(do_sub),
                               _ptr(ws), _stream(stream)))


def lh_gather_bwd(shape, idx, dq_sub, dk_sub, dv_sub, dq, dk, dv, stream=None):
    _check(_lib.lh_gather_bwd(ctypes.byref(shape.c()), _ptr(idx), _ptr(dq_sub), _ptr(dk_sub),
                              _ptr(dv_sub), _ptr(dq), _ptr(dk), _ptr(dv), _stream(stream)))


def lh_layer_fwd(shape, q, k, v, o, saved, ws, stream=None):
    _check(_lib.lh_layer_fwd(ctypes.byref(shape.c()), _ptr(q), _ptr(k), _ptr(v), _ptr(o),
                             _ptr(saved), _ptr(ws), _stream(stream)))


def lh_layer_bwd(shape, saved, d_o, dq, dk, dv, ws, stream=None):
    _check(_lib.lh_layer_bwd(ctypes.byref(shape.c()), _ptr(saved), _ptr(d_o), _ptr(dq), _ptr(dk),
                             _ptr(dv), _ptr(ws), _stream(stream)))


LH_STATIC_SCRATCH_ROWS = 1 << 20


def lh_attn_bwd_static(shape, q_sub, k_sub, v_sub, o_sub, lse, do_sub, dq_sub, dk_sub, dv_sub,
                       stream=None):
    """lh_attn_bwd for callers that cannot allocate: scratch in the library's static array."""
    _check(_lib.lh_attn_bwd_static(ctypes.byref(shape.c()), _ptr(q_sub), _ptr(k_sub),
                                   _ptr(v_sub), _ptr(o_sub), _ptr(lse), _ptr(do_sub),
                                   _ptr(dq_sub), _ptr(dk_sub), _ptr(dv_sub), _stream(stream)))


def lh_check_static(stream=None):
    """(status, fault flags) of lh_attn_bwd_static's static status word; clears it."""
    flags = ctypes.c_uint32(0)
    rc = _lib.lh_check_static(_stream(stream), ctypes.byref(flags))
    return rc, flags.value
