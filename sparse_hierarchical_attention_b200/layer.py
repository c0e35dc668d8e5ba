"""User-facing layer: device buffers from PyTorch, every step in liblh.so."""
from __future__ import annotations

import torch

from . import _lib
from ._lib import Shape


def saved_views(shape: Shape, saved: torch.Tensor):
    """Views of the forward context: idx, q_sub, k_sub, v_sub, o_sub, lse."""
    offs = _lib.lh_saved_offsets(shape)
    rows = shape.B * shape.H * shape.S

    def view(off, n, dtype, shp):
        nbytes = n * torch.tensor([], dtype=dtype).element_size()
        return saved[off:off + nbytes].view(dtype).view(*shp)

    sub = (shape.B, shape.H, shape.S, shape.d)
    return dict(
        idx=view(offs[0], rows, torch.int32, (shape.B, shape.H, shape.S)),
        q_sub=view(offs[1], rows * shape.d, shape.dtype, sub),
        k_sub=view(offs[2], rows * shape.d, shape.dtype, sub),
        v_sub=view(offs[3], rows * shape.d, shape.dtype, sub),
        o_sub=view(offs[4], rows * shape.d, torch.float32, sub),
        lse=view(offs[5], rows, torch.float32, (shape.B, shape.H, shape.S)),
    )


class LighthouseLayer:
    """Holds the workspace of one shape on one device and runs the layer's forward/backward."""

    def __init__(self, shape: Shape, device="cuda"):
        _lib.lh_validate(shape)
        self.shape = shape
        self.device = torch.device(device)
        self.ws = torch.zeros(_lib.lh_workspace_bytes(shape), dtype=torch.uint8, device=self.device)

    def new_saved(self):
        return torch.empty(_lib.lh_saved_bytes(self.shape), dtype=torch.uint8, device=self.device)

    def forward(self, q, k, v, o=None, saved=None):
        if o is None:
            o = torch.empty_like(q)
        if saved is None:
            saved = self.new_saved()
        _lib.lh_layer_fwd(self.shape, q, k, v, o, saved, self.ws)
        return o, saved

    def backward(self, saved, d_o, dq=None, dk=None, dv=None):
        s = self.shape
        kv = (s.B, s.kv_heads, s.N, s.d)  # K and V have the key/value heads
        dq = torch.empty_like(d_o) if dq is None else dq
        dk = torch.empty(kv, dtype=d_o.dtype, device=d_o.device) if dk is None else dk
        dv = torch.empty(kv, dtype=d_o.dtype, device=d_o.device) if dv is None else dv
        _lib.lh_layer_bwd(self.shape, saved, d_o, dq, dk, dv, self.ws)
        return dq, dk, dv

    def check(self):
        """Synchronises and raises if a kernel flagged a fault in the workspace status word."""
        rc, flags = _lib.lh_check(self.ws)
        if rc:
            raise _lib.LighthouseError(f"device fault flags {flags:#x}")


class _Fn(torch.autograd.Function):
    @staticmethod
    def forward(ctx, q, k, v, layer):
        o, saved = layer.forward(q.contiguous(), k.contiguous(), v.contiguous())
        ctx.layer, ctx.saved = layer, saved
        return o

    @staticmethod
    def backward(ctx, d_o):
        dq, dk, dv = ctx.layer.backward(ctx.saved, d_o.contiguous())
        return dq, dk, dv, None


class LighthouseAttention(torch.nn.Module):
    """Drop-in replacement of causal SDPA on [B, H, N, d] tensors during pre-training.

    k and v may have fewer heads than q (grouped-query heads, [B, Hkv, N, d] with H a multiple
    of Hkv). deterministic=True makes the backward bit-reproducible (no atomics; slower at
    d = 128)."""

    def __init__(self, p: int, L: int, S: int, deterministic: bool = False):
        super().__init__()
        self.p, self.L, self.S, self.deterministic = p, L, S, deterministic
        self._layers = {}

    def forward(self, q, k, v):
        B, H, N, d = q.shape
        Hkv = k.shape[1]
        shape = Shape(B, H, N, d, self.p, self.L, self.S, q.dtype, self.deterministic,
                      0 if Hkv == H else Hkv)
        key = (shape, q.device)
        if key not in self._layers:
            self._layers[key] = LighthouseLayer(shape, q.device)
        return _Fn.apply(q, k, v, self._layers[key])
