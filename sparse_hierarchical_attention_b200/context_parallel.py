"""Sequence-sharded context parallelism of the Lighthouse layer.

"Long Context Pre-Training with Lighthouse Attention" (gist.science summary, technical summary
section 4, scaling bullet) trains at 1M tokens on 32 GPUs with context parallelism. This module
holds the host side of that split: which tokens and which subsequence rows each rank owns, and
the two exchanges the layer needs. Every arithmetic step runs in the `ops` object it is given;
nothing here computes the method.

The split. The sequence is cut into W contiguous shards of N / W tokens, one per rank, each a
whole number of strata (runs of G chunks; see lh_sizes). A stratum's selection, gather and
scatter-back only touch its own tokens, so the pyramid, the scores, the top-K, the gather, the
scatter-back and their backward run on each shard alone, as a sequence of N / W tokens with
budget S / W. The subsequence is the strata's rows in order, so rank r owns the global rows
[r S/W, (r + 1) S/W). The causal attention is the one step that reaches across shards: a query
row sees every key row before it. Hence
  - forward: one all-gather of K_sub and V_sub (each rank's S / W rows); rank r runs attention
    for its own query rows against key rows [0, (r + 1) S/W);
  - backward: rank r's attention backward gives dQ_sub for its own rows and partial dK_sub,
    dV_sub for key rows [0, (r + 1) S/W); one reduce-scatter sums the partials of all ranks
    and leaves each rank its own rows.
The two exchanges carry 2 B H S d e bytes each way (e = bytes per element), against the
N-proportional bytes of the local stages. Remote rows arrive in local memory before any kernel
reads them.
"""
from __future__ import annotations

from dataclasses import dataclass

import torch


@dataclass(frozen=True)
class ShardPlan:
    """One rank's share of a layer call."""

    world: int
    rank: int
    N: int          # tokens of the whole sequence
    S: int          # subsequence rows of the whole sequence
    n_local: int    # tokens per rank, N / world
    s_local: int    # subsequence rows per rank, S / world
    tok0: int       # first token of this rank
    row0: int       # first subsequence row of this rank
    rows_seen: int  # key rows this rank's queries see: row0 + s_local


def plan(N, p, L, S, world, rank):
    """The shard of `rank` among `world` ranks, or ValueError if the strata do not split evenly.

    Strata are runs of G = C / gcd(S, C) chunks of p^(L-1) tokens with m = S G / C rows each;
    every rank must own a whole number of them."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("need 0 <= rank < world")
    T = p ** (L - 1)
    if N % T:
        raise ValueError("N must be a multiple of p^(L-1)")
    C = N // T
    a, b = S, C
    while b:
        a, b = b, a % b
    G = C // a
    strata = C // G
    if strata % world:
        raise ValueError(f"{strata} strata do not split over {world} ranks")
    n_local, s_local = N // world, S // world
    return ShardPlan(world, rank, N, S, n_local, s_local, rank * n_local, rank * s_local,
                     (rank + 1) * s_local)


def _reduce_scatter_rows(full, plan_, group):
    """Sums `full` [B, H, S, d] (zero outside the rows this rank produced) over the ranks and
    returns this rank's rows [B, H, S/W, d]. NCCL reduces and scatters in one collective; other
    backends sum the whole buffer and slice it."""
    import torch.distributed as dist
    rows = torch.split(full, plan_.s_local, dim=2)
    if dist.get_backend(group) == "nccl":
        out = torch.empty_like(rows[plan_.rank])
        dist.reduce_scatter(out, [r.contiguous() for r in rows], group=group)
        return out
    dist.all_reduce(full, group=group)
    return rows[plan_.rank].contiguous()


class ContextParallelLayer:
    """The layer over a sequence sharded by tokens across the ranks of `group`.

    `ops` runs the arithmetic of one rank (the library's kernels on a GPU; anything with the
    same contract elsewhere):
      local_fwd(q, k, v)            -> (idx, q_sub, k_sub, v_sub, state)   steps 1-4 on the shard
      attn_fwd(q_sub, k_seen, v_seen, row0)            -> (o_sub, lse)
      scatter(state, o_sub)         -> o                                      step 6 on the shard
      span_sums(state, d_o)         -> do_sub
      attn_bwd(q_sub, k_seen, v_seen, o_sub, lse, do_sub, row0) -> (dq_sub, dk_seen, dv_seen)
      gather_bwd(state, dq_sub, dk_sub, dv_sub) -> (dq, dk, dv)
    attn_fwd/attn_bwd take this rank's query rows (global rows row0 .. row0 + S/W - 1) and the
    key/value rows 0 .. row0 + S/W - 1 of the whole subsequence; the causal rule is on global
    rows. Tensors are [B, H, rows, d]."""

    def __init__(self, N, p, L, S, ops, group=None):
        import torch.distributed as dist
        self.group = group
        world = dist.get_world_size(group) if dist.is_initialized() else 1
        rank = dist.get_rank(group) if dist.is_initialized() else 0
        self.plan = plan(N, p, L, S, world, rank)
        self.ops = ops

    def _all_gather_rows(self, x):
        """[B, H, S/W, d] from every rank -> the rows 0 .. row0 + S/W - 1 of [B, H, S, d]."""
        import torch.distributed as dist
        pl = self.plan
        if pl.world == 1:
            return x
        parts = [torch.empty_like(x) for _ in range(pl.world)]
        dist.all_gather(parts, x.contiguous(), group=self.group)
        return torch.cat(parts[:pl.rank + 1], dim=2)

    def forward(self, q, k, v):
        """q, k, v: this rank's tokens [B, H, N/W, d]. Returns (o [B, H, N/W, d], context)."""
        pl = self.plan
        idx, q_sub, k_sub, v_sub, state = self.ops.local_fwd(q, k, v)
        k_seen, v_seen = self._all_gather_rows(k_sub), self._all_gather_rows(v_sub)
        o_sub, lse = self.ops.attn_fwd(q_sub, k_seen, v_seen, pl.row0)
        o = self.ops.scatter(state, o_sub)
        return o, (state, q_sub, k_seen, v_seen, o_sub, lse)

    def backward(self, ctx, d_o):
        """d_o: this rank's [B, H, N/W, d]. Returns (dq, dk, dv) for this rank's tokens."""
        pl = self.plan
        state, q_sub, k_seen, v_seen, o_sub, lse = ctx
        do_sub = self.ops.span_sums(state, d_o)
        dq_sub, dk_seen, dv_seen = self.ops.attn_bwd(q_sub, k_seen, v_seen, o_sub, lse, do_sub, pl.row0)
        if pl.world > 1:
            B, H, _, d = dk_seen.shape
            full_k = dk_seen.new_zeros(B, H, pl.S, d)
            full_v = dv_seen.new_zeros(B, H, pl.S, d)
            full_k[:, :, :pl.rows_seen] = dk_seen
            full_v[:, :, :pl.rows_seen] = dv_seen
            dk_sub = _reduce_scatter_rows(full_k, pl, self.group)
            dv_sub = _reduce_scatter_rows(full_v, pl, self.group)
        else:
            dk_sub, dv_sub = dk_seen, dv_seen
        return self.ops.gather_bwd(state, dq_sub, dk_sub, dv_sub)


class GpuOps:
    """One rank's stages on its GPU, every step a liblh kernel: the shard's pyramid, scores,
    top-K, gather, scatter-back and their backward through the single-GPU entry points on the
    shard's shape (N/W tokens, budget S/W), and the attention through lh_attn_fwd_cp /
    lh_attn_bwd_cp, which take the rank's query rows at a global offset. bf16, d = 128.
    With grouped heads (shape.Hkv) k, v and their pyramid levels and gradients have the
    key/value heads; the subsequence and the exchanges stay per query head."""

    def __init__(self, shape, device="cuda"):
        from . import _lib
        self.lib, self.shape = _lib, shape
        self.dev = torch.device(device)
        sz = _lib.lh_validate(shape)
        self.R = sz["R"]
        self.ws = torch.zeros(_lib.lh_workspace_bytes(shape), dtype=torch.uint8, device=self.dev)

    @staticmethod
    def _dense(*ts):
        for t in ts:  # the kernels read [B, H, rows, d] through raw pointers
            if not t.is_contiguous():
                raise ValueError("context-parallel operands must be contiguous [B, H, rows, d]")

    def _e(self, rows, dtype=None, heads=None):
        s = self.shape
        return torch.empty(s.B, heads or s.H, rows, s.d, dtype=dtype or s.dtype, device=self.dev)

    def local_fwd(self, q, k, v):
        s, L = self.shape, self.lib
        self._dense(q, k, v)
        R, kv = max(self.R, 1), s.kv_heads
        pq, pk, pv = self._e(R), self._e(R, heads=kv), self._e(R, heads=kv)
        score = torch.empty(s.B, s.H, s.N + self.R, dtype=torch.float32, device=self.dev)
        idx = torch.empty(s.B, s.H, s.S, dtype=torch.int32, device=self.dev)
        L.lh_build_pyramid(s, q, k, v, pq, pk, pv, score, self.ws)
        L.lh_select_topk(s, score, idx)
        subs = [self._e(s.S) for _ in range(3)]
        L.lh_gather(s, q, k, v, pq, pk, pv, idx, *subs, self.ws)
        return (idx, *subs, idx)

    def attn_fwd(self, q_sub, k_seen, v_seen, row0):
        s = self.shape
        self._dense(q_sub, k_seen, v_seen)
        o_sub = self._e(s.S, torch.float32)
        lse = torch.empty(s.B, s.H, s.S, dtype=torch.float32, device=self.dev)
        self.lib.lh_attn_fwd_cp(s, row0, q_sub, k_seen, v_seen, o_sub, lse, self.ws)
        return o_sub, lse

    def scatter(self, idx, o_sub):
        o = self._e(self.shape.N)
        self.lib.lh_scatter(self.shape, idx, o_sub, o)
        return o

    def span_sums(self, idx, d_o):
        self._dense(d_o)
        do_sub = self._e(self.shape.S)
        self.lib.lh_scatter_bwd(self.shape, idx, d_o, do_sub, self.ws)
        return do_sub

    def attn_bwd(self, q_sub, k_seen, v_seen, o_sub, lse, do_sub, row0):
        s = self.shape
        self._dense(q_sub, k_seen, v_seen, o_sub, lse, do_sub)
        dq_sub = self._e(s.S, torch.float32)
        dk_seen, dv_seen = (self._e(k_seen.shape[2], torch.float32) for _ in range(2))
        self.lib.lh_attn_bwd_cp(s, row0, q_sub, k_seen, v_seen, o_sub, lse, do_sub, dq_sub, dk_seen,
                                dv_seen, self.ws)
        return dq_sub, dk_seen, dv_seen

    def gather_bwd(self, idx, dq_sub, dk_sub, dv_sub):
        kv = self.shape.kv_heads
        out = [self._e(self.shape.N), self._e(self.shape.N, heads=kv), self._e(self.shape.N, heads=kv)]
        self.lib.lh_gather_bwd(self.shape, idx, dq_sub, dk_sub.contiguous(), dv_sub.contiguous(), *out)
        return tuple(out)

    def check(self):
        rc, flags = self.lib.lh_check(self.ws)
        if rc:
            raise self.lib.LighthouseError(f"device fault flags {flags:#x}")
