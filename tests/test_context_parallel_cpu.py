"""Sequence-sharded context parallelism (the layer's split over ranks by tokens) on CPU: two gloo
ranks run ContextParallelLayer with every arithmetic step done by the oracle on the rank's shard,
and each rank's outputs and gradients must equal the whole-sequence oracle layer on its tokens.
What is under test is the host side: the shard plan, the all-gather of K_sub/V_sub rows, the
global causal rule across shards, and the reduce-scatter of dK_sub/dV_sub."""
import multiprocessing as mp
import os
import socket

import numpy as np
import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


class OracleOps:
    """One rank's stages on the host, from the oracle (fp64), on a shard of N/W tokens."""

    def __init__(self, N_local, p, L, S_local):
        import oracle as O
        self.O = O
        self.geo = O.Geometry(N_local, p, L, S_local).check()

    def local_fwd(self, q, k, v):
        O, geo = self.O, self.geo
        q, k, v = (x.numpy() for x in (q, k, v))
        idx = O.select_topk(O.score(q, k, geo, 4), geo)
        hmap = O.kv_head_of(q.shape[1], k.shape[1])  # grouped heads: a query head's key head
        subs = [O.gather(q, O.build_pyramid(q, geo), idx)]
        subs += [O.gather(x[:, hmap], O.build_pyramid(x, geo)[:, hmap], idx) for x in (k, v)]
        self.heads = (q.shape[1], k.shape[1])
        return (idx, *(torch.from_numpy(s) for s in subs), idx)

    @staticmethod
    def _pad(x, row0):  # rows 0 .. row0 - 1 that this rank does not own: zeros
        B, H, _, d = x.shape
        return torch.cat([x.new_zeros(B, H, row0, d), x], dim=2)

    def attn_fwd(self, q_sub, k_seen, v_seen, row0):
        o, lse = self.O.attn_fwd(self._pad(q_sub, row0).numpy(), k_seen.numpy(), v_seen.numpy())
        return torch.from_numpy(o[:, :, row0:]), torch.from_numpy(lse[:, :, row0:])

    def scatter(self, idx, o_sub):
        return torch.from_numpy(self.O.scatter(idx, o_sub.numpy(), self.geo))

    def span_sums(self, idx, d_o):
        return torch.from_numpy(self.O.scatter_bwd(idx, d_o.numpy(), self.geo))

    def attn_bwd(self, q_sub, k_seen, v_seen, o_sub, lse, do_sub, row0):
        # rows before row0 carry dO = 0, so they add nothing to any gradient
        B, H, _, _ = q_sub.shape
        lse_p = torch.cat([lse.new_zeros(B, H, row0), lse], dim=2)
        dq, dk, dv = self.O.attn_bwd(self._pad(q_sub, row0).numpy(), k_seen.numpy(), v_seen.numpy(),
                                     self._pad(o_sub, row0).numpy(), lse_p.numpy(),
                                     self._pad(do_sub, row0).numpy())
        return torch.from_numpy(dq[:, :, row0:]), torch.from_numpy(dk), torch.from_numpy(dv)

    def gather_bwd(self, idx, dq, dk, dv):
        H, Hkv = self.heads
        out = [self.O.gather_bwd(idx, x.numpy(), self.geo) for x in (dq, dk, dv)]
        for i in (1, 2):  # a key/value head sums its query heads' gradients
            B, _, N, d = out[i].shape
            out[i] = out[i].reshape(B, Hkv, H // Hkv, N, d).sum(axis=2)
        return tuple(torch.from_numpy(x) for x in out)


CASES = [  # (N, p, L, S, Hkv): strata of G chunks, whole strata per rank; H = 2
    (64, 2, 3, 24, 2),    # C = 16, G = 2: 8 strata of 3 rows
    (128, 4, 3, 40, 2),   # C = 8, G = 1: 8 chunks of 5 rows
    (96, 2, 3, 26, 2),    # C = 24, G = 12: 2 strata of 13 rows (one per rank)
    (64, 2, 3, 24, 1),    # both query heads on one key/value head
]


def _worker(rank, world, port, case, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world),
                      RANK=str(rank))
    import sys
    sys.path.insert(0, ROOT)
    import datetime

    import torch.distributed as dist
    import oracle as O
    from sparse_hierarchical_attention_b200.context_parallel import ContextParallelLayer
    dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=120))
    N, p, L, S, Hkv = case
    B, H, d = 1, 2, 8
    g = torch.Generator().manual_seed(11)
    q, d_o = (torch.randn(B, H, N, d, generator=g, dtype=torch.float64) for _ in range(2))
    k, v = (torch.randn(B, Hkv, N, d, generator=g, dtype=torch.float64) for _ in range(2))
    layer = ContextParallelLayer(N, p, L, S, OracleOps(N // world, p, L, S // world))
    pl = layer.plan
    sl = slice(pl.tok0, pl.tok0 + pl.n_local)
    o, ctx = layer.forward(q[:, :, sl], k[:, :, sl], v[:, :, sl])
    grads = layer.backward(ctx, d_o[:, :, sl])
    # the whole sequence on one rank, by the oracle
    geo = O.Geometry(N, p, L, S).check()
    wo, sv = O.layer_fwd(q.numpy(), k.numpy(), v.numpy(), geo, 4)
    wg = O.layer_bwd(sv, d_o.numpy())
    err = max(float(np.abs(o.numpy() - wo[:, :, sl]).max()),
              *(float(np.abs(a.numpy() - b[:, :, sl]).max()) for a, b in zip(grads, wg)))
    dist.barrier()
    dist.destroy_process_group()
    out.put((rank, pl.row0, pl.rows_seen, err))


@pytest.mark.timeout(300)
@pytest.mark.parametrize("case", CASES)
def test_two_ranks_equal_the_whole_sequence(case):
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, case, out)) for r in range(world)]
    for pr in procs:
        pr.start()
    got = sorted(out.get(timeout=240) for _ in range(world))
    for pr in procs:
        pr.join(timeout=60)
        assert pr.exitcode == 0
    S = case[3]
    assert [(g[1], g[2]) for g in got] == [(0, S // 2), (S // 2, S)]  # row ranges of the ranks
    for rank, _, _, err in got:
        assert err < 1e-10, (rank, err)


def test_plan_rejects_strata_that_do_not_split():
    import sys
    sys.path.insert(0, ROOT)
    from sparse_hierarchical_attention_b200.context_parallel import plan
    assert plan(96, 2, 3, 26, 2, 1).row0 == 13
    with pytest.raises(ValueError):
        plan(96, 2, 3, 26, 4, 0)   # 2 strata over 4 ranks
    with pytest.raises(ValueError):
        plan(100, 2, 3, 25, 2, 0)  # N not a multiple of p^(L-1)
