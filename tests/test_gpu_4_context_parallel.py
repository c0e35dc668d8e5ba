"""The context-parallel split on one GPU: two ranks' shares run one after the other with the
library's kernels (GpuOps: the shard's stages and the offset attention lh_attn_fwd_cp /
lh_attn_bwd_cp), the all-gather and the reduce-scatter done on the host. The result must be the
single-GPU layer on the whole sequence: O bit for bit (each query block meets the same key
blocks in the same order), and the gradients within the acceptance rule of the oracle."""
import numpy as np
import pytest
import torch

import oracle as O

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    from sparse_hierarchical_attention_b200 import LighthouseLayer, Shape
    from sparse_hierarchical_attention_b200.context_parallel import GpuOps, plan

from gpu_util import assert_close, np64


@pytest.mark.parametrize("N,p,L,S,Hkv", [
    (8192, 4, 5, 32 * 32, 2),       # strata of one chunk: 16 per rank, 512 rows each
    (16384, 2, 3, 4096 + 256, 2),   # the p = 2, L = 3 ablation's strata (G = 16, 17 rows): 128 per rank
    (8192, 4, 5, 32 * 32, 1),       # grouped heads: both query heads on one key/value head
])
def test_two_ranks_equal_the_whole_sequence(N, p, L, S, Hkv):
    W, B, H, d = 2, 1, 2, 128
    g = torch.Generator(device="cuda").manual_seed(N + S)
    q, d_o = (torch.randn(B, H, N, d, generator=g, device="cuda").to(torch.bfloat16) for _ in range(2))
    k, v = (torch.randn(B, Hkv, N, d, generator=g, device="cuda").to(torch.bfloat16) for _ in range(2))
    whole = LighthouseLayer(Shape(B, H, N, d, p, L, S, Hkv=Hkv))
    o_ref, saved = whole.forward(q, k, v)
    dq_ref, dk_ref, dv_ref = whole.backward(saved, d_o)
    whole.check()

    plans = [plan(N, p, L, S, W, r) for r in range(W)]
    ops = [GpuOps(Shape(B, H, N // W, d, p, L, S // W, Hkv=Hkv)) for _ in range(W)]
    tok = [slice(pl.tok0, pl.tok0 + pl.n_local) for pl in plans]
    shard = lambda x, r: x[:, :, tok[r]].contiguous()  # what rank r holds  # noqa: E731
    local = [ops[r].local_fwd(shard(q, r), shard(k, r), shard(v, r)) for r in range(W)]
    k_all = torch.cat([x[2] for x in local], dim=2)  # the all-gather
    v_all = torch.cat([x[3] for x in local], dim=2)
    outs, ctx = [], []
    for r, pl in enumerate(plans):
        ks, vs = k_all[:, :, :pl.rows_seen].contiguous(), v_all[:, :, :pl.rows_seen].contiguous()
        o_sub, lse = ops[r].attn_fwd(local[r][1], ks, vs, pl.row0)
        outs.append(ops[r].scatter(local[r][4], o_sub))
        ctx.append((ks, vs, o_sub, lse))
    assert torch.equal(torch.cat(outs, dim=2), o_ref)

    dk_sum = torch.zeros(B, H, S, d, device="cuda")  # the reduce-scatter, summed on the host
    dv_sum = torch.zeros(B, H, S, d, device="cuda")
    dq_subs = []
    for r, pl in enumerate(plans):
        ks, vs, o_sub, lse = ctx[r]
        do_sub = ops[r].span_sums(local[r][4], shard(d_o, r))
        dq_sub, dk_seen, dv_seen = ops[r].attn_bwd(local[r][1], ks, vs, o_sub, lse, do_sub, pl.row0)
        dq_subs.append(dq_sub)
        dk_sum[:, :, :pl.rows_seen] += dk_seen
        dv_sum[:, :, :pl.rows_seen] += dv_seen
    grads = [[], [], []]
    for r, pl in enumerate(plans):
        rows = slice(pl.row0, pl.row0 + pl.s_local)
        for i, x in enumerate(ops[r].gather_bwd(local[r][4], dq_subs[r], dk_sum[:, :, rows], dv_sum[:, :, rows])):
            grads[i].append(x)
        ops[r].check()
    grads = [torch.cat(x, dim=2) for x in grads]

    geo = O.Geometry(N, p, L, S).check()
    # the oracle checks one head whole; a shared key/value head needs every query head of it
    h = (slice(0, 1), slice(1, 2)) if Hkv == H else (slice(0, 1), slice(0, H))
    hk = h if Hkv == H else (slice(0, 1), slice(0, Hkv))
    wo, sv = O.layer_fwd(np64(q[h]), np64(k[hk]), np64(v[hk]), geo, 8, store="bf16")
    want = O.layer_bwd(sv, np64(d_o[h]))
    for got, ref, w_, n, hh in zip(grads, (dq_ref, dk_ref, dv_ref), want, ("dQ", "dK", "dV"), (h, hk, hk)):
        assert_close(np64(got[hh]), w_, torch.bfloat16, n)
        x, y = got.float(), ref.float()  # and the whole-sequence GPU layer, to rounding
        rms = y.pow(2).mean().sqrt()
        assert ((x - y).abs() / torch.maximum(y.abs(), rms)).max().item() <= 2.0 ** -6, n
