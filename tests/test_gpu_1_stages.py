"""Stage-by-stage parity of the CUDA path (through the C ABI) with the CPU oracle.

Each entry point of include/lh.h is fed the same seeded inputs as the oracle function that
restates it. Sizes span several tiles and ragged tails; the oracle finishes in seconds.
"""
import numpy as np
import pytest
import torch

import oracle as O

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import sparse_hierarchical_attention_b200 as lh
    from sparse_hierarchical_attention_b200 import Shape

from gpu_util import assert_close, assert_pyramid, g_of, np64, store_of

DT = {"f32": torch.float32, "bf16": torch.bfloat16}

# (B, H, N, d, p, L, S)
POOL_SHAPES = [
    (1, 2, 4096, 128, 4, 5, 1024), (2, 3, 2048, 64, 4, 3, 512), (1, 2, 8192, 128, 4, 6, 512),
    (1, 1, 4096, 64, 4, 7, 256), (1, 2, 1024, 128, 2, 6, 512), (1, 2, 2187, 64, 3, 4, 243),
    (1, 3, 640, 128, 4, 1, 640), (2, 1, 1280, 64, 4, 4, 100), (1, 1, 65536, 128, 4, 8, 16),
    (1, 2, 4096, 64, 16, 3, 512), (1, 1, 2048, 128, 2, 11, 22),
]


def inputs(B, H, N, d, dtype, seed=0, scale=True):
    g = torch.Generator(device="cuda").manual_seed(seed)
    s = torch.exp(0.5 * torch.randn(B, H, N, 1, generator=g, device="cuda")) if scale else 1.0
    return [(torch.randn(B, H, N, d, generator=g, device="cuda") * s).to(dtype) for _ in range(3)]


def ws_for(shape):
    ws = torch.zeros(lh.lh_workspace_bytes(shape), dtype=torch.uint8, device="cuda")
    return ws


@pytest.mark.parametrize("dt", ["f32", "bf16"])
@pytest.mark.parametrize("B,H,N,d,p,L,S", POOL_SHAPES)
def test_pyramid_and_score(B, H, N, d, p, L, S, dt):
    dtype = DT[dt]
    shape = Shape(B, H, N, d, p, L, S, dtype)
    sz = lh.lh_validate(shape)
    q, k, v = inputs(B, H, N, d, dtype, seed=N + L)
    R = sz["R"]
    pq, pk, pv = (torch.empty(B, H, max(R, 1), d, dtype=dtype, device="cuda") for _ in range(3))
    score = torch.empty(B, H, N + R, dtype=torch.float32, device="cuda")
    ws = ws_for(shape)
    lh.lh_build_pyramid(shape, q, k, v, pq, pk, pv, score, ws)
    s_only = torch.empty_like(score)
    lh.lh_score(shape, q, k, s_only, ws)
    torch.cuda.synchronize()
    geo = O.Geometry(N, p, L, S).check()
    want_r = O.score(np64(q), np64(k), geo, g_of(dtype))
    got_r = s_only.cpu().numpy()
    assert np.array_equal(score.cpu().numpy(), got_r)
    bad = np.argwhere(got_r != want_r)
    assert bad.size == 0, f"{len(bad)} score mismatches, first {bad[:3]}"
    for x, px in ((q, pq), (k, pk), (v, pv)):
        got = np64(px)[:, :, :R]
        # the stored cells follow the fixed fp32 order and one rounding: bit-exact
        want = O.pool_stored(np64(x), geo, store_of(dtype))
        bad = np.argwhere(got != want)
        assert bad.size == 0, f"{len(bad)} pooled values differ, first {bad[:3]}"
        assert_pyramid(got, np64(x), geo, dtype)  # and within the bound of the exact mean


SEL_SHAPES = [(1, 2, 4096, 128, 4, 5, 1024), (2, 3, 2048, 64, 4, 3, 512),
              (1, 2, 8192, 128, 4, 6, 8 * 64), (1, 2, 1024, 128, 2, 6, 32 * 32),
              (1, 2, 2187, 64, 3, 4, 27 * 3), (1, 1, 1024, 64, 4, 4, 16 * 85),
              (1, 3, 640, 128, 4, 1, 640), (1, 2, 4096, 64, 4, 6, 4 * 1),
              # strata of G > 1 chunks (S no multiple of C): G = 16, 8, 2, and one stratum
              (1, 2, 4096, 64, 2, 3, 1024 + 64), (1, 2, 4096, 128, 4, 3, 256 + 96),
              (2, 2, 2048, 64, 4, 4, 32 * 5 + 16), (1, 1, 729, 64, 3, 4, 27 + 1)]


@pytest.mark.parametrize("quantised", [False, True])
@pytest.mark.parametrize("B,H,N,d,p,L,S", SEL_SHAPES)
def test_select_topk(B, H, N, d, p, L, S, quantised):
    shape = Shape(B, H, N, d, p, L, S, torch.bfloat16)
    sz = lh.lh_validate(shape)
    geo = O.Geometry(N, p, L, S).check()
    g = torch.Generator(device="cpu").manual_seed(7)
    if quantised:  # many exact ties exercise the total tie-break
        r = torch.randint(0, 6, (B, H, N + sz["R"]), generator=g).float()
    else:
        r = torch.rand(B, H, N + sz["R"], generator=g)
    idx = torch.empty(B, H, S, dtype=torch.int32, device="cuda")
    lh.lh_select_topk(shape, r.cuda(), idx)
    want = O.select_topk(r.numpy(), geo)
    assert np.array_equal(idx.cpu().numpy(), want)


def rand_sub(B, H, S, d, dtype, seed):
    g = torch.Generator(device="cuda").manual_seed(seed)
    return [torch.randn(B, H, S, d, generator=g, device="cuda").to(dtype) for _ in range(4)]


@pytest.mark.parametrize("det", [False, True])
@pytest.mark.parametrize("dt", ["f32", "bf16"])
@pytest.mark.parametrize("B,H,S,d", [(1, 2, 64, 64), (2, 2, 333, 128), (1, 3, 1000, 64),
                                     (1, 1, 1, 128), (1, 2, 4096, 128), (1, 1, 128, 128),
                                     (2, 3, 256, 64), (1, 2, 1024, 128), (1, 1, 2048, 64),
                                     (3, 5, 384, 128)])
def test_attention_fwd_bwd(B, H, S, d, dt, det):
    """Both backward modes (one pass with atomic dQ adds; deterministic two passes)."""
    dtype = DT[dt]
    N = S  # an L = 1 shape carries (S, d) to the attention entry points
    shape = Shape(B, H, N, d, 4, 1, S, dtype, det)
    qs, ks, vs, dos = rand_sub(B, H, S, d, dtype, seed=S)
    os_ = torch.empty(B, H, S, d, dtype=torch.float32, device="cuda")
    lse = torch.empty(B, H, S, dtype=torch.float32, device="cuda")
    ws = ws_for(shape)
    lh.lh_attn_fwd(shape, qs, ks, vs, os_, lse, ws)
    dq, dk, dv = (torch.empty(B, H, S, d, dtype=torch.float32, device="cuda") for _ in range(3))
    lh.lh_attn_bwd(shape, qs, ks, vs, os_, lse, dos, dq, dk, dv, ws)
    torch.cuda.synchronize()
    want_o, want_lse = O.attn_fwd(np64(qs), np64(ks), np64(vs))
    assert_close(np64(os_), want_o, dtype, "o_sub", mode="literal")
    np.testing.assert_allclose(np64(lse), want_lse, rtol=1e-5, atol=1e-5)
    # each side runs its backward on its own forward results
    wq, wk, wv = O.attn_bwd(np64(qs), np64(ks), np64(vs), want_o, want_lse, np64(dos))
    for got, want, n in ((dq, wq, "dq"), (dk, wk, "dk"), (dv, wv, "dv")):
        assert_close(np64(got), want, dtype, n, mode="literal")


@pytest.mark.parametrize("S,d", [(1024, 128), (1152, 128), (1024, 64), (1152, 64)])
def test_attention_running_max_grows(S, d):
    """The forward's lazy running max: O is rescaled only when a row's max grows by more than
    2^32, after the previous block's PV. Key blocks are scaled up part-way through the sequence
    (head 0 at odd blocks, head 1 at even ones), so that growth reaches both sets of softmax
    warps. Every other query row is scaled down, so that within one warp some rows grow and
    others do not. N(0,1) inputs never grow after the first block."""
    B, H = 1, 2
    dtype = torch.bfloat16
    shape = Shape(B, H, S, d, 4, 1, S, dtype)
    g = torch.Generator(device="cuda").manual_seed(11)
    nb = S // 128
    grow_at = [(1, 3), (2, 4)]  # blocks where the key scale goes up 4x, per head
    f = torch.ones(H, nb)
    for h, blocks in enumerate(grow_at):
        for b in blocks:
            f[h, b:] *= 4.0
    kscale = f.repeat_interleave(128, dim=1)[None, :, :, None].cuda()
    qscale = torch.where(torch.arange(S) % 2 == 0, 1.0, 0.1)[None, None, :, None].cuda()
    qs = (torch.randn(B, H, S, d, generator=g, device="cuda") * qscale).to(dtype)
    ks = (torch.randn(B, H, S, d, generator=g, device="cuda") * kscale).to(dtype)
    vs, dos = (torch.randn(B, H, S, d, generator=g, device="cuda").to(dtype) for _ in range(2))
    os_ = torch.empty(B, H, S, d, dtype=torch.float32, device="cuda")
    lse = torch.empty(B, H, S, dtype=torch.float32, device="cuda")
    ws = ws_for(shape)
    lh.lh_attn_fwd(shape, qs, ks, vs, os_, lse, ws)
    dq, dk, dv = (torch.empty(B, H, S, d, dtype=torch.float32, device="cuda") for _ in range(3))
    lh.lh_attn_bwd(shape, qs, ks, vs, os_, lse, dos, dq, dk, dv, ws)
    torch.cuda.synchronize()
    assert lh.lh_check(ws) == (0, 0)
    want_o, want_lse = O.attn_fwd(np64(qs), np64(ks), np64(vs))
    # the running max of an unscaled row that sees every block grows by more than 2^32
    qr = np64(qs)[0, :, S - 2]
    sc = np.einsum("hd,hjd->hj", qr, np64(ks)[0, :, :S - 1]) / np.sqrt(d)
    assert ((sc.max(-1) - sc[:, :128].max(-1)) * np.log2(np.e) > 32).all()
    assert_close(np64(os_), want_o, dtype, "o_sub", mode="literal")
    np.testing.assert_allclose(np64(lse), want_lse, rtol=1e-5, atol=1e-5)
    wq, wk, wv = O.attn_bwd(np64(qs), np64(ks), np64(vs), want_o, want_lse, np64(dos))
    for got, want, n in ((dq, wq, "dq"), (dk, wk, "dk"), (dv, wv, "dv")):
        assert_close(np64(got), want, dtype, n)


def valid_idx(B, H, N, p, L, S, seed):
    geo = O.Geometry(N, p, L, S).check()
    r = np.random.default_rng(seed).random((B, H, N + geo.R)).astype(np.float32)
    return geo, O.select_topk(r, geo)


SPREAD_SHAPES = [(1, 2, 4096, 128, 4, 5, 1024), (2, 3, 2048, 64, 4, 3, 512),
                 (1, 2, 1024, 128, 2, 6, 32 * 32), (1, 2, 2187, 64, 3, 4, 81),
                 (1, 3, 640, 128, 4, 1, 640), (1, 1, 16384, 128, 4, 7, 64),
                 (1, 2, 4096, 64, 2, 3, 1024 + 64), (2, 2, 2048, 128, 4, 4, 32 * 5 + 16)]


@pytest.mark.parametrize("dt", ["f32", "bf16"])
@pytest.mark.parametrize("B,H,N,d,p,L,S", SPREAD_SHAPES)
def test_gather_scatter_and_backward(B, H, N, d, p, L, S, dt):
    dtype = DT[dt]
    shape = Shape(B, H, N, d, p, L, S, dtype)
    geo, idx_np = valid_idx(B, H, N, p, L, S, seed=S)
    idx = torch.from_numpy(idx_np).cuda()
    ws = ws_for(shape)
    gen = torch.Generator(device="cuda").manual_seed(3)
    q, k, v = (torch.randn(B, H, N, d, generator=gen, device="cuda").to(dtype) for _ in range(3))
    R = max(geo.R, 1)
    pq, pk, pv = (torch.randn(B, H, R, d, generator=gen, device="cuda").to(dtype) for _ in range(3))
    subs = [torch.empty(B, H, S, d, dtype=dtype, device="cuda") for _ in range(3)]
    lh.lh_gather(shape, q, k, v, pq, pk, pv, idx, *subs, ws)
    o_sub = torch.randn(B, H, S, d, generator=gen, device="cuda")
    o = torch.empty(B, H, N, d, dtype=dtype, device="cuda")
    lh.lh_scatter(shape, idx, o_sub, o)
    d_o = torch.randn(B, H, N, d, generator=gen, device="cuda").to(dtype)
    do_sub = torch.empty(B, H, S, d, dtype=dtype, device="cuda")
    lh.lh_scatter_bwd(shape, idx, d_o, do_sub, ws)
    dsub = [torch.randn(B, H, S, d, generator=gen, device="cuda") for _ in range(3)]
    dx = [torch.empty(B, H, N, d, dtype=dtype, device="cuda") for _ in range(3)]
    lh.lh_gather_bwd(shape, idx, *dsub, *dx)
    torch.cuda.synchronize()
    assert lh.lh_check(ws) == (0, 0)
    for x, px, sub in zip((q, k, v), (pq, pk, pv), subs):  # a copy: bit-exact
        want = O.gather(np64(x), np64(px)[:, :, :geo.R], idx_np)
        assert np.array_equal(np64(sub), want)
    assert_close(np64(o), O.scatter(idx_np, np64(o_sub), geo), dtype, "scatter")
    assert_close(np64(do_sub), O.scatter_bwd(idx_np, np64(d_o), geo), dtype, "scatter_bwd")
    # the stored span sums follow the pyramid's fp32 order and one rounding: bit-exact
    full = np.concatenate([np64(d_o), O.pool_stored(np64(d_o), geo, store_of(dtype), mean=False)], 2)
    assert np.array_equal(np64(do_sub), np.take_along_axis(full, idx_np[..., None].astype(np.int64), 2))
    for got, ds in zip(dx, dsub):
        assert_close(np64(got), O.gather_bwd(idx_np, np64(ds), geo), dtype, "gather_bwd")


def test_out_of_range_ids_are_flagged_not_faulted():
    """A bad caller-supplied id gives a zero row and a status bit, never a memory fault."""
    B, H, N, d, p, L, S = 1, 1, 256, 64, 4, 3, 64
    shape = Shape(B, H, N, d, p, L, S, torch.bfloat16)
    ws = ws_for(shape)
    q, k, v = inputs(B, H, N, d, torch.bfloat16)
    R = lh.lh_validate(shape)["R"]
    pq, pk, pv = (torch.zeros(B, H, R, d, dtype=torch.bfloat16, device="cuda") for _ in range(3))
    idx = torch.zeros(B, H, S, dtype=torch.int32, device="cuda")
    idx[0, 0, 5] = N + R + 7
    idx[0, 0, 9] = -3
    subs = [torch.full((B, H, S, d), 1.0, dtype=torch.bfloat16, device="cuda") for _ in range(3)]
    lh.lh_gather(shape, q, k, v, pq, pk, pv, idx, *subs, ws)
    rc, flags = lh.lh_check(ws)
    assert rc != 0 and flags & 1
    assert (subs[0][0, 0, 5] == 0).all() and (subs[0][0, 0, 9] == 0).all()
    assert lh.lh_check(ws) == (0, 0)  # cleared by the read


@pytest.mark.parametrize("B,H,S,d", [(1, 2, 4096, 128), (1, 9, 1024, 128), (2, 3, 384, 128),
                                     (1, 2, 4096, 64), (1, 9, 1024, 64), (2, 3, 384, 64)])
def test_fused_backward_matches_the_deterministic_one(B, H, S, d):
    """The one-pass backward computes dK and dV exactly as the two-pass one (the same MMAs
    accumulate in the same order), so they agree bit for bit. Its dQ adds fp32 partial sums per
    128-key block in a varying order (atomic adds at d = 128, copy-engine reductions at d = 64):
    it agrees to fp32 rounding of those sums."""
    dtype = torch.bfloat16
    qs, ks, vs, dos = rand_sub(B, H, S, d, dtype, seed=S + 1)
    out = {}
    for det in (False, True):
        shape = Shape(B, H, S, d, 4, 1, S, dtype, det)
        ws = ws_for(shape)
        os_ = torch.empty(B, H, S, d, dtype=torch.float32, device="cuda")
        lse = torch.empty(B, H, S, dtype=torch.float32, device="cuda")
        lh.lh_attn_fwd(shape, qs, ks, vs, os_, lse, ws)
        g = [torch.empty(B, H, S, d, dtype=torch.float32, device="cuda") for _ in range(3)]
        lh.lh_attn_bwd(shape, qs, ks, vs, os_, lse, dos, *g, ws)
        assert lh.lh_check(ws) == (0, 0)
        out[det] = g
    (fq, fk, fv), (dq, dk, dv) = out[False], out[True]
    assert torch.equal(fk, dk) and torch.equal(fv, dv)
    rms = dq.pow(2).mean().sqrt()
    err = (fq - dq).abs() / torch.maximum(dq.abs(), rms)
    assert err.max().item() <= 1e-4, err.max().item()
