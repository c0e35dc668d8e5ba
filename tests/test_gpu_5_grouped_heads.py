"""Grouped-query heads on the GPU against the oracle: K and V with Hkv < H heads, query head h
using key/value head h // (H / Hkv). Every query head selects its own cells; a key/value head's
gradients sum those of its query heads. This is a reading: the pages describe no such model
(Llama-3-style grouped-query attention is the use)."""
import numpy as np
import pytest
import torch

import oracle as O
from workloads import WORKLOADS, make_inputs

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import sparse_hierarchical_attention_b200 as lh
    from sparse_hierarchical_attention_b200 import LighthouseAttention, LighthouseLayer, Shape, saved_views

from gpu_util import assert_close, g_of, np64, store_of

DT = {"f32": torch.float32, "bf16": torch.bfloat16}


def heads(B, H, Hkv, N, d, dtype, seed):
    g = torch.Generator(device="cuda").manual_seed(seed)
    s = torch.exp(0.5 * torch.randn(B, H, N, 1, generator=g, device="cuda"))
    q = (torch.randn(B, H, N, d, generator=g, device="cuda") * s).to(dtype)
    k, v = ((torch.randn(B, Hkv, N, d, generator=g, device="cuda") * s[:, ::H // Hkv]).to(dtype)
            for _ in range(2))
    return q, k, v


def ws_for(shape):
    return torch.zeros(lh.lh_workspace_bytes(shape), dtype=torch.uint8, device="cuda")


# (B, H, Hkv, N, d, p, L, S)
SHAPES = [
    (1, 4, 2, 4096, 128, 4, 5, 1024),   # one coarse pooling level beyond the tile
    (2, 4, 1, 2048, 64, 4, 3, 512),     # every query head on one key/value head
    (1, 6, 3, 8192, 128, 4, 6, 512),
    (1, 4, 2, 2187, 64, 3, 4, 243),
    (1, 8, 2, 4096, 64, 2, 3, 1024 + 64),  # strata of 16 chunks
]


@pytest.mark.parametrize("dt", ["f32", "bf16"])
@pytest.mark.parametrize("B,H,Hkv,N,d,p,L,S", SHAPES)
def test_grouped_pyramid_and_score(B, H, Hkv, N, d, p, L, S, dt):
    """Q pooled over the query heads, K and V over the key/value heads, all bit-exact; the
    score of query head h is |q| + |k| of its key/value head, bit-exact."""
    dtype = DT[dt]
    shape = Shape(B, H, N, d, p, L, S, dtype, Hkv=Hkv)
    R = lh.lh_validate(shape)["R"]
    q, k, v = heads(B, H, Hkv, N, d, dtype, seed=N + H)
    pq = torch.empty(B, H, max(R, 1), d, dtype=dtype, device="cuda")
    pk, pv = (torch.empty(B, Hkv, max(R, 1), d, dtype=dtype, device="cuda") for _ in range(2))
    score = torch.empty(B, H, N + R, dtype=torch.float32, device="cuda")
    ws = ws_for(shape)
    lh.lh_build_pyramid(shape, q, k, v, pq, pk, pv, score, ws)
    s_only = torch.empty_like(score)
    lh.lh_score(shape, q, k, s_only, ws)
    torch.cuda.synchronize()
    geo = O.Geometry(N, p, L, S).check()
    want = O.score(np64(q), np64(k), geo, g_of(dtype))
    assert np.array_equal(score.cpu().numpy(), want)
    assert np.array_equal(s_only.cpu().numpy(), want)
    for x, px in ((q, pq), (k, pk), (v, pv)):
        assert np.array_equal(np64(px)[:, :, :R], O.pool_stored(np64(x), geo, store_of(dtype)))


@pytest.mark.parametrize("dt", ["f32", "bf16"])
@pytest.mark.parametrize("B,H,Hkv,N,d,p,L,S", SHAPES)
def test_grouped_gather_and_its_backward(B, H, Hkv, N, d, p, L, S, dt):
    """k_sub / v_sub rows come from the key/value head (a copy: bit-exact); dK and dV of a
    key/value head sum the spread of every query head of its group."""
    dtype = DT[dt]
    shape = Shape(B, H, N, d, p, L, S, dtype, Hkv=Hkv)
    geo = O.Geometry(N, p, L, S).check()
    rng = np.random.default_rng(S + H)
    idx_np = O.select_topk(rng.random((B, H, N + geo.R)).astype(np.float32), geo)
    idx = torch.from_numpy(idx_np).cuda()
    gen = torch.Generator(device="cuda").manual_seed(7)
    R = max(geo.R, 1)
    q = torch.randn(B, H, N, d, generator=gen, device="cuda").to(dtype)
    k, v = (torch.randn(B, Hkv, N, d, generator=gen, device="cuda").to(dtype) for _ in range(2))
    pq = torch.randn(B, H, R, d, generator=gen, device="cuda").to(dtype)
    pk, pv = (torch.randn(B, Hkv, R, d, generator=gen, device="cuda").to(dtype) for _ in range(2))
    subs = [torch.empty(B, H, S, d, dtype=dtype, device="cuda") for _ in range(3)]
    ws = ws_for(shape)
    lh.lh_gather(shape, q, k, v, pq, pk, pv, idx, *subs, ws)
    dsub = [torch.randn(B, H, S, d, generator=gen, device="cuda") for _ in range(3)]
    dq = torch.empty(B, H, N, d, dtype=dtype, device="cuda")
    dk, dv = (torch.empty(B, Hkv, N, d, dtype=dtype, device="cuda") for _ in range(2))
    lh.lh_gather_bwd(shape, idx, *dsub, dq, dk, dv)
    torch.cuda.synchronize()
    assert lh.lh_check(ws) == (0, 0)
    hmap = O.kv_head_of(H, Hkv)
    assert np.array_equal(np64(subs[0]), O.gather(np64(q), np64(pq)[:, :, :geo.R], idx_np))
    for x, px, sub in ((k, pk, subs[1]), (v, pv, subs[2])):
        want = O.gather(np64(x)[:, hmap], np64(px)[:, hmap, :geo.R], idx_np)
        assert np.array_equal(np64(sub), want)
    assert_close(np64(dq), O.gather_bwd(idx_np, np64(dsub[0]), geo), dtype, "gather_bwd dQ")
    for got, ds, n in ((dk, dsub[1], "dK"), (dv, dsub[2], "dV")):
        per_q = O.gather_bwd(idx_np, np64(ds), geo)
        want = per_q.reshape(B, Hkv, H // Hkv, N, d).sum(axis=2)
        assert_close(np64(got), want, dtype, f"gather_bwd {n}")


# (workload recipe, B, H, Hkv, N, S): p, L, d and dtype of the named workload
LAYER = [
    ("tiny-2k-fp32", 1, 4, 2, 2048, 512),
    ("llama530m-98k", 1, 4, 1, 8192, 8 * 64),
    ("llama530m-98k", 1, 8, 2, 8192, 8 * 64),
    ("128k", 1, 4, 2, 8192, 8 * 64),
]


@pytest.mark.parametrize("det", [False, True])
@pytest.mark.parametrize("name,B,H,Hkv,N,S", LAYER)
def test_grouped_layer_matches_oracle(name, B, H, Hkv, N, S, det):
    w = WORKLOADS[name]
    shape = Shape(B, H, N, w.d, w.p, w.L, S, w.dtype, det, Hkv)
    q, _, _, d_o = make_inputs(w, "cuda", seed=0, B=B, H=H, N=N)
    _, k, v, _ = make_inputs(w, "cuda", seed=1, B=B, H=Hkv, N=N)
    layer = LighthouseLayer(shape)
    o, saved = layer.forward(q, k, v)
    dq, dk, dv = layer.backward(saved, d_o)
    layer.check()
    assert dk.shape == k.shape and dv.shape == v.shape
    geo = O.Geometry(N, w.p, w.L, S).check()
    wo, sv = O.layer_fwd(np64(q), np64(k), np64(v), geo, g_of(w.dtype), store=store_of(w.dtype))
    wgrads = O.layer_bwd(sv, np64(d_o))
    assert np.array_equal(saved_views(shape, saved)["idx"].cpu().numpy(), sv["idx"])
    assert_close(np64(o), wo, w.dtype, "O")
    for got, want, n in zip((dq, dk, dv), wgrads, ("dQ", "dK", "dV")):
        assert_close(np64(got), want, w.dtype, n)


def test_grouped_equals_the_layer_on_repeated_heads():
    """Forward: running the grouped layer, or the plain layer with every key/value head copied
    to its query heads, gives the same selection and the same O and dQ bit for bit (the same
    kernels see the same values); dK, dV then agree with the group sums within the roundings."""
    B, H, Hkv, N, d, p, L, S = 1, 4, 2, 4096, 128, 4, 5, 1024
    dtype = torch.bfloat16
    q, k, v = heads(B, H, Hkv, N, d, dtype, seed=3)
    d_o = torch.randn(B, H, N, d, device="cuda").to(dtype)
    g = H // Hkv
    kr, vr = (x.repeat_interleave(g, dim=1).contiguous() for x in (k, v))
    grouped = LighthouseLayer(Shape(B, H, N, d, p, L, S, dtype, True, Hkv))
    plain = LighthouseLayer(Shape(B, H, N, d, p, L, S, dtype, True))
    o1, s1 = grouped.forward(q, k, v)
    o2, s2 = plain.forward(q, kr, vr)
    dq1, dk1, dv1 = grouped.backward(s1, d_o)
    dq2, dk2, dv2 = plain.backward(s2, d_o)
    grouped.check()
    plain.check()
    assert torch.equal(o1, o2) and torch.equal(dq1, dq2)
    assert torch.equal(saved_views(grouped.shape, s1)["idx"], saved_views(plain.shape, s2)["idx"])
    for a, b in ((dk1, dk2), (dv1, dv2)):
        # the plain layer rounds each query head's share to bf16 (half an ulp, 2^-9 of that
        # share) before this sum; the grouped layer rounds the fp32 group sum once (2^-9 of it)
        shares = np64(b).reshape(B, Hkv, g, N, d)
        bound = 2.0 ** -8 * (np.abs(shares).sum(2) + np.abs(np64(a))) + 1e-30
        assert (np.abs(np64(a) - shares.sum(2)) <= bound).all()


def test_autograd_module_takes_fewer_key_heads():
    B, H, Hkv, N, d = 1, 4, 1, 2048, 64
    attn = LighthouseAttention(4, 3, 512)
    g = torch.Generator(device="cuda").manual_seed(9)
    q = torch.randn(B, H, N, d, generator=g, device="cuda").to(torch.bfloat16).requires_grad_()
    k, v = (torch.randn(B, Hkv, N, d, generator=g, device="cuda").to(torch.bfloat16).requires_grad_()
            for _ in range(2))
    o = attn(q, k, v)
    o.float().sum().backward()
    assert o.shape == q.shape and k.grad.shape == k.shape and v.grad.shape == v.shape
    assert torch.isfinite(k.grad.float()).all() and torch.isfinite(q.grad.float()).all()


def test_grouped_bad_ids_are_flagged_not_faulted():
    """A corrupted selection reaching the grouped backward (span sums, the dQ spread and the
    key/value group spread) sets status bit 1 instead of faulting."""
    B, H, Hkv, N, d, p, L, S = 1, 4, 2, 1024, 64, 4, 3, 256
    shape = Shape(B, H, N, d, p, L, S, torch.bfloat16, Hkv=Hkv)
    q, k, v = heads(B, H, Hkv, N, d, torch.bfloat16, seed=5)
    layer = LighthouseLayer(shape)
    o, saved = layer.forward(q, k, v)
    layer.check()
    idx = saved_views(shape, saved)["idx"]
    idx[0, 3, 5] = N + 10_000_000  # beyond the pyramid
    idx[0, 1, 9] = -3
    layer.backward(saved, torch.randn_like(q))
    rc, flags = lh.lh_check(layer.ws)
    assert rc != 0 and flags & 1
    assert lh.lh_check(layer.ws) == (0, 0)  # cleared by the read
