"""Pins of the CPU oracle against what the pages and the mathematics fix (CPU only).

Each test checks the oracle against something other than itself: brute force on tiny inputs,
closed forms, a hand-worked example, library routines on special cases, adjoint identities,
causality, and finite differences. The cited passages are in *Long Context Pre-Training with
Lighthouse Attention* (gist.science summary, technical summary sections 2.A-2.D, 5) and the
Nous Research article (edge.aivizor.me, four-stage paragraph).
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle as O

rng = np.random.default_rng(1234)


def rand(*shape, dtype=np.float32, scale=1.0):
    return (rng.standard_normal(shape) * scale).astype(dtype)


SMALL = [  # (N, p, L, S)
    (16, 2, 3, 8), (16, 2, 3, 16), (32, 4, 2, 16), (64, 4, 3, 16), (27, 3, 3, 9),
    (64, 2, 4, 40), (8, 2, 1, 8), (48, 4, 3, 12),
]
# budgets that are no multiple of the chunk count C: strata of G = C / gcd(S, C) chunks
STRATA = [  # (N, p, L, S): G
    (16, 2, 3, 6),     # C = 4: G = 2, 3 rows per stratum
    (64, 4, 3, 18),    # C = 4: G = 2, 9 rows
    (64, 2, 4, 12),    # C = 8: G = 2, 3 rows
    (27, 3, 3, 4),     # C = 3: G = 3, one stratum over the whole sequence
    (96, 2, 3, 26),    # C = 24: G = 12, 13 rows
    (128, 2, 3, 34),   # C = 32: G = 16, 17 rows (the structure of p = 2, L = 3, k = 1536 at 98K)
]


# ---------------------------------------------------------------- pyramid (section 2.A)
@pytest.mark.parametrize("N,p,L,S", SMALL)
def test_pyramid_cells_are_span_means(N, p, L, S):
    """A level-l cell is the mean of the p^l tokens it covers (closed form)."""
    geo = O.Geometry(N, p, L, S)
    x = rand(2, 2, N, 4)
    px = O.build_pyramid(x, geo)
    assert px.shape == (2, 2, geo.R, 4)
    for l in range(1, L):
        w = p ** l
        for j in range(N // w):
            want = [[sum(float(x[b, h, t, c]) for t in range(j * w, (j + 1) * w)) / w
                     for c in range(4)] for b in range(2) for h in range(2)]
            got = px[:, :, geo.offsets[l] - N + j].reshape(4, 4)
            np.testing.assert_allclose(got, np.array(want), rtol=1e-12, atol=1e-13)


# ---------------------------------------------------------------- scores (section 2.B)
@pytest.mark.parametrize("d,g", [(64, 8), (128, 8), (64, 4), (128, 4), (8, 4), (16, 8)])
def test_norm_matches_fp64_norm(d, g):
    """The fp32 norm in the fixed order is within a few fp32 ulps of the exact norm."""
    x = rand(500, d, scale=3.0)
    got = O.row_norm_f32(x, g).astype(np.float64)
    exact = np.sqrt((x.astype(np.float64) ** 2).sum(axis=1))
    assert np.max(np.abs(got - exact) / exact) < 4 * 2.0 ** -24 * math.log2(d)


def test_norm_closed_forms():
    """One-hot rows have norm |x|; constant rows of a power of two have norm c*sqrt(d)."""
    x = np.zeros((6, 128), np.float32)
    vals = [1.5, -3.0, 0.125, 7.0, -2.5, 100.0]
    for i, v in enumerate(vals):
        x[i, (37 * i) % 128] = v
    np.testing.assert_array_equal(O.row_norm_f32(x, 8), np.abs(np.array(vals, np.float32)))
    c = np.full((1, 64), 0.5, np.float32)
    assert O.row_norm_f32(c, 4)[0] == np.float32(0.5 * 8.0)
    assert O.row_norm_f32(np.zeros((1, 64), np.float32), 8)[0] == 0.0


def test_norm_order_is_the_fixed_one():
    """The tree order is not a sequential sum: a case where they differ must follow the tree."""
    # groups of g=4: group sums 2^24, 1, 1, 1 (as squares); sequential would round away the ones
    x = np.zeros((1, 16), np.float32)
    x[0, 0] = 4096.0  # square 2^24
    x[0, 4] = x[0, 8] = x[0, 12] = 1.0
    # tree: (2^24 + 1) + (1 + 1) -> 2^24 (tie to even) + 2 = 2^24 + 2
    got = O.row_norm_f32(x, 4)[0]
    assert got == np.sqrt(np.float32(2.0 ** 24 + 2.0))


@pytest.mark.parametrize("N,p,L,S", SMALL)
def test_coarse_score_is_max_over_span(N, p, L, S):
    """Coarse cells inherit each norm as the max over their tokens, then the two are summed."""
    geo = O.Geometry(N, p, L, S)
    q, k = rand(1, 3, N, 8, scale=2.0), rand(1, 3, N, 8)
    r = O.score(q, k, geo, 4)
    sq, sk = O.row_norm_f32(q, 4), O.row_norm_f32(k, 4)
    for h in range(3):
        for l in range(L):
            w = p ** l
            for j in range(N // w):
                want = np.float32(sq[0, h, j * w:(j + 1) * w].max()) + \
                    np.float32(sk[0, h, j * w:(j + 1) * w].max())
                assert r[0, h, geo.offsets[l] + j] == want


@pytest.mark.parametrize("N,p,L,S", [(16, 2, 3, 8), (64, 4, 3, 16), (27, 3, 3, 9)])
@pytest.mark.parametrize("H,Hkv", [(4, 2), (4, 1), (6, 3)])
def test_grouped_heads_score_with_their_key_head(N, p, L, S, H, Hkv):
    """Grouped-query heads: query head h ranks with its own q norms and the k norms of key head
    h // (H / Hkv), each max-pooled over the cell's span, then summed (brute force)."""
    geo = O.Geometry(N, p, L, S)
    q, k = rand(1, H, N, 8, scale=2.0), rand(1, Hkv, N, 8)
    r = O.score(q, k, geo, 4)
    sq, sk = O.row_norm_f32(q, 4), O.row_norm_f32(k, 4)
    for h in range(H):
        hk = h // (H // Hkv)
        for l in range(L):
            w = p ** l
            for j in range(N // w):
                want = np.float32(sq[0, h, j * w:(j + 1) * w].max()) + \
                    np.float32(sk[0, hk, j * w:(j + 1) * w].max())
                assert r[0, h, geo.offsets[l] + j] == want
    with pytest.raises(ValueError):
        O.score(q, rand(1, 3, N, 8) if H == 4 else rand(1, 4, N, 8), geo, 4)


# ---------------------------------------------------------------- selection (2.B, 2.C)
def brute_select(r, geo):
    """Every stratum of G chunks: full sort of all its candidates by the total key, the k best
    plus the G coarsest cells, then causal order."""
    out = []
    G = geo.C // math.gcd(geo.S, geo.C)  # restated here from the reading, not taken from geo
    k = geo.S * G // geo.C - G
    assert (G, k) == (geo.G, geo.k)
    for s in range(geo.C // G):
        cands = []
        for l in range(geo.L - 1):
            per = geo.p ** (geo.L - 1 - l)  # cells of level l in one chunk
            for j in range(s * G * per, (s + 1) * G * per):
                cands.append((float(r[geo.offsets[l] + j]), l, j))
        best = sorted(cands, key=lambda e: (-e[0], -e[1], e[2]))[:k]
        rows = [(l, j) for _, l, j in best] + [(geo.L - 1, c) for c in range(s * G, (s + 1) * G)]
        rows.sort(key=lambda e: ((e[1] + 1) * geo.p ** e[0], e[0]))
        out += [geo.offsets[l] + j for l, j in rows]
    return out


@pytest.mark.parametrize("N,p,L,S", SMALL + STRATA)
def test_topk_equals_full_sort(N, p, L, S):
    geo = O.Geometry(N, p, L, S).check()
    # quantised scores so that exact ties (and the tie-break) occur often
    q = np.round(rand(2, 2, N, 8) * 2) / 2
    k = np.round(rand(2, 2, N, 8) * 2) / 2
    r = O.score(q, k, geo, 8)
    idx = O.select_topk(r, geo)
    for b, h in itertools.product(range(2), range(2)):
        assert idx[b, h].tolist() == brute_select(r[b, h], geo)


@pytest.mark.parametrize("N,p,L,S", STRATA)
def test_topk_strata_invariants(N, p, L, S):
    """Every stratum keeps its G coarsest cells and k picks from inside it, in causal order;
    the rows of one chunk are contiguous and end with its coarsest cell."""
    geo = O.Geometry(N, p, L, S).check()
    assert geo.G > 1 and geo.C % geo.G == 0 and geo.m * (geo.C // geo.G) == S
    r = O.score(rand(1, 2, N, 8), rand(1, 2, N, 8), geo, 8)
    idx = O.select_topk(r, geo)
    level, cell = geo.decode(idx)
    end = (cell + 1) * geo.p ** level
    start = end - geo.p ** level
    span = geo.G * geo.T
    for h in range(2):
        assert len(set(idx[0, h].tolist())) == S
        for s in range(geo.C // geo.G):
            rows = slice(s * geo.m, (s + 1) * geo.m)
            lv, ce, st, en = level[0, h, rows], cell[0, h, rows], start[0, h, rows], end[0, h, rows]
            assert (st >= s * span).all() and (en <= (s + 1) * span).all()
            assert sorted(ce[lv == L - 1].tolist()) == list(range(s * geo.G, (s + 1) * geo.G))
            key = list(zip(en.tolist(), lv.tolist()))
            assert key == sorted(key) and len(set(key)) == len(key)
            chunk = st // geo.T
            assert (np.diff(chunk) >= 0).all()  # chunk segments are contiguous
            last = np.r_[chunk[1:] != chunk[:-1], True]
            assert (lv[last] == L - 1).all()  # each segment ends with its chunk's coarsest cell


@pytest.mark.parametrize("N,p,L,S", SMALL)
def test_topk_invariants(N, p, L, S):
    """Coarsest cell kept in every chunk as its last row; rows unique and causally ordered."""
    geo = O.Geometry(N, p, L, S).check()
    r = O.score(rand(1, 2, N, 8), rand(1, 2, N, 8), geo, 8)
    idx = O.select_topk(r, geo)
    assert idx.shape == (1, 2, S)
    level, cell = geo.decode(idx)
    end = (cell + 1) * geo.p ** level
    for h in range(2):
        assert len(set(idx[0, h].tolist())) == S
        for c in range(geo.C):
            rows = slice(c * geo.m, (c + 1) * geo.m)
            assert level[0, h, rows][-1] == L - 1 and cell[0, h, rows][-1] == c
            start = end[0, h, rows] - geo.p ** level[0, h, rows]
            assert (start >= c * geo.T).all() and (end[0, h, rows] <= (c + 1) * geo.T).all()
            key = list(zip(end[0, h, rows].tolist(), level[0, h, rows].tolist()))
            assert key == sorted(key) and len(set(key)) == len(key)


def test_topk_worked_example(golden_dir):
    ex = json.load(open(os.path.join(golden_dir, "topk_worked_example.json")))
    sh = ex["shape"]
    q = np.zeros((1, 1, sh["N"], sh["d"]), np.float32)
    k = np.zeros_like(q)
    q[0, 0, :, 0] = ex["q_norms"]
    k[0, 0, :, 1] = ex["k_norms"]
    for S, want in list(ex["idx"].items()) + list(ex["idx_strata"].items()):
        geo = O.Geometry(sh["N"], sh["p"], sh["L"], int(S)).check()
        r = O.score(q, k, geo, 4)
        assert r[0, 0].tolist() == ex["score"]
        assert O.select_topk(r, geo)[0, 0].tolist() == want


def test_select_everything_is_score_independent():
    """With m = M + 1 every cell is selected, whatever the scores."""
    geo = O.Geometry(32, 2, 3, 8 * 7).check()
    assert geo.m == geo.M + 1
    ids = []
    for seed in range(3):
        r = np.random.default_rng(seed).random((1, 1, geo.N + geo.R)).astype(np.float32)
        ids.append(O.select_topk(r, geo))
    assert (ids[0] == ids[1]).all() and (ids[0] == ids[2]).all()
    assert sorted(ids[0][0, 0].tolist()) == list(range(geo.N + geo.R))


# ---------------------------------------------------------------- attention (2.C)
def test_attention_closed_form_uniform():
    """Zero keys: uniform softmax, so O_i is the running mean of V and lse_i = ln(i+1)."""
    S, d = 37, 16
    qs = rand(1, 1, S, d).astype(np.float64)
    ks = np.zeros((1, 1, S, d))
    vs = rand(1, 1, S, d).astype(np.float64)
    o, lse = O.attn_fwd(qs, ks, vs)
    want = np.cumsum(vs[0, 0], axis=0) / np.arange(1, S + 1)[:, None]
    np.testing.assert_allclose(o[0, 0], want, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(lse[0, 0], np.log(np.arange(1, S + 1)), rtol=1e-13)


def test_attention_matches_torch_sdpa_and_autograd():
    """Forward equals torch's causal SDPA; backward equals torch autograd (fp64, CPU)."""
    B, H, S, d = 2, 3, 50, 16
    qs, ks, vs, dos = (rand(B, H, S, d).astype(np.float64) for _ in range(4))
    o, lse = O.attn_fwd(qs, ks, vs)
    dq, dk, dv = O.attn_bwd(qs, ks, vs, o, lse, dos)
    tq, tk, tv = (torch.tensor(a, requires_grad=True) for a in (qs, ks, vs))
    to = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, is_causal=True)
    to.backward(torch.tensor(dos))
    np.testing.assert_allclose(o, to.detach().numpy(), rtol=1e-10, atol=1e-12)
    for mine, ref in ((dq, tq), (dk, tk), (dv, tv)):
        np.testing.assert_allclose(mine, ref.grad.numpy(), rtol=1e-9, atol=1e-11)
    s = np.einsum("bhid,bhjd->bhij", qs, ks) / math.sqrt(d)
    s = np.where(np.tril(np.ones((S, S), bool)), s, -np.inf)
    np.testing.assert_allclose(lse, np.log(np.exp(s).sum(-1)), rtol=1e-12)


def by_definition_layer(q, k, v, geo, g):
    """The layer written without a subsequence: masked attention over selected pyramid cells.

    Cell e' is visible to cell e iff (end', level') <= (end, level). Each token's output is
    the sum of the outputs of the selected cells covering it. Plain loops, tiny inputs only.
    """
    B, H, N, d = q.shape
    r = O.score(q, k, geo, g)
    idx = O.select_topk(r, geo)
    out = np.zeros((B, H, N, d))
    for b, hq in itertools.product(range(B), range(H)):
        hk = hq * k.shape[1] // H  # the key/value head of query head hq (grouped-query heads)
        cells = [geo.decode(int(i)) for i in idx[b, hq]]
        cells = [(int(l), int(j)) for l, j in cells]
        rng_local = np.random.default_rng(b * 31 + hq)
        rng_local.shuffle(cells)  # the definition needs no particular order

        def mean_of(x, l, j):
            w = geo.p ** l
            h = hq if x.shape[1] == H else hk
            return np.asarray(x[b, h, j * w:(j + 1) * w], np.float64).mean(axis=0)

        for (l, j) in cells:
            key = ((j + 1) * geo.p ** l, l)
            qi = mean_of(q, l, j)
            vis = [(l2, j2) for (l2, j2) in cells if ((j2 + 1) * geo.p ** l2, l2) <= key]
            logits = [float(qi @ mean_of(k, l2, j2)) / math.sqrt(d) for l2, j2 in vis]
            mx = max(logits)
            wts = [math.exp(a - mx) for a in logits]
            z = sum(wts)
            oi = sum(w_ / z * mean_of(v, l2, j2) for w_, (l2, j2) in zip(wts, vis))
            out[b, hq, j * geo.p ** l:(j + 1) * geo.p ** l] += oi
    return out


@pytest.mark.parametrize("N,p,L,S", [(16, 2, 3, 8), (32, 4, 3, 8), (27, 3, 3, 9),
                                     (32, 2, 3, 8 * 7), (8, 2, 1, 8), (16, 2, 3, 6), (27, 3, 3, 4),
                                     (96, 2, 3, 26)])
def test_layer_equals_by_definition(N, p, L, S):
    geo = O.Geometry(N, p, L, S).check()
    q, k, v = (rand(1, 2, N, 8) for _ in range(3))
    o, _ = O.layer_fwd(q, k, v, geo, 4)
    np.testing.assert_allclose(o, by_definition_layer(q, k, v, geo, 4), rtol=1e-11, atol=1e-12)


@pytest.mark.parametrize("N,p,L,S", [(16, 2, 3, 8), (27, 3, 3, 9), (16, 2, 3, 6)])
@pytest.mark.parametrize("H,Hkv", [(4, 2), (4, 1)])
def test_grouped_heads_layer_equals_by_definition(N, p, L, S, H, Hkv):
    geo = O.Geometry(N, p, L, S).check()
    q = rand(1, H, N, 8)
    k, v = (rand(1, Hkv, N, 8) for _ in range(2))
    o, _ = O.layer_fwd(q, k, v, geo, 4)
    np.testing.assert_allclose(o, by_definition_layer(q, k, v, geo, 4), rtol=1e-11, atol=1e-12)


def test_recovery_identity_dense_sdpa():
    """With L = 1 the layer is plain dense causal SDPA (the recovery phase), fwd and bwd."""
    B, H, N, d = 1, 2, 64, 16
    geo = O.Geometry(N, 4, 1, N).check()
    q, k, v, do = (rand(B, H, N, d) for _ in range(4))
    o, saved = O.layer_fwd(q, k, v, geo, 4)
    dq, dk, dv = O.layer_bwd(saved, do.astype(np.float64))
    tq, tk, tv = (torch.tensor(a, dtype=torch.float64, requires_grad=True) for a in (q, k, v))
    to = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, is_causal=True)
    to.backward(torch.tensor(do, dtype=torch.float64))
    np.testing.assert_allclose(o, to.detach().numpy(), rtol=1e-10, atol=1e-12)
    for mine, ref in ((dq, tq), (dk, tk), (dv, tv)):
        np.testing.assert_allclose(mine, ref.grad.numpy(), rtol=1e-9, atol=1e-11)


# ---------------------------------------------------------------- scatter and adjoints (2.C)
@pytest.mark.parametrize("N,p,L,S", SMALL + STRATA)
def test_scatter_adjoints(N, p, L, S):
    """scatter_bwd is the adjoint of scatter; gather_bwd is the adjoint of pool-then-gather."""
    geo = O.Geometry(N, p, L, S).check()
    B, H, d = 2, 2, 4
    r = O.score(rand(B, H, N, 8), rand(B, H, N, 8), geo, 8)
    idx = O.select_topk(r, geo)
    xs, y = rand(B, H, S, d).astype(np.float64), rand(B, H, N, d).astype(np.float64)
    lhs = (O.scatter(idx, xs, geo) * y).sum()
    rhs = (xs * O.scatter_bwd(idx, y, geo)).sum()
    assert abs(lhs - rhs) <= 1e-10 * (abs(lhs) + 1)
    x = rand(B, H, N, d).astype(np.float64)
    g = O.gather(x, O.build_pyramid(x, geo), idx)
    lhs = (g * xs).sum()
    rhs = (x * O.gather_bwd(idx, xs, geo)).sum()
    assert abs(lhs - rhs) <= 1e-10 * (abs(lhs) + 1)


def test_every_token_covered_between_1_and_L_times():
    geo = O.Geometry(64, 2, 4, 40).check()
    r = O.score(rand(1, 3, 64, 8), rand(1, 3, 64, 8), geo, 8)
    idx = O.select_topk(r, geo)
    cover = O.scatter(idx, np.ones((1, 3, geo.S, 1)), geo)
    assert cover.min() >= 1 and cover.max() <= geo.L


# ---------------------------------------------------------------- causality (2.C, 5)
@pytest.mark.parametrize("N,p,L,S", [(64, 4, 3, 16), (64, 2, 4, 40), (16, 2, 1, 16),
                                     (64, 2, 4, 12), (96, 2, 3, 26)])
def test_future_chunks_do_not_change_the_past(N, p, L, S):
    """Perturbing the tokens of stratum s and later (a stratum is G chunks; G = 1 when S is a
    multiple of C) changes no output of the strata before s."""
    geo = O.Geometry(N, p, L, S).check()
    q, k, v = (rand(1, 2, N, 8) for _ in range(3))
    o, _ = O.layer_fwd(q, k, v, geo, 4)
    for c in range(1, geo.C // geo.G):
        q2, k2, v2 = q.copy(), k.copy(), v.copy()
        t0 = c * geo.G * geo.T
        for x in (q2, k2, v2):
            x[:, :, t0:] = rand(1, 2, N - t0, 8, scale=3.0)
        o2, _ = O.layer_fwd(q2, k2, v2, geo, 4)
        assert np.array_equal(o2[:, :, :t0], o[:, :, :t0])
        assert not np.allclose(o2[:, :, t0:], o[:, :, t0:])


# ---------------------------------------------------------------- gradients (2.B)
@pytest.mark.parametrize("N,p,L,S,H,Hkv", [(16, 2, 3, 8, 2, 2), (32, 4, 2, 16, 2, 2),
                                            (27, 3, 3, 9, 2, 2), (8, 2, 1, 8, 2, 2),
                                            (16, 2, 3, 6, 2, 2), (16, 2, 3, 8, 4, 2),
                                            (16, 2, 3, 6, 3, 1)])
def test_gradients_finite_differences(N, p, L, S, H, Hkv):
    """Central differences in fp64 with the selection held fixed (it is piecewise constant).
    With grouped-query heads (Hkv < H) a key/value element feeds every query head of its group,
    so its difference quotient checks the sum over the group."""
    geo = O.Geometry(N, p, L, S).check()
    B, d = 1, 4
    q = rand(B, H, N, d).astype(np.float64)
    k, v = (rand(B, Hkv, N, d).astype(np.float64) for _ in range(2))
    do = rand(B, H, N, d).astype(np.float64)
    o, saved = O.layer_fwd(q, k, v, geo, 4)
    idx = saved["idx"]
    grads = O.layer_bwd(saved, do)

    def loss(q_, k_, v_):
        return (O.layer_fwd(q_, k_, v_, geo, 4, idx=idx)[0] * do).sum()

    eps = 1e-6
    for which, gr in enumerate(grads):
        num = np.zeros_like(gr)
        for pos in itertools.product(*(range(n) for n in gr.shape)):
            args = [q.copy(), k.copy(), v.copy()]
            args[which][pos] += eps
            up = loss(*args)
            args[which][pos] -= 2 * eps
            num[pos] = (up - loss(*args)) / (2 * eps)
        np.testing.assert_allclose(gr, num, rtol=1e-6, atol=1e-7)


# ---------------------------------------------------------------- storage rounding
def test_bf16_rounding_matches_library_conversion():
    """Round-to-nearest-even to bf16 equals torch's fp32 -> bf16 conversion on fp32 values."""
    x = np.concatenate([rand(100000, scale=10.0), np.float32([1 + 2 ** -8, 1 + 3 * 2 ** -8,
                                                              -(1 + 2 ** -8), 0.0, 2 ** -20])])
    want = torch.from_numpy(x).to(torch.bfloat16).to(torch.float64).numpy()
    np.testing.assert_array_equal(O.round_to(x.astype(np.float64), "bf16"), want)
    assert O.round_to(np.float64(1 + 2 ** -8), "bf16") == 1.0  # tie goes to even
    assert O.round_to(np.float64(1 + 3 * 2 ** -8), "bf16") == 1 + 2 ** -6
    y = rand(1000).astype(np.float64) / 3
    np.testing.assert_array_equal(O.round_to(y, "f32"), y.astype(np.float32).astype(np.float64))


@pytest.mark.parametrize("N,p,L,S", SMALL)
@pytest.mark.parametrize("store", ["f32", "bf16"])
def test_stored_pyramid_is_the_rounded_mean(N, p, L, S, store):
    """The fp32-ordered stored cells are the exact span means up to a derived bound: fp32 sums
    at most (p-1)(L-1) additions deep, one scaling, one rounding to the storage type."""
    geo = O.Geometry(N, p, L, S)
    x = rand(2, 2, N, 8, scale=3.0)
    got = O.pool_stored(x, geo, store)
    exact = O.build_pyramid(x, geo)
    mean_abs = O.build_pyramid(np.abs(x), geo)
    u = 2.0 ** -8 if store == "bf16" else 2.0 ** -24
    depth = (p - 1) * (L - 1) + 1
    bound = depth * 2.0 ** -24 * mean_abs * (1 + u) + u * np.abs(exact) * (1 + 1e-6) + 1e-300
    assert (np.abs(got - exact) <= bound).all()
    sums = O.pool_stored(x, geo, store, mean=False)  # span sums: p^l times the mean
    scale = np.concatenate([np.full(N // p ** l, float(p ** l)) for l in range(1, L)]) if L > 1 \
        else np.zeros(0)
    np.testing.assert_allclose(sums, exact * scale[None, None, :, None],
                               rtol=8 * u + depth * 2.0 ** -23, atol=1e-5 * np.abs(x).max() * N)


def test_stored_pyramid_follows_the_fixed_order():
    """Children are added left to right in fp32: 2^24 + 1 + 1 + 1 stays 2^24 (ties to even)."""
    geo = O.Geometry(4, 4, 2, 1)
    x = np.array([2.0 ** 24, 1.0, 1.0, 1.0], np.float32).reshape(1, 1, 4, 1)
    assert O.pool_stored(x, geo, "f32", mean=False)[0, 0, 0, 0] == 2.0 ** 24
    assert O.build_pyramid(x, geo)[0, 0, 0, 0] * 4 == 2.0 ** 24 + 3
