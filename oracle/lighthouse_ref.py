"""Plain, slow CPU oracle of the Lighthouse selection layer (test infrastructure only).

This module is the checker, not the product. Only the tests, the smoke check and the CPU
baseline leg of the benchmark may import it. The CUDA library never calls it, and it calls
nothing of the CUDA library.

It computes the layer step by step, in float64 from the exact input values, with every
convention the pages leave open fixed as stated next to the step that takes it. The one
exception is the ranking score, which decides an integer result. It is computed in float32 in
one fixed order (row_norm_f32), so that the GPU path can match it bit for bit.

Sources: *Long Context Pre-Training with Lighthouse Attention* (gist.science summary,
technical summary section 2.A-2.D and section 5), and the Nous Research article on
edge.aivizor.me (the paragraph listing the layer's four stages).

All arrays are numpy, laid out [B, H, rows, d] with d fastest. Library primitives used as
single steps: matmul, exp/log, lexsort, add.at. Nothing here is blocked, fused or reordered
beyond what the definitions state, except that attention processes query rows in blocks to
bound memory. Each row's softmax is still the full definition.

Parity pins: every function here is pinned by a test under tests/test_oracle_*.py against
closed forms, brute force on tiny inputs, library routines on special cases, finite
differences, or invariants. The pages print no worked example, so there is no pin against
printed values.
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import numpy as np


# ---------------------------------------------------------------------------------------
# Shape bookkeeping (the pages' notation: p, L, N_l = N / p^l, budget S)
# ---------------------------------------------------------------------------------------
@dataclass(frozen=True)
class Geometry:
    """Derived sizes of one layer call: R pooled rows, C chunks of T = p^(L-1) tokens, M
    candidates per chunk; strata of G chunks, m = S G / C rows and k = m - G picks per stratum.

    The strata are the fewest consecutive chunks over which the budget S divides evenly:
    G = C / gcd(S, C). When S is a multiple of C (every configuration but the pages' p = 2,
    L = 3, k = 1536 ablation), G = 1 and a stratum is one chunk."""

    N: int
    p: int
    L: int
    S: int

    @property
    def n_level(self):  # N_l = N / p^l, l = 0..L-1
        return [self.N // self.p ** l for l in range(self.L)]

    @property
    def offsets(self):  # row-id offset of each level in the concatenated pyramid
        offs, acc = [0], self.N
        for l in range(1, self.L):
            offs.append(acc)
            acc += self.n_level[l]
        return offs

    @property
    def R(self):
        return sum(self.n_level[1:])

    @property
    def C(self):
        return self.n_level[-1]

    @property
    def T(self):
        return self.p ** (self.L - 1)

    @property
    def G(self):
        return self.C // math.gcd(self.S, self.C)

    @property
    def m(self):
        return self.S * self.G // self.C

    @property
    def k(self):
        return self.m - self.G

    @property
    def M(self):
        return sum(self.p ** (self.L - 1 - l) for l in range(self.L - 1))

    def check(self):
        if self.p < 2 or self.L < 1 or self.N < 1:
            raise ValueError("need p >= 2, L >= 1, N >= 1")
        if self.N % self.T:
            raise ValueError("N must be a multiple of p^(L-1)")
        if not (self.C <= self.S <= self.C * (self.M + 1)):
            raise ValueError("S must lie between C (the coarsest cells) and C (M + 1) (every cell)")
        return self

    def decode(self, rid):
        """Row id -> (level, cell index); vectorised over an int array."""
        rid = np.asarray(rid, dtype=np.int64)
        level = np.zeros_like(rid)
        cell = rid.copy()
        for l in range(1, self.L):
            sel = rid >= self.offsets[l]
            level[sel] = l
            cell[sel] = rid[sel] - self.offsets[l]
        return level, cell


# ---------------------------------------------------------------------------------------
# 1. Pyramid: each level is the mean of p consecutive entries of the level below
#    (Lighthouse summary, section 2.A; Nous Research article, four-stage paragraph).
# ---------------------------------------------------------------------------------------
def build_pyramid(x, geo: Geometry):
    """x: [B,H,N,d] -> pooled levels 1..L-1 concatenated, [B,H,R,d] float64."""
    B, H, N, d = x.shape
    level = np.asarray(x, dtype=np.float64)
    out = []
    for _ in range(1, geo.L):
        level = level.reshape(B, H, -1, geo.p, d).mean(axis=3)
        out.append(level)
    if not out:
        return np.zeros((B, H, 0, d))
    return np.concatenate(out, axis=2)


# ---------------------------------------------------------------------------------------
# 2. Scores: l2 norms of Q and K per head, max-pooled upward, summed (Lighthouse summary,
#    section 2.B; the article's "two scalar scores per cell").
# ---------------------------------------------------------------------------------------
def row_norm_f32(x, g):
    """fp32 l2 norm of each row of x[..., d] in one fixed order.

    Groups of g consecutive coordinates are summed in ascending order, each square rounded
    on its own; the group sums are then combined by a halving tree; then a rounded sqrt.
    """
    x = np.asarray(x, dtype=np.float32)
    d = x.shape[-1]
    G = d // g
    xg = x.reshape(*x.shape[:-1], G, g)
    acc = np.zeros(xg.shape[:-1], dtype=np.float32)
    for e in range(g):
        sq = xg[..., e] * xg[..., e]  # float32 product, rounded
        acc = acc + sq  # float32 sum, rounded
    while acc.shape[-1] > 1:
        s = acc.shape[-1] // 2
        acc = acc[..., :s] + acc[..., s:2 * s]
    return np.sqrt(acc[..., 0])


def kv_head_of(H, Hkv):
    """Grouped-query heads (a reading; the pages state none): with H query heads and Hkv
    key/value heads, H = g Hkv, query head h uses key/value head h // g, so g consecutive query
    heads share one. Hkv = H is the plain layer."""
    if Hkv < 1 or H % Hkv:
        raise ValueError("the query heads must split evenly over the key/value heads")
    return np.arange(H) // (H // Hkv)


def score(q, k, geo: Geometry, g):
    """Rank score r for every row id: float32 [B,H,N+R]. k may have fewer heads than q
    (grouped-query heads): query head h then scores with the norms of key head kv_head_of(h)."""
    B, H, N, _ = q.shape
    Hk = k.shape[1]
    sq, sk = row_norm_f32(q, g), row_norm_f32(k, g)
    levels_q, levels_k = [sq], [sk]
    for _ in range(1, geo.L):
        sq = sq.reshape(B, H, -1, geo.p).max(axis=3)
        sk = sk.reshape(B, Hk, -1, geo.p).max(axis=3)
        levels_q.append(sq)
        levels_k.append(sk)
    hmap = kv_head_of(H, Hk)
    r = [a + b[:, hmap] for a, b in zip(levels_q, levels_k)]  # float32 sum per cell
    return np.concatenate(r, axis=2).astype(np.float32)


# ---------------------------------------------------------------------------------------
# 3.-4. Stratified top-K and the causal order of the subsequence (Lighthouse summary,
#    sections 2.B-2.C; the article keeps the coarsest level always).
# ---------------------------------------------------------------------------------------
def select_topk(r, geo: Geometry):
    """r: float32 [B,H,N+R] -> idx int32 [B,H,S] (row ids, in subsequence order).

    Per stratum (G consecutive chunks): keep the G coarsest cells, pick the k best of the
    stratum's G M candidates (every cell of levels 0..L-2 inside it) by the total key (r
    descending, level descending, position ascending), and order the m rows by (end, level)."""
    B, H, _ = r.shape
    C, L, p, G, k = geo.C, geo.L, geo.p, geo.G, geo.k
    ns = C // G  # strata
    cand_r, cand_l, cand_j = [], [], []
    for l in range(L - 1):
        per = G * p ** (L - 1 - l)  # cells of level l per stratum
        lev = r[:, :, geo.offsets[l]:geo.offsets[l] + geo.n_level[l]].reshape(B, H, ns, per)
        cand_r.append(lev)
        cand_l.append(np.full(per, l))
        cand_j.append(np.arange(per))  # cell index within the stratum
    if L > 1:
        cr = np.concatenate(cand_r, axis=3)  # [B,H,ns,G*M]
        cl = np.concatenate(cand_l)
        cj = np.concatenate(cand_j)
        # total ranking key: r descending, level descending, position ascending
        order = np.lexsort((np.broadcast_to(cj, cr.shape),
                            np.broadcast_to(-cl, cr.shape),
                            -cr), axis=-1)
        top = order[..., :k]  # [B,H,ns,k] candidate numbers
        sel_l = cl[top]
        stratum = np.arange(ns).reshape(1, 1, ns, 1)
        sel_j = cj[top] + stratum * G * (p ** (L - 1 - sel_l))  # global cell index at its level
    else:
        sel_l = np.zeros((B, H, ns, 0), dtype=np.int64)
        sel_j = np.zeros((B, H, ns, 0), dtype=np.int64)
    # the G coarsest cells of every stratum
    coarse_l = np.full((B, H, ns, G), L - 1)
    coarse_j = np.broadcast_to(np.arange(C).reshape(1, 1, ns, G), (B, H, ns, G))
    all_l = np.concatenate([sel_l, coarse_l], axis=3)
    all_j = np.concatenate([sel_j, coarse_j], axis=3)
    # causal order inside the stratum: ascending (end, level)
    end = (all_j + 1) * (p ** all_l)
    order = np.lexsort((all_l, end), axis=-1)
    all_l = np.take_along_axis(all_l, order, axis=-1)
    all_j = np.take_along_axis(all_j, order, axis=-1)
    offs = np.asarray(geo.offsets)
    rid = offs[all_l] + all_j
    return rid.reshape(B, H, geo.S).astype(np.int32)


def gather(x, px, idx):
    """X_sub[i] = row idx[i] of the concatenated pyramid [x | px] (Lighthouse summary, 2.C)."""
    full = np.concatenate([np.asarray(x, dtype=np.float64), np.asarray(px, dtype=np.float64)],
                          axis=2)
    return np.take_along_axis(full, idx[..., None].astype(np.int64), axis=2)


# ---------------------------------------------------------------------------------------
# 5. Dense causal attention on the subsequence (Lighthouse summary, 2.C).
# ---------------------------------------------------------------------------------------
_ROW_BLOCK = 2048


def attn_fwd(qs, ks, vs):
    """Causal softmax attention over the S subsequence rows, scale 1/sqrt(d).

    Returns (O_sub [B,H,S,d] float64, lse [B,H,S] float64).
    """
    B, H, S, d = qs.shape
    sigma = 1.0 / np.sqrt(d)
    o = np.zeros((B, H, S, d))
    lse = np.zeros((B, H, S))
    for b in range(B):
        for h in range(H):
            for i0 in range(0, S, _ROW_BLOCK):
                i1 = min(S, i0 + _ROW_BLOCK)
                s = (qs[b, h, i0:i1] @ ks[b, h, :i1].T) * sigma
                visible = np.arange(i1)[None, :] <= np.arange(i0, i1)[:, None]
                s = np.where(visible, s, -np.inf)
                mx = s.max(axis=1, keepdims=True)
                e = np.exp(s - mx)
                z = e.sum(axis=1, keepdims=True)
                o[b, h, i0:i1] = (e / z) @ vs[b, h, :i1]
                lse[b, h, i0:i1] = (mx + np.log(z))[:, 0]
    return o, lse


def attn_bwd(qs, ks, vs, os_, lse, dos):
    """Gradients of attn_fwd w.r.t. Q_sub, K_sub, V_sub (Lighthouse summary, 2.B)."""
    B, H, S, d = qs.shape
    sigma = 1.0 / np.sqrt(d)
    dq, dk, dv = np.zeros_like(qs), np.zeros_like(ks), np.zeros_like(vs)
    for b in range(B):
        for h in range(H):
            D = (dos[b, h] * os_[b, h]).sum(axis=1)
            for i0 in range(0, S, _ROW_BLOCK):
                i1 = min(S, i0 + _ROW_BLOCK)
                s = (qs[b, h, i0:i1] @ ks[b, h, :i1].T) * sigma
                visible = np.arange(i1)[None, :] <= np.arange(i0, i1)[:, None]
                P = np.exp(np.where(visible, s - lse[b, h, i0:i1, None], -np.inf))
                dP = dos[b, h, i0:i1] @ vs[b, h, :i1].T
                dS = P * (dP - D[i0:i1, None])
                dv[b, h, :i1] += P.T @ dos[b, h, i0:i1]
                dq[b, h, i0:i1] = sigma * (dS @ ks[b, h, :i1])
                dk[b, h, :i1] += sigma * (dS.T @ qs[b, h, i0:i1])
    return dq, dk, dv


# ---------------------------------------------------------------------------------------
# 6. Scatter-back: every output row is added to each token of its span (Lighthouse
#    summary, 2.C).
# ---------------------------------------------------------------------------------------
def scatter(idx, os_, geo: Geometry):
    """O[t] = sum of O_sub[i] over subsequence rows whose span covers t."""
    B, H, S, d = os_.shape
    out = np.zeros((B, H, geo.N, d))
    level, cell = geo.decode(idx)
    bb, hh = np.meshgrid(np.arange(B), np.arange(H), indexing="ij")
    for l in range(geo.L):
        w = geo.p ** l
        acc = np.zeros((B, H, geo.n_level[l], d))
        sel = level == l  # rows of this level; add.at visits them in ascending (b, h, i)
        np.add.at(acc, (bb[..., None].repeat(S, 2)[sel], hh[..., None].repeat(S, 2)[sel],
                        cell[sel]), os_[sel])
        out += np.repeat(acc, w, axis=2)
    return out


# ---------------------------------------------------------------------------------------
# 7. Backward through scatter and gather/pooling (Lighthouse summary, 2.B).
# ---------------------------------------------------------------------------------------
def scatter_bwd(idx, d_o, geo: Geometry):
    """dO_sub[i] = sum of dO over the tokens of span(i)."""
    B, H, N, d = d_o.shape
    d_o = np.asarray(d_o, dtype=np.float64)
    sums = [d_o]
    for l in range(1, geo.L):
        sums.append(d_o.reshape(B, H, geo.n_level[l], geo.p ** l, d).sum(axis=3))
    full = np.concatenate(sums, axis=2)
    return np.take_along_axis(full, idx[..., None].astype(np.int64), axis=2)


def gather_bwd(idx, dx_sub, geo: Geometry):
    """dX[t] = sum over rows i whose span covers t of dX_sub[i] / p^level(i)."""
    B, H, S, d = dx_sub.shape
    out = np.zeros((B, H, geo.N, d))
    level, cell = geo.decode(idx)
    bb, hh = np.meshgrid(np.arange(B), np.arange(H), indexing="ij")
    for l in range(geo.L):
        w = geo.p ** l
        acc = np.zeros((B, H, geo.n_level[l], d))
        sel = level == l
        np.add.at(acc, (bb[..., None].repeat(S, 2)[sel], hh[..., None].repeat(S, 2)[sel],
                        cell[sel]), dx_sub[sel] / w)
        out += np.repeat(acc, w, axis=2)
    return out


# ---------------------------------------------------------------------------------------
# Storage rounding: the layer stores the pyramid and dO_sub in its dtype (O_sub stays fp32). Round to nearest, ties to even, from the exact value.
# ---------------------------------------------------------------------------------------
def round_to(x, store):
    """Exact value -> nearest value of the storage type ("bf16", "f32" or None = keep)."""
    x = np.asarray(x, dtype=np.float64)
    if store is None:
        return x
    if store == "f32":
        return x.astype(np.float32).astype(np.float64)
    if store == "bf16":  # 8 significant bits: scale the frexp mantissa to [128, 256), round
        m, e = np.frexp(x)
        return np.ldexp(np.rint(m * 256.0) / 256.0, e)
    raise ValueError(store)


def pool_stored(x, geo: Geometry, store, mean=True):
    """The stored pooled levels 1..L-1 of x, [B,H,R,d], as the layer rounds them.

    Rounding a pooled value to the storage type is a quantisation, so it is decided on the same
    fp32 value that the layer rounds: each level adds its p children's unrounded fp32 sums from
    left to right, in fp32; the cell is fl32(sum * fl32(1/p^l)) (mean=True) or the sum itself
    (mean=False, the span sums of the backward), then rounded once to `store`.
    """
    B, H, N, d = x.shape
    sums = np.asarray(x, dtype=np.float32)
    out = []
    for l in range(1, geo.L):
        ch = sums.reshape(B, H, -1, geo.p, d)
        acc = ch[:, :, :, 0, :]
        for c in range(1, geo.p):
            acc = acc + ch[:, :, :, c, :]  # float32, left to right
        sums = acc
        val = acc * (np.float32(1.0) / np.float32(geo.p ** l)) if mean else acc
        out.append(round_to(val.astype(np.float64), store))
    if not out:
        return np.zeros((B, H, 0, d))
    return np.concatenate(out, axis=2)


# ---------------------------------------------------------------------------------------
# Whole layer
# ---------------------------------------------------------------------------------------
def layer_fwd(q, k, v, geo: Geometry, g, idx=None, store=None):
    """Forward of the layer. g is the score group size (8 for bf16 inputs, 4 for fp32).

    idx may be given to force a selection (used for the dense recovery identity). store names
    the storage type of the stored intermediates: the pooled cells (and, in layer_bwd, the
    span sums dO_sub) are then the fp32 children sums of pool_stored rounded to it.
    k and v may have fewer heads than q (kv_head_of): each tensor is pooled over its own heads,
    every query head selects its own cells, and its subsequence takes the key and value rows
    of its key/value head.
    Returns (O [B,H,N,d] float64, saved dict for layer_bwd).
    """
    geo.check()
    if store is None:
        pq, pk, pv = (build_pyramid(x, geo) for x in (q, k, v))
    else:
        pq, pk, pv = (pool_stored(x, geo, store) for x in (q, k, v))
    r = None
    if idx is None:
        r = score(q, k, geo, g)
        idx = select_topk(r, geo)
    hmap = kv_head_of(q.shape[1], k.shape[1])
    qs = gather(q, pq, idx)
    ks, vs = gather(k[:, hmap], pk[:, hmap], idx), gather(v[:, hmap], pv[:, hmap], idx)
    os_, lse = attn_fwd(qs, ks, vs)  # O_sub is kept in fp32 by the layer: no storage rounding
    o = scatter(idx, os_, geo)
    saved = dict(idx=idx, score=r, qs=qs, ks=ks, vs=vs, os=os_, lse=lse, geo=geo, store=store,
                 kv_heads=k.shape[1])
    return o, saved


def layer_bwd(saved, d_o):
    """Backward of the layer: returns (dQ [B,H,N,d], dK, dV [B,Hkv,N,d]) float64. A key/value
    head's gradients are the sums of those reaching it from each of its query heads."""
    geo, idx, store = saved["geo"], saved["idx"], saved.get("store")
    if store is None:
        dos = scatter_bwd(idx, d_o, geo)
    else:  # the stored span sums: fp32 children sums in the pyramid's order, then rounded
        full = np.concatenate([np.asarray(d_o, np.float64),
                               pool_stored(d_o, geo, store, mean=False)], axis=2)
        dos = np.take_along_axis(full, idx[..., None].astype(np.int64), axis=2)
    dqs, dks, dvs = attn_bwd(saved["qs"], saved["ks"], saved["vs"], saved["os"], saved["lse"], dos)
    dq, dk, dv = gather_bwd(idx, dqs, geo), gather_bwd(idx, dks, geo), gather_bwd(idx, dvs, geo)
    B, H, N, d = dq.shape
    Hkv = saved.get("kv_heads", H)
    kv_head_of(H, Hkv)  # the same validation as the forward
    dk = dk.reshape(B, Hkv, H // Hkv, N, d).sum(axis=2)  # query heads j g .. j g + g - 1
    dv = dv.reshape(B, Hkv, H // Hkv, N, d).sum(axis=2)
    return dq, dk, dv
