"""Whole-layer parity of the CUDA path (lh_layer_fwd / lh_layer_bwd) with the CPU oracle.

Small shapes keep every parameter of the five workloads (p, L, m = S/C, d, dtype, row-scale
recipe) at sizes the oracle runs whole. The full-size workloads run on the GPU exactly as the
benchmark launches them; the oracle then checks sampled heads.
"""
import numpy as np
import pytest
import torch

import oracle as O

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import sparse_hierarchical_attention_b200 as lh
    from sparse_hierarchical_attention_b200 import LighthouseAttention, LighthouseLayer, Shape, saved_views
    from workloads import WORKLOADS, make_inputs

from gpu_util import assert_close, g_of, np64, store_of


def run_layer(shape, q, k, v, d_o):
    layer = LighthouseLayer(shape)
    o, saved = layer.forward(q, k, v)
    dq, dk, dv = layer.backward(saved, d_o)
    layer.check()
    return o, saved, (dq, dk, dv)


def oracle_layer(q, k, v, d_o, geo, dtype):
    """The oracle on the same inputs; stored intermediates rounded to the layer dtype."""
    o, sv = O.layer_fwd(np64(q), np64(k), np64(v), geo, g_of(dtype), store=store_of(dtype))
    return o, sv, O.layer_bwd(sv, np64(d_o))


# (workload recipe, B, H, N, S): same p, L, d, dtype and m = S/C as the named workload
SMALL = [
    ("tiny-2k-fp32", 1, 4, 2048, 512),
    ("32k", 1, 2, 4096, 16 * 32),
    ("llama530m-98k", 1, 2, 8192, 8 * 64),
    ("128k", 1, 2, 8192, 8 * 64),
    ("1m", 1, 1, 16384, 4 * 64),
]


@pytest.mark.parametrize("name,B,H,N,S", SMALL)
def test_layer_matches_oracle(name, B, H, N, S):
    w = WORKLOADS[name]
    shape = Shape(B, H, N, w.d, w.p, w.L, S, w.dtype)
    q, k, v, d_o = make_inputs(w, "cuda", seed=0, B=B, H=H, N=N)
    o, saved, grads = run_layer(shape, q, k, v, d_o)
    geo = O.Geometry(N, w.p, w.L, S).check()
    wo, sv, wgrads = oracle_layer(q, k, v, d_o, geo, w.dtype)
    idx = saved_views(shape, saved)["idx"].cpu().numpy()
    assert np.array_equal(idx, sv["idx"]), "selection differs from the oracle"
    assert_close(np64(o), wo, w.dtype, "O")
    for got, want, n in zip(grads, wgrads, ("dQ", "dK", "dV")):
        assert_close(np64(got), want, w.dtype, n)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("name,B,H,N,S", SMALL[:3])
def test_unit_variance_literal_thresholds(name, B, H, N, S, dtype):
    """The same shapes without row scales, checked against the literal thresholds."""
    w = WORKLOADS[name]
    shape = Shape(B, H, N, w.d, w.p, w.L, S, dtype)
    q, k, v, d_o = (t.to(dtype) for t in make_inputs(w, "cuda", seed=1, B=B, H=H, N=N, unit=True))
    o, saved, grads = run_layer(shape, q, k, v, d_o)
    geo = O.Geometry(N, w.p, w.L, S).check()
    wo, sv, wgrads = oracle_layer(q, k, v, d_o, geo, dtype)
    assert np.array_equal(saved_views(shape, saved)["idx"].cpu().numpy(), sv["idx"])
    assert_close(np64(o), wo, dtype, "O", mode="literal")
    for got, want, n in zip(grads, wgrads, ("dQ", "dK", "dV")):
        assert_close(np64(got), want, dtype, n, mode="scaled")


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("B,H,N,d,p,L,S", [
    (1, 2, 333, 64, 4, 1, 333),         # L = 1: dense causal SDPA, ragged tile tail
    (2, 2, 1024, 128, 4, 4, 16 * 85),   # m = M + 1: everything selected
    (1, 2, 4096, 128, 4, 6, 4),         # m = 1: only the coarsest cells
    (1, 2, 2048, 64, 2, 8, 128),        # p = 2
    (1, 2, 4096, 128, 2, 3, 1024 * 3),  # p = 2, L = 3 (the pages' best ablation): 4-token chunks, M = 6
    (1, 1, 2187, 128, 3, 4, 81 * 4),    # p = 3
    (1, 1, 1280, 64, 4, 4, 20 * 7),     # C = 20, S = 140: ragged attention tiles
    (1, 1, 2048, 64, 16, 3, 8 * 17),    # p = 16, the largest pooling factor
    (1, 1, 4096, 64, 2, 12, 2 * 64),    # L = 12, the most levels: five tree levels and a coarse pass
    (1, 1, 32768, 128, 4, 8, 2 * 64),   # M = 21844 candidates per chunk, near the shared-memory limit
    (1, 2, 4096, 64, 2, 3, 1024 + 64),  # strata of G = 16 chunks (p = 2, L = 3, one pick per stratum)
    (1, 2, 4096, 128, 4, 3, 256 + 96),  # G = 8, S = 352 (ragged attention tiles)
    (1, 1, 729, 64, 3, 4, 28),          # one stratum over the whole sequence
])
def test_layer_edge_cases(B, H, N, d, p, L, S, dtype):
    shape = Shape(B, H, N, d, p, L, S, dtype)
    g = torch.Generator(device="cuda").manual_seed(N + S)
    q, k, v, d_o = (torch.randn(B, H, N, d, generator=g, device="cuda").to(dtype) for _ in range(4))
    o, saved, grads = run_layer(shape, q, k, v, d_o)
    geo = O.Geometry(N, p, L, S).check()
    wo, sv, wgrads = oracle_layer(q, k, v, d_o, geo, dtype)
    assert np.array_equal(saved_views(shape, saved)["idx"].cpu().numpy(), sv["idx"])
    assert_close(np64(o), wo, dtype, "O")
    for got, want, n in zip(grads, wgrads, ("dQ", "dK", "dV")):
        assert_close(np64(got), want, dtype, n)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_dense_recovery_matches_torch_sdpa(dtype):
    """L = 1 is plain causal SDPA (the recovery phase); compare with torch on the GPU in fp32."""
    B, H, N, d = 1, 4, 1024, 128
    shape = Shape(B, H, N, d, 4, 1, N, dtype)
    g = torch.Generator(device="cuda").manual_seed(5)
    q, k, v, d_o = (torch.randn(B, H, N, d, generator=g, device="cuda").to(dtype) for _ in range(4))
    o, _, (dq, dk, dv) = run_layer(shape, q, k, v, d_o)
    tq, tk, tv = (x.float().requires_grad_() for x in (q, k, v))
    with torch.backends.cuda.sdp_kernel(enable_flash=False, enable_mem_efficient=False, enable_math=True):
        ref = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, is_causal=True)
    ref.backward(d_o.float())
    assert_close(np64(o), np64(ref), dtype, "O", mode="literal")
    for got, t, n in ((dq, tq, "dQ"), (dk, tk, "dK"), (dv, tv, "dV")):
        assert_close(np64(got), np64(t.grad), dtype, n)


@pytest.mark.parametrize("det", [True, False])
def test_deterministic_bits(det):
    """With LH_DETERMINISTIC every output is bit-identical run to run. Without it only dQ may
    differ, by the rounding of its atomic fp32 sums: at most one bf16 unit in the last place."""
    w = WORKLOADS["128k"]
    shape = Shape(1, 2, 8192, w.d, w.p, w.L, 512, w.dtype, det)
    q, k, v, d_o = make_inputs(w, "cuda", B=1, H=2, N=8192)
    a = run_layer(shape, q, k, v, d_o)
    b = run_layer(shape, q, k, v, d_o)
    assert torch.equal(a[0], b[0])
    assert torch.equal(a[2][1], b[2][1]) and torch.equal(a[2][2], b[2][2])
    if det:
        assert torch.equal(a[2][0], b[2][0])
    else:
        x, y = a[2][0].float(), b[2][0].float()
        assert ((x - y).abs() <= 2.0 ** -7 * torch.maximum(x.abs(), y.abs())).all()


def test_layer_replays_as_one_cuda_graph():
    """The layer allocates nothing and never synchronises, so a whole forward + backward step
    captures into one CUDA graph; replays with new inputs give the eager results bit for bit
    (in deterministic mode, so that bit equality is defined)."""
    w = WORKLOADS["128k"]
    shape = Shape(1, 2, 8192, w.d, w.p, w.L, 512, w.dtype, deterministic=True)
    layer = LighthouseLayer(shape)
    saved = layer.new_saved()
    ins = [torch.empty(1, 2, 8192, w.d, dtype=w.dtype, device="cuda") for _ in range(4)]
    outs = [torch.empty_like(ins[0]) for _ in range(4)]

    def step():
        layer.forward(ins[0], ins[1], ins[2], o=outs[0], saved=saved)
        layer.backward(saved, ins[3], dq=outs[1], dk=outs[2], dv=outs[3])

    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        step()  # warm the launch paths outside the capture
    torch.cuda.current_stream().wait_stream(side)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        step()
    for seed in (3, 4):
        for dst, src in zip(ins, make_inputs(w, "cuda", seed=seed, B=1, H=2, N=8192)):
            dst.copy_(src)
        g.replay()
        got = [t.clone() for t in outs]
        want = run_layer(shape, *ins)
        assert torch.equal(got[0], want[0])
        for x, y in zip(got[1:], want[2]):
            assert torch.equal(x, y)
    layer.check()


def test_future_chunks_do_not_change_the_past():
    w = WORKLOADS["llama530m-98k"]
    N, S = 8192, 8 * 64
    shape = Shape(1, 2, N, w.d, w.p, w.L, S, w.dtype)
    q, k, v, d_o = make_inputs(w, "cuda", B=1, H=2, N=N)
    o1 = run_layer(shape, q, k, v, d_o)[0]
    T = w.p ** (w.L - 1)
    for c in (1, 5):
        q2, k2, v2 = q.clone(), k.clone(), v.clone()
        for x in (q2, k2, v2):
            x[:, :, c * T:] = (3 * torch.randn_like(x[:, :, c * T:].float())).to(x.dtype)
        o2 = run_layer(shape, q2, k2, v2, d_o)[0]
        assert torch.equal(o1[:, :, :c * T], o2[:, :, :c * T])
        assert not torch.equal(o1[:, :, c * T:], o2[:, :, c * T:])


@pytest.mark.parametrize("unit", [False, True])
@pytest.mark.parametrize("name", ["32k", "llama530m-98k", "128k", "1m"])
def test_full_size_sampled_heads(name, unit):
    """Full-size workload in the benchmark's launch; the oracle checks the last head whole.

    unit=True drops the row scales, so the unit-variance acceptance limits apply literally.
    """
    w = WORKLOADS[name]
    shape = Shape(w.B, w.H, w.N, w.d, w.p, w.L, w.S, w.dtype)
    q, k, v, d_o = make_inputs(w, "cuda", seed=0, unit=unit)
    o, saved, grads = run_layer(shape, q, k, v, d_o)
    idx = saved_views(shape, saved)["idx"]
    geo = O.Geometry(w.N, w.p, w.L, w.S).check()
    for h in (0, w.H - 1):  # selection of two heads, bit-exact
        sl = (slice(0, 1), slice(h, h + 1))
        r = O.score(np64(q[sl]), np64(k[sl]), geo, g_of(w.dtype))
        assert np.array_equal(idx[sl].cpu().numpy(), O.select_topk(r, geo)), f"head {h}"
    h = w.H - 1
    sl = (slice(0, 1), slice(h, h + 1))
    wo, sv, wgrads = oracle_layer(q[sl], k[sl], v[sl], d_o[sl], geo, w.dtype)
    assert_close(np64(o[sl]), wo, w.dtype, "O", mode="literal" if unit else "scaled")
    for got, want, n in zip(grads, wgrads, ("dQ", "dK", "dV")):
        assert_close(np64(got[sl]), want, w.dtype, n)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_autograd_module_matches_layer_calls(dtype):
    """LighthouseAttention (nn.Module over a torch.autograd.Function) returns the O, dQ, dK and dV
    of explicit LighthouseLayer forward/backward calls on the same inputs, bit for bit: the same
    kernels run, and in deterministic mode the layer is bit-reproducible."""
    name, B, H, N, S = SMALL[1] if dtype == torch.bfloat16 else SMALL[0]
    w = WORKLOADS[name]
    shape = Shape(B, H, N, w.d, w.p, w.L, S, dtype, deterministic=True)
    q, k, v, d_o = (t.to(dtype) for t in make_inputs(w, "cuda", seed=3, B=B, H=H, N=N))
    o_ref, _, (dq_ref, dk_ref, dv_ref) = run_layer(shape, q, k, v, d_o)
    attn = LighthouseAttention(w.p, w.L, S, deterministic=True)
    qq, kk, vv = (x.clone().requires_grad_() for x in (q, k, v))
    o = attn(qq, kk, vv)
    o.backward(d_o)
    assert o.dtype == dtype and o.shape == q.shape
    assert torch.equal(o.detach(), o_ref)
    assert torch.equal(qq.grad, dq_ref)
    assert torch.equal(kk.grad, dk_ref)
    assert torch.equal(vv.grad, dv_ref)


@pytest.mark.parametrize("det", [False, True])
def test_pages_ablation_p2_L3_k1536(det):
    """The pages' best ablation (Lighthouse summary, technical summary 4, hyper-parameter bullet):
    p = 2, L = 3 and a top-K budget of k = 1536, at the 98K context of the 530M model (d = 64).
    The 24576 coarsest cells are all kept, so S = 24576 + 1536 = 26112 rows; the budget divides
    evenly over strata of 16 chunks (64 tokens), one pick each. One head is checked whole."""
    w = WORKLOADS["llama530m-98k"]
    N, p, L = 98304, 2, 3
    C = N // p ** (L - 1)
    S = C + 1536
    shape = Shape(1, 2, N, w.d, p, L, S, w.dtype, det)
    sz = lh.lh_validate(shape)
    assert (sz["C"], sz["G"], sz["m"], sz["k"]) == (24576, 16, 17, 1)
    q, k, v, d_o = make_inputs(w, "cuda", seed=0, B=1, H=2, N=N)
    o, saved, grads = run_layer(shape, q, k, v, d_o)
    geo = O.Geometry(N, p, L, S).check()
    sl = (slice(0, 1), slice(1, 2))
    wo, sv, wgrads = oracle_layer(q[sl], k[sl], v[sl], d_o[sl], geo, w.dtype)
    assert np.array_equal(saved_views(shape, saved)["idx"][sl].cpu().numpy(), sv["idx"])
    assert_close(np64(o[sl]), wo, w.dtype, "O")
    for got, want, n in zip(grads, wgrads, ("dQ", "dK", "dV")):
        assert_close(np64(got[sl]), want, w.dtype, n)
