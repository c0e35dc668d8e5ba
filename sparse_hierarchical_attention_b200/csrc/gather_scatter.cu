// Gather of the selected triples and the deterministic scatter-back ("Long Context Pre-Training
// with Lighthouse Attention", technical summary 2.C), and the backward of the gather through
// the pooling (technical summary 2.B: gradients reach Q, K, V through the gather).
//
// gather: one 16-byte lane per column slice, rows independent, a pure copy. With grouped heads
//   the K and V rows of query head h come from its key/value head h / grp.
// spread: one CTA per (b,h, chunk). The chunk's m row ids become a shared-memory map
//   (level, cell in chunk) -> subsequence row. Each token then adds the rows that cover it,
//   one per level at most, from the coarsest level down, sharing the partial sums of the
//   coarse levels among the tokens below them. fp32 accumulation, one
//   rounding, no atomics.
#include "common.cuh"

namespace lh {
namespace {

constexpr int kThreads = 256;

template <typename E, int D>
__global__ void __launch_bounds__(kThreads)
gather_kernel(const E* __restrict__ q, const E* __restrict__ k, const E* __restrict__ v,
              const E* __restrict__ pq, const E* __restrict__ pk, const E* __restrict__ pv,
              const int32_t* __restrict__ idx, E* qs, E* ks, E* vs, int64_t BH, int64_t N,
              int64_t R, int64_t S, int H, int grp, uint32_t* status) {
  constexpr int VEC = 16 / sizeof(E), LPR = D / VEC, RPC = kThreads / LPR;
  const int col = threadIdx.x % LPR;
  const int64_t row = (int64_t)blockIdx.x * RPC + threadIdx.x / LPR;  // over BH*S
  if (row >= BH * S) return;
  const int64_t bh = row / S;
  const int64_t bk = (bh / H) * (H / grp) + (bh % H) / grp;  // its key/value head
  const int64_t rid = idx[row];
  const E* src[3];
  E* dst[3] = {qs, ks, vs};
  bool ok = rid >= 0 && rid < N + R;
  if (!ok) {
    if (col == 0) raise_fault(status, kFaultIndex);
  } else if (rid < N) {
    src[0] = q + (bh * N + rid) * D; src[1] = k + (bk * N + rid) * D; src[2] = v + (bk * N + rid) * D;
  } else {
    src[0] = pq + (bh * R + (rid - N)) * D;
    src[1] = pk + (bk * R + (rid - N)) * D; src[2] = pv + (bk * R + (rid - N)) * D;
  }
#pragma unroll
  for (int xi = 0; xi < 3; ++xi) {
    const uint4 u = ok ? ldg16(src[xi] + col * VEC) : make_uint4(0, 0, 0, 0);
    stg16(dst[xi] + row * D + col * VEC, u);
  }
}

struct SpreadArgs {
  const void* src[3];
  void* dst[3];
  const int32_t* idx;
  uint32_t* status;
  int64_t N, R, S, T, m, G;  // m rows per stratum of G chunks
  int H, Hkv, grp;           // heads (grouped-head spread)
  int64_t off[16];
  float inv[16];  // per-level weight: 1 (scatter) or fl32(1/p^l) (gather backward)
  int p, L, ntensor;
};

template <typename E, typename SRC, int D>
__device__ inline void load_row(const SRC* src, int r, int col, float* x) {
  constexpr int VEC = 16 / sizeof(E);
  if constexpr (sizeof(SRC) == sizeof(E)) {
    Vec<E>::unpack(ldg16(src + (int64_t)r * D + col * VEC), x);
  } else {  // fp32 source: VEC elements = VEC/4 16-byte loads
#pragma unroll
    for (int h = 0; h < VEC / 4; ++h) Vec<float>::unpack(ldg16(src + (int64_t)r * D + col * VEC + 4 * h), x + 4 * h);
  }
}

// One CTA per (b,h, chunk). It maps the rows of its stratum (the m rows s*m .. s*m+m-1 of the
// chunk's stratum s) whose cells lie in this chunk; a row outside the stratum's cells raises the
// index fault. Covering cells are nested, so each token's sum is formed top-down:
// a stream of LPR lanes takes a group of p^A tokens (A = 2 when L >= 3), adds the rows of levels
// L-1..A that cover the whole group once, then the level-1 row once per p tokens, then the
// token's own level-0 row (the coarsest covering row first).
template <typename E, typename SRC, int D>
__global__ void __launch_bounds__(kThreads) spread_kernel(const SpreadArgs a) {
  constexpr int VEC = 16 / sizeof(E), LPR = D / VEC, STREAMS = kThreads / LPR;
  extern __shared__ int cmap[];  // (level, cell in chunk) -> subsequence row of this (b,h)
  const int tid = threadIdx.x, col = tid % LPR, stream = tid / LPR;
  const int64_t bh = blockIdx.y, c = blockIdx.x;
  const int L = a.L, p = a.p;

  int base[16], per[16];
  int tot = 0;
  {
    int cells = 1;
    for (int l = L - 1; l >= 0; --l) { per[l] = cells; cells *= p; }
    for (int l = 0; l < L; ++l) { base[l] = tot; tot += per[l]; }
  }
  for (int i = tid; i < tot; i += kThreads) cmap[i] = -1;
  __syncthreads();
  const int64_t st = c / a.G;  // this chunk's stratum
  for (int64_t i = st * a.m + tid; i < (st + 1) * a.m; i += kThreads) {
    const int64_t rid = a.idx[bh * a.S + i];
    int lvl = 0;
    if (rid < 0 || rid >= a.N + a.R) { raise_fault(a.status, kFaultIndex); continue; }
    for (int l = 1; l < L; ++l)
      if (rid >= a.off[l]) lvl = l;
    const int64_t in_stratum = rid - a.off[lvl] - st * a.G * per[lvl];
    if (in_stratum < 0 || in_stratum >= a.G * per[lvl]) { raise_fault(a.status, kFaultIndex); continue; }
    const int64_t local = rid - a.off[lvl] - c * per[lvl];
    if (local < 0 || local >= per[lvl]) continue;  // a cell of another chunk of the stratum
    cmap[base[lvl] + (int)local] = (int)i;
  }
  __syncthreads();

  const int A = L >= 3 ? 2 : L - 1;  // levels handled inside a group
  const int G = A == 2 ? p * p : (A == 1 ? p : 1);
  const int ngroups = (int)(a.T / G);
  for (int xi = 0; xi < a.ntensor; ++xi) {
    const SRC* src = static_cast<const SRC*>(a.src[xi]) + bh * a.S * D;
    E* dst = static_cast<E*>(a.dst[xi]) + (bh * a.N + c * a.T) * D + col * VEC;
    for (int g = stream; g < ngroups; g += STREAMS) {
      float coarse[VEC];
#pragma unroll
      for (int e = 0; e < VEC; ++e) coarse[e] = 0.f;
      // levels L-1 .. A cover the whole group: cell of level l = g / p^(l-A)
      int cells[16];
      cells[A] = g;
      for (int l = A + 1; l < L; ++l) cells[l] = cells[l - 1] / p;
      for (int l = L - 1; l >= A; --l) {
        const int r = cmap[base[l] + cells[l]];
        if (r >= 0) {
          float x[VEC];
          load_row<E, SRC, D>(src, r, col, x);
          const float w = a.inv[l];
#pragma unroll
          for (int e = 0; e < VEC; ++e) coarse[e] = __fadd_rn(coarse[e], __fmul_rn(x[e], w));
        }
      }
      const int n1 = A >= 1 ? p : 1;          // level-1 cells in the group (or 1)
      const int n0 = A == 2 ? p : (A == 1 ? p : 1);  // tokens per level-1 cell
      for (int c1 = 0; c1 < (A == 2 ? n1 : 1); ++c1) {
        float part[VEC];
#pragma unroll
        for (int e = 0; e < VEC; ++e) part[e] = coarse[e];
        if (A == 2) {
          const int r = cmap[base[1] + g * p + c1];
          if (r >= 0) {
            float x[VEC];
            load_row<E, SRC, D>(src, r, col, x);
            const float w = a.inv[1];
#pragma unroll
            for (int e = 0; e < VEC; ++e) part[e] = __fadd_rn(part[e], __fmul_rn(x[e], w));
          }
        }
        const int t0 = A == 2 ? (g * p + c1) * p : g * G;
        for (int c0 = 0; c0 < (A == 0 ? 1 : n0); ++c0) {
          const int t = t0 + c0;
          float out[VEC];
#pragma unroll
          for (int e = 0; e < VEC; ++e) out[e] = part[e];
          if (A >= 1) {  // with L = 1 the token is the coarsest level, already in `coarse`
            const int r = cmap[t];
            if (r >= 0) {
              float x[VEC];
              load_row<E, SRC, D>(src, r, col, x);
              const float w = a.inv[0];
#pragma unroll
              for (int e = 0; e < VEC; ++e) out[e] = __fadd_rn(out[e], __fmul_rn(x[e], w));
            }
          }
          stg16_stream(dst + (int64_t)t * D, Vec<E>::pack(out));  // O or dQ/dK/dV: final outputs
        }
      }
    }
  }
}

// Gather backward of K and V with grouped heads. One CTA per (b, key/value head, chunk). It maps
// the chunk's rows for each of the head's grp query heads (as spread_kernel does for one). The
// sums then take spread_kernel's top-down form, with the query heads inside each level: a stream
// takes a group of p^A tokens, adds the level L-1..A rows of every query head (levels in
// descending order, heads ascending within a level) once for the group, the level-1 rows once
// per p tokens, then each token's level-0 rows. With grp = 1 this is spread_kernel's order.
template <typename E, typename SRC, int D>
__global__ void __launch_bounds__(kThreads) spread_group_kernel(const SpreadArgs a) {
  constexpr int VEC = 16 / sizeof(E), LPR = D / VEC, STREAMS = kThreads / LPR;
  extern __shared__ int cmap[];  // [grp][(level, cell in chunk)] -> subsequence row
  const int tid = threadIdx.x, col = tid % LPR, stream = tid / LPR;
  const int64_t bk = blockIdx.y, c = blockIdx.x;  // b Hkv + j, chunk
  const int L = a.L, p = a.p, grp = a.grp;
  const int64_t bh0 = (bk / a.Hkv) * (int64_t)a.H + (bk % a.Hkv) * grp;  // its first query head

  int base[16], per[16];
  int tot = 0;
  {
    int cells = 1;
    for (int l = L - 1; l >= 0; --l) { per[l] = cells; cells *= p; }
    for (int l = 0; l < L; ++l) { base[l] = tot; tot += per[l]; }
  }
  for (int i = tid; i < grp * tot; i += kThreads) cmap[i] = -1;
  __syncthreads();
  const int64_t st = c / a.G;  // this chunk's stratum
  for (int hm = 0; hm < grp; ++hm) {
    for (int64_t i = st * a.m + tid; i < (st + 1) * a.m; i += kThreads) {
      const int64_t rid = a.idx[(bh0 + hm) * a.S + i];
      int lvl = 0;
      if (rid < 0 || rid >= a.N + a.R) { raise_fault(a.status, kFaultIndex); continue; }
      for (int l = 1; l < L; ++l)
        if (rid >= a.off[l]) lvl = l;
      const int64_t in_stratum = rid - a.off[lvl] - st * a.G * per[lvl];
      if (in_stratum < 0 || in_stratum >= a.G * per[lvl]) { raise_fault(a.status, kFaultIndex); continue; }
      const int64_t local = rid - a.off[lvl] - c * per[lvl];
      if (local < 0 || local >= per[lvl]) continue;  // a cell of another chunk of the stratum
      cmap[hm * tot + base[lvl] + (int)local] = (int)i;
    }
  }
  __syncthreads();

  const int A = L >= 3 ? 2 : L - 1;  // levels handled inside a group
  const int G = A == 2 ? p * p : (A == 1 ? p : 1);
  const int ngroups = (int)(a.T / G);
  for (int xi = 0; xi < a.ntensor; ++xi) {
    const SRC* src0 = static_cast<const SRC*>(a.src[xi]) + bh0 * a.S * D;  // head hm at + hm S D
    E* dst = static_cast<E*>(a.dst[xi]) + (bk * a.N + c * a.T) * D + col * VEC;
    // adds the (level l, cell) row of every query head of the group, scaled by 1/p^l
    auto add_level = [&](float (&acc)[VEC], int l, int cell) {
      for (int hm = 0; hm < grp; ++hm) {
        const int r = cmap[hm * tot + base[l] + cell];
        if (r >= 0) {
          float x[VEC];
          load_row<E, SRC, D>(src0 + (int64_t)hm * a.S * D, r, col, x);
          const float w = a.inv[l];
#pragma unroll
          for (int e = 0; e < VEC; ++e) acc[e] = __fadd_rn(acc[e], __fmul_rn(x[e], w));
        }
      }
    };
    for (int g = stream; g < ngroups; g += STREAMS) {
      float coarse[VEC];
#pragma unroll
      for (int e = 0; e < VEC; ++e) coarse[e] = 0.f;
      int cells[16];
      cells[A] = g;
      for (int l = A + 1; l < L; ++l) cells[l] = cells[l - 1] / p;
      for (int l = L - 1; l >= A; --l) add_level(coarse, l, cells[l]);
      const int n0 = A >= 1 ? p : 1;  // tokens per level-1 cell (per token with A = 1)
      for (int c1 = 0; c1 < (A == 2 ? p : 1); ++c1) {
        float part[VEC];
#pragma unroll
        for (int e = 0; e < VEC; ++e) part[e] = coarse[e];
        if (A == 2) add_level(part, 1, g * p + c1);
        const int t0 = A == 2 ? (g * p + c1) * p : g * G;
        for (int c0 = 0; c0 < (A == 0 ? 1 : n0); ++c0) {
          const int t = t0 + c0;
          float out[VEC];
#pragma unroll
          for (int e = 0; e < VEC; ++e) out[e] = part[e];
          if (A >= 1) add_level(out, 0, t);  // with L = 1 the token is the coarsest level, in `coarse`
          stg16_stream(dst + (int64_t)t * D, Vec<E>::pack(out));
        }
      }
    }
  }
}

template <typename E, typename SRC>
cudaError_t run_spread(const Geo& g, const SpreadArgs& a, cudaStream_t st) {
  const size_t smem = (size_t)(g.M + 1) * sizeof(int);
  dim3 grid((unsigned)g.C, (unsigned)g.BH);
  cudaError_t e;
  if (g.d == 64) {
    e = cudaFuncSetAttribute(spread_kernel<E, SRC, 64>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e == cudaSuccess) spread_kernel<E, SRC, 64><<<grid, kThreads, smem, st>>>(a);
  } else {
    e = cudaFuncSetAttribute(spread_kernel<E, SRC, 128>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e == cudaSuccess) spread_kernel<E, SRC, 128><<<grid, kThreads, smem, st>>>(a);
  }
  return e != cudaSuccess ? e : cudaGetLastError();
}

}  // namespace

cudaError_t launch_gather(const Geo& g, const void* q, const void* k, const void* v,
                          const void* pq, const void* pk, const void* pv, const int32_t* idx,
                          void* qs, void* ks, void* vs, uint32_t* status, cudaStream_t st) {
  const int vec = 16 / g.esize, lpr = g.d / vec, rpc = kThreads / lpr;
  const int64_t rows = g.BH * g.S;
  const unsigned grid = (unsigned)((rows + rpc - 1) / rpc);
#define LH_GATHER(E, D)                                                                      \
  gather_kernel<E, D><<<grid, kThreads, 0, st>>>(                                            \
      (const E*)q, (const E*)k, (const E*)v, (const E*)pq, (const E*)pk, (const E*)pv, idx, \
      (E*)qs, (E*)ks, (E*)vs, g.BH, g.N, g.R, g.S, g.H, g.grp, status)
  if (g.dtype == LH_BF16) {
    if (g.d == 64) LH_GATHER(__nv_bfloat16, 64); else LH_GATHER(__nv_bfloat16, 128);
  } else {
    if (g.d == 64) LH_GATHER(float, 64); else LH_GATHER(float, 128);
  }
#undef LH_GATHER
  return cudaGetLastError();
}

cudaError_t launch_spread(const Geo& g, const int32_t* idx, int ntensor, bool src_f32,
                          bool scale_by_level, const void* const* src, void* const* dst,
                          uint32_t* status, cudaStream_t st) {
  SpreadArgs a{};
  for (int i = 0; i < ntensor; ++i) { a.src[i] = src[i]; a.dst[i] = dst[i]; }
  a.idx = idx; a.status = status;
  a.N = g.N; a.R = g.R; a.S = g.S; a.T = g.T; a.m = g.m; a.G = g.G;
  a.p = g.p; a.L = g.L; a.ntensor = ntensor;
  for (int l = 0; l < 16; ++l) {
    a.off[l] = l < g.L ? g.off[l] : 0;
    double pw = 1.0;
    for (int q = 0; q < l; ++q) pw *= g.p;
    a.inv[l] = scale_by_level ? (float)(1.0 / pw) : 1.0f;
  }
  if (g.dtype == LH_BF16)
    return src_f32 ? run_spread<__nv_bfloat16, float>(g, a, st) : run_spread<__nv_bfloat16, __nv_bfloat16>(g, a, st);
  return run_spread<float, float>(g, a, st);
}

cudaError_t launch_spread_group(const Geo& g, const int32_t* idx, const void* const* src,
                                void* const* dst, uint32_t* status, cudaStream_t st) {
  SpreadArgs a{};
  for (int i = 0; i < 2; ++i) { a.src[i] = src[i]; a.dst[i] = dst[i]; }
  a.idx = idx; a.status = status;
  a.N = g.N; a.R = g.R; a.S = g.S; a.T = g.T; a.m = g.m; a.G = g.G;
  a.p = g.p; a.L = g.L; a.ntensor = 2;
  a.H = g.H; a.Hkv = g.Hkv; a.grp = g.grp;
  for (int l = 0; l < 16; ++l) {
    a.off[l] = l < g.L ? g.off[l] : 0;
    double pw = 1.0;
    for (int q = 0; q < l; ++q) pw *= g.p;
    a.inv[l] = (float)(1.0 / pw);
  }
  const size_t smem = (size_t)(g.M + 1) * g.grp * sizeof(int);
  dim3 grid((unsigned)g.C, (unsigned)g.BHkv);
  cudaError_t e;
#define LH_SPREAD_GROUP(E, D)                                                                        \
  e = cudaFuncSetAttribute(spread_group_kernel<E, float, D>, cudaFuncAttributeMaxDynamicSharedMemorySize, \
                           (int)smem);                                                               \
  if (e == cudaSuccess) spread_group_kernel<E, float, D><<<grid, kThreads, smem, st>>>(a)
  if (g.dtype == LH_BF16) {
    if (g.d == 64) { LH_SPREAD_GROUP(__nv_bfloat16, 64); } else { LH_SPREAD_GROUP(__nv_bfloat16, 128); }
  } else {
    if (g.d == 64) { LH_SPREAD_GROUP(float, 64); } else { LH_SPREAD_GROUP(float, 128); }
  }
#undef LH_SPREAD_GROUP
  return e != cudaSuccess ? e : cudaGetLastError();
}

}  // namespace lh
