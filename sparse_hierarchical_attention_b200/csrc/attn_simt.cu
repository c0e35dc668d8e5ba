// Causal attention on the gathered subsequence with fp32 FMA on the CUDA cores.
//
// This is the fp32 path (fp32 products and sums throughout, no TF32) and the bf16 fallback for shapes the
// tensor-core kernels do not take ("Long Context Pre-Training with Lighthouse Attention",
// technical summary 2.C: plain dense causal attention on the S rows; row j visible to row i
// iff j <= i).
//
// Tiles of 64 query x 64 key rows, 256 threads as a 16 x 16 grid. Thread (tr, tc) owns rows
// tr + 16*ii and columns tc + 16*jj, so that its shared-memory reads are either broadcasts or
// 16 consecutive words (conflict-free with a row pitch of D+1). Online softmax in the forward;
// the backward recomputes P from lse and runs two deterministic passes (dK,dV per key block;
// dQ per query block) so that no atomics decide a summation order.
#include "common.cuh"

namespace lh {
namespace {

constexpr int BM = 64, kThreads = 256;

template <typename E, int D>
__device__ inline void load_tile(float* dst, const E* src, int64_t row0, int64_t S, int tid) {
  // dst[r][c] with pitch D+1, rows >= S read as zero
  constexpr int VEC = 16 / sizeof(E), LPR = D / VEC;
  for (int it = tid; it < BM * LPR; it += kThreads) {
    const int r = it / LPR, cv = it % LPR;
    float x[VEC];
    uint4 u = make_uint4(0, 0, 0, 0);
    if (row0 + r < S) u = ldg16(src + (row0 + r) * D + cv * VEC);
    Vec<E>::unpack(u, x);
#pragma unroll
    for (int e = 0; e < VEC; ++e) dst[r * (D + 1) + cv * VEC + e] = x[e];
  }
}

template <typename E, int D>
__global__ void __launch_bounds__(kThreads)
attn_fwd_simt(const E* __restrict__ Q, const E* __restrict__ K, const E* __restrict__ V, float* O,
              float* lse, int64_t S, float sigma) {
  constexpr int P = D + 1, CC = D / 16;
  extern __shared__ float sm[];
  float* Qs = sm;
  float* Ks = Qs + BM * P;
  float* Vs = Ks + BM * P;
  float* Ps = Vs + BM * P;  // [64][65]
  const int tid = threadIdx.x, tr = tid / 16, tc = tid % 16;
  const int64_t bh = blockIdx.y;
  const int64_t nqb = (S + BM - 1) / BM;
  const int64_t qb = nqb - 1 - blockIdx.x;  // heaviest blocks first
  const E* q = Q + bh * S * D;
  const E* k = K + bh * S * D;
  const E* v = V + bh * S * D;
  load_tile<E, D>(Qs, q, qb * BM, S, tid);

  float m_i[4], l_i[4], o[4][CC];
#pragma unroll
  for (int ii = 0; ii < 4; ++ii) {
    m_i[ii] = -INFINITY; l_i[ii] = 0.f;
#pragma unroll
    for (int cc = 0; cc < CC; ++cc) o[ii][cc] = 0.f;
  }
  for (int64_t kb = 0; kb <= qb; ++kb) {
    __syncthreads();
    load_tile<E, D>(Ks, k, kb * BM, S, tid);
    load_tile<E, D>(Vs, v, kb * BM, S, tid);
    __syncthreads();
    float s[4][4];
#pragma unroll
    for (int ii = 0; ii < 4; ++ii)
#pragma unroll
      for (int jj = 0; jj < 4; ++jj) s[ii][jj] = 0.f;
#pragma unroll 8
    for (int c = 0; c < D; ++c) {
      float a[4], b[4];
#pragma unroll
      for (int ii = 0; ii < 4; ++ii) a[ii] = Qs[(tr + 16 * ii) * P + c];
#pragma unroll
      for (int jj = 0; jj < 4; ++jj) b[jj] = Ks[(tc + 16 * jj) * P + c];
#pragma unroll
      for (int ii = 0; ii < 4; ++ii)
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) s[ii][jj] = fmaf(a[ii], b[jj], s[ii][jj]);
    }
#pragma unroll
    for (int ii = 0; ii < 4; ++ii) {
      const int64_t i = qb * BM + tr + 16 * ii;
      float mx = -INFINITY;
#pragma unroll
      for (int jj = 0; jj < 4; ++jj) {
        const int64_t j = kb * BM + tc + 16 * jj;
        s[ii][jj] = (j <= i && j < S) ? s[ii][jj] * sigma : -INFINITY;
        mx = fmaxf(mx, s[ii][jj]);
      }
#pragma unroll
      for (int o2 = 8; o2 >= 1; o2 >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o2));
      const float m_new = fmaxf(m_i[ii], mx);
      const float m_use = m_new == -INFINITY ? 0.f : m_new;
      float rs = 0.f;
#pragma unroll
      for (int jj = 0; jj < 4; ++jj) {
        const float pv = expf(s[ii][jj] - m_use);
        rs += pv;
        Ps[(tr + 16 * ii) * 65 + tc + 16 * jj] = pv;
      }
#pragma unroll
      for (int o2 = 8; o2 >= 1; o2 >>= 1) rs += __shfl_xor_sync(0xffffffffu, rs, o2);
      const float alpha = expf(m_i[ii] - m_use);
      l_i[ii] = l_i[ii] * alpha + rs;
      m_i[ii] = m_new;
#pragma unroll
      for (int cc = 0; cc < CC; ++cc) o[ii][cc] *= alpha;
    }
    __syncthreads();
#pragma unroll 4
    for (int j = 0; j < BM; ++j) {
      float b[CC];
#pragma unroll
      for (int cc = 0; cc < CC; ++cc) b[cc] = Vs[j * P + tc + 16 * cc];
#pragma unroll
      for (int ii = 0; ii < 4; ++ii) {
        const float a = Ps[(tr + 16 * ii) * 65 + j];
#pragma unroll
        for (int cc = 0; cc < CC; ++cc) o[ii][cc] = fmaf(a, b[cc], o[ii][cc]);
      }
    }
  }
#pragma unroll
  for (int ii = 0; ii < 4; ++ii) {
    const int64_t i = qb * BM + tr + 16 * ii;
    if (i >= S) continue;
    const float inv = 1.f / l_i[ii];
#pragma unroll
    for (int cc = 0; cc < CC; ++cc) O[(bh * S + i) * D + tc + 16 * cc] = o[ii][cc] * inv;
    if (tc == 0) lse[bh * S + i] = m_i[ii] + logf(l_i[ii]);
  }
}

// D_i = dO_sub[i] . O_sub[i] in fp32 (O_sub kept in fp32); one warp per row.
template <typename E, int D>
__global__ void attn_delta(const float* __restrict__ O, const E* __restrict__ dO, float* delta,
                           int64_t rows) {
  const int64_t row = (int64_t)blockIdx.x * (blockDim.x / 32) + threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  if (row >= rows) return;
  float acc = 0.f;
  for (int c = lane; c < D; c += 32)
    acc = fmaf(O[row * D + c], to_f32(dO[row * D + c]), acc);
#pragma unroll
  for (int o2 = 16; o2 >= 1; o2 >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o2);
  if (lane == 0) delta[row] = acc;
}

// dK, dV for one 64-row key block, looping over the query blocks that can see it.
template <typename E, int D>
__global__ void __launch_bounds__(kThreads)
attn_bwd_dkdv_simt(const E* __restrict__ Q, const E* __restrict__ K, const E* __restrict__ V,
                   const E* __restrict__ dO, const float* __restrict__ lse,
                   const float* __restrict__ delta, float* dK, float* dV, int64_t S, float sigma) {
  constexpr int P = D + 1, CC = D / 16;
  extern __shared__ float sm[];
  float* Ks = sm;
  float* Vs = Ks + BM * P;
  float* Qs = Vs + BM * P;
  float* dOs = Qs + BM * P;
  float* Pt = dOs + BM * P;   // [key][query], pitch 65
  float* dSt = Pt + BM * 65;  // [key][query]
  float* ls = dSt + BM * 65;
  float* ds_ = ls + BM;
  const int tid = threadIdx.x, tr = tid / 16, tc = tid % 16;
  const int64_t bh = blockIdx.y;
  const int64_t nqb = (S + BM - 1) / BM;
  const int64_t kb = nqb - 1 - blockIdx.x;
  const E* q = Q + bh * S * D;
  const E* k = K + bh * S * D;
  const E* v = V + bh * S * D;
  const E* dout = dO + bh * S * D;
  load_tile<E, D>(Ks, k, kb * BM, S, tid);
  load_tile<E, D>(Vs, v, kb * BM, S, tid);
  float dv[4][CC], dk[4][CC];
#pragma unroll
  for (int jj = 0; jj < 4; ++jj)
#pragma unroll
    for (int cc = 0; cc < CC; ++cc) { dv[jj][cc] = 0.f; dk[jj][cc] = 0.f; }

  for (int64_t qb = kb; qb < nqb; ++qb) {
    __syncthreads();
    load_tile<E, D>(Qs, q, qb * BM, S, tid);
    load_tile<E, D>(dOs, dout, qb * BM, S, tid);
    if (tid < BM) {
      const int64_t i = qb * BM + tid;
      ls[tid] = i < S ? lse[bh * S + i] : 0.f;
      ds_[tid] = i < S ? delta[bh * S + i] : 0.f;
    }
    __syncthreads();
    float st[4][4], dpt[4][4];
#pragma unroll
    for (int jj = 0; jj < 4; ++jj)
#pragma unroll
      for (int ii = 0; ii < 4; ++ii) { st[jj][ii] = 0.f; dpt[jj][ii] = 0.f; }
#pragma unroll 4
    for (int c = 0; c < D; ++c) {
      float ka[4], va[4], qb_[4], ob[4];
#pragma unroll
      for (int jj = 0; jj < 4; ++jj) { ka[jj] = Ks[(tr + 16 * jj) * P + c]; va[jj] = Vs[(tr + 16 * jj) * P + c]; }
#pragma unroll
      for (int ii = 0; ii < 4; ++ii) { qb_[ii] = Qs[(tc + 16 * ii) * P + c]; ob[ii] = dOs[(tc + 16 * ii) * P + c]; }
#pragma unroll
      for (int jj = 0; jj < 4; ++jj)
#pragma unroll
        for (int ii = 0; ii < 4; ++ii) {
          st[jj][ii] = fmaf(ka[jj], qb_[ii], st[jj][ii]);
          dpt[jj][ii] = fmaf(va[jj], ob[ii], dpt[jj][ii]);
        }
    }
#pragma unroll
    for (int jj = 0; jj < 4; ++jj) {
      const int64_t j = kb * BM + tr + 16 * jj;
#pragma unroll
      for (int ii = 0; ii < 4; ++ii) {
        const int il = tc + 16 * ii;
        const int64_t i = qb * BM + il;
        const bool vis = i < S && j < S && j <= i;
        const float pv = vis ? expf(st[jj][ii] * sigma - ls[il]) : 0.f;
        Pt[(tr + 16 * jj) * 65 + il] = pv;
        dSt[(tr + 16 * jj) * 65 + il] = pv * (dpt[jj][ii] - ds_[il]);
      }
    }
    __syncthreads();
#pragma unroll 4
    for (int i = 0; i < BM; ++i) {
      float ob[CC], qv[CC];
#pragma unroll
      for (int cc = 0; cc < CC; ++cc) { ob[cc] = dOs[i * P + tc + 16 * cc]; qv[cc] = Qs[i * P + tc + 16 * cc]; }
#pragma unroll
      for (int jj = 0; jj < 4; ++jj) {
        const float pa = Pt[(tr + 16 * jj) * 65 + i], sa = dSt[(tr + 16 * jj) * 65 + i];
#pragma unroll
        for (int cc = 0; cc < CC; ++cc) {
          dv[jj][cc] = fmaf(pa, ob[cc], dv[jj][cc]);
          dk[jj][cc] = fmaf(sa, qv[cc], dk[jj][cc]);
        }
      }
    }
  }
#pragma unroll
  for (int jj = 0; jj < 4; ++jj) {
    const int64_t j = kb * BM + tr + 16 * jj;
    if (j >= S) continue;
#pragma unroll
    for (int cc = 0; cc < CC; ++cc) {
      dV[(bh * S + j) * D + tc + 16 * cc] = dv[jj][cc];
      dK[(bh * S + j) * D + tc + 16 * cc] = dk[jj][cc] * sigma;
    }
  }
}

// dQ for one 64-row query block, looping over the key blocks it sees.
template <typename E, int D>
__global__ void __launch_bounds__(kThreads)
attn_bwd_dq_simt(const E* __restrict__ Q, const E* __restrict__ K, const E* __restrict__ V,
                 const E* __restrict__ dO, const float* __restrict__ lse,
                 const float* __restrict__ delta, float* dQ, int64_t S, float sigma) {
  constexpr int P = D + 1, CC = D / 16;
  extern __shared__ float sm[];
  float* Qs = sm;
  float* dOs = Qs + BM * P;
  float* Ks = dOs + BM * P;
  float* Vs = Ks + BM * P;
  float* dSs = Vs + BM * P;  // [query][key], pitch 65
  const int tid = threadIdx.x, tr = tid / 16, tc = tid % 16;
  const int64_t bh = blockIdx.y;
  const int64_t nqb = (S + BM - 1) / BM;
  const int64_t qb = nqb - 1 - blockIdx.x;
  const E* q = Q + bh * S * D;
  const E* k = K + bh * S * D;
  const E* v = V + bh * S * D;
  load_tile<E, D>(Qs, q, qb * BM, S, tid);
  load_tile<E, D>(dOs, dO + bh * S * D, qb * BM, S, tid);
  float li[4], di[4];
#pragma unroll
  for (int ii = 0; ii < 4; ++ii) {
    const int64_t i = qb * BM + tr + 16 * ii;
    li[ii] = i < S ? lse[bh * S + i] : 0.f;
    di[ii] = i < S ? delta[bh * S + i] : 0.f;
  }
  float dq[4][CC];
#pragma unroll
  for (int ii = 0; ii < 4; ++ii)
#pragma unroll
    for (int cc = 0; cc < CC; ++cc) dq[ii][cc] = 0.f;
  for (int64_t kb = 0; kb <= qb; ++kb) {
    __syncthreads();
    load_tile<E, D>(Ks, k, kb * BM, S, tid);
    load_tile<E, D>(Vs, v, kb * BM, S, tid);
    __syncthreads();
    float s[4][4], dp[4][4];
#pragma unroll
    for (int ii = 0; ii < 4; ++ii)
#pragma unroll
      for (int jj = 0; jj < 4; ++jj) { s[ii][jj] = 0.f; dp[ii][jj] = 0.f; }
#pragma unroll 4
    for (int c = 0; c < D; ++c) {
      float qa[4], oa[4], kb_[4], vb[4];
#pragma unroll
      for (int ii = 0; ii < 4; ++ii) { qa[ii] = Qs[(tr + 16 * ii) * P + c]; oa[ii] = dOs[(tr + 16 * ii) * P + c]; }
#pragma unroll
      for (int jj = 0; jj < 4; ++jj) { kb_[jj] = Ks[(tc + 16 * jj) * P + c]; vb[jj] = Vs[(tc + 16 * jj) * P + c]; }
#pragma unroll
      for (int ii = 0; ii < 4; ++ii)
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) {
          s[ii][jj] = fmaf(qa[ii], kb_[jj], s[ii][jj]);
          dp[ii][jj] = fmaf(oa[ii], vb[jj], dp[ii][jj]);
        }
    }
#pragma unroll
    for (int ii = 0; ii < 4; ++ii) {
      const int64_t i = qb * BM + tr + 16 * ii;
#pragma unroll
      for (int jj = 0; jj < 4; ++jj) {
        const int64_t j = kb * BM + tc + 16 * jj;
        const bool vis = i < S && j < S && j <= i;
        const float pv = vis ? expf(s[ii][jj] * sigma - li[ii]) : 0.f;
        dSs[(tr + 16 * ii) * 65 + tc + 16 * jj] = pv * (dp[ii][jj] - di[ii]);
      }
    }
    __syncthreads();
#pragma unroll 4
    for (int j = 0; j < BM; ++j) {
      float kv[CC];
#pragma unroll
      for (int cc = 0; cc < CC; ++cc) kv[cc] = Ks[j * P + tc + 16 * cc];
#pragma unroll
      for (int ii = 0; ii < 4; ++ii) {
        const float a = dSs[(tr + 16 * ii) * 65 + j];
#pragma unroll
        for (int cc = 0; cc < CC; ++cc) dq[ii][cc] = fmaf(a, kv[cc], dq[ii][cc]);
      }
    }
  }
#pragma unroll
  for (int ii = 0; ii < 4; ++ii) {
    const int64_t i = qb * BM + tr + 16 * ii;
    if (i >= S) continue;
#pragma unroll
    for (int cc = 0; cc < CC; ++cc) dQ[(bh * S + i) * D + tc + 16 * cc] = dq[ii][cc] * sigma;
  }
}

template <typename E, int D>
cudaError_t fwd(const Geo& g, const void* qs, const void* ks, const void* vs, float* os, float* lse,
                cudaStream_t st) {
  const size_t smem = (size_t)(3 * BM * (D + 1) + BM * 65) * sizeof(float);
  cudaError_t e = cudaFuncSetAttribute(attn_fwd_simt<E, D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid((unsigned)((g.S + BM - 1) / BM), (unsigned)g.BH);
  attn_fwd_simt<E, D><<<grid, kThreads, smem, st>>>((const E*)qs, (const E*)ks, (const E*)vs, os, lse,
                                                    g.S, 1.0f / sqrtf((float)D));
  return cudaGetLastError();
}

template <typename E, int D>
cudaError_t bwd(const Geo& g, const void* qs, const void* ks, const void* vs, const float* os,
                const float* lse, const void* dos, float* dq, float* dk, float* dv, float* delta,
                cudaStream_t st) {
  const int64_t rows = g.BH * g.S;
  attn_delta<E, D><<<(unsigned)((rows + 7) / 8), 256, 0, st>>>(os, (const E*)dos, delta, rows);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const float sigma = 1.0f / sqrtf((float)D);
  dim3 grid((unsigned)((g.S + BM - 1) / BM), (unsigned)g.BH);
  const size_t smem1 = (size_t)(4 * BM * (D + 1) + 2 * BM * 65 + 2 * BM) * sizeof(float);
  e = cudaFuncSetAttribute(attn_bwd_dkdv_simt<E, D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem1);
  if (e != cudaSuccess) return e;
  attn_bwd_dkdv_simt<E, D><<<grid, kThreads, smem1, st>>>((const E*)qs, (const E*)ks, (const E*)vs,
                                                           (const E*)dos, lse, delta, dk, dv, g.S, sigma);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  const size_t smem2 = (size_t)(4 * BM * (D + 1) + BM * 65) * sizeof(float);
  e = cudaFuncSetAttribute(attn_bwd_dq_simt<E, D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem2);
  if (e != cudaSuccess) return e;
  attn_bwd_dq_simt<E, D><<<grid, kThreads, smem2, st>>>((const E*)qs, (const E*)ks, (const E*)vs,
                                                         (const E*)dos, lse, delta, dq, g.S, sigma);
  return cudaGetLastError();
}

}  // namespace

int attn_fwd_launches(const Geo&) { return 1; }
int attn_bwd_launches(const Geo& g) { return attn_bwd_fused(g) ? 2 : 3; }  // delta + one or two passes

cudaError_t launch_attn_fwd_simt(const Geo& g, const void* qs, const void* ks, const void* vs,
                                 float* os, float* lse, cudaStream_t st) {
  if (g.dtype == LH_BF16)
    return g.d == 64 ? fwd<__nv_bfloat16, 64>(g, qs, ks, vs, os, lse, st)
                     : fwd<__nv_bfloat16, 128>(g, qs, ks, vs, os, lse, st);
  return g.d == 64 ? fwd<float, 64>(g, qs, ks, vs, os, lse, st) : fwd<float, 128>(g, qs, ks, vs, os, lse, st);
}

cudaError_t launch_attn_bwd_simt(const Geo& g, const void* qs, const void* ks, const void* vs,
                                 const float* os, const float* lse, const void* dos, float* dq,
                                 float* dk, float* dv, float* delta, cudaStream_t st) {
  if (g.dtype == LH_BF16)
    return g.d == 64 ? bwd<__nv_bfloat16, 64>(g, qs, ks, vs, os, lse, dos, dq, dk, dv, delta, st)
                     : bwd<__nv_bfloat16, 128>(g, qs, ks, vs, os, lse, dos, dq, dk, dv, delta, st);
  return g.d == 64 ? bwd<float, 64>(g, qs, ks, vs, os, lse, dos, dq, dk, dv, delta, st)
                   : bwd<float, 128>(g, qs, ks, vs, os, lse, dos, dq, dk, dv, delta, st);
}

}  // namespace lh
