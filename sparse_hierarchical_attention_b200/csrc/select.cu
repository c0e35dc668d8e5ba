// Stratified top-K ("Long Context Pre-Training with Lighthouse Attention", technical summary
// 2.B: joint top-K over all levels; the Nous Research article's four-stage paragraph: the
// selection is stratified and always keeps the coarsest level).
//
// One CTA per (b,h, stratum of G chunks; G = 1 whenever S is a multiple of the chunk count).
// The stratum's G*M candidate scores become 64-bit keys that encode the total ranking order
// (score descending, then level descending, then position ascending): high word = the fp32 score
// bits (scores are >= +0, so the bit pattern orders like the value), then the level (higher
// wins), then the stratum-local position (lower wins). A most-significant-digit radix select
// (8-bit digits, shared-memory histograms, one warp scanning the 256 bins) finds the k-th
// largest key; it stops as soon as the bucket that holds the k-th key is taken whole. The k
// winners are then placed in causal order (end, level) by counting, each chunk's coarsest cell
// right after the winners of that chunk.
#include "common.cuh"

namespace lh {
namespace {

struct SelArgs {
  const float* score;
  int32_t* idx;
  int64_t N, R, S, m, k, M, G, T;
  int64_t off[16];
  int p, L;
};

template <int kSelThreads>
__global__ void __launch_bounds__(kSelThreads) select_kernel(const SelArgs a) {
  // [G*M] candidate keys, then [k] winners, then [G] winners per chunk of the stratum
  extern __shared__ unsigned long long keys[];
  __shared__ unsigned hist[256];
  __shared__ int s_digit, s_need, s_cnt, s_nsel;

  const int tid = threadIdx.x;
  const int64_t bh = blockIdx.y, st = blockIdx.x;  // stratum st: chunks st*G .. st*G + G-1
  const float* sc = a.score + bh * (a.N + a.R);
  int32_t* out = a.idx + bh * a.S + st * a.m;
  const int L = a.L, p = a.p, G = (int)a.G;
  const int M = (int)(a.G * a.M), k = (int)a.k;  // candidates and picks of the stratum
  int* per_chunk = reinterpret_cast<int*>(keys + M + k);

  // 1. candidate keys: level l holds G p^(L-1-l) cells per stratum. The key orders by score,
  //    then level (higher first), then stratum-local position (lower first).
  {
    int base = 0;
    for (int l = 0; l < L - 1; ++l) {
      int per = G;
      for (int q = l; q < L - 1; ++q) per *= p;
      for (int jl = tid; jl < per; jl += kSelThreads) {
        const float r = sc[a.off[l] + st * per + jl];
        const unsigned long long key = ((unsigned long long)__float_as_uint(r) << 32) |
                                       ((unsigned long long)l << 24) | (unsigned)(0xFFFFFF - jl);
        keys[base + jl] = key;
      }
      base += per;
    }
  }
  for (int i = tid; i < G; i += kSelThreads) per_chunk[i] = 0;
  if (tid == 0) s_nsel = 0;
  __syncthreads();

  if (k > 0) {
    // 2. radix select of the k-th largest key
    unsigned long long prefix = 0, mask = 0;
    int need = k;
    for (int shift = 56; shift >= 0; shift -= 8) {
      for (int i = tid; i < 256; i += kSelThreads) hist[i] = 0;
      __syncthreads();
      for (int q = tid; q < M; q += kSelThreads) {
        const unsigned long long key = keys[q];
        if ((key & mask) == prefix) atomicAdd(&hist[(key >> shift) & 255], 1u);
      }
      __syncthreads();
      if (tid < 32) {
        // lane l covers bins 255-8l .. 248-8l, taken from the top
        unsigned cnt[8], tot = 0;
#pragma unroll
        for (int i = 0; i < 8; ++i) { cnt[i] = hist[255 - 8 * tid - i]; tot += cnt[i]; }
        unsigned incl = tot;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const unsigned v = __shfl_up_sync(0xffffffffu, incl, o);
          if (tid >= o) incl += v;
        }
        const unsigned ball = __ballot_sync(0xffffffffu, incl >= (unsigned)need);
        const int first = __ffs(ball) - 1;
        if (ball == 0 && tid == 0) {  // cannot happen for a consistent histogram; stop safely
          s_digit = 0; s_need = need; s_cnt = -1;
        }
        if (tid == first) {
          unsigned cum = incl - tot;
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            if (cum + cnt[i] >= (unsigned)need) {
              s_digit = 255 - 8 * tid - i;
              s_need = need - (int)cum;
              s_cnt = (int)cnt[i];
              break;
            }
            cum += cnt[i];
          }
        }
      }
      __syncthreads();
      prefix |= (unsigned long long)s_digit << shift;
      mask |= 0xFFull << shift;
      need = s_need;
      const bool done = s_cnt == need || s_cnt < 0;
      __syncthreads();
      if (done) break;
    }
    // 3. winners: keys whose masked value is >= the prefix (exactly k of them)
    unsigned long long* win = keys + M;
    for (int q = tid; q < M; q += kSelThreads) {
      const unsigned long long key = keys[q];
      if ((key & mask) >= prefix) {
        const int pos = atomicAdd(&s_nsel, 1);
        if (pos < k) win[pos] = key;  // exactly k winners; the guard keeps shared memory safe
      }
    }
    __syncthreads();
    const int nsel = s_nsel < k ? s_nsel : k;
    for (int w = tid; w < nsel; w += kSelThreads) {  // winners per chunk of the stratum
      const int l = (int)((win[w] >> 24) & 0xFF);
      const int jl = 0xFFFFFF - (int)(win[w] & 0xFFFFFF);
      int64_t pw = 1;
      for (int q = 0; q < l; ++q) pw *= p;
      atomicAdd(&per_chunk[(int)((int64_t)jl * pw / a.T)], 1);
    }
    __syncthreads();
    // 4. causal order: a winner's row is its rank by (end, level) among the winners plus the
    //    coarsest cells of the chunks before its own (they end before it starts)
    for (int w = tid; w < nsel; w += kSelThreads) {
      const unsigned long long key = win[w];
      const int l = (int)((key >> 24) & 0xFF);
      const int jl = 0xFFFFFF - (int)(key & 0xFFFFFF);
      int64_t pw = 1;
      for (int q = 0; q < l; ++q) pw *= p;
      const int64_t ord = (((int64_t)jl + 1) * pw) * 16 + l;
      int rank = 0;
      for (int u = 0; u < nsel; ++u) {
        const unsigned long long k2 = win[u];
        const int l2 = (int)((k2 >> 24) & 0xFF);
        const int j2 = 0xFFFFFF - (int)(k2 & 0xFFFFFF);
        int64_t pw2 = 1;
        for (int q = 0; q < l2; ++q) pw2 *= p;
        rank += ((((int64_t)j2 + 1) * pw2) * 16 + l2) < ord;
      }
      int per = G;
      for (int q = l; q < L - 1; ++q) per *= p;
      const int row = rank + (int)((int64_t)jl * pw / a.T);
      if (row < a.m) out[row] = (int32_t)(a.off[l] + st * per + jl);
    }
  }
  // the coarsest cell of chunk cl comes after the winners of chunks 0..cl and the cl coarsest
  // cells before it
  for (int cl = tid; cl < G; cl += kSelThreads) {
    int before = cl;
    for (int u = 0; u <= cl; ++u) before += per_chunk[u];
    if (before < a.m) out[before] = (int32_t)(a.off[L - 1] + st * G + cl);
  }
}

}  // namespace

cudaError_t launch_select(const Geo& g, const float* score, int32_t* idx, cudaStream_t st) {
  SelArgs a{};
  a.score = score; a.idx = idx;
  a.N = g.N; a.R = g.R; a.S = g.S; a.m = g.m; a.k = g.k; a.M = g.M; a.G = g.G; a.T = g.T;
  a.p = g.p; a.L = g.L;
  for (int l = 0; l < 16; ++l) a.off[l] = l < g.L ? g.off[l] : 0;
  const size_t smem = (size_t)(g.G * g.M + g.k) * sizeof(unsigned long long) + (size_t)g.G * sizeof(int);
  dim3 grid((unsigned)(g.C / g.G), (unsigned)g.BH);
  // The kernel is bound by latency (shared-memory passes, synchronisations), so what counts is
  // how many strata an SM holds at once. Up to 16 KB of keys, 128-thread CTAs fit 16 per SM
  // (2048 threads); with more keys shared memory caps the CTAs per SM, and 256 threads each keep
  // the passes short (measured: 1364 keys 70 -> 59 us with 128 threads, 5460 keys 78 -> 91 us).
  cudaError_t e;
  if (smem <= 16384) {
    e = cudaFuncSetAttribute(select_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    select_kernel<128><<<grid, 128, smem, st>>>(a);
  } else {
    e = cudaFuncSetAttribute(select_kernel<256>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    select_kernel<256><<<grid, 256, smem, st>>>(a);
  }
  return cudaGetLastError();
}

}  // namespace lh
