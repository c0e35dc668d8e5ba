// Causal attention forward on the gathered subsequence with 5th-generation tensor cores
// (tcgen05, accumulators in tensor memory, operands staged by TMA). bf16 inputs, fp32 softmax
// and accumulation ("Long Context Pre-Training with Lighthouse Attention", technical summary
// 2.C: dense causal attention on the S selected rows; row j visible to row i iff j <= i).
//
// One CTA = 128 query rows of one (b,h) = 4 warps, thread t owning row t (TMEM lane t).
//  - Thread 0 also issues the TMA loads (Q once; K and V through two-stage rings) and the MMAs.
//  - S_j = Q K_j^T goes to one of two 128-column TMEM buffers, so S_{j+1} runs on the tensor
//    cores while the warps do the softmax of S_j.
//  - P_j goes to shared memory in the 128-byte-swizzled K-major layout as two bf16 terms,
//    P = hi + lo with hi = bf16(P) and lo = bf16(P - hi), and O += hi V_j + lo V_j accumulates
//    in TMEM (V read as an MN-major operand). The split keeps P to ~16 bits: the backward
//    recomputes P exactly and forms D_i = dO_i . O_i, so an O made from bf16-rounded P would
//    leave sum_j dS_ij off zero by dO . (O error), which is large on coarse rows whose dO sums
//    thousands of tokens.
//  - The running max is updated lazily: O and l are rescaled only when a row's max grows by more
//    than 2^8, which keeps every exponent bounded and skips most TMEM round trips.
//  - Key blocks above the diagonal are skipped; the diagonal block is masked.
// The output is fp32 O_sub and the natural-log lse. Shared memory per CTA: Q + 2 K + 2 V + 2 P
// tiles of 128 rows (224 KB at d = 128), one CTA per SM; tensor memory: 512 columns.
#include <mutex>

#include "tc.cuh"

namespace lh {
namespace {

using namespace tc;

constexpr int BM = 128, BN = 128, kThreads = 128;
constexpr int TILE = 128 * 128;  // bytes of one [128 rows][64 bf16] 128B-swizzled sub-tile

template <int D>
struct Layout {
  static constexpr int KB = D / 64;  // 64-column sub-tiles per row
  static constexpr int Q = 0;
  static constexpr int K = Q + KB * TILE;      // stage s at K + s * KB * TILE
  static constexpr int V = K + 2 * KB * TILE;  // stage s at V + s * KB * TILE
  static constexpr int P = V + 2 * KB * TILE;  // hi then lo, each 128 keys = 2 sub-tiles
  static constexpr int BAR = P + 4 * TILE;
  static constexpr int BYTES = BAR + 128;
};

// bars: 0 Q, 1-2 K stages, 3-4 V stages, 5-6 S buffers, 7 PV
template <int D>
__global__ void __launch_bounds__(kThreads, 1)
attn_fwd_tc(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
            const __grid_constant__ CUtensorMap tv, float* __restrict__ O, float* __restrict__ lse,
            int S, float scale_log2, uint32_t* status) {
  using Ly = Layout<D>;
  constexpr int KB = Ly::KB;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
  uint64_t* bar = reinterpret_cast<uint64_t*>(sm + Ly::BAR);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar + 8);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bar + 8) + 1;

  const int tid = threadIdx.x, warp = tid / 32;
  const int nqb = S / BM;
  const int qb = nqb - 1 - (int)blockIdx.y;  // heads vary fastest; heaviest tiles first
  const int bh = blockIdx.x;
  const int grow0 = bh * S;                  // first row of this (b,h) in the [BH*S, D] view
  const int nkb = qb + 1;

  if (tid == 0) {
    for (int i = 0; i < 8; ++i) mbar_init(bar + i, 1);
    *abort_flag = 0;
    fence_barrier_init();
    prefetch_tmap(&tq);
    prefetch_tmap(&tk);
    prefetch_tmap(&tv);
  }
  if (warp == 0) tmem_alloc(tmem_slot, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_slot;
  const uint32_t t_o = tbase + 256;
  const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
  const uint32_t s_q = smem_u32(sm + Ly::Q), s_k = smem_u32(sm + Ly::K);
  const uint32_t s_v = smem_u32(sm + Ly::V), s_p = smem_u32(sm + Ly::P);
  constexpr uint32_t IDESC_S = idesc_bf16(128, 128, false, false);
  constexpr uint32_t IDESC_PV = idesc_bf16(128, D, false, true);

  auto load_k = [&](int j) {  // K_j into stage j & 1
    uint64_t* b = bar + 1 + (j & 1);
    mbar_expect_tx(b, KB * TILE);
    for (int kb = 0; kb < KB; ++kb)
      tma_load_2d(sm + Ly::K + (j & 1) * KB * TILE + kb * TILE, &tk, kb * 64, grow0 + j * BN, b);
  };
  auto load_v = [&](int j) {
    uint64_t* b = bar + 3 + (j & 1);
    mbar_expect_tx(b, KB * TILE);
    for (int kb = 0; kb < KB; ++kb)
      tma_load_2d(sm + Ly::V + (j & 1) * KB * TILE + kb * TILE, &tv, kb * 64, grow0 + j * BN, b);
  };
  auto issue_s = [&](int j) {  // S_j = Q K_j^T into TMEM buffer j & 1
    const uint32_t kbase = s_k + (j & 1) * KB * TILE;
#pragma unroll
    for (int ks = 0; ks < D / 16; ++ks) {
      const uint32_t off = (ks / 4) * TILE + (ks % 4) * 32;
      mma_ss(tbase + (j & 1) * 128, sw128_desc(s_q + off, 16, 1024), sw128_desc(kbase + off, 16, 1024),
             IDESC_S, ks > 0);
    }
    mma_commit(bar + 5 + (j & 1));
  };
  auto issue_pv = [&](int j) {  // O += hi_j V_j + lo_j V_j
    const uint32_t vbase = s_v + (j & 1) * KB * TILE;
#pragma unroll
    for (int part = 0; part < 2; ++part) {
#pragma unroll
      for (int ks = 0; ks < BN / 16; ++ks) {
        const uint32_t poff = part * 2 * TILE + (ks / 4) * TILE + (ks % 4) * 32;
        mma_ss(t_o, sw128_desc(s_p + poff, 16, 1024), sw128_desc(vbase + ks * 2048, TILE, 1024),
               IDESC_PV, (j > 0 || part > 0 || ks > 0) ? 1u : 0u);
      }
    }
    mma_commit(bar + 7);
  };
  // all lanes of a warp wait together, so that the warp stays converged for tcgen05.ld/st
  auto wait_all = [&](uint64_t* b, uint32_t parity) {
    bool ok = mbar_wait(b, parity, abort_flag, status);
    return __all_sync(0xffffffffu, ok);
  };

  if (tid == 0) {
    mbar_expect_tx(bar, KB * TILE);
    for (int kb = 0; kb < KB; ++kb) tma_load_2d(sm + Ly::Q + kb * TILE, &tq, kb * 64, grow0 + qb * BM, bar);
    load_k(0);
    load_v(0);
    if (nkb > 1) { load_k(1); load_v(1); }
    if (mbar_wait(bar, 0, abort_flag, status) && mbar_wait(bar + 1, 0, abort_flag, status)) issue_s(0);
  }
  __syncwarp();

  const int row = tid;  // query row within the tile = TMEM lane
  float m_used = -INFINITY, l = 0.f;
  float s[BN];
  for (int j = 0; j < nkb; ++j) {
    // ---- S_j is ready; keep the tensor cores busy with S_{j+1}
    const bool ok_s = wait_all(bar + 5 + (j & 1), (j >> 1) & 1);
    tc_fence_after();
    if (tid == 0 && ok_s) {
      if (j + 2 < nkb) load_k(j + 2);  // K stage j&1 was consumed by S_j
      if (j + 1 < nkb && mbar_wait(bar + 1 + ((j + 1) & 1), ((j + 1) >> 1) & 1, abort_flag, status))
        issue_s(j + 1);
    }
    __syncwarp();
    // ---- softmax of S_j (row per thread)
    if (ok_s) {
      uint32_t r0[32], r1[32], r2[32], r3[32];
      const uint32_t ts = tbase + (j & 1) * 128 + lane_off;
      tmem_ld32(ts, r0);
      tmem_ld32(ts + 32, r1);
      tmem_ld32(ts + 64, r2);
      tmem_ld32(ts + 96, r3);
      tmem_wait_ld();
#pragma unroll
      for (int e = 0; e < 32; ++e) {
        s[e] = __uint_as_float(r0[e]) * scale_log2;
        s[32 + e] = __uint_as_float(r1[e]) * scale_log2;
        s[64 + e] = __uint_as_float(r2[e]) * scale_log2;
        s[96 + e] = __uint_as_float(r3[e]) * scale_log2;
      }
    }
    if (j == qb) {  // diagonal block: key column > query row is invisible
#pragma unroll
      for (int e = 0; e < BN; ++e)
        if (e > row) s[e] = -INFINITY;
    }
    float mt = -INFINITY;
#pragma unroll
    for (int e = 0; e < BN; ++e) mt = fmaxf(mt, s[e]);
    const bool grow = mt > m_used + 8.0f;
    const float m_new = grow ? mt : m_used;
    const float alpha = grow ? exp2f(m_used - m_new) : 1.0f;
    float sum = 0.f;
#pragma unroll
    for (int e = 0; e < BN; ++e) {
      s[e] = ex2(s[e] - m_new);
      sum += s[e];
    }
    l = l * alpha + sum;
    m_used = m_new;
    // ---- PV_{j-1} must be done before P and O are touched again
    bool ok_pv = true;
    if (j > 0) {
      ok_pv = wait_all(bar + 7, (j - 1) & 1);
      tc_fence_after();
      if (tid == 0 && ok_pv && j + 1 < nkb && j >= 1) load_v(j + 1);  // V stage (j+1)&1 is free
      __syncwarp();
    }
    if (ok_s && ok_pv && j > 0 && __any_sync(0xffffffffu, grow)) {  // rescale this warp's O rows
      uint32_t r[32];
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        tmem_ld32(t_o + lane_off + c * 32, r);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 32; ++e) r[e] = __float_as_uint(__uint_as_float(r[e]) * alpha);
        tmem_st32(t_o + lane_off + c * 32, r);
      }
      tmem_wait_st();
    }
    // P_j = hi + lo (bf16 each) -> shared memory, K-major, 128-byte swizzle
#pragma unroll
    for (int c = 0; c < BN / 8; ++c) {
      uint32_t wh[4], wl[4];
#pragma unroll
      for (int h = 0; h < 4; ++h) split_bf16x2(s[c * 8 + 2 * h], s[c * 8 + 2 * h + 1], wh[h], wl[h]);
      const uint32_t addr = s_p + (c / 8) * TILE + row * 128 + (((c % 8) ^ (row % 8)) * 16);
      asm volatile("st.shared.v4.b32 [%0], {%1,%2,%3,%4};" ::"r"(addr), "r"(wh[0]), "r"(wh[1]),
                   "r"(wh[2]), "r"(wh[3])
                   : "memory");
      asm volatile("st.shared.v4.b32 [%0], {%1,%2,%3,%4};" ::"r"(addr + 2 * TILE), "r"(wl[0]),
                   "r"(wl[1]), "r"(wl[2]), "r"(wl[3])
                   : "memory");
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (*abort_flag) break;
    if (tid == 0) {
      if (mbar_wait(bar + 3 + (j & 1), (j >> 1) & 1, abort_flag, status)) issue_pv(j);
    }
    __syncwarp();
  }

  // ---- epilogue: O / l and lse
  const bool ok_end = !*abort_flag && wait_all(bar + 7, (nkb - 1) & 1);
  tc_fence_after();
  if (ok_end) {
    const float inv = 1.0f / l;
    float* orow = O + (size_t)(grow0 + qb * BM + row) * D;
    uint32_t r[32];
#pragma unroll
    for (int c = 0; c < D / 32; ++c) {
      tmem_ld32(t_o + lane_off + c * 32, r);
      tmem_wait_ld();
#pragma unroll
      for (int e = 0; e < 32; e += 4) {
        float4 v = make_float4(__uint_as_float(r[e]) * inv, __uint_as_float(r[e + 1]) * inv,
                               __uint_as_float(r[e + 2]) * inv, __uint_as_float(r[e + 3]) * inv);
        *reinterpret_cast<float4*>(orow + c * 32 + e) = v;
      }
    }
    lse[grow0 + qb * BM + row] = (m_used + log2f(l)) * 0.69314718055994531f;
  }
  tc_fence_before();
  __syncthreads();
  if (*abort_flag) {  // let operations already in flight finish before the memory is released
    const uint64_t t0 = globaltimer();
    while (globaltimer() - t0 < 1000000ull) {
    }
  }
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tbase, 512);
}

// ---------------------------------------------------------------- host side
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

}  // namespace

// [rows, D] bf16 matrix, boxes of [box_rows][64 columns] with 128-byte swizzle.
bool make_tmap_rows_box(CUtensorMap* map, const void* base, int64_t rows, int D, int box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {(cuuint64_t)D, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)D * 2};
  cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool make_tmap_rows(CUtensorMap* map, const void* base, int64_t rows, int D) {
  return make_tmap_rows_box(map, base, rows, D, 128);
}

bool attn_tc_eligible(const Geo& g) {
  return g.dtype == LH_BF16 && (g.d == 64 || g.d == 128) && g.S % 128 == 0 &&
         g.BH * (int64_t)g.S < (int64_t)1 << 31;
}

cudaError_t launch_attn_fwd_tc(const Geo& g, const void* qs, const void* ks, const void* vs,
                               float* os, float* lse, uint32_t* status, cudaStream_t st) {
  CUtensorMap mq, mk, mv;
  const int64_t rows = g.BH * g.S;
  if (!make_tmap_rows(&mq, qs, rows, g.d) || !make_tmap_rows(&mk, ks, rows, g.d) ||
      !make_tmap_rows(&mv, vs, rows, g.d))
    return cudaErrorInvalidValue;
  const float scale_log2 = (1.0f / sqrtf((float)g.d)) * 1.4426950408889634f;
  dim3 grid((unsigned)g.BH, (unsigned)(g.S / BM));
  cudaError_t e;
  if (g.d == 128) {
    const int smem = Layout<128>::BYTES + 1024;
    e = cudaFuncSetAttribute(attn_fwd_tc<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e == cudaSuccess)
      attn_fwd_tc<128><<<grid, kThreads, smem, st>>>(mq, mk, mv, os, lse, g.S, scale_log2, status);
  } else {
    // padded so that two CTAs never share an SM (each holds all 512 TMEM columns)
    const int smem = Layout<64>::BYTES + 1024 > 120 * 1024 ? Layout<64>::BYTES + 1024 : 120 * 1024;
    e = cudaFuncSetAttribute(attn_fwd_tc<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e == cudaSuccess)
      attn_fwd_tc<64><<<grid, kThreads, smem, st>>>(mq, mk, mv, os, lse, g.S, scale_log2, status);
  }
  return e != cudaSuccess ? e : cudaGetLastError();
}

}  // namespace lh
