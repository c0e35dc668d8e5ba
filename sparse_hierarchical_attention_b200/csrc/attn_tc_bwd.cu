// Causal attention backward on the gathered subsequence with tcgen05 tensor cores ("Long Context
// Pre-Training with Lighthouse Attention", technical summary 2.B: gradients flow through the
// attention to Q, K and V). With D_i = dO_i . O_i and P_ij = exp(s Q_i . K_j - lse_i) for j <= i:
// dV_j = sum_i P_ij dO_i, dS_ij = P_ij (dO_i . V_j - D_i), dQ_i = s sum_j dS_ij K_j and
// dK_j = s sum_i dS_ij Q_i, with s = 1/sqrt(d).
//
// Two ways to run it:
//   fused (the default; the d = 64 form, with 128-row query blocks and dQ added by the copy
//     engine, is described above its kernel below): at d = 128 one CTA per 128-key block steps
//     through the 64-row query blocks that can see the keys:
//       S^T = K Q^T and dP^T = V dO^T;
//       P^T = exp2(S^T c - lse2) and dS^T = P^T (dP^T - D) in fp32 registers;
//       dV += P^T dO and dK += dS^T Q (accumulated in tensor memory over the whole block), and
//       dQ^T = K^T dS^T for this query block (fresh every step), which the warps add into the
//       fp32 dq_sub rows with atomic adds (red.global.add.f32). dq_sub is zeroed first.
//     P^T goes to tensor memory (A operand of dV). dS^T goes to one 128-byte-swizzled
//     shared-memory tile [128 keys][64 queries] that is at once the K-major A operand of dK and
//     the MN-major B operand of dQ^T; K^T is the CTA's K tile read MN-major. So each step's S and
//     dP are computed once for all three gradients. dV and dK are deterministic; the order in
//     which the key blocks' dQ terms reach a dq_sub row varies from run to run.
//   deterministic (LH_DETERMINISTIC): two kernels without atomics:
//     dkdv: the fused kernel's dV/dK part, with dS^T in tensor memory;
//     dq:   one CTA per 128-query block steps through the 64-row key blocks it sees:
//           S = Q K^T and dP = dO V^T, dS as above, dQ += dS K (dS from tensor memory).
//     This recomputes S and dP for dQ.
// Warp roles: warps 0-15 compute (warp w owns TMEM lanes 32(w%4)..+31 and column quarter w/4 of
// each step); warp 16 (one lane) issues the TMA loads; warp 17 (one lane) issues the S/dP MMAs and
// warp 18 (one lane) the accumulation MMAs, so that an MMA issue that waits for room in the tensor
// pipe never delays a load or the other stream, and the accumulation of a step is issued as soon
// as its P lands. The sides meet only at mbarriers (stage loaded, stage
// free, S ready, S buffer free, P written, accumulation done; one arrival per warp), so the tensor
// cores work on step it+1's S/dP and step it-1's accumulation while the warps do step it.
// Q/dO (fused, dkdv) and K/V (dq) come through TMA rings, with lse and D riding along as 1-D bulk
// copies. Tensor memory holds S/dP (single-buffered in dkdv and fused, whose warps read it at the
// start of a step; double-buffered in dq), the P/dS operands in their own columns (so that no MMA
// writes columns an earlier MMA may still read), and the accumulators until the epilogue writes
// fp32 results.
// dQ, dK and dV all sum P or dS against rows with mixed signs. Coarse rows carry dO_sub that
// sums thousands of tokens, and there those sums cancel by orders of magnitude. So P^T, dS^T and
// dS each enter their product as two bf16 terms, hi = bf16(x) and lo = bf16(x - hi). That is
// one extra MMA per product and keeps the operand to ~16 bits. With one bf16 term, single dV
// elements were off by 34% of their size.
// The warps' element arithmetic runs on key (or query) pairs with packed f32x2 FMA, subtract and
// multiply, each lane rounded as the scalar instruction is, so the results are those of the scalar
// sequence exp2(s c - lse2), (dP - D) p, hi/lo split, with half the issue slots.
// Every barrier that could run two phases ahead of a waiter is doubled, so that no parity wait
// is ambiguous. All waits are bounded and report through the status word; on an abort every role
// drains its own loads or MMAs before the CTA frees tensor memory (tc.cuh).
#include "tc.cuh"

namespace lh {

bool make_tmap_rows_box(CUtensorMap* map, const void* base, int64_t rows, int D, int box_rows);
// fp32 [rows][D] with 128-byte-swizzled boxes of 32 columns x box_rows rows (reductions into dq_sub)
bool make_tmap_f32_box(CUtensorMap* map, const void* base, int64_t rows, int D, int box_rows);

namespace {

using namespace tc;

constexpr int kCompute = 512;              // warps 0-15
constexpr int kThreads = kCompute + 96;    // + the TMA warp and two MMA warps (S/dP, accumulate)
constexpr int T128 = 128 * 128;  // [128 rows][64 bf16] sub-tile bytes
constexpr int T64 = 64 * 128;    // [64 rows][64 bf16] sub-tile bytes
constexpr float kLog2e = 1.4426950408889634f;

__device__ inline void red_add(float* p, float v) {
  asm volatile("red.global.add.f32 [%0], %1;" ::"l"(p), "f"(v) : "memory");
}

// One thread's share of a key-block step: key row kj, the 16 queries q0..q0+15 of its column
// quarter, their S^T and dP^T, and the step's lse and D from shared memory. Returns P^T and dS^T
// as query pairs (lower query in the low lane), zero where the key comes after the query.
__device__ inline void kv_step_elements(const float (&st)[16], const float (&dpt)[16],
                                        const float4* lv4, const float4* dv4, float scale_log2,
                                        int kj, int q0, bool diag, uint64_t (&p2)[8],
                                        uint64_t (&ds2)[8]) {
  const uint64_t c2 = f2_pack(scale_log2, scale_log2);
#pragma unroll
  for (int c4 = 0; c4 < 4; ++c4) {
    const float4 lv = lv4[c4], dv = dv4[c4];
    const uint64_t nla[2] = {f2_pack(-(lv.x * kLog2e), -(lv.y * kLog2e)),
                             f2_pack(-(lv.z * kLog2e), -(lv.w * kLog2e))};
    const uint64_t da[2] = {f2_pack(dv.x, dv.y), f2_pack(dv.z, dv.w)};
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int h = c4 * 2 + e;
      float a0, a1;
      f2_unpack(f2_fma(f2_pack(st[2 * h], st[2 * h + 1]), c2, nla[e]), a0, a1);
      p2[h] = f2_pack(ex2(a0), ex2(a1));
      ds2[h] = f2_mul(p2[h], f2_sub(f2_pack(dpt[2 * h], dpt[2 * h + 1]), da[e]));
    }
  }
  if (diag) {  // steps that reach the diagonal: keys after the query are invisible
#pragma unroll
    for (int h = 0; h < 8; ++h) {
      float x0, x1, y0, y1;
      f2_unpack(p2[h], x0, x1);
      f2_unpack(ds2[h], y0, y1);
      if (kj > q0 + 2 * h) { x0 = 0.f; y0 = 0.f; }
      if (kj > q0 + 2 * h + 1) { x1 = 0.f; y1 = 0.f; }
      p2[h] = f2_pack(x0, x1);
      ds2[h] = f2_pack(y0, y1);
    }
  }
}

// Writes one key-block's dV rows and sigma * dK rows (this thread's key row, its column quarter)
// from tensor memory.
template <int D>
__device__ inline void store_dkdv(float* dvrow, float* dkrow, uint32_t t_dv, uint32_t t_dk,
                                  uint32_t lane_off, int qtr, float sigma) {
  uint32_t r[16];
#pragma unroll
  for (int cc = 0; cc < D / 64; ++cc) {  // this quarter's D/4 columns, 16 at a time
    const int c = qtr * (D / 64) + cc;
    tmem_ld16(t_dv + lane_off + c * 16, r);
    tmem_wait_ld();
#pragma unroll
    for (int e = 0; e < 16; e += 4)
      *reinterpret_cast<float4*>(dvrow + c * 16 + e) =
          make_float4(__uint_as_float(r[e]), __uint_as_float(r[e + 1]), __uint_as_float(r[e + 2]),
                      __uint_as_float(r[e + 3]));
    tmem_ld16(t_dk + lane_off + c * 16, r);
    tmem_wait_ld();
#pragma unroll
    for (int e = 0; e < 16; e += 4)
      *reinterpret_cast<float4*>(dkrow + c * 16 + e) =
          make_float4(__uint_as_float(r[e]) * sigma, __uint_as_float(r[e + 1]) * sigma,
                      __uint_as_float(r[e + 2]) * sigma, __uint_as_float(r[e + 3]) * sigma);
  }
}

// ------------------------------------------------------------------------------------ dK, dV
constexpr int kStQ = 4;  // Q/dO stages of the dK/dV kernel

template <int D>
struct LayDKV {
  static constexpr int KB = D / 64;
  static constexpr int K = 0;                     // [128][D]
  static constexpr int V = K + KB * T128;         // [128][D]
  static constexpr int Q = V + KB * T128;         // kStQ stages of [64][D]
  static constexpr int DO = Q + kStQ * KB * T64;  // kStQ stages of [64][D]
  static constexpr int VEC = DO + kStQ * KB * T64;  // kStQ stages of lse[64], delta[64]
  static constexpr int BAR = VEC + kStQ * 512;
  static constexpr int BYTES = BAR + 256;
};

// bars: 0 K+V | 1-4 Q/dO stages loaded | 5 S ready | 6 S read | 7 P written | 8 acc done
//       | 9-12 Q/dO stages free | 13-14 drain of the two MMA issuers
// TMEM columns: S^T 0-63, dP^T 64-127, dV 128.., dK 128+D.., P^T hi 384, lo 416, dS^T hi 448,
// lo 480 (64 queries as bf16 pairs: 32 columns each)
template <int D>
__global__ void __launch_bounds__(kThreads, 1)
attn_bwd_dkdv_tc(const __grid_constant__ CUtensorMap tk, const __grid_constant__ CUtensorMap tv,
                 const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tdo,
                 const float* __restrict__ lse, const float* __restrict__ delta,
                 float* __restrict__ dK, float* __restrict__ dV, int S, int BH, float sigma,
                 float scale_log2, uint32_t* status, uint64_t wait_ns) {
  using Ly = LayDKV<D>;
  constexpr int KB = Ly::KB;
  constexpr int kBars = 11 + kStQ;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
  uint64_t* bar = reinterpret_cast<uint64_t*>(sm + Ly::BAR);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar + kBars);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bar + kBars) + 1;
  uint64_t* const bar_kv = bar;
  uint64_t* const bar_st = bar + 1;        // + stage
  uint64_t* const bar_s = bar + 5;
  uint64_t* const bar_sfree = bar + 6;
  uint64_t* const bar_p = bar + 7;
  uint64_t* const bar_acc = bar + 8;
  uint64_t* const bar_stfree = bar + 9;    // + stage
  uint64_t* const bar_drain = bar + 9 + kStQ;  // + issuer

  const int tid = threadIdx.x, warp = tid / 32;
  const int kb = blockIdx.y;  // low key blocks see the most queries: heaviest first in a group
  const int bh = (int)blockIdx.z * kHeadGroup + (int)blockIdx.x;
  if (bh >= BH) return;  // the last group may be partial
  const int g0 = bh * S;
  const int k0 = kb * 128;
  const int nit = (S - k0) / 64;  // 64-row query blocks starting at k0

  if (tid == 0) {
    for (int i = 0; i < kBars; ++i) mbar_init(bar + i, (i == 6 || i == 7) ? kCompute / 32 : 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0) tmem_alloc(tmem_slot, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_slot;
  const uint32_t t_st = tbase, t_dpt = tbase + 64, t_dv = tbase + 128, t_dk = tbase + 128 + D;
  const uint32_t t_pt = tbase + 384, t_dst = tbase + 448;
  const uint32_t s_k = smem_u32(sm + Ly::K), s_v = smem_u32(sm + Ly::V);
  const uint32_t s_q = smem_u32(sm + Ly::Q), s_do = smem_u32(sm + Ly::DO);
  constexpr uint32_t IDESC_S = idesc_bf16(128, 64, false, false);
  constexpr uint32_t IDESC_ACC = idesc_bf16(128, D, false, true);

  if (warp == kCompute / 32) {
    // ------------------------------------------------------------------ TMA warp
    if ((tid % 32) == 0) {
      prefetch_tmap(&tk); prefetch_tmap(&tv); prefetch_tmap(&tq); prefetch_tmap(&tdo);
      auto load_stage = [&](int it) {  // Q, dO, lse, D of query block it into stage it % kStQ
        const int sg = it % kStQ;
        uint64_t* b = bar_st + sg;
        mbar_expect_tx(b, 2 * KB * T64 + 512);
        for (int c = 0; c < KB; ++c) {
          tma_load_2d(sm + Ly::Q + sg * KB * T64 + c * T64, &tq, c * 64, g0 + k0 + it * 64, b);
          tma_load_2d(sm + Ly::DO + sg * KB * T64 + c * T64, &tdo, c * 64, g0 + k0 + it * 64, b);
        }
        bulk_load(sm + Ly::VEC + sg * 512, lse + g0 + k0 + it * 64, 256, b);
        bulk_load(sm + Ly::VEC + sg * 512 + 256, delta + g0 + k0 + it * 64, 256, b);
      };
      mbar_expect_tx(bar_kv, 2 * KB * T128);
      for (int c = 0; c < KB; ++c) {
        tma_load_2d(sm + Ly::K + c * T128, &tk, c * 64, g0 + k0, bar_kv);
        tma_load_2d(sm + Ly::V + c * T128, &tv, c * 64, g0 + k0, bar_kv);
      }
      int issued = 0;
      for (int it = 0; it < nit; ++it) {  // step it reuses the stage of step it - kStQ
        if (it >= kStQ && !mbar_wait(bar_stfree + it % kStQ, ((it - kStQ) / kStQ) & 1, abort_flag, status, wait_ns)) break;
        load_stage(it);
        ++issued;
      }
      mbar_drain(bar_kv, 0, status);
      drain_ring(bar_st, kStQ, issued, status);
    }
  } else if (warp == kCompute / 32 + 1 || warp == kCompute / 32 + 2) {
    // ------------------------------------------------------------------ MMA warps
    // warp 17 issues S^T/dP^T, warp 18 the accumulations; neither waits on the other's barriers
    if ((tid % 32) == 0) {
      const bool s_issuer = warp == kCompute / 32 + 1;
      // K-major operands: LBO 16, SBO 1024; MN-major Q/dO stages: LBO = one [64][64] sub-tile
      const uint64_t dK_ = desc_base(16, 1024) + (s_k >> 4), dV_ = desc_base(16, 1024) + (s_v >> 4);
      const uint64_t dQk = desc_base(16, 1024) + (s_q >> 4), dOk = desc_base(16, 1024) + (s_do >> 4);
      const uint64_t dQm = desc_base(T64, 1024) + (s_q >> 4), dOm = desc_base(T64, 1024) + (s_do >> 4);
      auto issue_s = [&](int it) {  // S^T = K Q^T, dP^T = V dO^T
        const uint32_t sg = (uint32_t)((it % kStQ) * KB * T64) >> 4;
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          const uint32_t offA = ((ks / 4) * T128 + (ks % 4) * 32) >> 4, offB = ((ks / 4) * T64 + (ks % 4) * 32) >> 4;
          mma_ss(t_st, dK_ + offA, dQk + sg + offB, IDESC_S, ks > 0);
          mma_ss(t_dpt, dV_ + offA, dOk + sg + offB, IDESC_S, ks > 0);
        }
        mma_commit(bar_s);
      };
      auto issue_acc = [&](int it) {  // dV += (P^T_hi + P^T_lo) dO, dK += (dS^T_hi + dS^T_lo) Q
        const uint32_t sg = (uint32_t)((it % kStQ) * KB * T64) >> 4;
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) {
          const uint64_t bq = dQm + sg + ks * 128, bo = dOm + sg + ks * 128;  // + ks * 2048 bytes
          mma_ts(t_dv, t_pt + ks * 8, bo, IDESC_ACC, (it > 0 || ks > 0) ? 1u : 0u);
          mma_ts(t_dv, t_pt + 32 + ks * 8, bo, IDESC_ACC, 1u);
          mma_ts(t_dk, t_dst + ks * 8, bq, IDESC_ACC, (it > 0 || ks > 0) ? 1u : 0u);
          mma_ts(t_dk, t_dst + 32 + ks * 8, bq, IDESC_ACC, 1u);
        }
        mma_commit(bar_acc);
        mma_commit(bar_stfree + it % kStQ);  // the stage of step it is free once this completes
      };
      if (s_issuer) {
        bool ok = mbar_wait(bar_kv, 0, abort_flag, status, wait_ns);
        for (int n = 0; n < nit && ok; ++n) {  // S^T/dP^T of step n once the warps have read step n-1's
          ok = mbar_wait(bar_st + n % kStQ, (n / kStQ) & 1, abort_flag, status, wait_ns) &&
               (n == 0 || mbar_wait(bar_sfree, (n - 1) & 1, abort_flag, status, wait_ns));
          if (!ok) break;
          tc_fence_after();
          issue_s(n);
        }
        mma_drain(bar_drain, status);
      } else {
        for (int it = 0; it < nit; ++it) {
          if (!mbar_wait(bar_p, it & 1, abort_flag, status, wait_ns)) break;  // P^T, dS^T of step it
          tc_fence_after();
          issue_acc(it);  // its stage-free commit also covers S(it): P(it) exists only after S(it)
        }
        mma_drain(bar_drain + 1, status);
      }
    }
  } else {
    // ------------------------------------------------------------------ compute warps
    const uint32_t lane_off = (uint32_t)((warp % 4) * 32) << 16;  // this warp's lane quarter
    const int row = (warp % 4) * 32 + (tid % 32);  // key row within the block = TMEM lane
    const int qtr = warp / 4;                       // this thread's 16 of the step's 64 columns
    const int kj = k0 + row;
    auto wait_all = [&](uint64_t* b, uint32_t parity) {
      bool ok = mbar_wait(b, parity, abort_flag, status, wait_ns);
      return __all_sync(0xffffffffu, ok);
    };
    for (int it = 0; it < nit; ++it) {
      if (!wait_all(bar_s, it & 1)) break;
      if (!wait_all(bar_st + it % kStQ, (it / kStQ) & 1)) break;  // lse, D of this step (visibility)
      tc_fence_after();
      float st[16], dpt[16];
      {
        uint32_t r0[16], r2[16];
        tmem_ld16(t_st + lane_off + qtr * 16, r0);
        tmem_ld16(t_dpt + lane_off + qtr * 16, r2);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          st[e] = __uint_as_float(r0[e]);
          dpt[e] = __uint_as_float(r2[e]);
        }
      }
      tc_fence_before();
      __syncwarp();
      if ((tid % 32) == 0) mbar_arrive(bar_sfree);  // S^T / dP^T may be overwritten
      const float4* lv4 = reinterpret_cast<const float4*>(sm + Ly::VEC + (it % kStQ) * 512) + qtr * 4;
      const float4* dv4 = reinterpret_cast<const float4*>(sm + Ly::VEC + (it % kStQ) * 512 + 256) + qtr * 4;
      const int q0 = k0 + it * 64 + qtr * 16;
      uint64_t p2[8], ds2[8];
      kv_step_elements(st, dpt, lv4, dv4, scale_log2, kj, q0, q0 < k0 + 128, p2, ds2);
      uint32_t wp[8], wq[8], wh[8], wl[8];
#pragma unroll
      for (int h = 0; h < 8; ++h) {
        split_bf16x2_f2(p2[h], wp[h], wq[h]);
        split_bf16x2_f2(ds2[h], wh[h], wl[h]);
      }
      // the accumulate MMAs of the previous step read P^T and dS^T
      if (it > 0 && !wait_all(bar_acc, (it - 1) & 1)) break;
      tc_fence_after();
      tmem_st8(t_pt + lane_off + qtr * 8, wp);
      tmem_st8(t_pt + lane_off + 32 + qtr * 8, wq);
      tmem_st8(t_dst + lane_off + qtr * 8, wh);
      tmem_st8(t_dst + lane_off + 32 + qtr * 8, wl);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if ((tid % 32) == 0) mbar_arrive(bar_p);  // P^T, dS^T of step it are written
    }
    // ---- epilogue: dV, dK rows
    const bool ok_end = !*abort_flag && wait_all(bar_acc, (nit - 1) & 1);
    tc_fence_after();
    if (ok_end)
      store_dkdv<D>(dV + (size_t)(g0 + kj) * D, dK + (size_t)(g0 + kj) * D, t_dv, t_dk, lane_off, qtr, sigma);
  }
  // every role has drained its own loads and MMAs: nothing still writes shared or tensor memory
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tbase, 512);
}

// ------------------------------------------------------------------------------------ fused
constexpr int kStF = 3;  // Q/dO stages of the fused kernel (four do not fit beside the dS tile)

template <int D>
struct LayFused {
  static constexpr int KB = D / 64;
  static constexpr int K = 0;                      // [128][D]
  static constexpr int V = K + KB * T128;          // [128][D]
  static constexpr int Q = V + KB * T128;          // kStF stages of [64][D]
  static constexpr int DO = Q + kStF * KB * T64;   // kStF stages of [64][D]
  static constexpr int DS = DO + kStF * KB * T64;  // dS^T hi, then lo: [128 keys][64 queries] each
  static constexpr int VEC = DS + 2 * T128;        // kStF stages of lse[64], delta[64]
  static constexpr int BAR = VEC + kStF * 512;
  static constexpr int BYTES = BAR + 256;
};

// bars: 0 K+V | 1-3 Q/dO stages loaded | 4 S ready | 5 S read | 6 P written | 7 acc done
//       | 8-10 Q/dO stages free | 11-12 drain of the two MMA issuers
// TMEM columns: S^T 0-63, dP^T 64-127, dV 128-255, dK 256-383, P^T hi 384, lo 416 (64 queries
// as bf16 pairs), dQ^T 448-511 (lanes = the D columns of dQ, columns = the step's 64 queries)
template <int D>
__global__ void __launch_bounds__(kThreads, 1)
attn_bwd_fused_tc(const __grid_constant__ CUtensorMap tk, const __grid_constant__ CUtensorMap tv,
                  const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tdo,
                  const float* __restrict__ lse, const float* __restrict__ delta,
                  float* __restrict__ dQ, float* __restrict__ dK, float* __restrict__ dV, int S,
                  int BH, int kb0, int Sk, float sigma, float scale_log2, uint32_t* status,
                  uint64_t wait_ns) {
  static_assert(D == 128, "dQ^T = K^T dS^T takes M = D = 128 tensor-memory lanes");
  using Ly = LayFused<D>;
  constexpr int KB = Ly::KB;
  constexpr int kBars = 10 + kStF;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
  uint64_t* bar = reinterpret_cast<uint64_t*>(sm + Ly::BAR);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar + kBars);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bar + kBars) + 1;
  uint64_t* const bar_kv = bar;
  uint64_t* const bar_st = bar + 1;              // + stage
  uint64_t* const bar_s = bar + 1 + kStF;
  uint64_t* const bar_sfree = bar + 2 + kStF;
  uint64_t* const bar_p = bar + 3 + kStF;
  uint64_t* const bar_acc = bar + 4 + kStF;
  uint64_t* const bar_stfree = bar + 5 + kStF;   // + stage
  uint64_t* const bar_drain = bar + 5 + 2 * kStF;  // + issuer

  const int tid = threadIdx.x, warp = tid / 32;
  const int kb = blockIdx.y;  // low key blocks see the most queries: heaviest first in a group
  const int bh = (int)blockIdx.z * kHeadGroup + (int)blockIdx.x;
  if (bh >= BH) return;  // the last group may be partial
  // S query rows and Sk key rows per (b,h); the queries are the global rows 128 kb0 .. Sk - 1 of
  // the keys' sequence (kb0 = 0, Sk = S on one GPU; a context-parallel rank owns a later slice)
  const int g0 = bh * S;                   // first query row of this (b,h)
  const int gk0 = bh * Sk;                 // first key row of this (b,h)
  const int k0 = kb * 128;                 // first key of the block (global row)
  const int qs = k0 > kb0 * 128 ? k0 : kb0 * 128;  // first query that sees the block (global)
  const int ql0 = qs - kb0 * 128;          // ... as a row of this CTA's query rows
  const int nit = (Sk - qs) / 64;          // 64-row query blocks from qs

  if (tid == 0) {
    for (int i = 0; i < kBars; ++i)
      mbar_init(bar + i, (bar + i == bar_sfree || bar + i == bar_p) ? kCompute / 32 : 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0) tmem_alloc(tmem_slot, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_slot;
  const uint32_t t_st = tbase, t_dpt = tbase + 64, t_dv = tbase + 128, t_dk = tbase + 256;
  const uint32_t t_pt = tbase + 384, t_dqt = tbase + 448;
  const uint32_t s_k = smem_u32(sm + Ly::K), s_v = smem_u32(sm + Ly::V);
  const uint32_t s_q = smem_u32(sm + Ly::Q), s_do = smem_u32(sm + Ly::DO);
  const uint32_t s_ds = smem_u32(sm + Ly::DS);
  constexpr uint32_t IDESC_S = idesc_bf16(128, 64, false, false);
  constexpr uint32_t IDESC_ACC = idesc_bf16(128, D, false, true);
  constexpr uint32_t IDESC_DQ = idesc_bf16(128, 64, true, true);  // A = K^T, B = dS^T: both MN-major

  if (warp == kCompute / 32) {
    // ------------------------------------------------------------------ TMA warp
    if ((tid % 32) == 0) {
      prefetch_tmap(&tk); prefetch_tmap(&tv); prefetch_tmap(&tq); prefetch_tmap(&tdo);
      auto load_stage = [&](int it) {  // Q, dO, lse, D of query block it into stage it % kStF
        const int sg = it % kStF;
        uint64_t* b = bar_st + sg;
        mbar_expect_tx(b, 2 * KB * T64 + 512);
        for (int c = 0; c < KB; ++c) {
          tma_load_2d(sm + Ly::Q + sg * KB * T64 + c * T64, &tq, c * 64, g0 + ql0 + it * 64, b);
          tma_load_2d(sm + Ly::DO + sg * KB * T64 + c * T64, &tdo, c * 64, g0 + ql0 + it * 64, b);
        }
        bulk_load(sm + Ly::VEC + sg * 512, lse + g0 + ql0 + it * 64, 256, b);
        bulk_load(sm + Ly::VEC + sg * 512 + 256, delta + g0 + ql0 + it * 64, 256, b);
      };
      mbar_expect_tx(bar_kv, 2 * KB * T128);
      for (int c = 0; c < KB; ++c) {
        tma_load_2d(sm + Ly::K + c * T128, &tk, c * 64, gk0 + k0, bar_kv);
        tma_load_2d(sm + Ly::V + c * T128, &tv, c * 64, gk0 + k0, bar_kv);
      }
      int issued = 0;
      for (int it = 0; it < nit; ++it) {  // step it reuses the stage of step it - kStF
        if (it >= kStF && !mbar_wait(bar_stfree + it % kStF, ((it - kStF) / kStF) & 1, abort_flag, status, wait_ns)) break;
        load_stage(it);
        ++issued;
      }
      mbar_drain(bar_kv, 0, status);
      drain_ring(bar_st, kStF, issued, status);
    }
  } else if (warp == kCompute / 32 + 1 || warp == kCompute / 32 + 2) {
    // ------------------------------------------------------------------ MMA warps
    if ((tid % 32) == 0) {
      const bool s_issuer = warp == kCompute / 32 + 1;
      // K-major operands: LBO 16, SBO 1024. MN-major operands: LBO = the distance between the
      // 64-element halves of the M or N extent, SBO = 1024 between 8-row groups along K.
      const uint64_t dK_ = desc_base(16, 1024) + (s_k >> 4), dV_ = desc_base(16, 1024) + (s_v >> 4);
      const uint64_t dQk = desc_base(16, 1024) + (s_q >> 4), dOk = desc_base(16, 1024) + (s_do >> 4);
      const uint64_t dQm = desc_base(T64, 1024) + (s_q >> 4), dOm = desc_base(T64, 1024) + (s_do >> 4);
      const uint64_t dSk = desc_base(16, 1024) + (s_ds >> 4);     // dS^T as A of dK, K-major
      const uint64_t dSm = desc_base(T128, 1024) + (s_ds >> 4);   // dS^T as B of dQ^T (N = 64)
      const uint64_t dKm = desc_base(T128, 1024) + (s_k >> 4);    // K^T as A of dQ^T (M = 128)
      auto issue_s = [&](int it) {  // S^T = K Q^T, dP^T = V dO^T
        const uint32_t sg = (uint32_t)((it % kStF) * KB * T64) >> 4;
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          const uint32_t offA = ((ks / 4) * T128 + (ks % 4) * 32) >> 4, offB = ((ks / 4) * T64 + (ks % 4) * 32) >> 4;
          mma_ss(t_st, dK_ + offA, dQk + sg + offB, IDESC_S, ks > 0);
          mma_ss(t_dpt, dV_ + offA, dOk + sg + offB, IDESC_S, ks > 0);
        }
        mma_commit(bar_s);
      };
      auto issue_acc = [&](int it) {
        const uint32_t sg = (uint32_t)((it % kStF) * KB * T64) >> 4;
        // dV += (P^T_hi + P^T_lo) dO and dK += (dS^T_hi + dS^T_lo) Q, 16 queries per MMA
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) {
          const uint64_t bq = dQm + sg + ks * 128, bo = dOm + sg + ks * 128;  // + ks * 2048 bytes
          const uint32_t acc = (it > 0 || ks > 0) ? 1u : 0u;
          mma_ts(t_dv, t_pt + ks * 8, bo, IDESC_ACC, acc);
          mma_ts(t_dv, t_pt + 32 + ks * 8, bo, IDESC_ACC, 1u);
          mma_ss(t_dk, dSk + ks * 2, bq, IDESC_ACC, acc);                     // + ks * 32 bytes
          mma_ss(t_dk, dSk + (T128 >> 4) + ks * 2, bq, IDESC_ACC, 1u);
        }
        // dQ^T = K^T (dS^T_hi + dS^T_lo), 16 keys per MMA, fresh for this query block
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint64_t a = dKm + kk * 128, b = dSm + kk * 128;  // + kk * 2048 bytes
          mma_ss(t_dqt, a, b, IDESC_DQ, kk > 0 ? 1u : 0u);
          mma_ss(t_dqt, a, b + (T128 >> 4), IDESC_DQ, 1u);
        }
        mma_commit(bar_acc);
        mma_commit(bar_stfree + it % kStF);  // the stage of step it is free once this completes
      };
      if (s_issuer) {
        bool ok = mbar_wait(bar_kv, 0, abort_flag, status, wait_ns);
        for (int n = 0; n < nit && ok; ++n) {  // S^T/dP^T of step n once the warps have read step n-1's
          ok = mbar_wait(bar_st + n % kStF, (n / kStF) & 1, abort_flag, status, wait_ns) &&
               (n == 0 || mbar_wait(bar_sfree, (n - 1) & 1, abort_flag, status, wait_ns));
          if (!ok) break;
          tc_fence_after();
          issue_s(n);
        }
        mma_drain(bar_drain, status);
      } else {
        for (int it = 0; it < nit; ++it) {
          if (!mbar_wait(bar_p, it & 1, abort_flag, status, wait_ns)) break;  // P^T, dS^T of step it
          tc_fence_after();
          issue_acc(it);  // its stage-free commit also covers S(it): P(it) exists only after S(it)
        }
        mma_drain(bar_drain + 1, status);
      }
    }
  } else {
    // ------------------------------------------------------------------ compute warps
    const uint32_t lane_off = (uint32_t)((warp % 4) * 32) << 16;  // this warp's lane quarter
    const int row = (warp % 4) * 32 + (tid % 32);  // key row of S^T, and the dQ^T column d
    const int qtr = warp / 4;                       // this thread's 16 of the step's 64 columns
    const int kj = k0 + row;
    // this thread's two 16-byte chunks of the swizzled dS^T row (queries qtr*16 .. +15)
    uint8_t* const ds_row = sm + Ly::DS + (row >> 3) * 1024 + (row & 7) * 128;
    const int ch0 = ((2 * qtr) ^ (row & 7)) * 16, ch1 = ((2 * qtr + 1) ^ (row & 7)) * 16;
    auto wait_all = [&](uint64_t* b, uint32_t parity) {
      bool ok = mbar_wait(b, parity, abort_flag, status, wait_ns);
      return __all_sync(0xffffffffu, ok);
    };
    // adds sigma * dQ^T[row][qtr*16 + j] of step `it` to dq_sub (query rows, column row)
    auto add_dq = [&](int it, const uint32_t (&r)[16]) {
      float* p = dQ + (size_t)(g0 + ql0 + it * 64 + qtr * 16) * D + row;
#pragma unroll
      for (int j = 0; j < 16; ++j) red_add(p + (size_t)j * D, __uint_as_float(r[j]) * sigma);
    };
    uint32_t dqr[16];
    for (int it = 0; it < nit; ++it) {
      if (!wait_all(bar_s, it & 1)) break;
      if (!wait_all(bar_st + it % kStF, (it / kStF) & 1)) break;  // lse, D of this step (visibility)
      tc_fence_after();
      float st[16], dpt[16];
      {
        uint32_t r0[16], r2[16];
        tmem_ld16(t_st + lane_off + qtr * 16, r0);
        tmem_ld16(t_dpt + lane_off + qtr * 16, r2);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          st[e] = __uint_as_float(r0[e]);
          dpt[e] = __uint_as_float(r2[e]);
        }
      }
      tc_fence_before();
      __syncwarp();
      if ((tid % 32) == 0) mbar_arrive(bar_sfree);  // S^T / dP^T may be overwritten
      const float4* lv4 = reinterpret_cast<const float4*>(sm + Ly::VEC + (it % kStF) * 512) + qtr * 4;
      const float4* dv4 = reinterpret_cast<const float4*>(sm + Ly::VEC + (it % kStF) * 512 + 256) + qtr * 4;
      const int q0 = qs + it * 64 + qtr * 16;  // global query row of this thread's first column
      uint64_t p2[8], ds2[8];
      kv_step_elements(st, dpt, lv4, dv4, scale_log2, kj, q0, q0 < k0 + 128, p2, ds2);
      uint32_t wp[8], wq[8], wh[8], wl[8];
#pragma unroll
      for (int h = 0; h < 8; ++h) {
        split_bf16x2_f2(p2[h], wp[h], wq[h]);
        split_bf16x2_f2(ds2[h], wh[h], wl[h]);
      }
      // the accumulate MMAs of the previous step read P^T and dS^T and wrote dQ^T
      if (it > 0) {
        if (!wait_all(bar_acc, (it - 1) & 1)) break;
        tc_fence_after();
        tmem_ld16(t_dqt + lane_off + qtr * 16, dqr);  // dQ^T of step it-1, before step it's MMAs
        tmem_wait_ld();
      }
      tmem_st8(t_pt + lane_off + qtr * 8, wp);
      tmem_st8(t_pt + lane_off + 32 + qtr * 8, wq);
      *reinterpret_cast<uint4*>(ds_row + ch0) = make_uint4(wh[0], wh[1], wh[2], wh[3]);
      *reinterpret_cast<uint4*>(ds_row + ch1) = make_uint4(wh[4], wh[5], wh[6], wh[7]);
      *reinterpret_cast<uint4*>(ds_row + T128 + ch0) = make_uint4(wl[0], wl[1], wl[2], wl[3]);
      *reinterpret_cast<uint4*>(ds_row + T128 + ch1) = make_uint4(wl[4], wl[5], wl[6], wl[7]);
      tmem_wait_st();
      fence_async_smem();  // the dS^T stores, visible to the MMAs that read them
      tc_fence_before();
      __syncwarp();
      if ((tid % 32) == 0) mbar_arrive(bar_p);  // P^T, dS^T of step it are written
      if (it > 0) add_dq(it - 1, dqr);
    }
    // ---- epilogue: the last step's dQ, then the dV, dK rows
    const bool ok_end = !*abort_flag && wait_all(bar_acc, (nit - 1) & 1);
    tc_fence_after();
    if (ok_end) {
      tmem_ld16(t_dqt + lane_off + qtr * 16, dqr);
      tmem_wait_ld();
      add_dq(nit - 1, dqr);
      store_dkdv<D>(dV + (size_t)(gk0 + kj) * D, dK + (size_t)(gk0 + kj) * D, t_dv, t_dk, lane_off, qtr, sigma);
    }
  }
  // every role has drained its own loads and MMAs: nothing still writes shared or tensor memory
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tbase, 512);
}

// P^T of one thread's 16 queries for its key kj: exp2(S^T c - lse log2 e), zero where the key
// comes after the query (only on steps that reach the diagonal). Query pairs, lower in the low lane.
__device__ inline void p_elements(const uint32_t (&st)[16], const float* lse, float scale_log2, int kj,
                                  int q0, bool diag, uint64_t (&p2)[8]) {
  const uint64_t c2 = f2_pack(scale_log2, scale_log2);
#pragma unroll
  for (int c4 = 0; c4 < 4; ++c4) {
    const float4 lv = reinterpret_cast<const float4*>(lse)[c4];
    const uint64_t nla[2] = {f2_pack(-(lv.x * kLog2e), -(lv.y * kLog2e)),
                             f2_pack(-(lv.z * kLog2e), -(lv.w * kLog2e))};
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int h = c4 * 2 + e;
      float a0, a1;
      f2_unpack(f2_fma(f2_pack(__uint_as_float(st[2 * h]), __uint_as_float(st[2 * h + 1])), c2, nla[e]), a0, a1);
      p2[h] = f2_pack(ex2(a0), ex2(a1));
    }
  }
  if (diag) {
#pragma unroll
    for (int h = 0; h < 8; ++h) {
      float x0, x1;
      f2_unpack(p2[h], x0, x1);
      if (kj > q0 + 2 * h) x0 = 0.f;
      if (kj > q0 + 2 * h + 1) x1 = 0.f;
      p2[h] = f2_pack(x0, x1);
    }
  }
}

// dS^T = P^T (dP^T - D) for the same 16 queries, zero where the key comes after the query.
__device__ inline void ds_elements(const uint64_t (&p2)[8], const uint32_t (&dpt)[16], const float* dlt,
                                   int kj, int q0, bool diag, uint64_t (&ds2)[8]) {
#pragma unroll
  for (int c4 = 0; c4 < 4; ++c4) {
    const float4 dv = reinterpret_cast<const float4*>(dlt)[c4];
    const uint64_t da[2] = {f2_pack(dv.x, dv.y), f2_pack(dv.z, dv.w)};
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int h = c4 * 2 + e;
      ds2[h] = f2_mul(p2[h], f2_sub(f2_pack(__uint_as_float(dpt[2 * h]), __uint_as_float(dpt[2 * h + 1])), da[e]));
    }
  }
  if (diag) {
#pragma unroll
    for (int h = 0; h < 8; ++h) {
      float y0, y1;
      f2_unpack(ds2[h], y0, y1);
      if (kj > q0 + 2 * h) y0 = 0.f;
      if (kj > q0 + 2 * h + 1) y1 = 0.f;
      ds2[h] = f2_pack(y0, y1);
    }
  }
}

// ------------------------------------------------------------------------------------ fused, d = 64
// One pass at d = 64: one CTA per 128-key block steps through the 128-row query blocks that see it.
//   S^T = K Q^T and dP^T = V dO^T (N = 128 queries); P^T = exp2(S^T c - lse2) written over S^T in
//   tensor memory; dS^T = P^T (dP^T - D) into a shared-memory tile;
//   dV += P^T dO and dK += dS^T Q (N = d = 64, accumulated over the block);
//   dQ = dS K for the step's 128 queries (M = 128 queries, so no 64-row MMA), into one of two
//   tensor-memory buffers; the warps stage sigma dQ in shared memory (128-byte swizzled fp32
//   boxes of 32 columns) and one thread adds it into dq_sub with two TMA tensor reductions
//   (cp.reduce.async.bulk.tensor .add), so the atomic traffic runs in the copy engine while the
//   warps go on. dq_sub is zeroed by the D kernel first; the order of the key blocks' terms in a
//   dq_sub row varies from run to run, as in the d = 128 one-pass kernel.
template <int D>
struct LayFused64 {
  static constexpr int K = 0;                 // [128 keys][64]
  static constexpr int V = K + T128;          // [128 keys][64]
  static constexpr int ST = V + T128;         // two stages of Q [128][64], dO [128][64]
  static constexpr int DS = ST + 4 * T128;    // dS^T hi, then lo: [128 keys][128 queries] each
  static constexpr int STG = DS + 4 * T128;   // sigma dQ staging: two [128 rows][32 fp32] boxes
  static constexpr int VEC = STG + 2 * T128;  // two stages of lse[128], D[128]
  static constexpr int BAR = VEC + 2 * 1024;
  static constexpr int BYTES = BAR + 256;
};
static_assert(LayFused64<64>::BYTES + 1024 <= 232448, "d = 64 one-pass backward shared memory");

__device__ inline void tma_reduce_add_2d(const CUtensorMap* map, const void* src, int32_t x, int32_t y) {
  asm volatile("cp.reduce.async.bulk.tensor.2d.global.shared::cta.add.tile.bulk_group [%0, {%2, %3}], [%1];"
               ::"l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(src)), "r"(x), "r"(y) : "memory");
}
__device__ inline void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
__device__ inline void bulk_wait_read_all() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
__device__ inline void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }
__device__ inline void compute_sync() { asm volatile("bar.sync 1, %0;" ::"n"(kCompute) : "memory"); }

// bars: 0 K+V | 1-2 stages loaded | 3-4 stages free | 5 S^T done | 6 dP^T done | 7 P^T written
//       | 8 dS^T written | 9-10 dQ buffer done | 11-12 dQ buffer read | 13 dV done | 14 dK done
//       | 15 drain of the MMA issuer
// TMEM columns: S^T 0-127 (P^T written over it: 16 queries per 16 columns, hi then lo), dP^T
// 128-255, dV 256-319, dK 320-383, dQ buffers 384 and 448 (lanes = queries, columns = d).
template <int D>
__global__ void __launch_bounds__(kThreads, 1)
attn_bwd_fused64_tc(const __grid_constant__ CUtensorMap tk, const __grid_constant__ CUtensorMap tv,
                    const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tdo,
                    const __grid_constant__ CUtensorMap tdq, const float* __restrict__ lse,
                    const float* __restrict__ delta, float* __restrict__ dK, float* __restrict__ dV,
                    int S, int BH, float sigma, float scale_log2, uint32_t* status, uint64_t wait_ns) {
  static_assert(D == 64, "the d = 64 one-pass kernel");
  using Ly = LayFused64<D>;
  constexpr int kBars = 16;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
  uint64_t* bar = reinterpret_cast<uint64_t*>(sm + Ly::BAR);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar + kBars);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bar + kBars) + 1;
  uint64_t* const bar_kv = bar;
  uint64_t* const bar_st = bar + 1;      // + stage
  uint64_t* const bar_stfree = bar + 3;  // + stage
  uint64_t* const bar_s = bar + 5;
  uint64_t* const bar_dp = bar + 6;
  uint64_t* const bar_p = bar + 7;
  uint64_t* const bar_ds = bar + 8;
  uint64_t* const bar_dq = bar + 9;      // + buffer
  uint64_t* const bar_dqr = bar + 11;    // + buffer
  uint64_t* const bar_vdone = bar + 13;
  uint64_t* const bar_kdone = bar + 14;
  uint64_t* const bar_drain = bar + 15;

  const int tid = threadIdx.x, warp = tid / 32;
  const int kb = blockIdx.y;  // low key blocks see the most queries: heaviest first in a group
  const int bh = (int)blockIdx.z * kHeadGroup + (int)blockIdx.x;
  if (bh >= BH) return;  // the last group may be partial
  const int g0 = bh * S;         // first row of this (b,h)
  const int k0 = kb * 128;       // first key of the block; its first query block too
  const int nit = (S - k0) / 128;

  if (tid == 0) {
    for (int i = 0; i < kBars; ++i) {
      uint64_t* b = bar + i;
      mbar_init(b, (b == bar_p || b == bar_ds || b == bar_dqr || b == bar_dqr + 1) ? kCompute / 32 : 1);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0) tmem_alloc(tmem_slot, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_slot;
  const uint32_t t_s = tbase, t_dp = tbase + 128, t_dv = tbase + 256, t_dk = tbase + 320;
  const uint32_t t_dq = tbase + 384;  // + 64 * buffer
  constexpr uint32_t kLo = (2 * T128) >> 4;  // dS^T lo tile, in descriptor units

  if (warp == kCompute / 32) {
    // ------------------------------------------------------------------ TMA: K, V, then Q/dO stages
    if ((tid % 32) == 0) {
      prefetch_tmap(&tk); prefetch_tmap(&tv); prefetch_tmap(&tq); prefetch_tmap(&tdo);
      mbar_expect_tx(bar_kv, 2 * T128);
      tma_load_2d(sm + Ly::K, &tk, 0, g0 + k0, bar_kv);
      tma_load_2d(sm + Ly::V, &tv, 0, g0 + k0, bar_kv);
      int issued = 0;
      for (int j = 0; j < nit; ++j) {  // step j into stage j % 2 once dK(j - 2) is done
        if (j >= 2 && !mbar_wait(bar_stfree + (j & 1), ((j - 2) >> 1) & 1, abort_flag, status, wait_ns)) break;
        uint64_t* b = bar_st + (j & 1);
        uint8_t* stg = sm + Ly::ST + (j & 1) * 2 * T128;
        mbar_expect_tx(b, 2 * T128 + 1024);
        tma_load_2d(stg, &tq, 0, g0 + k0 + j * 128, b);
        tma_load_2d(stg + T128, &tdo, 0, g0 + k0 + j * 128, b);
        bulk_load(sm + Ly::VEC + (j & 1) * 1024, lse + g0 + k0 + j * 128, 512, b);
        bulk_load(sm + Ly::VEC + (j & 1) * 1024 + 512, delta + g0 + k0 + j * 128, 512, b);
        ++issued;
      }
      mbar_drain(bar_kv, 0, status);
      drain_ring(bar_st, 2, issued, status);
    }
  } else if (warp == kCompute / 32 + 1) {
    // ------------------------------------------------------------------ MMA issuer
    if ((tid % 32) == 0) {
      const uint32_t s_k = smem_u32(sm + Ly::K), s_v = smem_u32(sm + Ly::V);
      const uint32_t s_st = smem_u32(sm + Ly::ST), s_ds = smem_u32(sm + Ly::DS);
      // K-major: LBO 16, SBO 1024. MN-major: LBO = the distance between 64-element halves of the
      // M or N extent (one [128][64] sub-tile), SBO = 1024 between 8-row groups along K.
      const uint64_t aK = desc_base(16, 1024) + (s_k >> 4), aV = desc_base(16, 1024) + (s_v >> 4);
      const uint64_t bKm = desc_base(T128, 1024) + (s_k >> 4);  // K as B of dQ (N = d), MN-major
      const uint64_t bStK = desc_base(16, 1024) + (s_st >> 4);   // Q, dO as B of S^T, dP^T
      const uint64_t bStM = desc_base(T128, 1024) + (s_st >> 4); // Q, dO as B of dK, dV (N = d)
      const uint64_t aSk = desc_base(16, 1024) + (s_ds >> 4);    // dS^T as A of dK, K-major
      const uint64_t aSm = desc_base(T128, 1024) + (s_ds >> 4);  // dS as A of dQ (M = queries), MN-major
      constexpr uint32_t IDESC_S = idesc_bf16(128, 128, false, false);
      constexpr uint32_t IDESC_ACC = idesc_bf16(128, D, false, true);
      constexpr uint32_t IDESC_DQ = idesc_bf16(128, D, true, true);
      auto stage = [](int j, int which) { return (uint32_t)(((j & 1) * 2 + which) * T128) >> 4; };
      auto issue_s = [&](int j) {  // S^T = K Q^T
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks)
          mma_ss(t_s, aK + ks * 2, bStK + stage(j, 0) + ks * 2, IDESC_S, ks > 0);  // + ks * 32 bytes
        mma_commit(bar_s);
      };
      auto issue_dp = [&](int j) {  // dP^T = V dO^T
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks)
          mma_ss(t_dp, aV + ks * 2, bStK + stage(j, 1) + ks * 2, IDESC_S, ks > 0);
        mma_commit(bar_dp);
      };
      auto issue_dv = [&](int j) {  // dV += (P^T_hi + P^T_lo) dO, 16 queries per MMA
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
          const uint64_t b = bStM + stage(j, 1) + ks * 128;  // + ks * 2048 bytes: 16 query rows
          mma_ts(t_dv, t_s + ks * 16, b, IDESC_ACC, (j > 0 || ks > 0) ? 1u : 0u);
          mma_ts(t_dv, t_s + ks * 16 + 8, b, IDESC_ACC, 1u);
        }
        mma_commit(bar_vdone);  // P^T's columns are free once this completes
      };
      auto issue_dq = [&](int j) {  // dQ = (dS_hi + dS_lo) K, 16 keys per MMA, fresh each step
        const uint32_t t = t_dq + (j & 1) * 64;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint64_t a = aSm + kk * 128, b = bKm + kk * 128;  // + kk * 2048 bytes: 16 keys
          mma_ss(t, a, b, IDESC_DQ, kk > 0 ? 1u : 0u);
          mma_ss(t, a + kLo, b, IDESC_DQ, 1u);
        }
        mma_commit(bar_dq + (j & 1));
      };
      auto issue_dk = [&](int j) {  // dK += (dS^T_hi + dS^T_lo) Q
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
          const uint64_t b = bStM + stage(j, 0) + ks * 128;
          const uint32_t offA = ((ks / 4) * T128 + (ks % 4) * 32) >> 4;
          mma_ss(t_dk, aSk + offA, b, IDESC_ACC, (j > 0 || ks > 0) ? 1u : 0u);
          mma_ss(t_dk, aSk + offA + kLo, b, IDESC_ACC, 1u);
        }
        mma_commit(bar_stfree + (j & 1));  // the stage of step j is free once this completes
        mma_commit(bar_kdone);
      };
      // Per step j: dV(j); S^T(j+1) once dV(j) has read P^T(j); dP^T(j+1) once the warps have
      // read dP^T(j); then dQ(j) and dK(j), which fill the pipe while the warps start step j+1.
      bool ok = mbar_wait(bar_kv, 0, abort_flag, status, wait_ns) &&
                mbar_wait(bar_st, 0, abort_flag, status, wait_ns);
      if (ok) {
        tc_fence_after();
        issue_s(0);
        issue_dp(0);
      }
      for (int j = 0; j < nit && ok; ++j) {
        if (!mbar_wait(bar_p, j & 1, abort_flag, status, wait_ns)) break;
        tc_fence_after();
        issue_dv(j);
        if (j + 1 < nit) {
          if (!mbar_wait(bar_st + ((j + 1) & 1), ((j + 1) >> 1) & 1, abort_flag, status, wait_ns) ||
              !mbar_wait(bar_vdone, j & 1, abort_flag, status, wait_ns))
            break;
          tc_fence_after();
          issue_s(j + 1);
        }
        if (!mbar_wait(bar_ds, j & 1, abort_flag, status, wait_ns)) break;  // dS^T(j); dP^T(j) read
        tc_fence_after();
        if (j + 1 < nit) issue_dp(j + 1);
        if (j >= 2 && !mbar_wait(bar_dqr + (j & 1), ((j - 2) >> 1) & 1, abort_flag, status, wait_ns)) break;
        tc_fence_after();
        issue_dq(j);
        issue_dk(j);
      }
      mma_drain(bar_drain, status);
    }
  } else if (warp < kCompute / 32) {
    // ------------------------------------------------------------------ compute warps
    const uint32_t lane_off = (uint32_t)((warp % 4) * 32) << 16;  // this warp's lane quarter
    const int row = (warp % 4) * 32 + (tid % 32);  // key row of S^T; query row of dQ
    const int qtr = warp / 4;                       // this thread's 32 of the step's 128 queries
    const int kj = k0 + row;
    uint8_t* const ds_row = sm + Ly::DS + (qtr >> 1) * T128 + (row >> 3) * 1024 + (row & 7) * 128;
    const int cb = (qtr & 1) * 4;
    // this thread's 16 columns of sigma dQ in the staging box qtr / 2 (32 fp32 per 128-byte row)
    uint8_t* const stg_row = sm + Ly::STG + (qtr >> 1) * T128 + row * 128;
    auto wait_all = [&](uint64_t* b, uint32_t parity) {
      bool w = mbar_wait(b, parity, abort_flag, status, wait_ns);
      return __all_sync(0xffffffffu, w);
    };
    // dQ of step i: read it, stage sigma dQ, and add it into dq_sub rows with the copy engine.
    // Every compute warp reaches both barriers whatever `ok` is, so none waits alone.
    auto flush_dq = [&](int i, bool& ok) {
      uint32_t r[16];
      ok = ok && wait_all(bar_dq + (i & 1), (i >> 1) & 1);
      tc_fence_after();
      if (ok) {
        tmem_ld16(t_dq + (i & 1) * 64 + lane_off + qtr * 16, r);
        tmem_wait_ld();
      }
      tc_fence_before();
      __syncwarp();
      if (ok && (tid % 32) == 0) mbar_arrive(bar_dqr + (i & 1));
      if (tid == 0) bulk_wait_read_all();  // the previous reduction has read the staging
      compute_sync();
      if (ok) {
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const int ch = (cb + c) ^ (row & 7);
          *reinterpret_cast<float4*>(stg_row + ch * 16) =
              make_float4(__uint_as_float(r[4 * c]) * sigma, __uint_as_float(r[4 * c + 1]) * sigma,
                          __uint_as_float(r[4 * c + 2]) * sigma, __uint_as_float(r[4 * c + 3]) * sigma);
        }
      }
      fence_async_smem();  // the staging stores, visible to the copy engine
      compute_sync();
      if (ok && tid == 0) {
        tma_reduce_add_2d(&tdq, sm + Ly::STG, 0, g0 + k0 + i * 128);
        tma_reduce_add_2d(&tdq, sm + Ly::STG + T128, 32, g0 + k0 + i * 128);
        bulk_commit();
      }
    };
    bool ok = true;
    for (int j = 0; j < nit; ++j) {
      const int q0 = k0 + j * 128 + qtr * 32;  // query row of this thread's first column
      const bool diag = j == 0;                // the first step holds the diagonal block
      const float* vec = reinterpret_cast<const float*>(sm + Ly::VEC + (j & 1) * 1024);
      // P^T, written over this thread's S^T columns
      ok = ok && wait_all(bar_s, j & 1) && wait_all(bar_st + (j & 1), (j >> 1) & 1);
      tc_fence_after();
      uint64_t p2[2][8];
      if (ok) {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          uint32_t r[16];
          tmem_ld16(t_s + lane_off + qtr * 32 + h * 16, r);
          tmem_wait_ld();
          p_elements(r, vec + qtr * 32 + h * 16, scale_log2, kj, q0 + h * 16, diag, p2[h]);
          uint32_t wp[8], wq[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) split_bf16x2_f2(p2[h][e], wp[e], wq[e]);
          tmem_st8(t_s + lane_off + (2 * qtr + h) * 16, wp);
          tmem_st8(t_s + lane_off + (2 * qtr + h) * 16 + 8, wq);
        }
        tmem_wait_st();
      }
      tc_fence_before();
      __syncwarp();
      if (ok && (tid % 32) == 0) mbar_arrive(bar_p);
      // dS^T into shared memory, once dQ(j-1) and dK(j-1) have read the previous one
      ok = ok && wait_all(bar_dp, j & 1) && (j == 0 || wait_all(bar_kdone, (j - 1) & 1));
      tc_fence_after();
      if (ok) {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          uint32_t r[16];
          tmem_ld16(t_dp + lane_off + qtr * 32 + h * 16, r);
          tmem_wait_ld();
          uint64_t ds2[8];
          ds_elements(p2[h], r, vec + 128 + qtr * 32 + h * 16, kj, q0 + h * 16, diag, ds2);
          uint32_t wh[8], wl[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) split_bf16x2_f2(ds2[e], wh[e], wl[e]);
          const int c0 = ((cb + 2 * h) ^ (row & 7)) * 16, c1 = ((cb + 2 * h + 1) ^ (row & 7)) * 16;
          *reinterpret_cast<uint4*>(ds_row + c0) = make_uint4(wh[0], wh[1], wh[2], wh[3]);
          *reinterpret_cast<uint4*>(ds_row + c1) = make_uint4(wh[4], wh[5], wh[6], wh[7]);
          *reinterpret_cast<uint4*>(ds_row + 2 * T128 + c0) = make_uint4(wl[0], wl[1], wl[2], wl[3]);
          *reinterpret_cast<uint4*>(ds_row + 2 * T128 + c1) = make_uint4(wl[4], wl[5], wl[6], wl[7]);
        }
      }
      fence_async_smem();  // the dS^T stores, visible to the MMAs that read them
      tc_fence_before();
      __syncwarp();
      if (ok && (tid % 32) == 0) mbar_arrive(bar_ds);
      if (j > 0) flush_dq(j - 1, ok);
    }
    flush_dq(nit - 1, ok);
    // ---- epilogue: dV, dK rows (dK(nit-1) is the CTA's last MMA)
    ok = ok && !*abort_flag && wait_all(bar_kdone, (nit - 1) & 1);
    tc_fence_after();
    if (ok)
      store_dkdv<D>(dV + (size_t)(g0 + kj) * D, dK + (size_t)(g0 + kj) * D, t_dv, t_dk, lane_off, qtr, sigma);
    if (tid == 0) bulk_wait_all();  // every reduction has finished reading the staging
  }
  // every role has drained its own loads and MMAs: nothing still writes shared or tensor memory
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tbase, 512);
}

// ------------------------------------------------------------------------------------ dQ
constexpr int kStK = 4;  // K/V stages of the dQ kernel

template <int D>
struct LayDQ {
  static constexpr int KB = D / 64;
  static constexpr int Q = 0;                    // [128][D]
  static constexpr int DO = Q + KB * T128;       // [128][D]
  static constexpr int K = DO + KB * T128;       // kStK stages of [64][D]
  static constexpr int V = K + kStK * KB * T64;  // kStK stages of [64][D]
  static constexpr int BAR = V + kStK * KB * T64;
  static constexpr int BYTES = BAR + 256;
};

// bars: 0 Q+dO | 1-4 K/V stages | 5-6 S buffers | 7-8 S buffers free | 9 dS written | 10-11 acc
//       | 12-15 K/V stages free | 16-17 drain of the two MMA issuers
// TMEM columns: S / dP buffer b at 128b / 128b + 64, dQ at 256, dS hi at 384, lo at 416
template <int D>
__global__ void __launch_bounds__(kThreads, 1)
attn_bwd_dq_tc(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tdo,
               const __grid_constant__ CUtensorMap tk, const __grid_constant__ CUtensorMap tv,
               const float* __restrict__ lse, const float* __restrict__ delta,
               float* __restrict__ dQ, int S, int BH, float sigma, float scale_log2, uint32_t* status,
               uint64_t wait_ns) {
  using Ly = LayDQ<D>;
  constexpr int KB = Ly::KB;
  constexpr int kBars = 18;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
  uint64_t* bar = reinterpret_cast<uint64_t*>(sm + Ly::BAR);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar + kBars);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bar + kBars) + 1;

  const int tid = threadIdx.x, warp = tid / 32;
  const int nqb = S / 128;
  const int qb = nqb - 1 - (int)blockIdx.y;  // heaviest blocks first within a head group
  const int bh = (int)blockIdx.z * kHeadGroup + (int)blockIdx.x;
  if (bh >= BH) return;  // the last group may be partial
  const int g0 = bh * S;
  const int q0 = qb * 128;
  const int nit = (q0 + 128) / 64;  // 64-row key blocks up to the diagonal

  if (tid == 0) {
    for (int i = 0; i < kBars; ++i) mbar_init(bar + i, (i == 7 || i == 8 || i == 9) ? kCompute / 32 : 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0) tmem_alloc(tmem_slot, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_slot;
  const uint32_t t_dq = tbase + 256, t_ds = tbase + 384;
  const uint32_t s_q = smem_u32(sm + Ly::Q), s_do = smem_u32(sm + Ly::DO);
  const uint32_t s_k = smem_u32(sm + Ly::K), s_v = smem_u32(sm + Ly::V);
  constexpr uint32_t IDESC_S = idesc_bf16(128, 64, false, false);
  constexpr uint32_t IDESC_ACC = idesc_bf16(128, D, false, true);

  if (warp == kCompute / 32) {
    // ------------------------------------------------------------------ TMA warp
    if ((tid % 32) == 0) {
      prefetch_tmap(&tq); prefetch_tmap(&tdo); prefetch_tmap(&tk); prefetch_tmap(&tv);
      auto load_kv = [&](int it) {  // K, V of key block it into stage it % kStK
        const int sg = it % kStK;
        uint64_t* b = bar + 1 + sg;
        mbar_expect_tx(b, 2 * KB * T64);
        for (int c = 0; c < KB; ++c) {
          tma_load_2d(sm + Ly::K + sg * KB * T64 + c * T64, &tk, c * 64, g0 + it * 64, b);
          tma_load_2d(sm + Ly::V + sg * KB * T64 + c * T64, &tv, c * 64, g0 + it * 64, b);
        }
      };
      mbar_expect_tx(bar, 2 * KB * T128);
      for (int c = 0; c < KB; ++c) {
        tma_load_2d(sm + Ly::Q + c * T128, &tq, c * 64, g0 + q0, bar);
        tma_load_2d(sm + Ly::DO + c * T128, &tdo, c * 64, g0 + q0, bar);
      }
      int issued = 0;
      for (int it = 0; it < nit; ++it) {  // step it reuses the stage of step it - kStK
        if (it >= kStK && !mbar_wait(bar + 12 + it % kStK, ((it - kStK) / kStK) & 1, abort_flag, status, wait_ns)) break;
        load_kv(it);
        ++issued;
      }
      mbar_drain(bar, 0, status);
      drain_ring(bar + 1, kStK, issued, status);
    }
  } else if (warp == kCompute / 32 + 1 || warp == kCompute / 32 + 2) {
    // ------------------------------------------------------------------ MMA warps
    // warp 17 issues S/dP, warp 18 the accumulations
    if ((tid % 32) == 0) {
      const bool s_issuer = warp == kCompute / 32 + 1;
      const uint64_t dQ_ = desc_base(16, 1024) + (s_q >> 4), dO_ = desc_base(16, 1024) + (s_do >> 4);
      const uint64_t dKk = desc_base(16, 1024) + (s_k >> 4), dVk = desc_base(16, 1024) + (s_v >> 4);
      const uint64_t dKm = desc_base(T64, 1024) + (s_k >> 4);
      auto issue_s = [&](int it) {  // S = Q K^T, dP = dO V^T into TMEM buffer it & 1
        const uint32_t sg = (uint32_t)((it % kStK) * KB * T64) >> 4;
        const uint32_t t_s = tbase + (it & 1) * 128, t_dp = t_s + 64;
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          const uint32_t offA = ((ks / 4) * T128 + (ks % 4) * 32) >> 4, offB = ((ks / 4) * T64 + (ks % 4) * 32) >> 4;
          mma_ss(t_s, dQ_ + offA, dKk + sg + offB, IDESC_S, ks > 0);
          mma_ss(t_dp, dO_ + offA, dVk + sg + offB, IDESC_S, ks > 0);
        }
        mma_commit(bar + 5 + (it & 1));
      };
      auto issue_acc = [&](int it) {  // dQ += (dS_hi + dS_lo) K, dS from tensor memory
        const uint32_t sg = (uint32_t)((it % kStK) * KB * T64) >> 4;
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) {
          const uint64_t bk = dKm + sg + ks * 128;  // + ks * 2048 bytes
          mma_ts(t_dq, t_ds + ks * 8, bk, IDESC_ACC, (it > 0 || ks > 0) ? 1u : 0u);
          mma_ts(t_dq, t_ds + 32 + ks * 8, bk, IDESC_ACC, 1u);
        }
        mma_commit(bar + 10 + (it & 1));
        mma_commit(bar + 12 + it % kStK);  // the stage of step it is free once this completes
      };
      if (s_issuer) {
        bool ok = mbar_wait(bar, 0, abort_flag, status, wait_ns);
        for (int n = 0; n < nit && ok; ++n) {  // S/dP of step n into buffer n & 1 once it is free
          ok = mbar_wait(bar + 1 + n % kStK, (n / kStK) & 1, abort_flag, status, wait_ns);
          if (ok && n >= 2) ok = mbar_wait(bar + 7 + (n & 1), ((n >> 1) - 1) & 1, abort_flag, status, wait_ns);
          if (!ok) break;
          tc_fence_after();
          issue_s(n);
        }
        mma_drain(bar + 16, status);
      } else {
        for (int it = 0; it < nit; ++it) {
          if (!mbar_wait(bar + 9, it & 1, abort_flag, status, wait_ns)) break;  // dS of step it
          tc_fence_after();
          issue_acc(it);  // its stage-free commit also covers S(it): dS(it) exists only after S(it)
        }
        mma_drain(bar + 17, status);
      }
    }
  } else {
    // ------------------------------------------------------------------ compute warps
    const uint32_t lane_off = (uint32_t)((warp % 4) * 32) << 16;  // this warp's lane quarter
    const int row = (warp % 4) * 32 + (tid % 32);  // query row within the block = TMEM lane
    const int qtr = warp / 4;                       // this thread's 16 of the step's 64 columns
    const int qi = q0 + row;
    const float l2 = lse[g0 + qi] * kLog2e;
    const float dl = delta[g0 + qi];
    auto wait_all = [&](uint64_t* b, uint32_t parity) {
      bool ok = mbar_wait(b, parity, abort_flag, status, wait_ns);
      return __all_sync(0xffffffffu, ok);
    };
    for (int it = 0; it < nit; ++it) {
      if (!wait_all(bar + 5 + (it & 1), (it >> 1) & 1)) break;
      tc_fence_after();
      float s[16], dp[16];
      {
        uint32_t r0[16], r2[16];
        const uint32_t t_s = tbase + (it & 1) * 128, t_dp = t_s + 64;
        tmem_ld16(t_s + lane_off + qtr * 16, r0);
        tmem_ld16(t_dp + lane_off + qtr * 16, r2);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          s[e] = __uint_as_float(r0[e]);
          dp[e] = __uint_as_float(r2[e]);
        }
      }
      tc_fence_before();
      __syncwarp();
      if ((tid % 32) == 0) mbar_arrive(bar + 7 + (it & 1));  // this S buffer may be overwritten
      const int kj0 = it * 64 + qtr * 16;
      uint64_t ds2[8];  // key pairs (2h, 2h+1), one f32x2 instruction per pair
      {
        const uint64_t c2 = f2_pack(scale_log2, scale_log2), nl2 = f2_pack(-l2, -l2), dl2 = f2_pack(dl, dl);
#pragma unroll
        for (int h = 0; h < 8; ++h) {
          float a0, a1;
          f2_unpack(f2_fma(f2_pack(s[2 * h], s[2 * h + 1]), c2, nl2), a0, a1);
          ds2[h] = f2_mul(f2_pack(ex2(a0), ex2(a1)), f2_sub(f2_pack(dp[2 * h], dp[2 * h + 1]), dl2));
        }
      }
      if (kj0 + 16 > q0) {  // steps that reach the diagonal: keys after the query are invisible
#pragma unroll
        for (int h = 0; h < 8; ++h) {
          float y0, y1;
          f2_unpack(ds2[h], y0, y1);
          if (kj0 + 2 * h > qi) y0 = 0.f;
          if (kj0 + 2 * h + 1 > qi) y1 = 0.f;
          ds2[h] = f2_pack(y0, y1);
        }
      }
      uint32_t wh[8], wl[8];  // dS = hi + lo: this quarter's 16 keys as 8 columns of pairs each
#pragma unroll
      for (int h = 0; h < 8; ++h) split_bf16x2_f2(ds2[h], wh[h], wl[h]);
      // the accumulate MMAs of the previous step read dS
      if (it > 0 && !wait_all(bar + 10 + ((it - 1) & 1), ((it - 1) >> 1) & 1)) break;
      tc_fence_after();
      tmem_st8(t_ds + lane_off + qtr * 8, wh);
      tmem_st8(t_ds + lane_off + 32 + qtr * 8, wl);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if ((tid % 32) == 0) mbar_arrive(bar + 9);  // dS of step it is written
    }
    const bool ok_end = !*abort_flag && wait_all(bar + 10 + ((nit - 1) & 1), ((nit - 1) >> 1) & 1);
    tc_fence_after();
    if (ok_end) {
      float* dqrow = dQ + (size_t)(g0 + qi) * D;
      uint32_t r[16];
#pragma unroll
      for (int cc = 0; cc < D / 64; ++cc) {  // this quarter's D/4 columns, 16 at a time
        const int c = qtr * (D / 64) + cc;
        tmem_ld16(t_dq + lane_off + c * 16, r);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 16; e += 4)
          *reinterpret_cast<float4*>(dqrow + c * 16 + e) =
              make_float4(__uint_as_float(r[e]) * sigma, __uint_as_float(r[e + 1]) * sigma,
                          __uint_as_float(r[e + 2]) * sigma, __uint_as_float(r[e + 3]) * sigma);
      }
    }
  }
  // every role has drained its own loads and MMAs: nothing still writes shared or tensor memory
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tbase, 512);
}

// D_i = dO_sub[i] . O_sub[i] (fp32 O_sub); one warp per row. If dq is given, the row of dq is
// zeroed too (the fused kernel adds into it).
__global__ void delta_kernel(const float* __restrict__ O, const __nv_bfloat16* __restrict__ dO,
                             float* __restrict__ delta, float* __restrict__ dq, int64_t rows, int D) {
  const int64_t row = (int64_t)blockIdx.x * (blockDim.x / 32) + threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  if (row >= rows) return;
  float acc = 0.f;
  for (int c = lane * 4; c < D; c += 128) {
    const float4 o = *reinterpret_cast<const float4*>(O + row * D + c);
    const __nv_bfloat162 a = *reinterpret_cast<const __nv_bfloat162*>(dO + row * D + c);
    const __nv_bfloat162 b = *reinterpret_cast<const __nv_bfloat162*>(dO + row * D + c + 2);
    acc = fmaf(o.x, __low2float(a), acc);
    acc = fmaf(o.y, __high2float(a), acc);
    acc = fmaf(o.z, __low2float(b), acc);
    acc = fmaf(o.w, __high2float(b), acc);
    if (dq) *reinterpret_cast<float4*>(dq + row * D + c) = make_float4(0.f, 0.f, 0.f, 0.f);
  }
#pragma unroll
  for (int o2 = 16; o2 >= 1; o2 >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o2);
  if (lane == 0) delta[row] = acc;
}

// both kernels of a pass hold all 512 TMEM columns: padded so that two CTAs never share an SM
int padded_smem(int bytes) { return bytes + 1024 > 120 * 1024 ? bytes + 1024 : 120 * 1024; }

template <int D>
cudaError_t run_bwd(const Geo& g, const void* qs, const void* ks, const void* vs, const float* os,
                    const float* lse, const void* dos, float* dq, float* dk, float* dv, float* delta,
                    uint32_t* status, cudaStream_t st) {
  const bool fused = !(g.flags & LH_DETERMINISTIC);
  const int64_t rows = g.BH * g.S;
  CUtensorMap q64, do64, k128, v128;
  if (!make_tmap_rows_box(&q64, qs, rows, D, 64) || !make_tmap_rows_box(&do64, dos, rows, D, 64) ||
      !make_tmap_rows_box(&k128, ks, rows, D, 128) || !make_tmap_rows_box(&v128, vs, rows, D, 128))
    return cudaErrorInvalidValue;
  delta_kernel<<<(unsigned)((rows + 7) / 8), 256, 0, st>>>(os, (const __nv_bfloat16*)dos, delta,
                                                           fused ? dq : nullptr, rows, D);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const float sigma = 1.0f / sqrtf((float)D);
  const float scale_log2 = sigma * kLog2e;
  const dim3 grid((unsigned)(g.BH < kHeadGroup ? g.BH : kHeadGroup), (unsigned)(g.S / 128),
                  (unsigned)((g.BH + kHeadGroup - 1) / kHeadGroup));
  if constexpr (D == 64) {
    if (fused) {
      CUtensorMap q128f, do128f, dq32;
      if (!make_tmap_rows_box(&q128f, qs, rows, D, 128) || !make_tmap_rows_box(&do128f, dos, rows, D, 128) ||
          !make_tmap_f32_box(&dq32, dq, rows, D, 128))
        return cudaErrorInvalidValue;
      const int smem = padded_smem(LayFused64<D>::BYTES);
      e = cudaFuncSetAttribute(attn_bwd_fused64_tc<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
      if (e != cudaSuccess) return e;
      attn_bwd_fused64_tc<D><<<grid, kThreads, smem, st>>>(k128, v128, q128f, do128f, dq32, lse, delta, dk, dv,
                                                            g.S, (int)g.BH, sigma, scale_log2, status,
                                                            g.wait_ns);
      return cudaGetLastError();
    }
  }
  if constexpr (D == 128) {
    if (fused) {
      const int smem = padded_smem(LayFused<D>::BYTES);
      e = cudaFuncSetAttribute(attn_bwd_fused_tc<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
      if (e != cudaSuccess) return e;
      attn_bwd_fused_tc<D><<<grid, kThreads, smem, st>>>(k128, v128, q64, do64, lse, delta, dq, dk, dv,
                                                          g.S, (int)g.BH, 0, g.S, sigma, scale_log2, status,
                                                          g.wait_ns);
      return cudaGetLastError();
    }
  }
  const int smem1 = padded_smem(LayDKV<D>::BYTES);
  e = cudaFuncSetAttribute(attn_bwd_dkdv_tc<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem1);
  if (e != cudaSuccess) return e;
  attn_bwd_dkdv_tc<D><<<grid, kThreads, smem1, st>>>(
      k128, v128, q64, do64, lse, delta, dk, dv, g.S, (int)g.BH, sigma, scale_log2, status, g.wait_ns);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  CUtensorMap q128, do128, k64, v64;
  if (!make_tmap_rows_box(&q128, qs, rows, D, 128) || !make_tmap_rows_box(&do128, dos, rows, D, 128) ||
      !make_tmap_rows_box(&k64, ks, rows, D, 64) || !make_tmap_rows_box(&v64, vs, rows, D, 64))
    return cudaErrorInvalidValue;
  const int smem2 = padded_smem(LayDQ<D>::BYTES);
  e = cudaFuncSetAttribute(attn_bwd_dq_tc<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem2);
  if (e != cudaSuccess) return e;
  attn_bwd_dq_tc<D><<<grid, kThreads, smem2, st>>>(
      q128, do128, k64, v64, lse, delta, dq, g.S, (int)g.BH, sigma, scale_log2, status, g.wait_ns);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attn_bwd_tc_rows(const Geo& g, int kb0, int Sk, const void* qs, const void* ks,
                                    const void* vs, const float* os, const float* lse,
                                    const void* dos, float* dq, float* dk, float* dv, float* delta,
                                    uint32_t* status, cudaStream_t st) {
  if (g.d != 128) return cudaErrorNotSupported;  // the one-pass kernel takes d = 128
  constexpr int D = 128;
  const int64_t rows = g.BH * g.S, krows = g.BH * (int64_t)Sk;
  CUtensorMap q64, do64, k128, v128;
  if (!make_tmap_rows_box(&q64, qs, rows, D, 64) || !make_tmap_rows_box(&do64, dos, rows, D, 64) ||
      !make_tmap_rows_box(&k128, ks, krows, D, 128) || !make_tmap_rows_box(&v128, vs, krows, D, 128))
    return cudaErrorInvalidValue;
  delta_kernel<<<(unsigned)((rows + 7) / 8), 256, 0, st>>>(os, (const __nv_bfloat16*)dos, delta, dq, rows, D);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const float sigma = 1.0f / sqrtf((float)D);
  const float scale_log2 = sigma * kLog2e;
  const dim3 grid((unsigned)(g.BH < kHeadGroup ? g.BH : kHeadGroup), (unsigned)(Sk / 128),
                  (unsigned)((g.BH + kHeadGroup - 1) / kHeadGroup));
  const int smem = padded_smem(LayFused<D>::BYTES);
  e = cudaFuncSetAttribute(attn_bwd_fused_tc<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  attn_bwd_fused_tc<D><<<grid, kThreads, smem, st>>>(k128, v128, q64, do64, lse, delta, dq, dk, dv, g.S,
                                                      (int)g.BH, kb0, Sk, sigma, scale_log2, status,
                                                      g.wait_ns);
  return cudaGetLastError();
}

bool attn_bwd_fused(const Geo& g) {
  return attn_tc_eligible(g) && !(g.flags & LH_DETERMINISTIC);
}

cudaError_t launch_attn_bwd_tc(const Geo& g, const void* qs, const void* ks, const void* vs,
                               const float* os, const float* lse, const void* dos, float* dq,
                               float* dk, float* dv, float* delta, uint32_t* status, cudaStream_t st) {
  return g.d == 128 ? run_bwd<128>(g, qs, ks, vs, os, lse, dos, dq, dk, dv, delta, status, st)
                    : run_bwd<64>(g, qs, ks, vs, os, lse, dos, dq, dk, dv, delta, status, st);
}

}  // namespace lh
