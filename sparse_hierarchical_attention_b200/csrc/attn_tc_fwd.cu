// Causal attention forward on the gathered subsequence with 5th-generation tensor cores
// (tcgen05, accumulators in tensor memory, operands staged by TMA). bf16 inputs, fp32 softmax
// and accumulation ("Long Context Pre-Training with Lighthouse Attention", technical summary
// 2.C: dense causal attention on the S selected rows; row j visible to row i iff j <= i).
//
// One CTA = 128 query rows of one (b,h). Warp roles:
//  - warps 0-15 (softmax), in two sets: set 0 (warps 0-7) takes the even key blocks, set 1
//    (warps 8-15) the odd ones, so that one set's exponentials run while the other set loads its
//    scores, takes its maxima and waits. Warps w, w+4, w+8, w+12 share the TMEM lanes
//    32(w%4)..+31 (query rows); within a set, warp w takes keys 0-63 of its block and warp w+4
//    keys 64-127;
//  - warp 16, one lane: TMA loads (Q once; K through a three-stage ring, V through two or three,
//    the two rings advancing independently);
//  - warp 17, one lane: the S MMAs; warp 18, one lane: the PV MMAs.
// Tensor memory (512 columns): three S/P buffers at 0, 128 and 256 and O at 384. S_j = Q K_j^T
// goes to buffer j % 3; once the softmax warps hold S_j in registers they write P_j over it, and
// PV_j reads P_j there. S_{j+3} waits for PV_j.
//  - P_j = hi + lo with hi = bf16(P) and lo = bf16(P - hi), and O += hi V_j + lo V_j takes the
//    A operand from tensor memory (hi of keys 16i..16i+15 in 8 columns, their lo in the next 8).
//    The split keeps P to ~16 bits: the backward recomputes P exactly and forms
//    D_i = dO_i . O_i, so an O made from bf16-rounded P would leave sum_j dS_ij off zero by
//    dO . (O error), which is large on coarse rows whose dO sums thousands of tokens.
//  - The running max is updated lazily: O is rescaled only when a row's max grows by more than
//    2^kGrow (2^32), which keeps every exponent bounded and skips most rescales, each of which
//    waits for the previous PV. P <= 2^32, l <= 2^32 S and |O| <= 2^32 S max|V| stay inside the
//    fp32 range while S max|V| < 2^96 (S = 2^20 rows leave |V| up to 2^76). The max of block j
//    goes from one set to the other through shared memory and a named barrier per set and lane
//    quarter, on which the set of block j syncs and the set of block j - 1 arrives; the same
//    barrier swaps the two halves' block maxima. Each warp keeps its own row sum, relative to
//    the max it last used, and the four sums of a row meet in the epilogue.
//  - The softmax warps are bound by instruction issue and the ex2 unit, so their arithmetic is
//    counted: the row max is taken over the raw scores with three-input max (exact, as the scale is
//    positive), the scale enters the exponent through one packed f32x2 FMA per pair of keys, and
//    the row sums and the lo residuals are packed f32x2 adds and subtracts.
//  - Key blocks above the diagonal are skipped; the diagonal block is masked.
// The output is fp32 O_sub and the natural-log lse. Shared memory per CTA: Q + 3 K + 2 V tiles of
// 128 rows at d = 128 (192 KB; 3 V tiles at d = 64), one CTA per SM.
#include <mutex>

#include "tc.cuh"

namespace lh {
namespace {

using namespace tc;

constexpr int BM = 128, BN = 128;
constexpr int kSoftmax = 512, kThreads = kSoftmax + 96;  // + the TMA warp and two MMA warps
constexpr int kStages = 3;  // K ring
constexpr int kSBuf = 3;    // S/P buffers in tensor memory
template <int D> constexpr int v_stages() { return D == 128 ? 2 : 3; }
constexpr int TILE = 128 * 128;  // bytes of one [128 rows][64 bf16] 128B-swizzled sub-tile

template <int D>
struct Layout {
  static constexpr int KB = D / 64;  // 64-column sub-tiles per row
  static constexpr int Q = 0;
  static constexpr int K = Q + KB * TILE;            // stage s at K + s * KB * TILE
  static constexpr int V = K + kStages * KB * TILE;  // stage s at V + s * KB * TILE
  static constexpr int BAR = V + v_stages<D>() * KB * TILE;
  // floats [.][128 rows]: XM [2] the max block j used, at j & 1; XC [4][2 halves] the halves'
  // maxima of block j, at j & 3 (a warp can store block j + 2's maximum before its partner has
  // read block j's, but not block j + 4's: that needs PV_{j+1}, after the partner's arrival);
  // XL, XE [4 warps] partial row sums and the max each is relative to
  static constexpr int XM = BAR + 256;
  static constexpr int XC = XM + 2 * 128 * 4;
  static constexpr int XL = XC + 8 * 128 * 4;
  static constexpr int XE = XL + 4 * 128 * 4;
  static constexpr int BYTES = XE + 4 * 128 * 4;
};

// bars: 0 Q | 1-3 K loaded | 4-6 V loaded | 7-9 K free | 10-12 V free | 13-15 S ready
//       | 16-18 P written | 19-21 PV done | 22 last PV done | 23-24 drain of the two MMA issuers
constexpr int kBars = 25;
// O is rescaled when a row's max grows by more than 2^kGrow (log2 units). Rows of the
// gathered subsequences span hundreds of log2 units: with 8 instead, 69% of the 128x128
// blocks of a 32K head rescale some row, with 32, 22%.
constexpr float kGrow = 32.0f;

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
attn_fwd_tc(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
            const __grid_constant__ CUtensorMap tv, float* __restrict__ O, float* __restrict__ lse,
            int S, int BH, int kb0, int Sk, float scale_log2, uint32_t* status, uint64_t wait_ns) {
  using Ly = Layout<D>;
  constexpr int KB = Ly::KB;
  constexpr int kStV = v_stages<D>();
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
  uint64_t* bar = reinterpret_cast<uint64_t*>(sm + Ly::BAR);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar + kBars);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bar + kBars) + 1;
  uint64_t* const bar_q = bar;
  uint64_t* const bar_k = bar + 1;
  uint64_t* const bar_v = bar + 4;
  uint64_t* const bar_kfree = bar + 7;
  uint64_t* const bar_vfree = bar + 10;
  uint64_t* const bar_s = bar + 13;
  uint64_t* const bar_p = bar + 16;
  uint64_t* const bar_pv = bar + 19;
  uint64_t* const bar_fin = bar + 22;

  const int tid = threadIdx.x, warp = tid / 32;
  // S query rows and Sk key rows per (b,h); the queries are the global rows 128 kb0 .. of the
  // keys' sequence (kb0 = 0, Sk = S on one GPU; a context-parallel rank owns a later slice)
  const int nqb = S / BM;
  const int qb = nqb - 1 - (int)blockIdx.y;  // heaviest tiles first within a head group
  const int bh = (int)blockIdx.z * kHeadGroup + (int)blockIdx.x;
  if (bh >= BH) return;  // the last group may be partial
  const int grow0 = bh * S;                  // first query row of this (b,h) in the [BH*S, D] view
  const int krow0 = bh * Sk;                 // first key row of this (b,h)
  const int nkb = kb0 + qb + 1;              // key blocks up to the diagonal

  if (tid == 0) {
    for (int i = 0; i < kBars; ++i)
      mbar_init(bar + i, (i >= 16 && i <= 18) ? 8 : 1);  // P written: the eight warps of one set
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0) tmem_alloc(tmem_slot, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_slot;
  const uint32_t t_o = tbase + kSBuf * 128;

  if (warp == kSoftmax / 32) {
    // ------------------------------------------------------------------ TMA warp
    if ((tid % 32) == 0) {
      prefetch_tmap(&tq); prefetch_tmap(&tk); prefetch_tmap(&tv);
      auto load_k = [&](int j) {
        uint64_t* b = bar_k + j % kStages;
        mbar_expect_tx(b, KB * TILE);
        for (int c = 0; c < KB; ++c)
          tma_load_2d(sm + Ly::K + (j % kStages) * KB * TILE + c * TILE, &tk, c * 64, krow0 + j * BN, b);
      };
      auto load_v = [&](int j) {
        uint64_t* b = bar_v + j % kStV;
        mbar_expect_tx(b, KB * TILE);
        for (int c = 0; c < KB; ++c)
          tma_load_2d(sm + Ly::V + (j % kStV) * KB * TILE + c * TILE, &tv, c * 64, krow0 + j * BN, b);
      };
      mbar_expect_tx(bar_q, KB * TILE);
      for (int c = 0; c < KB; ++c) tma_load_2d(sm + Ly::Q + c * TILE, &tq, c * 64, grow0 + qb * BM, bar_q);
      // The two rings advance independently: K_j reuses the stage of K_{j-3} once S_{j-3} has read
      // it, V_j that of V_{j-kStV} once PV_{j-kStV} has, and a K load never waits behind a V stage.
      int nk = 0, nv = 0;  // loads issued into each ring
      uint64_t t_moved = globaltimer();
      for (uint32_t it = 1; nk < nkb || nv < nkb; ++it) {
        bool moved = false;
        if (nk < nkb && (nk < kStages || mbar_try(bar_kfree + nk % kStages, ((nk - kStages) / kStages) & 1))) {
          load_k(nk++);
          moved = true;
        }
        if (nv < nk && (nv < kStV || mbar_try(bar_vfree + nv % kStV, ((nv - kStV) / kStV) & 1))) {
          load_v(nv++);
          moved = true;
        }
        if (moved) {
          t_moved = globaltimer();
        } else if ((it & 255) == 0) {  // no stage freed for wait_ns: the bound of every other wait
          if (*abort_flag) break;
          if (globaltimer() - t_moved > wait_ns) {
            *abort_flag = 1;
            raise_fault(status, kFaultTimeout);
            break;
          }
        }
      }
      // every load issued has landed before this thread leaves (on the normal path they were
      // all consumed already, so these return at once)
      mbar_drain(bar_q, 0, status);
      drain_ring(bar_k, kStages, nk, status);
      drain_ring(bar_v, kStV, nv, status);
    }
  } else if (warp == kSoftmax / 32 + 1 || warp == kSoftmax / 32 + 2) {
    // ------------------------------------------------------------------ MMA warps
    if ((tid % 32) == 0) {
      const bool s_issuer = warp == kSoftmax / 32 + 1;
      const uint32_t s_q = smem_u32(sm + Ly::Q), s_k = smem_u32(sm + Ly::K), s_v = smem_u32(sm + Ly::V);
      const uint64_t dQ = desc_base(16, 1024) + (s_q >> 4), dK = desc_base(16, 1024) + (s_k >> 4);
      const uint64_t dV = desc_base(TILE, 1024) + (s_v >> 4);  // MN-major: LBO = one sub-tile
      constexpr uint32_t IDESC_S = idesc_bf16(128, 128, false, false);
      constexpr uint32_t IDESC_PV = idesc_bf16(128, D, false, true);
      auto issue_s = [&](int j) {  // S_j = Q K_j^T into TMEM buffer j % 3
        const uint32_t sg = (uint32_t)((j % kStages) * KB * TILE) >> 4;
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          const uint32_t off = ((ks / 4) * TILE + (ks % 4) * 32) >> 4;
          mma_ss(tbase + (j % kSBuf) * 128, dQ + off, dK + sg + off, IDESC_S, ks > 0);
        }
        mma_commit(bar_s + j % kSBuf);
        mma_commit(bar_kfree + j % kStages);
      };
      auto issue_pv = [&](int j) {  // O += hi_j V_j + lo_j V_j, P_j over S_j in buffer j % 3
        const uint32_t sg = (uint32_t)((j % kStV) * KB * TILE) >> 4;
        const uint32_t tp = tbase + (j % kSBuf) * 128;
#pragma unroll
        for (int part = 0; part < 2; ++part) {
#pragma unroll
          for (int ks = 0; ks < BN / 16; ++ks)  // keys 16 ks ..: hi at column 16 ks, lo at 16 ks + 8
            mma_ts(t_o, tp + ks * 16 + part * 8, dV + sg + ks * (2048 >> 4), IDESC_PV,
                   (j > 0 || part > 0 || ks > 0) ? 1u : 0u);
        }
        mma_commit(bar_pv + j % kSBuf);
        mma_commit(bar_vfree + j % kStV);
      };
      if (s_issuer) {
        bool ok = mbar_wait(bar_q, 0, abort_flag, status, wait_ns);
        for (int n = 0; n < nkb && ok; ++n) {  // S_n into buffer n % 3 once PV_{n-3} has read P_{n-3} there
          ok = mbar_wait(bar_k + n % kStages, (n / kStages) & 1, abort_flag, status, wait_ns);
          if (ok && n >= kSBuf) ok = mbar_wait(bar_pv + n % kSBuf, ((n / kSBuf) - 1) & 1, abort_flag, status, wait_ns);
          if (!ok) break;
          tc_fence_after();
          issue_s(n);
        }
        mma_drain(bar + 23, status);
      } else {
        int j = 0;
        for (; j < nkb; ++j) {
          const bool ok = mbar_wait(bar_p + j % kSBuf, (j / kSBuf) & 1, abort_flag, status, wait_ns) &&
                          mbar_wait(bar_v + j % kStV, (j / kStV) & 1, abort_flag, status, wait_ns);
          if (!ok) break;
          tc_fence_after();
          issue_pv(j);
        }
        if (j == nkb) mma_commit(bar_fin);
        mma_drain(bar + 24, status);
      }
    }
  } else {
    // ------------------------------------------------------------------ softmax warps
    // Set 0 (warps 0-7) takes the even key blocks, set 1 (warps 8-15) the odd ones. Warps
    // w, w + 4, w + 8, w + 12 own the same 32 query rows (TMEM lanes 32 (w % 4) ..); within a set,
    // warp w + 4 h takes keys 64 h .. 64 h + 63 of the block. One set's exponentials thus overlap
    // the other set's loads, maxima and waits.
    constexpr int DQ = D / 4;  // O columns each of the four warps of a lane quarter stores
    const int q4 = warp % 4, half = (warp / 4) & 1, set = warp / 8;
    const uint32_t lane_off = (uint32_t)(q4 * 32) << 16;
    const int row = q4 * 32 + (tid % 32);  // query row within the tile = TMEM lane
    float* const xm = reinterpret_cast<float*>(sm + Ly::XM);
    float* const xc = reinterpret_cast<float*>(sm + Ly::XC);
    float* const xl = reinterpret_cast<float*>(sm + Ly::XL);
    float* const xe = reinterpret_cast<float*>(sm + Ly::XE);
    // Block j meets on the named barrier of its set and lane quarter: the set's two warps sync,
    // having stored their halves' maxima, and the other set's two warps arrive, having stored
    // the max block j - 1 used (block 0 has no predecessor: its two warps alone). Every warp
    // takes these steps for every block of its set whatever its waits returned, so a failed wait
    // never strands another warp at a barrier.
    const int bar_in = 1 + 4 * set + q4, bar_out = 1 + 4 * (set ^ 1) + q4;
    auto wait_all = [&](uint64_t* b, uint32_t parity) {  // the whole warp waits, converged
      bool ok = mbar_wait(b, parity, abort_flag, status, wait_ns);
      return __all_sync(0xffffffffu, ok);
    };
    float m_mine = -INFINITY, l = 0.f;  // this warp's partial row sum, relative to m_mine
    bool ok = true;
    for (int j = set; j < nkb; j += 2) {
      ok = ok && wait_all(bar_s + j % kSBuf, (j / kSBuf) & 1);
      tc_fence_after();
      const uint32_t ts = tbase + (j % kSBuf) * 128 + half * 64 + lane_off;  // this warp's 64 keys
      float s[64];
      if (ok) {
        uint32_t r0[32], r1[32];
        tmem_ld32(ts, r0);
        tmem_ld32(ts + 32, r1);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 32; ++e) {  // raw scores: the scale goes into the exponent's FMA
          s[e] = __uint_as_float(r0[e]);
          s[32 + e] = __uint_as_float(r1[e]);
        }
      } else {
#pragma unroll
        for (int e = 0; e < 64; ++e) s[e] = 0.f;
      }
      if (j == kb0 + qb) {  // diagonal block: key column > query row is invisible
#pragma unroll
        for (int e = 0; e < 64; ++e)
          if (half * 64 + e > row) s[e] = -INFINITY;
      }
      float m4[4];
#pragma unroll
      for (int c = 0; c < 4; ++c) {  // four chains of 16; the scale is positive, so max commutes with it
        m4[c] = max3(s[16 * c], s[16 * c + 1], s[16 * c + 2]);
#pragma unroll
        for (int e = 16 * c + 3; e < 16 * c + 15; e += 2) m4[c] = max3(m4[c], s[e], s[e + 1]);
        m4[c] = fmaxf(m4[c], s[16 * c + 15]);
      }
      const float mloc = max3(m4[0], m4[1], fmaxf(m4[2], m4[3])) * scale_log2;
      xc[((j & 3) * 2 + half) * 128 + row] = mloc;
      if (j == 0) asm volatile("bar.sync %0, 64;" ::"r"(bar_in) : "memory");
      else asm volatile("bar.sync %0, 128;" ::"r"(bar_in) : "memory");
      const float mt = fmaxf(mloc, xc[((j & 3) * 2 + (half ^ 1)) * 128 + row]);
      const float m_prev = j > 0 ? xm[((j - 1) & 1) * 128 + row] : -INFINITY;  // the max block j - 1 used
      const bool grow = mt > m_prev + kGrow;
      const float m_new = grow ? mt : m_prev;
      if (j + 1 < nkb) {
        if (half == 0) xm[(j & 1) * 128 + row] = m_new;
        asm volatile("bar.arrive %0, 128;" ::"r"(bar_out) : "memory");
      }
      const uint64_t c2 = f2_pack(scale_log2, scale_log2), nm2 = f2_pack(-m_new, -m_new);
      uint64_t sum2[2] = {f2_pack(0.f, 0.f), f2_pack(0.f, 0.f)};
#pragma unroll
      for (int c = 0; c < 4; ++c) {  // keys 64 half + 16 c ..: P hi in columns 16 c .. + 7, lo in 16 c + 8 ..
        uint32_t h[8], w[8];
#pragma unroll
        for (int e = 0; e < 16; e += 2) {  // p = 2^(s * scale - m), a pair per instruction
          float a0, a1;
          f2_unpack(f2_fma(f2_pack(s[16 * c + e], s[16 * c + e + 1]), c2, nm2), a0, a1);
          const uint64_t x = f2_pack(ex2(a0), ex2(a1));
          sum2[(e >> 1) & 1] = f2_add(sum2[(e >> 1) & 1], x);
          split_bf16x2_f2(x, h[e / 2], w[e / 2]);
        }
        if (ok) {  // S_j of these columns is in registers already: P goes over it
          tmem_st8(ts + 16 * c, h);
          tmem_st8(ts + 16 * c + 8, w);
        }
      }
      float sa0, sa1, sb0, sb1;
      f2_unpack(sum2[0], sa0, sa1);
      f2_unpack(sum2[1], sb0, sb1);
      if (m_new != m_mine) l *= exp2f(m_mine - m_new);  // l = 0 before this warp's first block
      l += (sa0 + sa1) + (sb0 + sb1);
      m_mine = m_new;
      // O holds sum_{i<j} P_i V_i relative to m_prev: rescale this warp's half of it once PV_{j-1}
      // is done (both warps of the set see the same grow flags)
      if (j > 0 && __any_sync(0xffffffffu, grow)) {
        ok = ok && wait_all(bar_pv + (j - 1) % kSBuf, ((j - 1) / kSBuf) & 1);
        tc_fence_after();
        if (ok) {
          const float alpha = grow ? exp2f(m_prev - m_new) : 1.0f;
          uint32_t r[32];
#pragma unroll
          for (int c = 0; c < D / 64; ++c) {
            const uint32_t to = t_o + lane_off + half * (D / 2) + c * 32;
            tmem_ld32(to, r);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e) r[e] = __float_as_uint(__uint_as_float(r[e]) * alpha);
            tmem_st32(to, r);
          }
        }
      }
      if (ok) tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (ok && (tid % 32) == 0) mbar_arrive(bar_p + j % kSBuf);
    }
    // ---- epilogue: O / l and lse (the four warps' partial sums brought to the last max)
    ok = ok && wait_all(bar_fin, 0);
    tc_fence_after();
    const int k4 = set * 2 + half;
    xl[k4 * 128 + row] = l;
    xe[k4 * 128 + row] = m_mine;
    asm volatile("bar.sync %0, 128;" ::"r"(9 + q4) : "memory");
    float m_fin = xe[row];
#pragma unroll
    for (int k = 1; k < 4; ++k) m_fin = fmaxf(m_fin, xe[k * 128 + row]);
    float lt = 0.f;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float lk = xl[k * 128 + row], mk = xe[k * 128 + row];
      lt += mk == m_fin ? lk : lk * exp2f(mk - m_fin);
    }
    if (ok) {
      const float inv = 1.0f / lt;
      float* orow = O + (size_t)(grow0 + qb * BM + row) * D + k4 * DQ;
      if constexpr (DQ == 32) {
        uint32_t r[32];
        tmem_ld32(t_o + lane_off + k4 * DQ, r);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 32; e += 4)
          *reinterpret_cast<float4*>(orow + e) =
              make_float4(__uint_as_float(r[e]) * inv, __uint_as_float(r[e + 1]) * inv,
                          __uint_as_float(r[e + 2]) * inv, __uint_as_float(r[e + 3]) * inv);
      } else {
        uint32_t r[16];
        tmem_ld16(t_o + lane_off + k4 * DQ, r);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 16; e += 4)
          *reinterpret_cast<float4*>(orow + e) =
              make_float4(__uint_as_float(r[e]) * inv, __uint_as_float(r[e + 1]) * inv,
                          __uint_as_float(r[e + 2]) * inv, __uint_as_float(r[e + 3]) * inv);
      }
      if (k4 == 0) lse[grow0 + qb * BM + row] = (m_fin + log2f(lt)) * 0.69314718055994531f;
    }
  }
  // every role has drained its own loads and MMAs, so nothing still writes shared or tensor
  // memory once all threads are here
  tc_fence_before();
  __syncthreads();
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

bool make_tmap_f32_box(CUtensorMap* map, const void* base, int64_t rows, int D, int box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {(cuuint64_t)D, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)D * 4};
  cuuint32_t box[2] = {32, (cuuint32_t)box_rows};  // 32 fp32 = one 128-byte swizzle row
  cuuint32_t estr[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<void*>(base), dims, strides, box,
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

cudaError_t launch_attn_fwd_tc_rows(const Geo& g, int kb0, int Sk, const void* qs, const void* ks,
                                    const void* vs, float* os, float* lse, uint32_t* status,
                                    cudaStream_t st) {
  CUtensorMap mq, mk, mv;
  if (!make_tmap_rows(&mq, qs, g.BH * g.S, g.d) || !make_tmap_rows(&mk, ks, g.BH * Sk, g.d) ||
      !make_tmap_rows(&mv, vs, g.BH * Sk, g.d))
    return cudaErrorInvalidValue;
  const float scale_log2 = (1.0f / sqrtf((float)g.d)) * 1.4426950408889634f;
  const unsigned gx = g.BH < kHeadGroup ? (unsigned)g.BH : (unsigned)kHeadGroup;
  dim3 grid(gx, (unsigned)(g.S / BM), (unsigned)((g.BH + kHeadGroup - 1) / kHeadGroup));
  cudaError_t e;
  if (g.d == 128) {
    const int smem = Layout<128>::BYTES + 1024;
    e = cudaFuncSetAttribute(attn_fwd_tc<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e == cudaSuccess)
      attn_fwd_tc<128><<<grid, kThreads, smem, st>>>(mq, mk, mv, os, lse, g.S, (int)g.BH, kb0, Sk, scale_log2,
                                                      status, g.wait_ns);
  } else {
    // padded so that two CTAs never share an SM (each holds all 512 TMEM columns)
    const int smem = Layout<64>::BYTES + 1024 > 120 * 1024 ? Layout<64>::BYTES + 1024 : 120 * 1024;
    e = cudaFuncSetAttribute(attn_fwd_tc<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e == cudaSuccess)
      attn_fwd_tc<64><<<grid, kThreads, smem, st>>>(mq, mk, mv, os, lse, g.S, (int)g.BH, kb0, Sk, scale_log2,
                                                     status, g.wait_ns);
  }
  return e != cudaSuccess ? e : cudaGetLastError();
}

cudaError_t launch_attn_fwd_tc(const Geo& g, const void* qs, const void* ks, const void* vs,
                               float* os, float* lse, uint32_t* status, cudaStream_t st) {
  return launch_attn_fwd_tc_rows(g, 0, g.S, qs, ks, vs, os, lse, status, st);
}

}  // namespace lh
