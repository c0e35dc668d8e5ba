// Streaming pooling kernels.
//
// MODE_PYRAMID: the symmetric average-pooling pyramid over Q, K, V and the l2 rank score of
//   every cell, in one pass over the inputs ("Long Context Pre-Training with Lighthouse
//   Attention", technical summary 2.A and 2.B; the Nous Research article's four-stage
//   paragraph: Theta(N) pyramid, two scalar scores per cell, max-pooled upward). With grouped
//   query heads (fewer key/value heads) it takes two passes: K and V over their heads, leaving
//   the max-pooled key norms in scratch, then Q, whose scores add its key head's norms.
// MODE_SPANSUM: dO_sub[i] = sum of dO over span(i) for the selected cells only, the backward
//   of the scatter-back (technical summary 2.B: gradients flow through scatter-back).
//
// Structure (per (b,h)):
//   tile kernel  - 256 threads; each row of d elements is covered by LPR lanes holding 16 bytes
//                  each. A "stream" (LPR lanes) walks W = p^A consecutive tokens and keeps fp32
//                  partial sums of levels 1..A in registers. The STREAMS level-A cells of the
//                  CTA then go through a shared-memory tree up to level A2. If A2 < L-1 the
//                  level-A2 fp32 sums (and score maxima) go to a small scratch buffer.
//   coarse kernel - one CTA per chunk finishes levels A2+1..L-1 from that scratch.
// Sums are fp32 in ascending child order, never re-read from rounded storage; a stored cell is
// fl32(sum * fl32(1/p^l)) rounded once. Norms take one fixed fp32 order so that the selection is
// reproducible bit for bit: each 16-byte group of a row is summed in ascending coordinate order
// (every square rounded on its own, no FMA), the group sums are folded by a halving tree, and
// the root is a correctly rounded square root.
#include <algorithm>

#include "common.cuh"

namespace lh {
namespace {

constexpr int kThreads = 256;
enum { MODE_PYRAMID = 0, MODE_SPANSUM = 1 };
// Rows one stream walks with register carries: p^A <= 16 for the three-tensor pyramid, <= 64 for
// the one-tensor span sums (fewer live registers, so longer streams and fewer tile setups).
constexpr int kWMaxPyr = 16, kWMaxSpan = 64;
// Rows fetched ahead per thread, and the CTAs per SM the register budget is sized for (a sweep
// of 4 or 8 rows against 2, 3 or 4 CTAs per SM at 128K picked these; A >= 3, which only p = 2
// or 3 reaches, carries more level sums and gets a larger budget).
template <int MODE> constexpr int rows_ahead() { return MODE == 0 ? 8 : 4; }
template <int MODE, int A> constexpr int ctas_per_sm() {
  return MODE == 0 ? (A >= 3 ? 2 : 3) : (A >= 4 ? 3 : 4);
}

struct PoolArgs {
  const void* x[3];  // q, k, v (pyramid) or d_o (span sums)
  void* px[3];       // pooled outputs [BH, R, D] (pyramid) or do_sub [BH, S, D] (span sums)
  float* score;      // [BH, N+R] or null
  float* tmp;        // level-A2 fp32 sums [BH, N/p^A2, ntensor, D] then maxima [BH, N/p^A2, 2]
  const int32_t* idx;  // span sums: the selection [BH, S]
  uint32_t* status;
  int64_t N, R, S, T, m, C, G;  // m rows per stratum of G chunks
  int64_t off[16];    // row id offsets of levels
  float inv[16];      // fl32(1 / p^l)
  int wdiv[8];        // W / p^l for l = 1..A: level-l cells per stream
  int p, L, W, A2, U;
  int do_pyr, do_score;
  // Pyramid: the nx tensors streamed, and what the score of a cell is:
  //   0: |x[0]| + |x[1]| (q, k: each query head has its own key head);
  //   1: |x[0]| (grouped heads, key/value pass: the max-pooled key norms);
  //   2: |x[0]| + partner row of the key head (grouped heads, query pass).
  int nx, score_mode;
  const float* partner;  // mode 2: [B Hkv, N+R] max-pooled key norms
  int H, grp;            // mode 2: query heads per batch, query heads per key/value head
};

// Mode 2's partner row: the key/value head of query head bh (b H + h -> b Hkv + h / grp).
__device__ inline const float* partner_row(const PoolArgs& a, int64_t bh) {
  return a.partner + ((bh / a.H) * (a.H / a.grp) + (bh % a.H) / a.grp) * (a.N + a.R);
}
// A cell's score from the query-side and key-side maxima (see score_mode); rid its row id.
__device__ inline float cell_score(const PoolArgs& a, const float* prow, float sq, float sk, int64_t rid) {
  return a.score_mode == 0 ? __fadd_rn(sq, sk) : a.score_mode == 1 ? sq : __fadd_rn(sq, prow[rid]);
}

// fp32 l2 norm in that fixed order. Each lane of a row sums the squares of its 16-byte
// group in ascending order (products rounded on their own) and leaves that partial in shared
// memory; one lane then folds the LPR partials of the row with the halving tree (partial i
// pairs with i + s for s = LPR/2 .. 1, the pairs a lane butterfly would form) and takes the root.
template <int VEC>
__device__ inline float group_sumsq(const float* x) {
  float a = 0.f;
#pragma unroll
  for (int e = 0; e < VEC; ++e) a = __fadd_rn(a, __fmul_rn(x[e], x[e]));
  return a;
}
template <int LPR>
__device__ inline float tree_norm(const float* part) {
  float t[LPR];
#pragma unroll
  for (int i = 0; i < LPR; ++i) t[i] = part[i];
#pragma unroll
  for (int s = LPR / 2; s >= 1; s >>= 1)
#pragma unroll
    for (int i = 0; i < s; ++i) t[i] = __fadd_rn(t[i], t[i + s]);
  return __fsqrt_rn(t[0]);
}

// Two-lane fp32 add (sm_100 f32x2): each lane rounds to nearest exactly as __fadd_rn does. Products
// stay scalar (__fmul_rn): a packed multiply feeding a packed add did not reproduce the separately
// rounded scalar pair on fp32 inputs.
__device__ inline void add2(float& a0, float& a1, float b0, float b1) {
  asm("{\n\t.reg .b64 ra, rb;\n\tmov.b64 ra, {%0, %1};\n\tmov.b64 rb, {%2, %3};\n\t"
      "add.rn.f32x2 ra, ra, rb;\n\tmov.b64 {%0, %1}, ra;\n\t}"
      : "+f"(a0), "+f"(a1)
      : "f"(b0), "f"(b1));
}

// Row id -> level and cell index, from the level offsets.
__device__ inline void decode_rid(int64_t rid, const int64_t* off, int L, int& lvl, int64_t& cell) {
  lvl = 0;
#pragma unroll 1
  for (int l = 1; l < L; ++l)
    if (rid >= off[l]) lvl = l;
  cell = rid - off[lvl];
}

template <typename E, int D, int A, int MODE>
__global__ void __launch_bounds__(kThreads, (ctas_per_sm<MODE, A>())) pool_tile_kernel(const PoolArgs a) {
  using V = Vec<E>;
  constexpr int VEC = V::N, LPR = D / VEC, STREAMS = kThreads / LPR;
  constexpr int NX = MODE == MODE_PYRAMID ? 3 : 1;
  constexpr int AR = A > 0 ? A : 1;
  constexpr bool NORMS = MODE == MODE_PYRAMID;
  constexpr int PSTR = LPR + 1;  // partials row stride (conflict-free column reads)
  __shared__ float stage[NX][STREAMS][D];
  __shared__ float smax[2][STREAMS];
  __shared__ int smap[MODE == MODE_SPANSUM ? 2 * STREAMS * kWMaxSpan + 64 : 1];  // (level, cell) -> row
  // norms: per-lane partial sums of squares [2][STREAMS][16 rows][PSTR], then per stream the row
  // norms and the level maxima [2][STREAMS][32] (W + W/p + ... + 1 <= 32 entries)
  extern __shared__ float dyn[];
  float* const part = dyn;
  float* const lev = dyn + 2 * STREAMS * 16 * PSTR;

  const int tid = threadIdx.x, col = tid % LPR, s = tid / LPR;
  const int64_t bh = blockIdx.y;
  const int W = a.W, p = a.p;
  const int64_t tile = (int64_t)W * STREAMS;
  const int64_t t_tile = (int64_t)blockIdx.x * tile;
  const int64_t tok0 = t_tile + (int64_t)s * W;
  const bool active = tok0 < a.N;
  const int nx = MODE == MODE_PYRAMID ? a.nx : 1;
  const int64_t NR = a.N + a.R;
  const float* const prow = MODE == MODE_PYRAMID && a.score_mode == 2 ? partner_row(a, bh) : nullptr;

  // Span sums: map every selected cell of level <= A2 inside this tile to its subsequence row.
  // Map layout: level l occupies tile/p^l slots starting at moff(l).
  int map_base[16];
  if constexpr (MODE == MODE_SPANSUM) {
    int acc = 0;
    int64_t cells = tile;
    for (int l = 0; l <= a.A2; ++l) {
      map_base[l] = acc;
      acc += (int)cells;
      cells /= p;
    }
    for (int i = tid; i < acc; i += kThreads) smap[i] = -1;
    __syncthreads();
    // the rows of the strata that hold this tile's chunks; cells outside the tile are skipped
    const int64_t c0 = t_tile / a.T;
    const int64_t c1 = std::min<int64_t>((t_tile + tile - 1) / a.T, a.C - 1);
    const int64_t r0 = (c0 / a.G) * a.m, r1 = (c1 / a.G + 1) * a.m;
    for (int64_t i = r0 + tid; i < r1; i += kThreads) {
      const int64_t rid = a.idx[bh * a.S + i];
      if (rid < 0 || rid >= NR) { raise_fault(a.status, kFaultIndex); continue; }
      int lvl; int64_t cell;
      decode_rid(rid, a.off, a.L, lvl, cell);
      if (lvl > a.A2) continue;
      int64_t pw = 1;
      for (int l = 0; l < lvl; ++l) pw *= p;
      const int64_t first = t_tile / pw;  // first cell of this level inside the tile
      if (cell >= first && cell < first + tile / pw)
        smap[map_base[lvl] + (int)(cell - first)] = (int)i;
    }
    __syncthreads();
  }

  // The tensors go through the tile one after another, so that the registers hold the level
  // partial sums and the fetched rows of one tensor only (more CTAs per SM, more rows in flight).
  constexpr int U = rows_ahead<MODE>();
#pragma unroll 1
  for (int xi = 0; xi < nx; ++xi) {
    float acc[AR][VEC];
#pragma unroll
    for (int l = 0; l < AR; ++l)
#pragma unroll
      for (int e = 0; e < VEC; ++e) acc[l][e] = 0.f;
    // Level l+1 completes after p completions of level l (level 0: rows); cellj[l] is the global
    // index of the level-(l+1) cell being summed. W = p^A divides the tile, so the first cell of
    // a stream is a product of small integers.
    int left[AR];
    int64_t cellj[AR];
#pragma unroll
    for (int l = 0; l < AR; ++l) {
      left[l] = p;
      cellj[l] = ((int64_t)blockIdx.x * STREAMS + s) * (A > 0 ? a.wdiv[l] : 0);
    }
    const E* const X = static_cast<const E*>(a.x[xi]) + (bh * a.N + tok0) * D + col * VEC;
    E* const PX = static_cast<E*>(a.px[MODE == MODE_PYRAMID ? xi : 0]);
    const bool norm_of = NORMS && a.do_score && xi < (a.score_mode == 0 ? 2 : 1);  // the scored rows
    // L2 prefetch ahead of the loads. The kernel waits mostly on load latency, and the rows a
    // warp holds in flight are capped by its registers (the span-sum kernel sits at the register
    // limit of 4 CTAs per SM). A bulk prefetch into L2 holds no registers: one lane of the group
    // asks for the stream's rows PF ahead (contiguous, U rows per request), so the loads then hit
    // L2. Measured per mode: PF = 16 for the pyramid (U = 8), PF = 4 for the span sums (U = 4).
    constexpr int PF = MODE == MODE_PYRAMID ? 16 : 4;
    if (active && col == 0)
      prefetch_l2(X, (uint32_t)((W < PF ? W : PF) * D * sizeof(E)));
#pragma unroll 1
    for (int row0 = 0; row0 < W; row0 += U) {
      if (active && col == 0 && row0 + PF < W)  // an active stream's W rows all lie inside x
        prefetch_l2(X + (int64_t)(row0 + PF) * D, (uint32_t)(min(U, W - (row0 + PF)) * D * sizeof(E)));
      uint4 raw[U];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        raw[u] = make_uint4(0, 0, 0, 0);
        if (active && row0 + u < W) raw[u] = ldg16(X + (int64_t)(row0 + u) * D);
      }
      // one row: the span-sum level-0 store, the level sums, and the cells they complete
      auto take_row = [&](int row, const float (&x)[VEC]) {
        if constexpr (MODE == MODE_SPANSUM) {
          if (active) {
            const int r = smap[s * W + row];
            if (r >= 0) stg16(PX + (bh * a.S + r) * D + col * VEC, V::pack(x));
          }
        }
        if constexpr (A > 0) {
          if constexpr (MODE == MODE_PYRAMID) {
#pragma unroll
            for (int e = 0; e < VEC; e += 2) add2(acc[0][e], acc[0][e + 1], x[e], x[e + 1]);
          } else {  // scalar adds measured faster for the one-tensor span sums
#pragma unroll
            for (int e = 0; e < VEC; ++e) acc[0][e] += x[e];
          }
#pragma unroll
          for (int l = 0; l < A; ++l) {  // a finished level-l cell may finish level l+1, and so on
            if (--left[l] != 0) break;
            left[l] = p;
            const int lv = l + 1;
            if (active) {
              if constexpr (MODE == MODE_PYRAMID) {
                if (a.do_pyr) {
                  const int64_t prow = bh * a.R + (a.off[lv] - a.N) + cellj[l];
                  float o[VEC];
#pragma unroll
                  for (int e = 0; e < VEC; ++e) o[e] = __fmul_rn(acc[l][e], a.inv[lv]);
                  stg16(PX + prow * D + col * VEC, V::pack(o));
                }
              } else {
                const int local = (int)(cellj[l] - (int64_t)blockIdx.x * STREAMS * a.wdiv[l]);
                const int r = smap[map_base[lv] + local];
                if (r >= 0) stg16(PX + (bh * a.S + r) * D + col * VEC, V::pack(acc[l]));
              }
            }
            ++cellj[l];
            if (l + 1 < A) {
#pragma unroll
              for (int e = 0; e < VEC; e += 2)
                add2(acc[l + 1 < A ? l + 1 : l][e], acc[l + 1 < A ? l + 1 : l][e + 1], acc[l][e], acc[l][e + 1]);
            } else {
#pragma unroll
              for (int e = 0; e < VEC; ++e) stage[xi][s][col * VEC + e] = acc[l][e];
            }
#pragma unroll
            for (int e = 0; e < VEC; ++e) acc[l][e] = 0.f;
          }
        }
      };
      if constexpr (MODE == MODE_SPANSUM) {
#pragma unroll
        for (int u = 0; u < U; ++u) {
          const int row = row0 + u;
          if (row >= W) break;  // the same for every thread of the CTA
          float x[VEC];
          V::unpack(raw[u], x);
          take_row(row, x);
        }
      } else {
#pragma unroll
      for (int u = 0; u < U; u += 2) {  // rows in pairs: their sums of squares run as f32x2
        const int row = row0 + u;
        if (row >= W) break;  // the same for every thread of the CTA
        const bool second = row + 1 < W;
        float x0[VEC], x1[VEC];
        V::unpack(raw[u], x0);
        V::unpack(raw[u + 1], x1);
        if (norm_of) {
          float a0 = 0.f, a1 = 0.f;  // each row's group in ascending order
#pragma unroll
          for (int e = 0; e < VEC; ++e) add2(a0, a1, __fmul_rn(x0[e], x0[e]), __fmul_rn(x1[e], x1[e]));
          part[((xi * STREAMS + s) * 16 + row) * PSTR + col] = a0;
          if (second) part[((xi * STREAMS + s) * 16 + row + 1) * PSTR + col] = a1;
        }
        take_row(row, x0);
        if (second) take_row(row + 1, x1);
      }
      }
    }
  }

  // Norms of the stream's W rows (lane c takes rows c, c + LPR, ...), the level-0 scores, and the
  // max-pooled scores of levels 1..A.
  if constexpr (NORMS) {
    if (a.do_score) {
      __syncwarp();
      float* const lq = lev + s * 32;
      float* const lk = lev + (STREAMS + s) * 32;
      for (int r = col; r < W; r += LPR) {
        const float nq = tree_norm<LPR>(part + (s * 16 + r) * PSTR);
        const float nk = a.score_mode == 0 ? tree_norm<LPR>(part + ((STREAMS + s) * 16 + r) * PSTR) : 0.f;
        if (active) a.score[bh * NR + tok0 + r] = cell_score(a, prow, nq, nk, tok0 + r);
        lq[r] = nq;
        lk[r] = nk;
      }
      __syncwarp();
      int base = 0, n = W;
#pragma unroll 1
      for (int l = 1; l <= A; ++l) {
        const int nc = n / p;
        const int64_t first = ((int64_t)blockIdx.x * STREAMS + s) * a.wdiv[l - 1];
        for (int c = col; c < nc; c += LPR) {
          float mq = 0.f, mk = 0.f;
          for (int ch = 0; ch < p; ++ch) {
            mq = fmaxf(mq, lq[base + c * p + ch]);
            mk = fmaxf(mk, lk[base + c * p + ch]);
          }
          lq[base + n + c] = mq;
          lk[base + n + c] = mk;
          if (active) a.score[bh * NR + a.off[l] + first + c] = cell_score(a, prow, mq, mk, a.off[l] + first + c);
        }
        base += n;
        n = nc;
        __syncwarp();
      }
      if (A > 0 && col == 0) { smax[0][s] = lq[base]; smax[1][s] = lk[base]; }
    }
  }
  if (A == 0 || (a.U == 0 && a.A2 >= a.L - 1)) return;
  __syncthreads();

  // Shared-memory tree: levels A+1..A2 from the STREAMS level-A cells of this tile.
  int cells = STREAMS;
  int64_t pw = W;  // p^level of the current stage
  for (int u = 1; u <= a.U; ++u) {
    const int lvl = A + u;
    const int nc = cells / p;
    pw *= p;
    const int nitems = nx * nc * D;
    float v[(NX * STREAMS * D + kThreads - 1) / kThreads];
    float vmax[2] = {0.f, 0.f};
    int n = 0;
    for (int it = tid; it < nitems; it += kThreads, ++n) {
      const int xi = it / (nc * D), rem = it % (nc * D), c = rem / D, dd = rem % D;
      float sum = 0.f;
      for (int ch = 0; ch < p; ++ch) sum += stage[xi][c * p + ch][dd];
      v[n] = sum;
    }
    if (tid < nc) {
      for (int ch = 0; ch < p; ++ch) {
        vmax[0] = fmaxf(vmax[0], smax[0][tid * p + ch]);
        vmax[1] = fmaxf(vmax[1], smax[1][tid * p + ch]);
      }
    }
    __syncthreads();
    n = 0;
    for (int it = tid; it < nitems; it += kThreads, ++n) {
      const int xi = it / (nc * D), rem = it % (nc * D), c = rem / D, dd = rem % D;
      stage[xi][c][dd] = v[n];
      const int64_t j = t_tile / pw + c;
      if (j * pw < a.N) {
        if constexpr (MODE == MODE_PYRAMID) {
          if (a.do_pyr)
            static_cast<E*>(a.px[xi])[(bh * a.R + (a.off[lvl] - a.N) + j) * D + dd] =
                from_f32<E>(__fmul_rn(v[n], a.inv[lvl]));
        } else {
          const int r = smap[map_base[lvl] + c];
          if (r >= 0) static_cast<E*>(a.px[0])[(bh * a.S + r) * D + dd] = from_f32<E>(v[n]);
        }
      }
    }
    if (tid < nc) {
      smax[0][tid] = vmax[0];
      smax[1][tid] = vmax[1];
      const int64_t j = t_tile / pw + tid;
      if (MODE == MODE_PYRAMID && a.do_score && j * pw < a.N)
        a.score[bh * NR + a.off[lvl] + j] = cell_score(a, prow, vmax[0], vmax[1], a.off[lvl] + j);
    }
    __syncthreads();
    cells = nc;
  }

  // Hand the level-A2 sums to the coarse kernel.
  if (a.A2 < a.L - 1) {
    const int64_t n_a2 = a.N / pw;  // cells of level A2 per (b,h)
    for (int it = tid; it < nx * cells * D; it += kThreads) {
      const int xi = it / (cells * D), rem = it % (cells * D), c = rem / D, dd = rem % D;
      const int64_t j = t_tile / pw + c;
      if (j < n_a2) a.tmp[((bh * n_a2 + j) * NX + xi) * D + dd] = stage[xi][c][dd];
    }
    if (tid < cells) {
      const int64_t j = t_tile / pw + tid;
      float* mx = a.tmp + (int64_t)gridDim.y * n_a2 * NX * D;
      if (j < n_a2) {
        mx[(bh * n_a2 + j) * 2 + 0] = smax[0][tid];
        mx[(bh * n_a2 + j) * 2 + 1] = smax[1][tid];
      }
    }
  }
}

// Levels A2+1..L-1 of one chunk from the level-A2 fp32 sums. Thread (xi, dd) walks the
// chunk's level-A2 cells in order with one partial sum per coarser level; thread NX*D takes the
// score maxima the same way. Each fetches the cells eight at a time (independent loads), since
// the kernel is bound by load latency.
template <typename E, int MODE>
__global__ void pool_coarse_kernel(const PoolArgs a, int D, int NX) {
  const int64_t bh = blockIdx.y, chunk = blockIdx.x;
  const int tid = threadIdx.x;
  const int p = a.p;
  const int nlev = a.L - 1 - a.A2;  // levels to build here
  int64_t pw_a2 = 1;
  for (int l = 0; l < a.A2; ++l) pw_a2 *= p;
  const int64_t n_a2 = a.N / pw_a2;
  int64_t ncell = 1;
  for (int l = 0; l < nlev; ++l) ncell *= p;  // level-A2 cells per chunk
  const int64_t first = chunk * ncell;

  // Span sums: (level above A2, cell inside the chunk) -> subsequence row, or -1.
  extern __shared__ int cmap[];
  int cbase[16];
  if constexpr (MODE == MODE_SPANSUM) {
    int tot = 0;
    int64_t per = ncell;
    for (int u = 0; u < nlev; ++u) {
      per /= p;
      cbase[u] = tot;
      tot += (int)per;
    }
    for (int i = tid; i < tot; i += blockDim.x) cmap[i] = -1;
    __syncthreads();
    const int64_t st = chunk / a.G;  // the rows of this chunk's stratum; other chunks' cells skipped
    for (int64_t i = st * a.m + tid; i < (st + 1) * a.m; i += blockDim.x) {
      const int64_t rid = a.idx[bh * a.S + i];
      if (rid < 0 || rid >= a.N + a.R) { raise_fault(a.status, kFaultIndex); continue; }
      int lvl; int64_t cell;
      decode_rid(rid, a.off, a.L, lvl, cell);
      if (lvl <= a.A2) continue;
      const int u = lvl - a.A2 - 1;
      int64_t cells_per_chunk = 1;
      for (int q = lvl; q < a.L - 1; ++q) cells_per_chunk *= p;
      const int64_t local = cell - chunk * cells_per_chunk;
      if (local >= 0 && local < cells_per_chunk) cmap[cbase[u] + (int)local] = (int)i;
    }
    __syncthreads();
  }

  constexpr int kBatch = 8;
  if (tid < (MODE == MODE_PYRAMID ? a.nx : 1) * D) {
    const int xi = tid / D, dd = tid % D;
    const float* src = a.tmp + ((bh * n_a2 + first) * NX + xi) * D + dd;  // cell c at c NX D
    float acc[16];
    for (int u = 0; u < 16; ++u) acc[u] = 0.f;
    for (int64_t c0 = 0; c0 < ncell; c0 += kBatch) {
      float x[kBatch];
#pragma unroll
      for (int i = 0; i < kBatch; ++i) x[i] = c0 + i < ncell ? __ldg(src + (c0 + i) * NX * D) : 0.f;
      for (int i = 0; i < kBatch && c0 + i < ncell; ++i) {
        const int64_t c = c0 + i;
        acc[0] += x[i];
        int64_t pw = 1;
        for (int u = 0; u < nlev; ++u) {
          pw *= p;
          if ((c + 1) % pw != 0) break;
          const int lvl = a.A2 + 1 + u;
          const int64_t j = (first + c + 1) / pw - 1;
          if constexpr (MODE == MODE_PYRAMID) {
            if (a.do_pyr)
              static_cast<E*>(a.px[xi])[(bh * a.R + (a.off[lvl] - a.N) + j) * D + dd] =
                  from_f32<E>(__fmul_rn(acc[u], a.inv[lvl]));
          } else {
            int64_t cells_per_chunk = ncell / pw;
            const int r = cmap[cbase[u] + (int)(j - chunk * cells_per_chunk)];
            if (r >= 0) static_cast<E*>(a.px[0])[(bh * a.S + r) * D + dd] = from_f32<E>(acc[u]);
          }
          if (u + 1 < nlev) acc[u + 1] += acc[u];
          acc[u] = 0.f;
        }
      }
    }
  }
  if (MODE == MODE_PYRAMID && a.do_score && tid == NX * D) {
    const float* mx = a.tmp + (int64_t)gridDim.y * n_a2 * NX * D + (bh * n_a2 + first) * 2;
    const float* const prow = a.score_mode == 2 ? partner_row(a, bh) : nullptr;
    float q[16], k[16];
    for (int u = 0; u < 16; ++u) { q[u] = 0.f; k[u] = 0.f; }
    for (int64_t c0 = 0; c0 < ncell; c0 += kBatch) {
      float xq[kBatch], xk[kBatch];
#pragma unroll
      for (int i = 0; i < kBatch; ++i) {
        xq[i] = c0 + i < ncell ? __ldg(mx + (c0 + i) * 2) : 0.f;
        xk[i] = c0 + i < ncell ? __ldg(mx + (c0 + i) * 2 + 1) : 0.f;
      }
      for (int i = 0; i < kBatch && c0 + i < ncell; ++i) {
        const int64_t c = c0 + i;
        q[0] = fmaxf(q[0], xq[i]);
        k[0] = fmaxf(k[0], xk[i]);
        int64_t pw = 1;
        for (int u = 0; u < nlev; ++u) {
          pw *= p;
          if ((c + 1) % pw != 0) break;
          const int lvl = a.A2 + 1 + u;
          const int64_t j = (first + c + 1) / pw - 1;
          a.score[bh * (a.N + a.R) + a.off[lvl] + j] = cell_score(a, prow, q[u], k[u], a.off[lvl] + j);
          if (u + 1 < nlev) { q[u + 1] = fmaxf(q[u + 1], q[u]); k[u + 1] = fmaxf(k[u + 1], k[u]); }
          q[u] = 0.f; k[u] = 0.f;
        }
      }
    }
  }
}

// Register levels A for a pooling factor: the largest A <= min(L-1, 4) with p^A <= wmax.
int pick_A(int p, int L, int wmax) {
  int A = 0, pw = 1;
  while (A < L - 1 && A < 4 && pw * p <= wmax) { pw *= p; ++A; }
  return A;
}

struct Plan {
  int A, W, streams, U, A2;
};

Plan make_plan(const Geo& g, int wmax) {
  Plan pl;
  pl.A = pick_A(g.p, g.L, wmax);
  pl.W = 1;
  for (int i = 0; i < pl.A; ++i) pl.W *= g.p;
  const int vec = 16 / g.esize, lpr = g.d / vec;
  pl.streams = kThreads / lpr;
  pl.U = 0;
  if (pl.A > 0) {
    int sc = pl.streams;
    while (pl.A + pl.U < g.L - 1 && sc % g.p == 0) { sc /= g.p; ++pl.U; }
  }
  pl.A2 = pl.A + pl.U;
  return pl;
}

template <typename E, int D, int A, int MODE>
cudaError_t launch_tile_a(dim3 grid, const PoolArgs& a, cudaStream_t st) {
  constexpr int LPR = D / Vec<E>::N, STREAMS = kThreads / LPR;
  const size_t smem = MODE == MODE_PYRAMID ? (size_t)(2 * STREAMS * 16 * (LPR + 1) + 2 * STREAMS * 32) * sizeof(float) : 0;
  cudaError_t e = cudaFuncSetAttribute(pool_tile_kernel<E, D, A, MODE>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  pool_tile_kernel<E, D, A, MODE><<<grid, kThreads, smem, st>>>(a);
  return cudaGetLastError();
}

template <typename E, int D, int MODE>
cudaError_t launch_tile(const Plan& pl, const PoolArgs& a, int64_t BH, cudaStream_t st) {
  const int64_t tile = (int64_t)pl.W * pl.streams;
  dim3 grid((unsigned)((a.N + tile - 1) / tile), (unsigned)BH);
  switch (pl.A) {
    case 0: return launch_tile_a<E, D, 0, MODE>(grid, a, st);
    case 1: return launch_tile_a<E, D, 1, MODE>(grid, a, st);
    case 2: return launch_tile_a<E, D, 2, MODE>(grid, a, st);
    case 3: return launch_tile_a<E, D, 3, MODE>(grid, a, st);
    default: return launch_tile_a<E, D, 4, MODE>(grid, a, st);
  }
}

// heads: the (b,h) rows of the streamed tensors (B H, or B Hkv for the key/value pass)
template <int MODE>
cudaError_t run_pool(const Geo& g, PoolArgs& a, int64_t heads, cudaStream_t st) {
  const Plan pl = make_plan(g, MODE == MODE_SPANSUM ? kWMaxSpan : kWMaxPyr);
  a.N = g.N; a.R = g.R; a.S = g.S; a.T = g.T; a.m = g.m; a.C = g.C; a.G = g.G;
  a.p = g.p; a.L = g.L; a.W = pl.W; a.A2 = pl.A2; a.U = pl.U;
  for (int l = 0, w = pl.W; l < 8; ++l) {  // level-(l+1) cells per stream
    w = l < pl.A ? w / g.p : 0;
    a.wdiv[l] = w;
  }
  for (int l = 0; l < 16; ++l) {
    a.off[l] = l < g.L ? g.off[l] : 0;
    double pw = 1.0;
    for (int q = 0; q < l; ++q) pw *= g.p;
    a.inv[l] = l < g.L ? 1.0f / (float)pw : 0.f;
  }
  cudaError_t e;
  const bool bf = g.dtype == LH_BF16;
  if (g.d == 64)
    e = bf ? launch_tile<__nv_bfloat16, 64, MODE>(pl, a, heads, st) : launch_tile<float, 64, MODE>(pl, a, heads, st);
  else
    e = bf ? launch_tile<__nv_bfloat16, 128, MODE>(pl, a, heads, st) : launch_tile<float, 128, MODE>(pl, a, heads, st);
  if (e != cudaSuccess || pl.A2 >= g.L - 1) return e;
  const int nx = MODE == MODE_PYRAMID ? 3 : 1;
  dim3 grid((unsigned)g.C, (unsigned)heads);
  const int threads = ((nx * g.d + (MODE == MODE_PYRAMID ? 1 : 0) + 31) / 32) * 32;  // + the score thread
  // span sums: one map slot per cell of the levels above A2 inside a chunk
  size_t smem = 0;
  if (MODE == MODE_SPANSUM) {
    int64_t per = 1, tot = 0;
    for (int l = g.L - 1; l > pl.A2; --l) { tot += per; per *= g.p; }
    smem = (size_t)tot * sizeof(int);
  }
  if (bf) pool_coarse_kernel<__nv_bfloat16, MODE><<<grid, threads, smem, st>>>(a, g.d, nx);
  else pool_coarse_kernel<float, MODE><<<grid, threads, smem, st>>>(a, g.d, nx);
  return cudaGetLastError();
}

size_t tmp_bytes(const Geo& g, int nx, int wmax) {
  const Plan pl = make_plan(g, wmax);
  if (pl.A2 >= g.L - 1) return 0;
  int64_t pw = 1;
  for (int l = 0; l < pl.A2; ++l) pw *= g.p;
  const int64_t n = g.BH * (g.N / pw);
  return (size_t)(n * nx * g.d + n * 2) * sizeof(float);
}

}  // namespace

size_t pyramid_tmp_bytes(const Geo& g) { return tmp_bytes(g, 3, kWMaxPyr); }
int pool_launches(const Geo& g) {
  return (make_plan(g, kWMaxPyr).A2 >= g.L - 1 ? 1 : 2) * (g.grp > 1 ? 2 : 1);
}
size_t span_sum_tmp_bytes(const Geo& g) { return tmp_bytes(g, 1, kWMaxSpan); }
int span_sum_launches(const Geo& g) { return make_plan(g, kWMaxSpan).A2 >= g.L - 1 ? 1 : 2; }

cudaError_t launch_pyramid(const Geo& g, const void* q, const void* k, const void* v, void* pq,
                           void* pk, void* pv, float* score, void* tmp, float* kscore,
                           cudaStream_t st) {
  if (g.grp == 1) {  // q, k, v of each head in one pass; score = |q| + |k|
    PoolArgs a{};
    a.x[0] = q; a.x[1] = k; a.x[2] = v;
    a.px[0] = pq; a.px[1] = pk; a.px[2] = pv;
    a.score = score;
    a.tmp = static_cast<float*>(tmp);
    a.do_pyr = pq != nullptr;
    a.do_score = score != nullptr;
    a.nx = a.do_pyr ? 3 : 2;
    a.score_mode = 0;
    return run_pool<MODE_PYRAMID>(g, a, g.BH, st);
  }
  // Grouped heads: the key/value heads first (K and V pooled, the max-pooled |k| of every cell
  // into kscore), then the query heads (Q pooled, score = |q| + the kscore row of the head's
  // key/value head, the same fp32 sum as in one pass).
  PoolArgs a{};
  a.x[0] = k; a.x[1] = v;
  a.px[0] = pk; a.px[1] = pv;
  a.score = score ? kscore : nullptr;
  a.tmp = static_cast<float*>(tmp);
  a.do_pyr = pq != nullptr;
  a.do_score = score != nullptr;
  a.nx = a.do_pyr ? 2 : 1;
  a.score_mode = 1;
  cudaError_t e = run_pool<MODE_PYRAMID>(g, a, g.BHkv, st);
  if (e != cudaSuccess) return e;
  PoolArgs b{};
  b.x[0] = q;
  b.px[0] = pq;
  b.score = score;
  b.tmp = static_cast<float*>(tmp);
  b.do_pyr = pq != nullptr;
  b.do_score = score != nullptr;
  b.nx = 1;
  b.score_mode = 2;
  b.partner = kscore;
  b.H = g.H; b.grp = g.grp;
  return run_pool<MODE_PYRAMID>(g, b, g.BH, st);
}

cudaError_t launch_span_sum(const Geo& g, const int32_t* idx, const void* d_o, void* do_sub,
                            void* tmp, uint32_t* status, cudaStream_t st) {
  PoolArgs a{};
  a.x[0] = d_o;
  a.px[0] = do_sub;
  a.idx = idx;
  a.status = status;
  a.tmp = static_cast<float*>(tmp);
  a.do_pyr = 1;
  return run_pool<MODE_SPANSUM>(g, a, g.BH, st);
}

}  // namespace lh
