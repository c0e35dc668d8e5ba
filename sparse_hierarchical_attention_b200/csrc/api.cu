// C ABI of the Lighthouse selection layer: validation, workspace layout, dispatch and the
// layer-level orchestration of the five steps (declared in include/lh.h).
#include <atomic>
#include <cstdio>
#include <cstring>

#include "common.cuh"

namespace lh {

namespace {
thread_local char g_last_error[256] = "";
constexpr uint64_t kDefaultWaitNs = 2000000000ull;
std::atomic<uint64_t> g_wait_ns{kDefaultWaitNs};
}  // namespace

int fail_cuda(cudaError_t e) {
  std::snprintf(g_last_error, sizeof(g_last_error), "%s", cudaGetErrorString(e));
  return LH_ERR_CUDA;
}

// Fills g from a shape; returns LH_OK or the reason the GPU path cannot take it.
int make_geo(const lh_shape* s, Geo& g) {
  if (!s) return LH_ERR_INVALID_ARG;
  std::memset(&g, 0, sizeof(g));
  g.B = s->B; g.H = s->H; g.N = s->N; g.d = s->d; g.p = s->p; g.L = s->L; g.S = s->S;
  g.dtype = s->dtype;
  g.flags = s->flags;
  g.Hkv = s->Hkv ? s->Hkv : s->H;
  g.wait_ns = g_wait_ns.load(std::memory_order_relaxed);
  if (s->flags & ~LH_DETERMINISTIC) return LH_ERR_INVALID_ARG;
  if (g.B < 1 || g.H < 1 || g.N < 1 || g.d < 1 || g.p < 2 || g.L < 1 || g.S < 1)
    return LH_ERR_INVALID_ARG;
  if (g.dtype != LH_F32 && g.dtype != LH_BF16) return LH_ERR_INVALID_ARG;
  if (g.Hkv < 1 || g.H % g.Hkv) return LH_ERR_INVALID_ARG;
  g.grp = g.H / g.Hkv;
  if (g.L > 12 || g.p > 16) return LH_ERR_UNSUPPORTED;
  int64_t T = 1;
  for (int l = 1; l < g.L; ++l) {
    T *= g.p;
    if (T > (1 << 20)) return LH_ERR_UNSUPPORTED;
  }
  if (g.N % T) return LH_ERR_INVALID_ARG;
  g.T = T;
  g.C = g.N / T;
  // Strata: the fewest consecutive chunks over which the budget S divides evenly.
  {
    int64_t a = g.S, b = g.C;
    while (b) { const int64_t t = a % b; a = b; b = t; }
    g.G = g.C / a;  // C / gcd(S, C): 1 whenever S is a multiple of C
  }
  g.m = g.S * g.G / g.C;  // rows per stratum
  g.k = g.m - g.G;        // picks per stratum besides its G coarsest cells
  g.M = 0;
  for (int l = 0; l + 1 < g.L; ++l) {
    g.cand_off[l] = g.M;
    int64_t per = 1;
    for (int q = l; q + 1 < g.L; ++q) per *= g.p;
    g.M += per;
  }
  if (g.S < g.C || g.S > g.C * (g.M + 1)) return LH_ERR_INVALID_ARG;
  g.BH = (int64_t)g.B * g.H;
  g.BHkv = (int64_t)g.B * g.Hkv;
  g.R = 0;
  int64_t nl = g.N;
  for (int l = 0; l < g.L; ++l) {
    g.nlev[l] = nl;
    g.off[l] = l == 0 ? 0 : g.N + g.R;
    if (l > 0) g.R += nl;
    nl /= g.p;
  }
  if (g.N + g.R >= (int64_t)1 << 31) return LH_ERR_UNSUPPORTED;
  if (g.d != 64 && g.d != 128) return LH_ERR_UNSUPPORTED;
  g.esize = g.dtype == LH_BF16 ? 2 : 4;
  if (g.BH > 65535 || g.C > 0x7fffffff) return LH_ERR_UNSUPPORTED;
  // shared-memory limits of the selection and spread kernels
  // shared-memory limits of the selection (a stratum's candidate keys, its winners and per-chunk
  // counts) and spread kernels; the key packs a cell's stratum-local index into 24 bits
  // (the spread of grouped heads maps the cells of all grp query heads of a chunk at once)
  if ((size_t)(g.G * g.M + g.k) * 8 + (size_t)g.G * 4 > 200 * 1024 ||
      (size_t)(g.M + 1) * 4 * g.grp > 200 * 1024)
    return LH_ERR_UNSUPPORTED;
  if (g.G * g.T >= ((int64_t)1 << 24)) return LH_ERR_UNSUPPORTED;
  return LH_OK;
}

namespace {

size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

bool aligned(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Workspace layout: [status 256 B | forward region or backward region (they never overlap in
// time)]. Forward: pq, pk, pv, score, pooling scratch. Backward: do_sub, delta, dq_sub,
// dk_sub, dv_sub, span-sum scratch.
struct WsLayout {
  size_t status, pq, pk, pv, score, ptmp, kscore, fwd_end;
  size_t do_sub, delta, dq, dk, dv, stmp, bwd_end;
  size_t total;
};

WsLayout ws_layout(const Geo& g) {
  WsLayout w{};
  const size_t pyr = align256((size_t)(g.BH * g.R * g.d) * g.esize);
  const size_t pyr_kv = align256((size_t)(g.BHkv * g.R * g.d) * g.esize);
  const size_t sub = align256((size_t)(g.BH * g.S * g.d) * g.esize);
  const size_t sub32 = align256((size_t)(g.BH * g.S * g.d) * 4);
  const size_t row32 = align256((size_t)(g.BH * g.S) * 4);
  size_t o = 0;
  w.status = o; o += 256;
  const size_t base = o;
  w.pq = o; o += pyr;
  w.pk = o; o += pyr_kv;
  w.pv = o; o += pyr_kv;
  w.score = o; o += align256((size_t)(g.BH * (g.N + g.R)) * 4);
  w.ptmp = o; o += align256(pyramid_tmp_bytes(g));
  w.kscore = o;  // grouped heads: the max-pooled key norms of every key/value head
  if (g.grp > 1) o += align256((size_t)(g.BHkv * (g.N + g.R)) * 4);
  w.fwd_end = o;
  o = base;
  w.do_sub = o; o += sub;
  w.delta = o; o += row32;
  w.dq = o; o += sub32;
  w.dk = o; o += sub32;
  w.dv = o; o += sub32;
  w.stmp = o; o += align256(span_sum_tmp_bytes(g));
  w.bwd_end = o;
  w.total = w.fwd_end > w.bwd_end ? w.fwd_end : w.bwd_end;
  return w;
}

struct SavedLayout {
  size_t idx, qs, ks, vs, os, lse, total;
};

SavedLayout saved_layout(const Geo& g) {
  SavedLayout s{};
  const size_t sub = align256((size_t)(g.BH * g.S * g.d) * g.esize);
  size_t o = 0;
  s.idx = o; o += align256((size_t)(g.BH * g.S) * 4);
  s.qs = o; o += sub;
  s.ks = o; o += sub;
  s.vs = o; o += sub;
  s.os = o; o += align256((size_t)(g.BH * g.S * g.d) * 4);  // fp32 o_sub
  s.lse = o; o += align256((size_t)(g.BH * g.S) * 4);
  s.total = o;
  return s;
}

template <typename T> T* at(void* base, size_t off) {
  return reinterpret_cast<T*>(static_cast<char*>(base) + off);
}
template <typename T> const T* at(const void* base, size_t off) {
  return reinterpret_cast<const T*>(static_cast<const char*>(base) + off);
}

#define LH_CHECK_GEO(shape, g)        \
  Geo g;                              \
  {                                   \
    const int rc_ = make_geo(shape, g); \
    if (rc_ != LH_OK) return rc_;     \
  }
#define LH_REQUIRE_PTR(p) \
  if (!(p) || !aligned(p)) return LH_ERR_INVALID_ARG
#define LH_CUDA(call)                       \
  {                                         \
    const cudaError_t e_ = (call);          \
    if (e_ != cudaSuccess) return fail_cuda(e_); \
  }

cudaError_t attn_fwd(const Geo& g, const void* qs, const void* ks, const void* vs, float* os,
                     float* lse, uint32_t* status, cudaStream_t st) {
  if (attn_tc_eligible(g)) return launch_attn_fwd_tc(g, qs, ks, vs, os, lse, status, st);
  return launch_attn_fwd_simt(g, qs, ks, vs, os, lse, st);
}

// dQ, dK, dV from the fp32 sub-gradients: one spread of the three when every query head has its
// own key/value head; with grouped heads dQ per query head, then dK and dV per key/value head
// over its group's selections.
cudaError_t spread_grads(const Geo& g, const int32_t* idx, const float* dqs, const float* dks,
                         const float* dvs, void* dq, void* dk, void* dv, uint32_t* status,
                         cudaStream_t st) {
  if (g.grp == 1) {
    const void* src[3] = {dqs, dks, dvs};
    void* dst[3] = {dq, dk, dv};
    return launch_spread(g, idx, 3, true, true, src, dst, status, st);
  }
  const void* src_q[1] = {dqs};
  void* dst_q[1] = {dq};
  cudaError_t e = launch_spread(g, idx, 1, true, true, src_q, dst_q, status, st);
  if (e != cudaSuccess) return e;
  const void* src_kv[2] = {dks, dvs};
  void* dst_kv[2] = {dk, dv};
  return launch_spread_group(g, idx, src_kv, dst_kv, status, st);
}

cudaError_t attn_bwd(const Geo& g, const void* qs, const void* ks, const void* vs,
                     const float* os, const float* lse, const void* dos, float* dq, float* dk,
                     float* dv, float* delta, uint32_t* status, cudaStream_t st) {
  return attn_bwd_dispatch(g, qs, ks, vs, os, lse, dos, dq, dk, dv, delta, status, st);
}

}  // namespace

cudaError_t attn_bwd_dispatch(const Geo& g, const void* qs, const void* ks, const void* vs,
                              const float* os, const float* lse, const void* dos, float* dq,
                              float* dk, float* dv, float* delta, uint32_t* status, cudaStream_t st) {
  if (attn_tc_eligible(g))
    return launch_attn_bwd_tc(g, qs, ks, vs, os, lse, dos, dq, dk, dv, delta, status, st);
  return launch_attn_bwd_simt(g, qs, ks, vs, os, lse, dos, dq, dk, dv, delta, st);
}

}  // namespace lh

using namespace lh;

extern "C" {

const char* lh_status_string(int status) {
  switch (status) {
    case LH_OK: return "ok";
    case LH_ERR_INVALID_ARG: return "invalid argument";
    case LH_ERR_UNSUPPORTED: return "unsupported by the GPU path";
    case LH_ERR_WORKSPACE: return "workspace too small";
    case LH_ERR_CUDA: return g_last_error[0] ? g_last_error : "CUDA error";
    case LH_ERR_DEVICE: return "a kernel reported a fault (see lh_check flags)";
    default: return "unknown status";
  }
}

const char* lh_version(void) { return "lighthouse-b200 0.1 (sm_100a)"; }

int lh_validate(const lh_shape* shape, lh_sizes* out) {
  LH_CHECK_GEO(shape, g);
  if (out) {
    out->R = g.R; out->C = g.C; out->T = g.T; out->m = g.m; out->k = g.k; out->M = g.M;
    out->G = g.G;
  }
  return LH_OK;
}

size_t lh_workspace_bytes(const lh_shape* shape) {
  Geo g;
  if (make_geo(shape, g) != LH_OK) return 0;
  return ws_layout(g).total;
}

size_t lh_saved_bytes(const lh_shape* shape) {
  Geo g;
  if (make_geo(shape, g) != LH_OK) return 0;
  return saved_layout(g).total;
}

int lh_launches(const lh_shape* shape, int* fwd, int* bwd) {
  LH_CHECK_GEO(shape, g);
  // forward: pyramid (+coarse; a key/value pass first with grouped heads), select, gather,
  // attention, scatter
  if (fwd) *fwd = pool_launches(g) + 1 + 1 + attn_fwd_launches(g) + 1;
  // backward: span sums (+coarse), attention backward, gather backward (two with grouped heads)
  if (bwd) *bwd = span_sum_launches(g) + attn_bwd_launches(g) + (g.grp > 1 ? 2 : 1);
  return LH_OK;
}

int lh_saved_offsets(const lh_shape* shape, size_t offsets[6]) {
  LH_CHECK_GEO(shape, g);
  if (!offsets) return LH_ERR_INVALID_ARG;
  const SavedLayout s = saved_layout(g);
  offsets[0] = s.idx; offsets[1] = s.qs; offsets[2] = s.ks;
  offsets[3] = s.vs; offsets[4] = s.os; offsets[5] = s.lse;
  return LH_OK;
}

uint64_t lh_set_wait_limit_ns(uint64_t ns) {
  return g_wait_ns.exchange(ns ? ns : kDefaultWaitNs);
}

int lh_workspace_init(void* ws, void* stream) {
  LH_REQUIRE_PTR(ws);
  LH_CUDA(cudaMemsetAsync(ws, 0, 256, static_cast<cudaStream_t>(stream)));
  return LH_OK;
}

int lh_check(void* ws, void* stream, uint32_t* flags) {
  LH_REQUIRE_PTR(ws);
  uint32_t h = 0;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  LH_CUDA(cudaStreamSynchronize(st));
  LH_CUDA(cudaMemcpy(&h, ws, sizeof(h), cudaMemcpyDeviceToHost));
  LH_CUDA(cudaMemset(ws, 0, sizeof(uint32_t)));
  if (flags) *flags = h;
  return h ? LH_ERR_DEVICE : LH_OK;
}

int lh_build_pyramid(const lh_shape* shape, const void* q, const void* k, const void* v,
                     void* pq, void* pk, void* pv, float* score, void* ws, void* stream) {
  LH_CHECK_GEO(shape, g);
  LH_REQUIRE_PTR(q); LH_REQUIRE_PTR(k); LH_REQUIRE_PTR(ws);
  const bool pyr = pq || pk || pv;
  if (pyr && g.R > 0) { LH_REQUIRE_PTR(v); LH_REQUIRE_PTR(pq); LH_REQUIRE_PTR(pk); LH_REQUIRE_PTR(pv); }
  if (!pyr && !score) return LH_ERR_INVALID_ARG;
  if (score && !aligned(score)) return LH_ERR_INVALID_ARG;
  const WsLayout w = ws_layout(g);
  LH_CUDA(launch_pyramid(g, q, k, v, (pyr && g.R > 0) ? pq : nullptr, pk, pv, score,
                         at<char>(ws, w.ptmp), at<float>(ws, w.kscore), static_cast<cudaStream_t>(stream)));
  return LH_OK;
}

int lh_score(const lh_shape* shape, const void* q, const void* k, float* score, void* ws,
             void* stream) {
  return lh_build_pyramid(shape, q, k, nullptr, nullptr, nullptr, nullptr, score, ws, stream);
}

int lh_select_topk(const lh_shape* shape, const float* score, int32_t* idx, void* stream) {
  LH_CHECK_GEO(shape, g);
  LH_REQUIRE_PTR(score); LH_REQUIRE_PTR(idx);
  LH_CUDA(launch_select(g, score, idx, static_cast<cudaStream_t>(stream)));
  return LH_OK;
}

int lh_gather(const lh_shape* shape, const void* q, const void* k, const void* v,
              const void* pq, const void* pk, const void* pv, const int32_t* idx,
              void* q_sub, void* k_sub, void* v_sub, void* ws, void* stream) {
  LH_CHECK_GEO(shape, g);
  LH_REQUIRE_PTR(q); LH_REQUIRE_PTR(k); LH_REQUIRE_PTR(v); LH_REQUIRE_PTR(idx);
  LH_REQUIRE_PTR(q_sub); LH_REQUIRE_PTR(k_sub); LH_REQUIRE_PTR(v_sub); LH_REQUIRE_PTR(ws);
  if (g.R > 0) { LH_REQUIRE_PTR(pq); LH_REQUIRE_PTR(pk); LH_REQUIRE_PTR(pv); }
  LH_CUDA(launch_gather(g, q, k, v, pq, pk, pv, idx, q_sub, k_sub, v_sub,
                        at<uint32_t>(ws, 0), static_cast<cudaStream_t>(stream)));
  return LH_OK;
}

int lh_attn_fwd(const lh_shape* shape, const void* q_sub, const void* k_sub, const void* v_sub,
                float* o_sub, float* lse, void* ws, void* stream) {
  LH_CHECK_GEO(shape, g);
  LH_REQUIRE_PTR(q_sub); LH_REQUIRE_PTR(k_sub); LH_REQUIRE_PTR(v_sub);
  LH_REQUIRE_PTR(o_sub); LH_REQUIRE_PTR(lse); LH_REQUIRE_PTR(ws);
  LH_CUDA(attn_fwd(g, q_sub, k_sub, v_sub, o_sub, lse, at<uint32_t>(ws, 0),
                   static_cast<cudaStream_t>(stream)));
  return LH_OK;
}

int lh_attn_bwd(const lh_shape* shape, const void* q_sub, const void* k_sub, const void* v_sub,
                const float* o_sub, const float* lse, const void* do_sub, float* dq_sub,
                float* dk_sub, float* dv_sub, void* ws, void* stream) {
  LH_CHECK_GEO(shape, g);
  LH_REQUIRE_PTR(q_sub); LH_REQUIRE_PTR(k_sub); LH_REQUIRE_PTR(v_sub); LH_REQUIRE_PTR(o_sub);
  LH_REQUIRE_PTR(lse); LH_REQUIRE_PTR(do_sub); LH_REQUIRE_PTR(dq_sub); LH_REQUIRE_PTR(dk_sub);
  LH_REQUIRE_PTR(dv_sub); LH_REQUIRE_PTR(ws);
  const WsLayout w = ws_layout(g);
  LH_CUDA(attn_bwd(g, q_sub, k_sub, v_sub, o_sub, lse, do_sub, dq_sub, dk_sub, dv_sub,
                   at<float>(ws, w.delta), at<uint32_t>(ws, 0), static_cast<cudaStream_t>(stream)));
  return LH_OK;
}

namespace {
// Shapes the context-parallel attention takes; fills the key rows per (b,h).
int cp_check(const Geo& g, int64_t row0, int* kb0, int* Sk) {
  if (row0 < 0) return LH_ERR_INVALID_ARG;
  if (g.dtype != LH_BF16 || g.d != 128 || g.S % 128 || row0 % 128) return LH_ERR_UNSUPPORTED;
  if (g.BH * (row0 + g.S) >= ((int64_t)1 << 31)) return LH_ERR_UNSUPPORTED;
  *kb0 = (int)(row0 / 128);
  *Sk = (int)(row0 + g.S);
  return LH_OK;
}
}  // namespace

int lh_attn_fwd_cp(const lh_shape* shape, int64_t row0, const void* q_sub, const void* k_seen,
                   const void* v_seen, float* o_sub, float* lse, void* ws, void* stream) {
  LH_CHECK_GEO(shape, g);
  int kb0 = 0, Sk = 0;
  const int rc = cp_check(g, row0, &kb0, &Sk);
  if (rc != LH_OK) return rc;
  LH_REQUIRE_PTR(q_sub); LH_REQUIRE_PTR(k_seen); LH_REQUIRE_PTR(v_seen);
  LH_REQUIRE_PTR(o_sub); LH_REQUIRE_PTR(lse); LH_REQUIRE_PTR(ws);
  LH_CUDA(launch_attn_fwd_tc_rows(g, kb0, Sk, q_sub, k_seen, v_seen, o_sub, lse, at<uint32_t>(ws, 0),
                                  static_cast<cudaStream_t>(stream)));
  return LH_OK;
}

int lh_attn_bwd_cp(const lh_shape* shape, int64_t row0, const void* q_sub, const void* k_seen,
                   const void* v_seen, const float* o_sub, const float* lse, const void* do_sub,
                   float* dq_sub, float* dk_seen, float* dv_seen, void* ws, void* stream) {
  LH_CHECK_GEO(shape, g);
  int kb0 = 0, Sk = 0;
  const int rc = cp_check(g, row0, &kb0, &Sk);
  if (rc != LH_OK) return rc;
  LH_REQUIRE_PTR(q_sub); LH_REQUIRE_PTR(k_seen); LH_REQUIRE_PTR(v_seen); LH_REQUIRE_PTR(o_sub);
  LH_REQUIRE_PTR(lse); LH_REQUIRE_PTR(do_sub); LH_REQUIRE_PTR(dq_sub); LH_REQUIRE_PTR(dk_seen);
  LH_REQUIRE_PTR(dv_seen); LH_REQUIRE_PTR(ws);
  const WsLayout w = ws_layout(g);
  LH_CUDA(launch_attn_bwd_tc_rows(g, kb0, Sk, q_sub, k_seen, v_seen, o_sub, lse, do_sub, dq_sub, dk_seen,
                                  dv_seen, at<float>(ws, w.delta), at<uint32_t>(ws, 0),
                                  static_cast<cudaStream_t>(stream)));
  return LH_OK;
}

int lh_scatter(const lh_shape* shape, const int32_t* idx, const float* o_sub, void* o,
               void* stream) {
  LH_CHECK_GEO(shape, g);
  LH_REQUIRE_PTR(idx); LH_REQUIRE_PTR(o_sub); LH_REQUIRE_PTR(o);
  const void* src[1] = {o_sub};
  void* dst[1] = {o};
  LH_CUDA(launch_spread(g, idx, 1, true, false, src, dst, nullptr, static_cast<cudaStream_t>(stream)));
  return LH_OK;
}

int lh_scatter_bwd(const lh_shape* shape, const int32_t* idx, const void* d_o, void* do_sub,
                   void* ws, void* stream) {
  LH_CHECK_GEO(shape, g);
  LH_REQUIRE_PTR(idx); LH_REQUIRE_PTR(d_o); LH_REQUIRE_PTR(do_sub); LH_REQUIRE_PTR(ws);
  const WsLayout w = ws_layout(g);
  LH_CUDA(launch_span_sum(g, idx, d_o, do_sub, at<char>(ws, w.stmp), at<uint32_t>(ws, 0),
                          static_cast<cudaStream_t>(stream)));
  return LH_OK;
}

int lh_gather_bwd(const lh_shape* shape, const int32_t* idx, const float* dq_sub,
                  const float* dk_sub, const float* dv_sub, void* dq, void* dk, void* dv,
                  void* stream) {
  LH_CHECK_GEO(shape, g);
  LH_REQUIRE_PTR(idx); LH_REQUIRE_PTR(dq_sub); LH_REQUIRE_PTR(dk_sub); LH_REQUIRE_PTR(dv_sub);
  LH_REQUIRE_PTR(dq); LH_REQUIRE_PTR(dk); LH_REQUIRE_PTR(dv);
  LH_CUDA(spread_grads(g, idx, dq_sub, dk_sub, dv_sub, dq, dk, dv, nullptr,
                       static_cast<cudaStream_t>(stream)));
  return LH_OK;
}

int lh_layer_fwd(const lh_shape* shape, const void* q, const void* k, const void* v, void* o,
                 void* saved, void* ws, void* stream) {
  LH_CHECK_GEO(shape, g);
  LH_REQUIRE_PTR(q); LH_REQUIRE_PTR(k); LH_REQUIRE_PTR(v); LH_REQUIRE_PTR(o);
  LH_REQUIRE_PTR(saved); LH_REQUIRE_PTR(ws);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const WsLayout w = ws_layout(g);
  const SavedLayout s = saved_layout(g);
  uint32_t* status = at<uint32_t>(ws, 0);
  void* pq = g.R > 0 ? at<char>(ws, w.pq) : nullptr;
  void* pk = g.R > 0 ? at<char>(ws, w.pk) : nullptr;
  void* pv = g.R > 0 ? at<char>(ws, w.pv) : nullptr;
  float* score = at<float>(ws, w.score);
  int32_t* idx = at<int32_t>(saved, s.idx);
  LH_CUDA(launch_pyramid(g, q, k, v, pq, pk, pv, score, at<char>(ws, w.ptmp), at<float>(ws, w.kscore), st));
  LH_CUDA(launch_select(g, score, idx, st));
  LH_CUDA(launch_gather(g, q, k, v, pq, pk, pv, idx, at<char>(saved, s.qs), at<char>(saved, s.ks),
                        at<char>(saved, s.vs), status, st));
  LH_CUDA(attn_fwd(g, at<char>(saved, s.qs), at<char>(saved, s.ks), at<char>(saved, s.vs),
                   at<float>(saved, s.os), at<float>(saved, s.lse), status, st));
  const void* src[1] = {at<float>(saved, s.os)};
  void* dst[1] = {o};
  LH_CUDA(launch_spread(g, idx, 1, true, false, src, dst, status, st));
  return LH_OK;
}

int lh_layer_bwd(const lh_shape* shape, const void* saved, const void* d_o, void* dq, void* dk,
                 void* dv, void* ws, void* stream) {
  LH_CHECK_GEO(shape, g);
  LH_REQUIRE_PTR(saved); LH_REQUIRE_PTR(d_o); LH_REQUIRE_PTR(dq); LH_REQUIRE_PTR(dk);
  LH_REQUIRE_PTR(dv); LH_REQUIRE_PTR(ws);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const WsLayout w = ws_layout(g);
  const SavedLayout s = saved_layout(g);
  uint32_t* status = at<uint32_t>(ws, 0);
  const int32_t* idx = at<int32_t>(saved, s.idx);
  void* dos = at<char>(ws, w.do_sub);
  float* dqs = at<float>(ws, w.dq);
  float* dks = at<float>(ws, w.dk);
  float* dvs = at<float>(ws, w.dv);
  LH_CUDA(launch_span_sum(g, idx, d_o, dos, at<char>(ws, w.stmp), status, st));
  LH_CUDA(attn_bwd(g, at<char>(saved, s.qs), at<char>(saved, s.ks), at<char>(saved, s.vs),
                   at<float>(saved, s.os), at<float>(saved, s.lse), dos, dqs, dks, dvs,
                   at<float>(ws, w.delta), status, st));
  LH_CUDA(spread_grads(g, idx, dqs, dks, dvs, dq, dk, dv, status, st));
  return LH_OK;
}

}  // extern "C"
