// Shared device helpers and the internal launch interface of the Lighthouse library.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "lh.h"

namespace lh {

constexpr uint32_t kFaultIndex = 1u;    // a row id outside [0, N+R)
constexpr uint32_t kFaultTimeout = 2u;  // a bounded wait ran out
constexpr uint32_t kFaultDrain = 4u;    // an abort-path wait for the CTA's own operations ran out

// Sizes derived from one layer shape (N_l = N/p^l cells per level, R pooled rows, C chunks of
// T = p^(L-1) tokens, M candidates per chunk; strata of G chunks with m = S G / C rows and
// k = m - G picks each), computed on the host.
struct Geo {
  int B, H, N, d, p, L, S, dtype;
  int flags;          // lh_shape.flags (LH_DETERMINISTIC)
  int Hkv, grp;       // key/value heads and query heads per key/value head (grp = H / Hkv)
  int64_t BHkv;       // B * Hkv
  uint64_t wait_ns;   // bound of every wait inside a kernel (lh_set_wait_limit_ns)
  int64_t BH, R, C, T, m, k, M;
  int64_t G;          // chunks per stratum (C / gcd(S, C))
  int64_t nlev[16];  // N_l = N / p^l
  int64_t off[16];   // row id of the first cell of level l (off[0] = 0, off[1] = N, ...)
  int64_t cand_off[16];  // offset of level l inside a chunk's candidate list (levels 0..L-2)
  int esize;          // bytes per element of the storage dtype
};

// Raw element <-> fp32 helpers. Loads and stores move 16 bytes per thread.
template <typename E> struct Vec;
template <> struct Vec<float> {
  static constexpr int N = 4;
  __device__ static inline void unpack(const uint4& u, float* f) {
    f[0] = __uint_as_float(u.x); f[1] = __uint_as_float(u.y);
    f[2] = __uint_as_float(u.z); f[3] = __uint_as_float(u.w);
  }
  __device__ static inline uint4 pack(const float* f) {
    return make_uint4(__float_as_uint(f[0]), __float_as_uint(f[1]), __float_as_uint(f[2]),
                      __float_as_uint(f[3]));
  }
};
template <> struct Vec<__nv_bfloat16> {
  static constexpr int N = 8;
  __device__ static inline void unpack(const uint4& u, float* f) {
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      f[2 * i] = __uint_as_float(w[i] << 16);
      f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
  }
  __device__ static inline uint4 pack(const float* f) {
    uint32_t w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      __nv_bfloat162 h = __floats2bfloat162_rn(f[2 * i], f[2 * i + 1]);
      w[i] = *reinterpret_cast<uint32_t*>(&h);
    }
    return make_uint4(w[0], w[1], w[2], w[3]);
  }
};

__device__ inline float to_f32(float x) { return x; }
__device__ inline float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }
template <typename E> __device__ inline E from_f32(float x);
template <> __device__ inline float from_f32<float>(float x) { return x; }
template <> __device__ inline __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);
}

__device__ inline uint4 ldg16(const void* p) { return __ldg(reinterpret_cast<const uint4*>(p)); }
// Bulk prefetch of [p, p + bytes) into L2 (16-byte aligned, size a multiple of 16); a hint that
// holds no registers and changes no result.
__device__ inline void prefetch_l2(const void* p, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}
__device__ inline void stg16(void* p, uint4 v) { *reinterpret_cast<uint4*>(p) = v; }
// Store with the evict-first (streaming) policy, for final outputs that no later kernel of the
// step reads back: the L2 then keeps the lines that are reused (the covering rows in the spread).
__device__ inline void stg16_stream(void* p, uint4 v) {
  asm volatile("st.global.cs.v4.b32 [%0], {%1, %2, %3, %4};" ::"l"(p), "r"(v.x), "r"(v.y), "r"(v.z),
               "r"(v.w) : "memory");
}

__device__ inline void raise_fault(uint32_t* status, uint32_t bit) {
  if (status) atomicOr(status, bit);
}

// Fills g from a shape: LH_OK, or the lh_status that says why the GPU path cannot take it.
int make_geo(const lh_shape* s, Geo& g);
// Records the CUDA error's text for lh_status_string and returns LH_ERR_CUDA.
int fail_cuda(cudaError_t e);

// ---- internal launchers (one per kernel family); all return cudaError_t of the launch ----
// kscore: [B Hkv, N+R] scratch for the max-pooled key norms when heads are grouped (grp > 1)
cudaError_t launch_pyramid(const Geo& g, const void* q, const void* k, const void* v, void* pq,
                           void* pk, void* pv, float* score, void* tmp, float* kscore,
                           cudaStream_t st);
size_t pyramid_tmp_bytes(const Geo& g);
int pool_launches(const Geo& g);  // 1 or 2: the tile kernel, plus the coarse kernel if needed
cudaError_t launch_select(const Geo& g, const float* score, int32_t* idx, cudaStream_t st);
cudaError_t launch_gather(const Geo& g, const void* q, const void* k, const void* v,
                          const void* pq, const void* pk, const void* pv, const int32_t* idx,
                          void* qs, void* ks, void* vs, uint32_t* status, cudaStream_t st);
cudaError_t launch_spread(const Geo& g, const int32_t* idx, int ntensor, bool from_f32,
                          bool scale_by_level, const void* const* src, void* const* dst,
                          uint32_t* status, cudaStream_t st);
// gather backward of K and V with grouped heads: dX of key/value head j adds, per token, the
// level-scaled fp32 rows of its query heads j grp .. j grp + grp - 1 (two tensors)
cudaError_t launch_spread_group(const Geo& g, const int32_t* idx, const void* const* src,
                                void* const* dst, uint32_t* status, cudaStream_t st);
cudaError_t launch_span_sum(const Geo& g, const int32_t* idx, const void* d_o, void* do_sub,
                            void* tmp, uint32_t* status, cudaStream_t st);
size_t span_sum_tmp_bytes(const Geo& g);
int span_sum_launches(const Geo& g);  // 1 or 2, as pool_launches
bool attn_tc_eligible(const Geo& g);  // bf16, d in {64,128}, S % 128 == 0
// The one-pass dK/dV/dQ backward runs (d = 128 on the tensor-core path, LH_DETERMINISTIC unset).
bool attn_bwd_fused(const Geo& g);
cudaError_t launch_attn_fwd_tc(const Geo& g, const void* qs, const void* ks, const void* vs,
                               float* os, float* lse, uint32_t* status, cudaStream_t st);
cudaError_t launch_attn_bwd_tc(const Geo& g, const void* qs, const void* ks, const void* vs,
                               const float* os, const float* lse, const void* dos, float* dq,
                               float* dk, float* dv, float* delta, uint32_t* status, cudaStream_t st);
// The attention backward as the library runs it: tensor cores where eligible, else fp32 FMA.
cudaError_t attn_bwd_dispatch(const Geo& g, const void* qs, const void* ks, const void* vs,
                              const float* os, const float* lse, const void* dos, float* dq,
                              float* dk, float* dv, float* delta, uint32_t* status, cudaStream_t st);
// Context-parallel forms: g.S query rows per (b,h) at global rows 128 kb0 .. of a key sequence of
// Sk rows per (b,h) (Sk = 128 kb0 + g.S); bf16, S % 128 == 0. The backward's dk, dv have Sk rows.
cudaError_t launch_attn_fwd_tc_rows(const Geo& g, int kb0, int Sk, const void* qs, const void* ks,
                                    const void* vs, float* os, float* lse, uint32_t* status,
                                    cudaStream_t st);
cudaError_t launch_attn_bwd_tc_rows(const Geo& g, int kb0, int Sk, const void* qs, const void* ks,
                                    const void* vs, const float* os, const float* lse,
                                    const void* dos, float* dq, float* dk, float* dv, float* delta,
                                    uint32_t* status, cudaStream_t st);
int attn_fwd_launches(const Geo& g);
int attn_bwd_launches(const Geo& g);
cudaError_t launch_attn_fwd_simt(const Geo& g, const void* qs, const void* ks, const void* vs,
                                 float* os, float* lse, cudaStream_t st);
cudaError_t launch_attn_bwd_simt(const Geo& g, const void* qs, const void* ks, const void* vs,
                                 const float* os, const float* lse, const void* dos, float* dq,
                                 float* dk, float* dv, float* delta, cudaStream_t st);

}  // namespace lh
