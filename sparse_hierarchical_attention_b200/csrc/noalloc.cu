// lh_attn_bwd_static and lh_check_static: the attention backward without a caller-supplied
// workspace.
//
// Some callers cannot allocate device memory at all. Examples are a plugin whose host
// framework owns every device allocation, and code running where the allocator is off limits.
// Those callers cannot provide the workspace that lh_attn_bwd takes for its per-row
// D_i = dO_sub[i] . O_sub[i] and its status word. This entry point keeps that scratch in a
// file-scope device array instead:
//   - its size is fixed at compile time;
//   - every GPU that loads this library holds it until the process exits.
// The caller still passes every input and output buffer.
//
// The paper has no counterpart: this is a deployment variant of the same kernels.
#include <mutex>

#include "common.cuh"

namespace lh {
namespace {

// 256 bytes of status word, then D for up to LH_STATIC_SCRATCH_ROWS rows (4 MiB).
constexpr size_t kStatusBytes = 256;
constexpr size_t kStaticBytes = kStatusBytes + (size_t)LH_STATIC_SCRATCH_ROWS * sizeof(float);

static __device__ __align__(256) unsigned char g_static_scratch[kStaticBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_dev_ptr[kMaxDevices] = {};  // device address of g_static_scratch, per device ordinal

// Device address of the static scratch on the current device. In host code the array's name
// is only a host-side stand-in, so the address must come from cudaGetSymbolAddress, with the
// device current. The first call on a device resolves it and clears the status word (a
// synchronous set-up, so that first call must not be inside a stream capture); later calls
// reuse the cached address.
cudaError_t scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_dev_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_static_scratch);
    if (e != cudaSuccess) return e;
    // the status word starts at zero (set once here; lh_check_static clears it after a read)
    e = cudaMemset(p, 0, kStatusBytes);
    if (e != cudaSuccess) return e;
    e = cudaDeviceSynchronize();
    if (e != cudaSuccess) return e;
    g_dev_ptr[dev] = p;
  }
  *out = g_dev_ptr[dev];
  return cudaSuccess;
}

}  // namespace
}  // namespace lh

using namespace lh;

extern "C" int lh_attn_bwd_static(const lh_shape* shape, const void* q_sub, const void* k_sub,
                                  const void* v_sub, const float* o_sub, const float* lse,
                                  const void* do_sub, float* dq_sub, float* dk_sub, float* dv_sub,
                                  void* stream) {
  Geo g;
  const int rc = make_geo(shape, g);
  if (rc != LH_OK) return rc;
  if (g.BH * g.S > (int64_t)LH_STATIC_SCRATCH_ROWS) return LH_ERR_WORKSPACE;
  const void* ptrs[] = {q_sub, k_sub, v_sub, o_sub, lse, do_sub, dq_sub, dk_sub, dv_sub};
  for (const void* p : ptrs)
    if (!p || (reinterpret_cast<uintptr_t>(p) & 15u)) return LH_ERR_INVALID_ARG;
  void* base = nullptr;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e = scratch_address(&base);
  if (e != cudaSuccess) return fail_cuda(e);
  // D is written in full before it is read. The status word is not cleared here: a fault of an
  // earlier call stays latched until lh_check_static reads and clears it.
  float* delta = reinterpret_cast<float*>(static_cast<char*>(base) + kStatusBytes);
  uint32_t* dev_status = reinterpret_cast<uint32_t*>(base);
  e = attn_bwd_dispatch(g, q_sub, k_sub, v_sub, o_sub, lse, do_sub, dq_sub, dk_sub, dv_sub, delta,
                        dev_status, st);
  if (e != cudaSuccess) return fail_cuda(e);
  return LH_OK;
}

extern "C" int lh_check_static(void* stream, uint32_t* flags) {
  void* base = nullptr;
  cudaError_t e = scratch_address(&base);
  if (e != cudaSuccess) return fail_cuda(e);
  uint32_t h = 0;
  if ((e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream))) != cudaSuccess) return fail_cuda(e);
  if ((e = cudaMemcpy(&h, base, sizeof(h), cudaMemcpyDeviceToHost)) != cudaSuccess) return fail_cuda(e);
  if ((e = cudaMemset(base, 0, sizeof(h))) != cudaSuccess) return fail_cuda(e);
  if (flags) *flags = h;
  return h ? LH_ERR_DEVICE : LH_OK;
}
