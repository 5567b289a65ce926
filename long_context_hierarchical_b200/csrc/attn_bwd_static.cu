// lh_attn_bwd_static: the attention backward for callers that cannot
// allocate device memory.  The only scratch lh_attn_bwd needs is the row term
// D = rowsum(dOg * Og) when the caller does not pass it; here D lives in a
// fixed array compiled into the library instead of a caller workspace.
#include <mutex>

#include "host.h"

namespace lh {

cudaError_t launch_rowdot(int64_t rows, int d, int dtype, const void* dO, const void* O, float* D,
                          cudaStream_t st);

namespace {

constexpr int64_t kStaticRows = LH_ATTN_BWD_STATIC_MAX_ROWS;

// Scratch for D: one float per (problem, row), shared by every call.
__device__ __align__(256) float g_attn_bwd_scratch[kStaticRows];

constexpr int kMaxDevices = 64;
float* g_scratch_ptr[kMaxDevices] = {};
std::mutex g_scratch_mu;

// Device address of the scratch array on the current device.  In host code
// the array's name is only a host-side handle, so the address is looked up
// once per device, with that device current, and cached.
cudaError_t scratch_on_current_device(float** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (g_scratch_ptr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_attn_bwd_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_ptr[dev] = static_cast<float*>(p);
  }
  *out = g_scratch_ptr[dev];
  return cudaSuccess;
}

}  // namespace
}  // namespace lh

using namespace lh;

extern "C" lh_status lh_attn_bwd_static(int64_t BH, int64_t S, int32_t d, int32_t dtype,
                                        const void* Qg, const void* Kg, const void* Vg,
                                        const void* Og, const float* lse, const void* dOg,
                                        void* dQg, void* dKg, void* dVg, lh_stream_t stream) {
  if (BH < 1 || S < 1) return fail(LH_ERR_INVALID_ARG, "BH and S must be >= 1");
  if (dtype != LH_F32 && dtype != LH_BF16)
    return fail(LH_ERR_UNSUPPORTED, "dtype must be LH_F32 or LH_BF16");
  if (d != 64 && d != 128) return fail(LH_ERR_UNSUPPORTED, "only d in {64, 128} is built");
  if (BH > kStaticRows / S)
    return fail(LH_ERR_WORKSPACE,
                "lh_attn_bwd_static: BH * S exceeds LH_ATTN_BWD_STATIC_MAX_ROWS (1048576 rows)");
  const void* ptrs[] = {Qg, Kg, Vg, Og, lse, dOg, dQg, dKg, dVg};
  for (const void* q : ptrs)
    if (!aligned16(q)) return fail(LH_ERR_INVALID_ARG, "a pointer is null or not 16-byte aligned");
  float* D = nullptr;
  lh_status s = cuda_status(scratch_on_current_device(&D), "lh_attn_bwd_static/scratch");
  if (s != LH_OK) return s;
  cudaStream_t st = as_cuda(stream);
  s = cuda_status(launch_rowdot(BH * S, d, dtype, dOg, Og, D, st), "lh_attn_bwd_static/rowdot");
  if (s != LH_OK) return s;
  s = cuda_status(launch_attn_bwd(BH, S, d, dtype, Qg, Kg, Vg, Og, lse, dOg, D, dQg, dKg, dVg,
                                  nullptr, st),
                  "lh_attn_bwd_static");
  if (s != LH_OK) return s;
  return ok();
}
