// lh_attn_bwd_static: the attention backward for callers that cannot
// allocate device memory.  The only scratch lh_attn_bwd needs is the row term
// D = rowsum(dOg * Og) when the caller does not pass it; here D lives in a
// fixed array compiled into the library instead of a caller workspace.
#include "host.h"

namespace lh {

cudaError_t launch_rowdot(int64_t rows, int d, int dtype, const void* dO, const void* O, float* D,
                          cudaStream_t st);

namespace {

constexpr int64_t kStaticRows = LH_ATTN_BWD_STATIC_MAX_ROWS;

// Scratch for D: one float per (problem, row), shared by every call.
__device__ __align__(256) float g_attn_bwd_scratch[kStaticRows];

// Device address of the scratch array in the current device's context.  In
// host code the array's name is only a host-side handle; the address is
// looked up on every call (a host-side call), so it stays right after a
// device reset, in another context and on every device.
cudaError_t scratch_on_current_device(float** out) {
  void* p = nullptr;
  cudaError_t e = cudaGetSymbolAddress(&p, g_attn_bwd_scratch);
  if (e != cudaSuccess) return e;
  *out = static_cast<float*>(p);
  return cudaSuccess;
}

}  // namespace
}  // namespace lh

using namespace lh;

extern "C" lh_status lh_attn_bwd_static(int64_t BH, int64_t S, int32_t d, int32_t dtype,
                                        const void* Qg, const void* Kg, const void* Vg,
                                        const void* Og, const float* lse, const void* dOg,
                                        void* dQg, void* dKg, void* dVg, lh_stream_t stream) {
  Range range("lh_attn_bwd_static");
  lh_status s = check_attn(BH, S, d, dtype);
  if (s != LH_OK) return s;
  if (BH > kStaticRows / S)
    return fail(LH_ERR_WORKSPACE,
                "lh_attn_bwd_static: BH * S exceeds LH_ATTN_BWD_STATIC_MAX_ROWS (1048576 rows)");
  const void* ptrs[] = {Qg, Kg, Vg, Og, lse, dOg, dQg, dKg, dVg};
  for (const void* q : ptrs)
    if (!aligned16(q)) return fail(LH_ERR_INVALID_ARG, "a pointer is null or not 16-byte aligned");
  float* D = nullptr;
  s = cuda_status(scratch_on_current_device(&D), "lh_attn_bwd_static/scratch");
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
