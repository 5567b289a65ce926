// Internal host-side declarations shared by the entry points and the kernels.
#pragma once

#include <cuda_runtime.h>
#include <nvtx3/nvToolsExt.h>
#include <stdint.h>

#include <string>

#include "lh.h"
#include "common.cuh"

namespace lh {

// NVTX range over one entry point or stage (a no-op unless a profiler is
// attached), so a trace shows the stages by name around their launches.
struct Range {
  explicit Range(const char* name) { nvtxRangePushA(name); }
  ~Range() { nvtxRangePop(); }
  Range(const Range&) = delete;
  Range& operator=(const Range&) = delete;
};

// Thread-local reason for the last non-OK status.
lh_status fail(lh_status s, const std::string& why);
lh_status ok();
// Map a CUDA error (from a launch or a runtime call) to a status.
lh_status cuda_status(cudaError_t e, const char* where);

Geo make_geo(const lh_plan& p);
// Argument checks shared by the attention entry points (sizes, dtype, d).
lh_status check_attn(int64_t BH, int64_t S, int32_t d, int32_t dtype);

// Calls f.template operator()<T, D>() for the plan's storage type and head
// dimension (d in {64, 128}, validated by lh_plan_init).
template <typename F>
void with_type_dim(const lh_plan& plan, F&& f) {
  const bool bf = plan.c.dtype == LH_BF16;
  if (plan.c.d == 128) {
    if (bf) f.template operator()<__nv_bfloat16, 128>();
    else f.template operator()<float, 128>();
  } else {
    if (bf) f.template operator()<__nv_bfloat16, 64>();
    else f.template operator()<float, 64>();
  }
}
// Device address of the status word that bounded waits set on timeout.
unsigned int* device_status_ptr();
bool aligned16(const void* ptr);
inline cudaStream_t as_cuda(lh_stream_t s) { return reinterpret_cast<cudaStream_t>(s); }

// Kernel launchers: enqueue only, return the launch error.
cudaError_t launch_pyramid_score(const lh_plan& plan, const void* Q, const void* K,
                                 const void* V, void* pyrQ, void* pyrK, void* pyrV,
                                 float* scores, bool pool, bool score, cudaStream_t st);
cudaError_t launch_topk(const lh_plan& plan, const float* scores, int32_t* sel_idx,
                        int32_t* slot_of, void* ws, cudaStream_t st);
int64_t topk_ws_bytes(const lh_plan& plan);
cudaError_t launch_gather(const lh_plan& plan, const void* Q, const void* K, const void* V,
                          const void* pyrQ, const void* pyrK, const void* pyrV,
                          const int32_t* sel_idx, void* Qg, void* Kg, void* Vg, cudaStream_t st);
cudaError_t launch_scatter(const lh_plan& plan, const void* Og, const int32_t* slot_of, void* O,
                           cudaStream_t st);
cudaError_t launch_scatter_bwd(const lh_plan& plan, const void* dO, const void* Og,
                               const int32_t* sel_idx, void* dOg, float* D, cudaStream_t st);
cudaError_t launch_gather_bwd(const lh_plan& plan, const void* dQg, const void* dKg,
                              const void* dVg, const int32_t* slot_of, void* dQ, void* dK,
                              void* dV, cudaStream_t st);
cudaError_t launch_attn_fwd(int64_t BH, int64_t S, int d, int dtype, const void* Qg, const void* Kg,
                            const void* Vg, void* Og, float* lse, cudaStream_t st);
int64_t attn_bwd_ws_bytes(int64_t BH, int64_t S, int d, int dtype);
void set_deterministic(int on);
int deterministic();
cudaError_t launch_attn_bwd(int64_t BH, int64_t S, int d, int dtype, const void* Qg, const void* Kg,
                            const void* Vg, const void* Og, const float* lse, const void* dOg,
                            const float* D, void* dQg, void* dKg, void* dVg, void* ws,
                            cudaStream_t st);
// bf16 attention with d = 128 (tcgen05).
cudaError_t launch_attn_fwd_tc128(int64_t BH, int64_t S, const void* Q, const void* K,
                                  const void* V, void* O, float* lse, cudaStream_t st);
// One CTA waiting on a barrier nothing signals (the failure-path self-test).
cudaError_t launch_wait_timeout_selftest(cudaStream_t st);

}  // namespace lh
