// Stage-3 attention dispatch: the storage dtype picks the kernel family.
#include <atomic>

#include "host.h"

namespace lh {

cudaError_t launch_attn_fwd_f32(int64_t BH, int64_t S, int d, const float* Q, const float* K,
                                const float* V, float* O, float* lse, cudaStream_t st);
cudaError_t launch_attn_bwd_f32(int64_t BH, int64_t S, int d, const float* Q, const float* K,
                                const float* V, const float* lse, const float* dO,
                                const float* D, float* dQ, float* dK, float* dV, cudaStream_t st);
cudaError_t launch_rowdot(int64_t rows, int d, int dtype, const void* dO, const void* O, float* D,
                          cudaStream_t st);
cudaError_t launch_attn_fwd_tc(int64_t BH, int64_t S, const void* Q, const void* K, const void* V,
                               void* O, float* lse, cudaStream_t st);
cudaError_t launch_attn_bwd_tc(int64_t BH, int64_t S, const void* Q, const void* K, const void* V,
                               const float* lse, const void* dO, const float* D, void* dQ,
                               void* dK, void* dV, float* dq_acc, cudaStream_t st);
cudaError_t launch_attn_bwd_tc128(int64_t BH, int64_t S, const void* Q, const void* K, const void* V,
                                  const float* lse, const void* dO, const float* D, void* dQ,
                                  void* dK, void* dV, float* dq_acc, cudaStream_t st);

namespace {
std::atomic<int> g_deterministic{0};
int64_t align256(int64_t x) { return (x + 255) & ~int64_t(255); }
}  // namespace

void set_deterministic(int on) { g_deterministic.store(on != 0); }
int deterministic() { return g_deterministic.load(); }

// [D when the caller passes none | bf16: fp32 dQ accumulator of the fused
// schedule, BH * S * d floats]
int64_t attn_bwd_ws_bytes(int64_t BH, int64_t S, int d, int dtype) {
  const int64_t d_bytes = align256(BH * S * 4);
  return dtype == LH_BF16 ? d_bytes + align256(BH * S * d * 4) : d_bytes;
}

cudaError_t launch_attn_fwd(int64_t BH, int64_t S, int d, int dtype, const void* Qg, const void* Kg,
                            const void* Vg, void* Og, float* lse, cudaStream_t st) {
  if (dtype == LH_F32)
    return launch_attn_fwd_f32(BH, S, d, (const float*)Qg, (const float*)Kg, (const float*)Vg,
                               (float*)Og, lse, st);
  if (d == 128) return launch_attn_fwd_tc128(BH, S, Qg, Kg, Vg, Og, lse, st);
  return launch_attn_fwd_tc(BH, S, Qg, Kg, Vg, Og, lse, st);
}

cudaError_t launch_attn_bwd(int64_t BH, int64_t S, int d, int dtype, const void* Qg, const void* Kg,
                            const void* Vg, const void* Og, const float* lse, const void* dOg,
                            const float* D, void* dQg, void* dKg, void* dVg, void* ws,
                            cudaStream_t st) {
  if (D == nullptr) {
    float* Dw = static_cast<float*>(ws);
    cudaError_t e = launch_rowdot(BH * S, d, dtype, dOg, Og, Dw, st);
    if (e != cudaSuccess) return e;
    D = Dw;
  }
  if (dtype == LH_F32)
    return launch_attn_bwd_f32(BH, S, d, (const float*)Qg, (const float*)Kg, (const float*)Vg, lse,
                               (const float*)dOg, D, (float*)dQg, (float*)dKg, (float*)dVg, st);
  // Without a workspace (the allocation-free entry point) or in deterministic
  // mode the two-kernel schedule runs; otherwise the fused one.
  float* dq_acc = (ws != nullptr && !deterministic())
                      ? reinterpret_cast<float*>(static_cast<char*>(ws) + align256(BH * S * 4))
                      : nullptr;
  if (d == 128)
    return launch_attn_bwd_tc128(BH, S, Qg, Kg, Vg, lse, dOg, D, dQg, dKg, dVg, dq_acc, st);
  return launch_attn_bwd_tc(BH, S, Qg, Kg, Vg, lse, dOg, D, dQg, dKg, dVg, dq_acc, st);
}

}  // namespace lh
