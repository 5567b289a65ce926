// Dense causal attention on the gathered sub-sequence, fp32 storage.
//
// Stage 3 runs plain causal softmax attention on the [S, d] sub-sequence
// (skill card "lighthouse-attention", stage 3: a standard S x S causal mask).
// The fp32 path is the accuracy path: tf32 tensor cores cannot hold a 1e-4
// tolerance, so it runs on the CUDA cores in fp32.  One warp owns one row
// (a query row forward and for dQ, a key row for dK/dV); lane l holds
// channels {l, l+32}; the dot products reduce across the warp.  Cost is
// O(S^2 d) with no tiling: this path serves short fp32 sequences.
#include "host.h"

namespace lh {
namespace {

constexpr int kWarps = 8;

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__global__ void __launch_bounds__(kWarps * 32)
attn_fwd_f32_kernel(int64_t BH, int64_t S, const float* __restrict__ Q, const float* __restrict__ K,
                    const float* __restrict__ V, float* __restrict__ O, float* __restrict__ lse,
                    float scale) {
  const int lane = threadIdx.x & 31;
  const int64_t row = (int64_t)blockIdx.x * kWarps + (threadIdx.x >> 5);
  if (row >= BH * S) return;
  const int64_t bh = row / S, i = row - bh * S;
  const float* q = Q + row * kD;
  const float q0 = q[lane], q1 = q[lane + 32];
  const float* kb = K + bh * S * kD;
  const float* vb = V + bh * S * kD;
  float m = -INFINITY, l = 0.f, o0 = 0.f, o1 = 0.f;
  for (int64_t j = 0; j <= i; ++j) {
    const float s = warp_sum(q0 * kb[j * kD + lane] + q1 * kb[j * kD + lane + 32]) * scale;
    const float mn = fmaxf(m, s);
    const float a = expf(m - mn);  // 0 on the first key
    const float p = expf(s - mn);
    l = l * a + p;
    o0 = o0 * a + p * vb[j * kD + lane];
    o1 = o1 * a + p * vb[j * kD + lane + 32];
    m = mn;
  }
  O[row * kD + lane] = o0 / l;
  O[row * kD + lane + 32] = o1 / l;
  if (lane == 0) lse[row] = m + logf(l);
}

// D[i] = sum_c dO[i,c] * O[i,c]
template <typename T>
__global__ void __launch_bounds__(kWarps * 32)
rowdot_kernel(int64_t rows, const T* __restrict__ dO, const T* __restrict__ O, float* __restrict__ D) {
  const int lane = threadIdx.x & 31;
  const int64_t row = (int64_t)blockIdx.x * kWarps + (threadIdx.x >> 5);
  if (row >= rows) return;
  float a = 0.f;
  for (int c = lane; c < kD; c += 32)
    a = fmaf((float)dO[row * kD + c], (float)O[row * kD + c], a);
  a = warp_sum(a);
  if (lane == 0) D[row] = a;
}

// dQ_i = scale * sum_{j<=i} P_ij (dP_ij - D_i) K_j
__global__ void __launch_bounds__(kWarps * 32)
attn_bwd_dq_f32_kernel(int64_t BH, int64_t S, const float* __restrict__ Q, const float* __restrict__ K,
                       const float* __restrict__ V, const float* __restrict__ lse,
                       const float* __restrict__ dO, const float* __restrict__ D,
                       float* __restrict__ dQ, float scale) {
  const int lane = threadIdx.x & 31;
  const int64_t row = (int64_t)blockIdx.x * kWarps + (threadIdx.x >> 5);
  if (row >= BH * S) return;
  const int64_t bh = row / S, i = row - bh * S;
  const float q0 = Q[row * kD + lane], q1 = Q[row * kD + lane + 32];
  const float g0 = dO[row * kD + lane], g1 = dO[row * kD + lane + 32];
  const float li = lse[row], Di = D[row];
  const float* kb = K + bh * S * kD;
  const float* vb = V + bh * S * kD;
  float a0 = 0.f, a1 = 0.f;
  for (int64_t j = 0; j <= i; ++j) {
    const float k0 = kb[j * kD + lane], k1 = kb[j * kD + lane + 32];
    const float s = warp_sum(q0 * k0 + q1 * k1) * scale;
    const float dp = warp_sum(g0 * vb[j * kD + lane] + g1 * vb[j * kD + lane + 32]);
    const float ds = expf(s - li) * (dp - Di);
    a0 = fmaf(ds, k0, a0);
    a1 = fmaf(ds, k1, a1);
  }
  dQ[row * kD + lane] = a0 * scale;
  dQ[row * kD + lane + 32] = a1 * scale;
}

// dV_j = sum_{i>=j} P_ij dO_i ;  dK_j = scale * sum_{i>=j} P_ij (dP_ij - D_i) Q_i
__global__ void __launch_bounds__(kWarps * 32)
attn_bwd_dkv_f32_kernel(int64_t BH, int64_t S, const float* __restrict__ Q, const float* __restrict__ K,
                        const float* __restrict__ V, const float* __restrict__ lse,
                        const float* __restrict__ dO, const float* __restrict__ D,
                        float* __restrict__ dK, float* __restrict__ dV, float scale) {
  const int lane = threadIdx.x & 31;
  const int64_t row = (int64_t)blockIdx.x * kWarps + (threadIdx.x >> 5);
  if (row >= BH * S) return;
  const int64_t bh = row / S, j = row - bh * S;
  const float k0 = K[row * kD + lane], k1 = K[row * kD + lane + 32];
  const float v0 = V[row * kD + lane], v1 = V[row * kD + lane + 32];
  const float* qb = Q + bh * S * kD;
  const float* gb = dO + bh * S * kD;
  const float* lb = lse + bh * S;
  const float* db = D + bh * S;
  float dk0 = 0.f, dk1 = 0.f, dv0 = 0.f, dv1 = 0.f;
  for (int64_t i = j; i < S; ++i) {
    const float q0 = qb[i * kD + lane], q1 = qb[i * kD + lane + 32];
    const float g0 = gb[i * kD + lane], g1 = gb[i * kD + lane + 32];
    const float s = warp_sum(q0 * k0 + q1 * k1) * scale;
    const float p = expf(s - lb[i]);
    const float dp = warp_sum(g0 * v0 + g1 * v1);
    const float ds = p * (dp - db[i]);
    dv0 = fmaf(p, g0, dv0);
    dv1 = fmaf(p, g1, dv1);
    dk0 = fmaf(ds, q0, dk0);
    dk1 = fmaf(ds, q1, dk1);
  }
  dK[row * kD + lane] = dk0 * scale;
  dK[row * kD + lane + 32] = dk1 * scale;
  dV[row * kD + lane] = dv0;
  dV[row * kD + lane + 32] = dv1;
}

}  // namespace

cudaError_t launch_attn_fwd_f32(int64_t BH, int64_t S, const float* Q, const float* K,
                                const float* V, float* O, float* lse, cudaStream_t st) {
  const unsigned blocks = (unsigned)((BH * S + kWarps - 1) / kWarps);
  attn_fwd_f32_kernel<<<blocks, kWarps * 32, 0, st>>>(BH, S, Q, K, V, O, lse, 0.125f);
  return cudaGetLastError();
}

cudaError_t launch_rowdot(int64_t rows, int dtype, const void* dO, const void* O, float* D,
                          cudaStream_t st) {
  const unsigned blocks = (unsigned)((rows + kWarps - 1) / kWarps);
  if (dtype == LH_BF16)
    rowdot_kernel<__nv_bfloat16><<<blocks, kWarps * 32, 0, st>>>(
        rows, (const __nv_bfloat16*)dO, (const __nv_bfloat16*)O, D);
  else
    rowdot_kernel<float><<<blocks, kWarps * 32, 0, st>>>(rows, (const float*)dO, (const float*)O, D);
  return cudaGetLastError();
}

cudaError_t launch_attn_bwd_f32(int64_t BH, int64_t S, const float* Q, const float* K,
                                const float* V, const float* lse, const float* dO,
                                const float* D, float* dQ, float* dK, float* dV, cudaStream_t st) {
  const unsigned blocks = (unsigned)((BH * S + kWarps - 1) / kWarps);
  attn_bwd_dq_f32_kernel<<<blocks, kWarps * 32, 0, st>>>(BH, S, Q, K, V, lse, dO, D, dQ, 0.125f);
  attn_bwd_dkv_f32_kernel<<<blocks, kWarps * 32, 0, st>>>(BH, S, Q, K, V, lse, dO, D, dK, dV, 0.125f);
  return cudaGetLastError();
}

}  // namespace lh
