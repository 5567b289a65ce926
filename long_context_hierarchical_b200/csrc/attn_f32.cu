// Dense causal attention on the gathered sub-sequence, fp32 storage.
//
// Stage 3 runs plain causal softmax attention on the [S, d] sub-sequence
// (skill card "lighthouse-attention", stage 3: a standard S x S causal mask).
// The fp32 path is the accuracy path: tf32 tensor cores cannot hold a 1e-4
// tolerance, so it runs on the CUDA cores in fp32.  One warp owns one row
// (a query row forward and for dQ, a key row for dK/dV); lane l holds
// channels {l, l+32, ...} (d/32 of them); the dot products reduce across the
// warp.  Cost is O(S^2 d) with no tiling: this path serves short fp32
// sequences.
#include <math.h>

#include "host.h"

namespace lh {
namespace {

constexpr int kWarps = 8;

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// This lane's d/32 channels of one row.
template <int D>
struct Lane {
  static constexpr int C = D / 32;
  float v[C];
  __device__ __forceinline__ void load(const float* row, int lane) {
#pragma unroll
    for (int k = 0; k < C; ++k) v[k] = row[lane + 32 * k];
  }
  __device__ __forceinline__ void store(float* row, int lane, float s) const {
#pragma unroll
    for (int k = 0; k < C; ++k) row[lane + 32 * k] = v[k] * s;
  }
  __device__ __forceinline__ void zero() {
#pragma unroll
    for (int k = 0; k < C; ++k) v[k] = 0.f;
  }
  // Dot product of the whole row (every lane gets it).
  __device__ __forceinline__ float dot(const Lane& o) const {
    float a = 0.f;
#pragma unroll
    for (int k = 0; k < C; ++k) a = fmaf(v[k], o.v[k], a);
    return warp_sum(a);
  }
};

template <int D>
__global__ void __launch_bounds__(kWarps * 32)
attn_fwd_f32_kernel(int64_t BH, int64_t S, const float* __restrict__ Q, const float* __restrict__ K,
                    const float* __restrict__ V, float* __restrict__ O, float* __restrict__ lse,
                    float scale) {
  const int lane = threadIdx.x & 31;
  const int64_t row = (int64_t)blockIdx.x * kWarps + (threadIdx.x >> 5);
  if (row >= BH * S) return;
  const int64_t bh = row / S, i = row - bh * S;
  Lane<D> q, o;
  q.load(Q + row * D, lane);
  o.zero();
  const float* kb = K + bh * S * D;
  const float* vb = V + bh * S * D;
  float m = -INFINITY, l = 0.f;
  for (int64_t j = 0; j <= i; ++j) {
    Lane<D> k, v;
    k.load(kb + j * D, lane);
    v.load(vb + j * D, lane);
    const float s = q.dot(k) * scale;
    const float mn = fmaxf(m, s);
    const float a = expf(m - mn);  // 0 on the first key
    const float p = expf(s - mn);
    l = l * a + p;
#pragma unroll
    for (int c = 0; c < Lane<D>::C; ++c) o.v[c] = o.v[c] * a + p * v.v[c];
    m = mn;
  }
#pragma unroll
  for (int c = 0; c < Lane<D>::C; ++c) O[row * D + lane + 32 * c] = o.v[c] / l;
  if (lane == 0) lse[row] = m + logf(l);
}

// D[i] = sum_c dO[i,c] * O[i,c]
template <typename T>
__global__ void __launch_bounds__(kWarps * 32)
rowdot_kernel(int64_t rows, int d, const T* __restrict__ dO, const T* __restrict__ O,
              float* __restrict__ D) {
  const int lane = threadIdx.x & 31;
  const int64_t row = (int64_t)blockIdx.x * kWarps + (threadIdx.x >> 5);
  if (row >= rows) return;
  float a = 0.f;
  for (int c = lane; c < d; c += 32)
    a = fmaf((float)dO[row * d + c], (float)O[row * d + c], a);
  a = warp_sum(a);
  if (lane == 0) D[row] = a;
}

// dQ_i = scale * sum_{j<=i} P_ij (dP_ij - D_i) K_j
template <int D>
__global__ void __launch_bounds__(kWarps * 32)
attn_bwd_dq_f32_kernel(int64_t BH, int64_t S, const float* __restrict__ Q, const float* __restrict__ K,
                       const float* __restrict__ V, const float* __restrict__ lse,
                       const float* __restrict__ dO, const float* __restrict__ Drow,
                       float* __restrict__ dQ, float scale) {
  const int lane = threadIdx.x & 31;
  const int64_t row = (int64_t)blockIdx.x * kWarps + (threadIdx.x >> 5);
  if (row >= BH * S) return;
  const int64_t bh = row / S, i = row - bh * S;
  Lane<D> q, g, a;
  q.load(Q + row * D, lane);
  g.load(dO + row * D, lane);
  a.zero();
  const float li = lse[row], Di = Drow[row];
  const float* kb = K + bh * S * D;
  const float* vb = V + bh * S * D;
  for (int64_t j = 0; j <= i; ++j) {
    Lane<D> k, v;
    k.load(kb + j * D, lane);
    v.load(vb + j * D, lane);
    const float s = q.dot(k) * scale;
    const float dp = g.dot(v);
    const float ds = expf(s - li) * (dp - Di);
#pragma unroll
    for (int c = 0; c < Lane<D>::C; ++c) a.v[c] = fmaf(ds, k.v[c], a.v[c]);
  }
  a.store(dQ + row * D, lane, scale);
}

// dV_j = sum_{i>=j} P_ij dO_i ;  dK_j = scale * sum_{i>=j} P_ij (dP_ij - D_i) Q_i
template <int D>
__global__ void __launch_bounds__(kWarps * 32)
attn_bwd_dkv_f32_kernel(int64_t BH, int64_t S, const float* __restrict__ Q, const float* __restrict__ K,
                        const float* __restrict__ V, const float* __restrict__ lse,
                        const float* __restrict__ dO, const float* __restrict__ Drow,
                        float* __restrict__ dK, float* __restrict__ dV, float scale) {
  const int lane = threadIdx.x & 31;
  const int64_t row = (int64_t)blockIdx.x * kWarps + (threadIdx.x >> 5);
  if (row >= BH * S) return;
  const int64_t bh = row / S, j = row - bh * S;
  Lane<D> k, v, dk, dv;
  k.load(K + row * D, lane);
  v.load(V + row * D, lane);
  dk.zero();
  dv.zero();
  const float* qb = Q + bh * S * D;
  const float* gb = dO + bh * S * D;
  const float* lb = lse + bh * S;
  const float* db = Drow + bh * S;
  for (int64_t i = j; i < S; ++i) {
    Lane<D> q, g;
    q.load(qb + i * D, lane);
    g.load(gb + i * D, lane);
    const float s = q.dot(k) * scale;
    const float p = expf(s - lb[i]);
    const float dp = g.dot(v);
    const float ds = p * (dp - db[i]);
#pragma unroll
    for (int c = 0; c < Lane<D>::C; ++c) {
      dv.v[c] = fmaf(p, g.v[c], dv.v[c]);
      dk.v[c] = fmaf(ds, q.v[c], dk.v[c]);
    }
  }
  dk.store(dK + row * D, lane, scale);
  dv.store(dV + row * D, lane, 1.f);
}

// 1/sqrt(d), rounded once to fp32.
float softmax_scale(int d) { return (float)(1.0 / sqrt((double)d)); }

}  // namespace

cudaError_t launch_attn_fwd_f32(int64_t BH, int64_t S, int d, const float* Q, const float* K,
                                const float* V, float* O, float* lse, cudaStream_t st) {
  const unsigned blocks = (unsigned)((BH * S + kWarps - 1) / kWarps);
  if (d == 128)
    attn_fwd_f32_kernel<128><<<blocks, kWarps * 32, 0, st>>>(BH, S, Q, K, V, O, lse, softmax_scale(d));
  else
    attn_fwd_f32_kernel<64><<<blocks, kWarps * 32, 0, st>>>(BH, S, Q, K, V, O, lse, softmax_scale(d));
  return cudaGetLastError();
}

cudaError_t launch_rowdot(int64_t rows, int d, int dtype, const void* dO, const void* O, float* D,
                          cudaStream_t st) {
  const unsigned blocks = (unsigned)((rows + kWarps - 1) / kWarps);
  if (dtype == LH_BF16)
    rowdot_kernel<__nv_bfloat16><<<blocks, kWarps * 32, 0, st>>>(
        rows, d, (const __nv_bfloat16*)dO, (const __nv_bfloat16*)O, D);
  else
    rowdot_kernel<float><<<blocks, kWarps * 32, 0, st>>>(rows, d, (const float*)dO, (const float*)O, D);
  return cudaGetLastError();
}

cudaError_t launch_attn_bwd_f32(int64_t BH, int64_t S, int d, const float* Q, const float* K,
                                const float* V, const float* lse, const float* dO,
                                const float* D, float* dQ, float* dK, float* dV, cudaStream_t st) {
  const unsigned blocks = (unsigned)((BH * S + kWarps - 1) / kWarps);
  const float sc = softmax_scale(d);
  if (d == 128) {
    attn_bwd_dq_f32_kernel<128><<<blocks, kWarps * 32, 0, st>>>(BH, S, Q, K, V, lse, dO, D, dQ, sc);
    attn_bwd_dkv_f32_kernel<128><<<blocks, kWarps * 32, 0, st>>>(BH, S, Q, K, V, lse, dO, D, dK, dV, sc);
  } else {
    attn_bwd_dq_f32_kernel<64><<<blocks, kWarps * 32, 0, st>>>(BH, S, Q, K, V, lse, dO, D, dQ, sc);
    attn_bwd_dkv_f32_kernel<64><<<blocks, kWarps * 32, 0, st>>>(BH, S, Q, K, V, lse, dO, D, dK, dV, sc);
  }
  return cudaGetLastError();
}

}  // namespace lh
