// Stage 3 gather, stage 4 scatter-back, and their backward passes.
//
// Gather (skill card "lighthouse-attention", stage 3; gist.science Technical
// Summary 2.C): the selected pyramid rows are copied into dense [S, d]
// tensors in the causal order fixed by lh_topk.
// Scatter-back (stage 4 "Scatter-back 重建"; gist.science 2.C "deterministic
// scatter kernel"): output row t sums, over levels, the attention output of
// the entry whose range R(l, i) = [i p^l + p^l - 1, i p^l + 2 p^l - 2]
// contains t, i.e. i = floor((t+1)/p^l) - 1; at most L rows per token.
// Backward ("梯度流": dL -> scatter -> attention -> gather): the adjoints of
// those two maps, plus the softmax-backward row term D.
//
// All four kernels are "one 8-lane group per row": lane c of a group moves
// channels [8c, 8c+8) with 16-byte accesses, so a warp touches 4 whole rows
// per instruction.  The scatter and gather-backward kernels are
// token-centric and sum in a fixed (ascending-level) order: no atomics, and
// the result does not depend on scheduling.
#include "host.h"

namespace lh {
namespace {

constexpr int kThreads = 256;
constexpr int kRowsPerBlock = kThreads / 8;

template <typename T>
__device__ __forceinline__ void copy_chunk(T* dst, const T* src) {
  // 8 elements: 16 bytes for bf16, 32 for fp32.
  const uint4* s = reinterpret_cast<const uint4*>(src);
  uint4* d = reinterpret_cast<uint4*>(dst);
#pragma unroll
  for (int i = 0; i < (int)(8 * sizeof(T) / 16); ++i) d[i] = __ldg(s + i);
}

template <typename T>
__global__ void __launch_bounds__(kThreads)
gather_kernel(Geo g, const T* __restrict__ Q, const T* __restrict__ K, const T* __restrict__ V,
              const T* __restrict__ pQ, const T* __restrict__ pK, const T* __restrict__ pV,
              const int32_t* __restrict__ sel_idx, T* __restrict__ Qg, T* __restrict__ Kg,
              T* __restrict__ Vg) {
  const int64_t row = (int64_t)blockIdx.x * kRowsPerBlock + (threadIdx.x >> 3);
  const int c = threadIdx.x & 7;
  if (row >= g.BH * g.S) return;
  const int64_t bh = row / g.S;
  const int64_t f = sel_idx[row];
  const int64_t dst = row * kD + c * 8;
  if (f < 0 || f >= g.Ntot) {  // not a pyramid index: write zeros, read nothing
    const float z[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    Vec8<T>::store(Qg + dst, z);
    Vec8<T>::store(Kg + dst, z);
    Vec8<T>::store(Vg + dst, z);
    return;
  }
  const int l = level_of(g, f);
  const int64_t i = f - g.flat_off[l];
  int64_t src;
  const T *sq, *sk, *sv;
  if (l == 0) {
    src = (bh * g.N + i) * kD;
    sq = Q; sk = K; sv = V;
  } else {
    src = (bh * g.Npyr + g.pyr_off[l] + i) * kD;
    sq = pQ; sk = pK; sv = pV;
  }
  copy_chunk(Qg + dst, sq + src + c * 8);
  copy_chunk(Kg + dst, sk + src + c * 8);
  copy_chunk(Vg + dst, sv + src + c * 8);
}

template <typename T>
__device__ __forceinline__ void store_stream(T* p, const float (&x)[8]);
template <>
__device__ __forceinline__ void store_stream<__nv_bfloat16>(__nv_bfloat16* p, const float (&x)[8]) {
  uint32_t w[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    __nv_bfloat162 h = __floats2bfloat162_rn(x[2 * i], x[2 * i + 1]);
    w[i] = *reinterpret_cast<uint32_t*>(&h);
  }
  __stcs(reinterpret_cast<uint4*>(p), make_uint4(w[0], w[1], w[2], w[3]));
}
template <>
__device__ __forceinline__ void store_stream<float>(float* p, const float (&x)[8]) {
  __stcs(reinterpret_cast<float4*>(p), make_float4(x[0], x[1], x[2], x[3]));
  __stcs(reinterpret_cast<float4*>(p) + 1, make_float4(x[4], x[5], x[6], x[7]));
}

// L is a template parameter so the per-level index loads and row loads are
// all issued before the first one is used.
template <typename T, int L>
__global__ void __launch_bounds__(kThreads)
scatter_kernel(Geo g, const T* __restrict__ Og, const int32_t* __restrict__ slot_of,
               T* __restrict__ O) {
  const int64_t row = (int64_t)blockIdx.x * kRowsPerBlock + (threadIdx.x >> 3);
  const int c = threadIdx.x & 7;
  if (row >= g.BH * g.N) return;
  const int64_t bh = row / g.N;
  const int64_t t = row - bh * g.N;
  const int32_t* inv = slot_of + bh * g.Ntot;
  const T* og = Og + bh * g.S * kD + c * 8;
  int32_t slot[L];
#pragma unroll
  for (int l = 0; l < L; ++l) {
    const int64_t i = ((t + 1) >> (g.logp * l)) - 1;
    slot[l] = i >= 0 ? __ldg(inv + g.flat_off[l] + i) : -1;
  }
  float x[L][8];
#pragma unroll
  for (int l = 0; l < L; ++l) {
    if (slot[l] >= 0 && slot[l] < g.S) Vec8<T>::load(og + (int64_t)slot[l] * kD, x[l]);
    else {
#pragma unroll
      for (int e = 0; e < 8; ++e) x[l][e] = 0.f;
    }
  }
  float acc[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    acc[e] = 0.f;
#pragma unroll
    for (int l = 0; l < L; ++l) acc[e] += x[l][e];  // ascending level
  }
  store_stream<T>(O + row * kD + c * 8, acc);
}

template <typename T>
__global__ void __launch_bounds__(kThreads)
scatter_bwd_kernel(Geo g, const T* __restrict__ dO, const T* __restrict__ Og,
                   const int32_t* __restrict__ sel_idx, T* __restrict__ dOg, float* __restrict__ D) {
  const int64_t row = (int64_t)blockIdx.x * kRowsPerBlock + (threadIdx.x >> 3);
  const int c = threadIdx.x & 7;
  const bool live = row < g.BH * g.S;
  const int64_t r = live ? row : 0;
  const int64_t bh = r / g.S;
  int64_t f = sel_idx[r];
  if (f < 0 || f >= g.Ntot) f = g.Ntot - 1;  // unreachable for a valid selection
  const int l = level_of(g, f);
  const int64_t i = f - g.flat_off[l];
  const int sh = g.logp * l;
  const int64_t lo = ((i + 1) << sh) - 1;
  const int64_t hi = min(lo + (int64_t(1) << sh) - 1, g.N - 1);
  const T* src = dO + bh * g.N * kD + c * 8;
  float acc[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) acc[e] = 0.f;
  for (int64_t t = lo; t <= hi; ++t) {
    float x[8];
    Vec8<T>::load(src + t * kD, x);
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] += x[e];
  }
  float o[8];
  Vec8<T>::load(Og + r * kD + c * 8, o);
  float dsum = 0.f;
#pragma unroll
  for (int e = 0; e < 8; ++e) dsum = fmaf(Vec8<T>::rounded(acc[e]), o[e], dsum);
  dsum += __shfl_xor_sync(0xffffffffu, dsum, 1);
  dsum += __shfl_xor_sync(0xffffffffu, dsum, 2);
  dsum += __shfl_xor_sync(0xffffffffu, dsum, 4);
  if (!live) return;
  Vec8<T>::store(dOg + r * kD + c * 8, acc);
  if (c == 0) D[r] = dsum;
}

template <typename T, int L>
__global__ void __launch_bounds__(kThreads)
gather_bwd_kernel(Geo g, const T* __restrict__ dQg, const T* __restrict__ dKg,
                  const T* __restrict__ dVg, const int32_t* __restrict__ slot_of,
                  T* __restrict__ dQ, T* __restrict__ dK, T* __restrict__ dV) {
  const int64_t row = (int64_t)blockIdx.x * kRowsPerBlock + (threadIdx.x >> 3);
  const int c = threadIdx.x & 7;
  if (row >= g.BH * g.N) return;
  const int64_t bh = row / g.N;
  const int64_t t = row - bh * g.N;
  const int32_t* inv = slot_of + bh * g.Ntot;
  const int64_t base = bh * g.S * kD + c * 8;
  int32_t slot[L];
#pragma unroll
  for (int l = 0; l < L; ++l) slot[l] = __ldg(inv + g.flat_off[l] + (t >> (g.logp * l)));
  const T* src[3] = {dQg, dKg, dVg};
  T* dst[3] = {dQ, dK, dV};
#pragma unroll
  for (int w = 0; w < 3; ++w) {
    float x[L][8];
#pragma unroll
    for (int l = 0; l < L; ++l) {
      if (slot[l] >= 0 && slot[l] < g.S) Vec8<T>::load(src[w] + base + (int64_t)slot[l] * kD, x[l]);
      else {
#pragma unroll
        for (int e = 0; e < 8; ++e) x[l][e] = 0.f;
      }
    }
    float acc[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      acc[e] = 0.f;
#pragma unroll
      for (int l = 0; l < L; ++l)  // ascending level; 1/p^l is a power of two: exact
        acc[e] = fmaf(x[l][e], 1.f / (float)(1 << (g.logp * l)), acc[e]);
    }
    store_stream<T>(dst[w] + row * kD + c * 8, acc);
  }
}

unsigned blocks_for(int64_t rows) { return (unsigned)((rows + kRowsPerBlock - 1) / kRowsPerBlock); }

}  // namespace

cudaError_t launch_gather(const lh_plan& plan, const void* Q, const void* K, const void* V,
                          const void* pyrQ, const void* pyrK, const void* pyrV,
                          const int32_t* sel_idx, void* Qg, void* Kg, void* Vg, cudaStream_t st) {
  const Geo g = make_geo(plan);
  const unsigned b = blocks_for(g.BH * g.S);
  if (plan.c.dtype == LH_BF16) {
    using T = __nv_bfloat16;
    gather_kernel<T><<<b, kThreads, 0, st>>>(g, (const T*)Q, (const T*)K, (const T*)V,
                                             (const T*)pyrQ, (const T*)pyrK, (const T*)pyrV,
                                             sel_idx, (T*)Qg, (T*)Kg, (T*)Vg);
  } else {
    using T = float;
    gather_kernel<T><<<b, kThreads, 0, st>>>(g, (const T*)Q, (const T*)K, (const T*)V,
                                             (const T*)pyrQ, (const T*)pyrK, (const T*)pyrV,
                                             sel_idx, (T*)Qg, (T*)Kg, (T*)Vg);
  }
  return cudaGetLastError();
}

template <typename T, int L>
void scatter_l(const Geo& g, unsigned b, const void* Og, const int32_t* slot_of, void* O, cudaStream_t st) {
  scatter_kernel<T, L><<<b, kThreads, 0, st>>>(g, (const T*)Og, slot_of, (T*)O);
}

template <typename T>
void scatter_t(const Geo& g, unsigned b, const void* Og, const int32_t* slot_of, void* O, cudaStream_t st) {
  switch (g.L) {
    case 1: scatter_l<T, 1>(g, b, Og, slot_of, O, st); break;
    case 2: scatter_l<T, 2>(g, b, Og, slot_of, O, st); break;
    case 3: scatter_l<T, 3>(g, b, Og, slot_of, O, st); break;
    case 4: scatter_l<T, 4>(g, b, Og, slot_of, O, st); break;
    default: scatter_l<T, 5>(g, b, Og, slot_of, O, st); break;
  }
}

cudaError_t launch_scatter(const lh_plan& plan, const void* Og, const int32_t* slot_of, void* O,
                           cudaStream_t st) {
  const Geo g = make_geo(plan);
  const unsigned b = blocks_for(g.BH * g.N);
  if (plan.c.dtype == LH_BF16) scatter_t<__nv_bfloat16>(g, b, Og, slot_of, O, st);
  else scatter_t<float>(g, b, Og, slot_of, O, st);
  return cudaGetLastError();
}

cudaError_t launch_scatter_bwd(const lh_plan& plan, const void* dO, const void* Og,
                               const int32_t* sel_idx, void* dOg, float* D, cudaStream_t st) {
  const Geo g = make_geo(plan);
  const unsigned b = blocks_for(g.BH * g.S);
  if (plan.c.dtype == LH_BF16) {
    using T = __nv_bfloat16;
    scatter_bwd_kernel<T><<<b, kThreads, 0, st>>>(g, (const T*)dO, (const T*)Og, sel_idx, (T*)dOg, D);
  } else {
    using T = float;
    scatter_bwd_kernel<T><<<b, kThreads, 0, st>>>(g, (const T*)dO, (const T*)Og, sel_idx, (T*)dOg, D);
  }
  return cudaGetLastError();
}

template <typename T, int L>
void gather_bwd_l(const Geo& g, unsigned b, const void* dQg, const void* dKg, const void* dVg,
                  const int32_t* slot_of, void* dQ, void* dK, void* dV, cudaStream_t st) {
  gather_bwd_kernel<T, L><<<b, kThreads, 0, st>>>(g, (const T*)dQg, (const T*)dKg, (const T*)dVg,
                                                  slot_of, (T*)dQ, (T*)dK, (T*)dV);
}

template <typename T>
void gather_bwd_t(const Geo& g, unsigned b, const void* dQg, const void* dKg, const void* dVg,
                  const int32_t* slot_of, void* dQ, void* dK, void* dV, cudaStream_t st) {
  switch (g.L) {
    case 1: gather_bwd_l<T, 1>(g, b, dQg, dKg, dVg, slot_of, dQ, dK, dV, st); break;
    case 2: gather_bwd_l<T, 2>(g, b, dQg, dKg, dVg, slot_of, dQ, dK, dV, st); break;
    case 3: gather_bwd_l<T, 3>(g, b, dQg, dKg, dVg, slot_of, dQ, dK, dV, st); break;
    case 4: gather_bwd_l<T, 4>(g, b, dQg, dKg, dVg, slot_of, dQ, dK, dV, st); break;
    default: gather_bwd_l<T, 5>(g, b, dQg, dKg, dVg, slot_of, dQ, dK, dV, st); break;
  }
}

cudaError_t launch_gather_bwd(const lh_plan& plan, const void* dQg, const void* dKg,
                              const void* dVg, const int32_t* slot_of, void* dQ, void* dK,
                              void* dV, cudaStream_t st) {
  const Geo g = make_geo(plan);
  const unsigned b = blocks_for(g.BH * g.N);
  if (plan.c.dtype == LH_BF16) gather_bwd_t<__nv_bfloat16>(g, b, dQg, dKg, dVg, slot_of, dQ, dK, dV, st);
  else gather_bwd_t<float>(g, b, dQg, dKg, dVg, slot_of, dQ, dK, dV, st);
  return cudaGetLastError();
}

}  // namespace lh
