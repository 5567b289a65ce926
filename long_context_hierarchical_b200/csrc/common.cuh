// Shared device helpers of the Lighthouse kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "lh.h"

namespace lh {

constexpr int kD = 64;  // head dimension built here

// ---------------------------------------------------------------------------
// 8-element row chunks: one 16-byte load for bf16, two for fp32.
// ---------------------------------------------------------------------------

template <typename T>
struct Vec8;

template <>
struct Vec8<__nv_bfloat16> {
  static __device__ __forceinline__ void load(const __nv_bfloat16* p, float (&x)[8]) {
    uint4 u = __ldg(reinterpret_cast<const uint4*>(p));
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      x[2 * i] = __uint_as_float(w[i] << 16);
      x[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
  }
  // Streaming load for data read once.
  static __device__ __forceinline__ void load_stream(const __nv_bfloat16* p, float (&x)[8]) {
    uint4 u = __ldcs(reinterpret_cast<const uint4*>(p));
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      x[2 * i] = __uint_as_float(w[i] << 16);
      x[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
  }
  static __device__ __forceinline__ void store(__nv_bfloat16* p, const float (&x)[8]) {
    uint32_t w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      __nv_bfloat162 h = __floats2bfloat162_rn(x[2 * i], x[2 * i + 1]);
      w[i] = *reinterpret_cast<uint32_t*>(&h);
    }
    *reinterpret_cast<uint4*>(p) = make_uint4(w[0], w[1], w[2], w[3]);
  }
  // Round to the storage type and back (the value a store would keep).
  static __device__ __forceinline__ float rounded(float x) {
    return __bfloat162float(__float2bfloat16_rn(x));
  }
};

template <>
struct Vec8<float> {
  static __device__ __forceinline__ void load(const float* p, float (&x)[8]) {
    float4 a = __ldg(reinterpret_cast<const float4*>(p));
    float4 b = __ldg(reinterpret_cast<const float4*>(p) + 1);
    x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
    x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
  }
  static __device__ __forceinline__ void load_stream(const float* p, float (&x)[8]) {
    float4 a = __ldcs(reinterpret_cast<const float4*>(p));
    float4 b = __ldcs(reinterpret_cast<const float4*>(p) + 1);
    x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
    x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
  }
  static __device__ __forceinline__ void store(float* p, const float (&x)[8]) {
    reinterpret_cast<float4*>(p)[0] = make_float4(x[0], x[1], x[2], x[3]);
    reinterpret_cast<float4*>(p)[1] = make_float4(x[4], x[5], x[6], x[7]);
  }
  static __device__ __forceinline__ float rounded(float x) { return x; }
};

// Device-side view of the plan fields the kernels need (passed by value).
struct Geo {
  int64_t BH, N, S, Ntot, Npyr, M, Ksel;
  int L, p, logp;
  int k, select;  // per-level budget and lh_select rule
  int64_t n[LH_MAX_LEVELS];
  int64_t flat_off[LH_MAX_LEVELS + 1];
  int64_t pyr_off[LH_MAX_LEVELS];
};

// Level of a level-major flat index (L <= LH_MAX_LEVELS, a short scan).
__device__ __forceinline__ int level_of(const Geo& g, int64_t f) {
  int l = 0;
#pragma unroll
  for (int j = 1; j < LH_MAX_LEVELS; ++j)
    if (j < g.L && f >= g.flat_off[j]) l = j;
  return l;
}

}  // namespace lh
