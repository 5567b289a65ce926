// Stages 1 and 2a: the symmetric average-pool pyramid and the l2-norm scores,
// fused into one pass over Q, K and V.
//
// Pyramid (skill card "lighthouse-attention", stage 1 "金字塔构建";
// gist.science Technical Summary 2.A): level l entry i of X in {Q, K, V} is
// the mean of tokens [i p^l, (i+1) p^l).  Scores (stage 2 "打分与选择";
// gist.science 2.B): level-0 token t scores ||Q_t||_2 + ||K_t||_2, and a
// coarse entry inherits the max of the level-0 scores in its span.
//
// Work split: one warp owns W = max(p^(L-1), 16) consecutive tokens of one
// (batch, head), so every pyramid entry it writes lies inside its rows.  Per
// step the warp covers 16 rows: lane = 8*rr + c holds column chunk c (8
// channels, one 16-byte load for bf16) of the 4-row block rr, rows
// [4 rr, 4 rr + 4), for each 64-channel group of the row in turn (one group
// for d = 64, two for d = 128; the norm sums run over all groups).  Sums over 2 or 4 rows stay in the lane, sums over 8 and
// 16 rows take one or two xor-shuffles across rr, and longer spans
// accumulate across steps in registers.  Sums are fp32 and rounded once;
// p^l is a power of two, so the mean's scaling is exact.  The norm sums run
// in fp64: for bf16 inputs every square is exact in fp64, so the fp32 score
// does not depend on the order of the sum.
#include "host.h"

namespace lh {
namespace {

template <typename T>
struct Packed;
template <>
struct Packed<__nv_bfloat16> {
  uint4 u;
  __device__ __forceinline__ void load(const __nv_bfloat16* p) { u = __ldcs(reinterpret_cast<const uint4*>(p)); }
  __device__ __forceinline__ void zero() { u = make_uint4(0, 0, 0, 0); }
  __device__ __forceinline__ void unpack(float (&x)[8]) const {
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      x[2 * i] = __uint_as_float(w[i] << 16);
      x[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
  }
};
template <>
struct Packed<float> {
  float4 a, b;
  __device__ __forceinline__ void load(const float* p) {
    a = __ldcs(reinterpret_cast<const float4*>(p));
    b = __ldcs(reinterpret_cast<const float4*>(p) + 1);
  }
  __device__ __forceinline__ void zero() { a = b = make_float4(0.f, 0.f, 0.f, 0.f); }
  __device__ __forceinline__ void unpack(float (&x)[8]) const {
    x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
    x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
  }
};

__device__ __forceinline__ void shfl_add8(float (&s)[8], int mask) {
#pragma unroll
  for (int e = 0; e < 8; ++e) s[e] += __shfl_xor_sync(0xffffffffu, s[e], mask);
}

template <typename T>
__device__ __forceinline__ void store_mean(T* dst, const float (&s)[8], float inv) {
  float m[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) m[e] = s[e] * inv;
  Vec8<T>::store(dst, m);
}

template <typename T, int D, int LOGP, int L>
__global__ void __launch_bounds__(128)
pyramid_score_kernel(Geo g, const T* __restrict__ Q, const T* __restrict__ K,
                     const T* __restrict__ V, T* __restrict__ pyrQ, T* __restrict__ pyrK,
                     T* __restrict__ pyrV, float* __restrict__ scores, int pool, int score,
                     int64_t groups_per_head) {
  constexpr int PC = 1 << (LOGP * (L - 1));  // tokens of one coarsest entry
  constexpr int W = PC > 16 ? PC : 16;       // rows owned by one warp
  constexpr int STEPS = W / 16;
  const int lane = threadIdx.x & 31;
  const int rr = lane >> 3, c = lane & 7;
  const int64_t gw = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (gw >= g.BH * groups_per_head) return;  // whole warp leaves together
  const int64_t bh = gw / groups_per_head;
  const int64_t row0 = (gw % groups_per_head) * W;
  const int64_t N = g.N;

  constexpr int G = D / 64;  // 64-channel groups per row
  const T* src[3] = {Q + bh * N * D, K + bh * N * D, V ? V + bh * N * D : nullptr};
  T* dst[3] = {pyrQ ? pyrQ + bh * g.Npyr * D : nullptr, pyrK ? pyrK + bh * g.Npyr * D : nullptr,
               pyrV ? pyrV + bh * g.Npyr * D : nullptr};
  float* sc = scores ? scores + bh * g.M : nullptr;
  const int ntens = pool ? 3 : 2;

  // Cross-step state: running sums of levels whose span exceeds 16 rows
  // (only p = 4, levels 3 and 4) and the running max of level 3's score.
  float acc3[G][3][8], acc4[G][3][8];
  float runmax3 = -INFINITY;
#pragma unroll
  for (int h = 0; h < G; ++h)
#pragma unroll
    for (int t = 0; t < 3; ++t)
#pragma unroll
      for (int e = 0; e < 8; ++e) acc3[h][t][e] = acc4[h][t][e] = 0.f;

#pragma unroll 1
  for (int s = 0; s < STEPS; ++s) {
    const int64_t blk = row0 + s * 16 + rr * 4;  // first row of this lane's block
    double ssq[8];  // [0..3]: ||Q_row||^2 partials, [4..7]: ||K_row||^2 partials
#pragma unroll
    for (int j = 0; j < 8; ++j) ssq[j] = 0.0;

#pragma unroll
    for (int h = 0; h < G; ++h) {
      const int col = c * 8 + 64 * h;  // first channel of this lane's chunk
      Packed<T> raw[3][4];
#pragma unroll
      for (int t = 0; t < 3; ++t)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          if (t < ntens && blk + j < N) raw[t][j].load(src[t] + (blk + j) * D + col);
          else raw[t][j].zero();
        }

#pragma unroll
      for (int t = 0; t < 3; ++t) {
        if (t >= ntens) break;
        float x[4][8];
#pragma unroll
        for (int j = 0; j < 4; ++j) raw[t][j].unpack(x[j]);
        if (score && t < 2) {
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            double a = 0.0;
#pragma unroll
            for (int e = 0; e < 8; ++e) a = fma((double)x[j][e], (double)x[j][e], a);
            ssq[t * 4 + j] += a;
          }
        }
        if (!pool) continue;
        // Level sums.  s2a/s2b: rows {0,1}/{2,3}; s4: the 4-row block.
        float s2a[8], s2b[8], s4[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          s2a[e] = x[0][e] + x[1][e];
          s2b[e] = x[2][e] + x[3][e];
          s4[e] = s2a[e] + s2b[e];
        }
        T* out = dst[t];
        if (LOGP == 1) {
          // p = 2: P = 2, 4, 8, 16 for levels 1..4.
          if (L >= 2) {
            const int64_t i = blk / 2;
            if (blk < N) store_mean<T>(out + (g.pyr_off[1] + i) * D + col, s2a, 0.5f);
            if (blk + 2 < N) store_mean<T>(out + (g.pyr_off[1] + i + 1) * D + col, s2b, 0.5f);
          }
          if (L >= 3 && blk < N) store_mean<T>(out + (g.pyr_off[2] + blk / 4) * D + col, s4, 0.25f);
          if (L >= 4) {
            float s8[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) s8[e] = s4[e];
            shfl_add8(s8, 8);
            if ((rr & 1) == 0 && blk < N)
              store_mean<T>(out + (g.pyr_off[3] + blk / 8) * D + col, s8, 0.125f);
            if (L >= 5) {
              shfl_add8(s8, 16);
              if (rr == 0 && blk < N)
                store_mean<T>(out + (g.pyr_off[4] + blk / 16) * D + col, s8, 0.0625f);
            }
          }
        } else {
          // p = 4: P = 4, 16, 64, 256 for levels 1..4.
          if (L >= 2 && blk < N) store_mean<T>(out + (g.pyr_off[1] + blk / 4) * D + col, s4, 0.25f);
          if (L >= 3) {
            float s16[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) s16[e] = s4[e];
            shfl_add8(s16, 8);
            shfl_add8(s16, 16);
            if (rr == 0 && blk < N)
              store_mean<T>(out + (g.pyr_off[2] + blk / 16) * D + col, s16, 1.f / 16.f);
            if (L >= 4) {
#pragma unroll
              for (int e = 0; e < 8; ++e) acc3[h][t][e] += s16[e];
              if ((s & 3) == 3) {
                if (rr == 0) {
                  const int64_t i = (row0 + s * 16) / 64;
                  store_mean<T>(out + (g.pyr_off[3] + i) * D + col, acc3[h][t], 1.f / 64.f);
                }
                if (L >= 5) {
#pragma unroll
                  for (int e = 0; e < 8; ++e) acc4[h][t][e] += acc3[h][t][e];
                }
#pragma unroll
                for (int e = 0; e < 8; ++e) acc3[h][t][e] = 0.f;
              }
              if (L >= 5 && (s & 15) == 15) {
                if (rr == 0) {
                  const int64_t i = (row0 + s * 16) / 256;
                  store_mean<T>(out + (g.pyr_off[4] + i) * D + col, acc4[h][t], 1.f / 256.f);
                }
#pragma unroll
                for (int e = 0; e < 8; ++e) acc4[h][t][e] = 0.f;
              }
            }
          }
        }
      }
    }  // 64-channel groups

    if (score) {
      // Reduce-scatter the 8 partials over the 8 column lanes: afterwards
      // lane c holds the full sum of ssq[c].
      const bool b2 = c & 4, b1 = c & 2, b0 = c & 1;
      double w4[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const double send = b2 ? ssq[i] : ssq[i + 4];
        const double keep = b2 ? ssq[i + 4] : ssq[i];
        w4[i] = keep + __shfl_xor_sync(0xffffffffu, send, 4);
      }
      double w2[2];
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        const double send = b1 ? w4[i] : w4[i + 2];
        const double keep = b1 ? w4[i + 2] : w4[i];
        w2[i] = keep + __shfl_xor_sync(0xffffffffu, send, 2);
      }
      const double send1 = b0 ? w2[0] : w2[1];
      const double keep1 = b0 ? w2[1] : w2[0];
      const double tot = keep1 + __shfl_xor_sync(0xffffffffu, send1, 1);
      const double nrm = sqrt(tot);
      const double other = __shfl_xor_sync(0xffffffffu, nrm, 4);
      // Lanes c < 4: score of row blk + c.
      const int64_t row = blk + c;
      float sv = (c < 4 && row < N) ? __double2float_rn(nrm + other) : 0.f;
      if (c < 4 && row < N) sc[row] = sv;
      // Max-pool over spans of 2, 4, 8 and 16 rows (levels <= L-2 only).
      const float m2 = fmaxf(sv, __shfl_xor_sync(0xffffffffu, sv, 1));
      const float m4 = fmaxf(m2, __shfl_xor_sync(0xffffffffu, m2, 2));
      const float m8 = fmaxf(m4, __shfl_xor_sync(0xffffffffu, m4, 8));
      const float m16 = fmaxf(m8, __shfl_xor_sync(0xffffffffu, m8, 16));
      if (LOGP == 1) {
        if (L >= 3 && (c == 0 || c == 2) && row < N) sc[g.flat_off[1] + row / 2] = m2;
        if (L >= 4 && c == 0 && blk < N) sc[g.flat_off[2] + blk / 4] = m4;
        if (L >= 5 && c == 0 && (rr & 1) == 0 && blk < N) sc[g.flat_off[3] + blk / 8] = m8;
      } else {
        if (L >= 3 && c == 0 && blk < N) sc[g.flat_off[1] + blk / 4] = m4;
        if (L >= 4 && lane == 0 && blk < N) sc[g.flat_off[2] + blk / 16] = m16;
        if (L >= 5) {
          runmax3 = fmaxf(runmax3, m16);
          if ((s & 3) == 3) {
            if (lane == 0) sc[g.flat_off[3] + (row0 + s * 16) / 64] = runmax3;
            runmax3 = -INFINITY;
          }
        }
      }
    }
  }
}

template <typename T, int D, int LOGP, int L>
cudaError_t launch_typed(const lh_plan& plan, const void* Q, const void* K, const void* V,
                         void* pyrQ, void* pyrK, void* pyrV, float* scores, bool pool,
                         bool score, cudaStream_t st) {
  const Geo g = make_geo(plan);
  constexpr int PC = 1 << (LOGP * (L - 1));
  constexpr int W = PC > 16 ? PC : 16;
  const int64_t groups = (g.N + W - 1) / W;
  const int64_t warps = g.BH * groups;
  const int64_t blocks = (warps + 3) / 4;
  pyramid_score_kernel<T, D, LOGP, L><<<(unsigned)blocks, 128, 0, st>>>(
      g, static_cast<const T*>(Q), static_cast<const T*>(K), static_cast<const T*>(V),
      static_cast<T*>(pyrQ), static_cast<T*>(pyrK), static_cast<T*>(pyrV), scores, pool ? 1 : 0,
      score ? 1 : 0, groups);
  return cudaGetLastError();
}

template <typename T, int D>
cudaError_t launch_levels(const lh_plan& plan, const void* Q, const void* K, const void* V,
                          void* pyrQ, void* pyrK, void* pyrV, float* scores, bool pool,
                          bool score, cudaStream_t st) {
  const int L = plan.c.L;
#define LH_CASE(LOGP, LL)                                                                   \
  if (L == LL) return launch_typed<T, D, LOGP, LL>(plan, Q, K, V, pyrQ, pyrK, pyrV, scores, pool, \
                                                score, st);
  if (plan.c.p == 2) {
    LH_CASE(1, 2) LH_CASE(1, 3) LH_CASE(1, 4) LH_CASE(1, 5)
  } else {
    LH_CASE(2, 2) LH_CASE(2, 3) LH_CASE(2, 4) LH_CASE(2, 5)
  }
#undef LH_CASE
  return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_pyramid_score(const lh_plan& plan, const void* Q, const void* K,
                                 const void* V, void* pyrQ, void* pyrK, void* pyrV,
                                 float* scores, bool pool, bool score, cudaStream_t st) {
  if (plan.c.L < 2) return cudaSuccess;  // no coarse level and no candidates
  cudaError_t e = cudaSuccess;
  with_type_dim(plan, [&]<typename T, int D>() {
    e = launch_levels<T, D>(plan, Q, K, pool ? V : nullptr, pyrQ, pyrK, pyrV, scores, pool, score,
                            st);
  });
  return e;
}

}  // namespace lh
