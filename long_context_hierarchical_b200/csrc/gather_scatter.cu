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
// Every kernel is a template on the head dimension D (64 or 128).  The gather
// kernel gives each row to 8 lanes: lane c moves channels [8c, 8c+8) of each
// 64-channel group with 16-byte accesses, so a warp touches 4 whole rows per
// instruction (the split of the other kernels is below).  The scatter and gather-backward kernels are
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

template <typename T, int D>
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
  const int64_t dst = row * D + c * 8;
  if (f < 0 || f >= g.Ntot) {  // not a pyramid index: write zeros, read nothing
    const float z[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int h = 0; h < D / 64; ++h) {
      Vec8<T>::store(Qg + dst + 64 * h, z);
      Vec8<T>::store(Kg + dst + 64 * h, z);
      Vec8<T>::store(Vg + dst + 64 * h, z);
    }
    return;
  }
  const int l = level_of(g, f);
  const int64_t i = f - g.flat_off[l];
  int64_t src;
  const T *sq, *sk, *sv;
  if (l == 0) {
    src = (bh * g.N + i) * D;
    sq = Q; sk = K; sv = V;
  } else {
    src = (bh * g.Npyr + g.pyr_off[l] + i) * D;
    sq = pQ; sk = pK; sv = pV;
  }
#pragma unroll
  for (int h = 0; h < D / 64; ++h) {
    copy_chunk(Qg + dst + 64 * h, sq + src + c * 8 + 64 * h);
    copy_chunk(Kg + dst + 64 * h, sk + src + c * 8 + 64 * h);
    copy_chunk(Vg + dst + 64 * h, sv + src + c * 8 + 64 * h);
  }
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

// p = 2^LOGP and L are template parameters, the head comes from blockIdx.y
// and indices inside a head are 32-bit, so the per-token index arithmetic is
// a handful of shifts and adds.  The token-centric kernels (scatter, gather
// backward) give each row to R lanes, lane c moving chunks c, c + R, ...,
// so the per-token index work is shared by fewer lanes (these kernels are
// instruction-bound with 8 lanes per row) while every store instruction
// still covers whole 32-byte sectors.
constexpr int kLanesPerRow = 4;
template <int D>
constexpr int kChunks = D / 8 / kLanesPerRow;  // 8-element chunks per lane
constexpr int kRowsPerBlock4 = kThreads / kLanesPerRow;

// Two forms of the token-centric kernels, with the same sums in the same
// order.  kAll: the row loads of every level are issued before any of them
// is used, so all L are in flight together (a level whose entry is not
// selected reads row 0 of the head instead, valid cached memory, and drops
// the value with a select); this is faster where most tokens have several
// selected levels (98K tokens, k = 1536: S/N = 0.19).  Otherwise a branch per
// level loads only the selected rows, faster for sparse selections (512K,
// k = 2048: S/N = 0.06).  The launch picks kAll for S/N >= 1/8.
template <typename T, int D, int LOGP, int L, bool kAll>
__global__ void __launch_bounds__(kThreads)
scatter_kernel(Geo g, const T* __restrict__ Og, const int32_t* __restrict__ slot_of,
               T* __restrict__ O) {
  const int t = blockIdx.x * kRowsPerBlock4 + (int)(threadIdx.x / kLanesPerRow);
  const int c = threadIdx.x % kLanesPerRow;
  if (t >= (int)g.N) return;
  const int64_t bh = blockIdx.y;
  const int32_t* inv = slot_of + bh * g.Ntot;
  const T* og = Og + bh * g.S * D + c * 8;
  const int S = (int)g.S;
  int32_t slot[L];
  bool hit[L];
#pragma unroll
  for (int l = 0; l < L; ++l) {
    const int i = ((t + 1) >> (LOGP * l)) - 1;
    const int32_t sl = i >= 0 ? __ldg(inv + (int)g.flat_off[l] + i) : -1;
    hit[l] = (unsigned)sl < (unsigned)S;
    slot[l] = hit[l] ? sl : 0;
  }
  float a[kChunks<D>][8];
#pragma unroll
  for (int k = 0; k < kChunks<D>; ++k)
#pragma unroll
    for (int e = 0; e < 8; ++e) a[k][e] = 0.f;
  if constexpr (kAll) {
    float x[L][kChunks<D>][8];
#pragma unroll
    for (int l = 0; l < L; ++l)
#pragma unroll
      for (int k = 0; k < kChunks<D>; ++k)
        Vec8<T>::load(og + (int64_t)slot[l] * D + 8 * kLanesPerRow * k, x[l][k]);
#pragma unroll
    for (int l = 0; l < L; ++l)  // ascending level
#pragma unroll
      for (int k = 0; k < kChunks<D>; ++k)
#pragma unroll
        for (int e = 0; e < 8; ++e) a[k][e] = hit[l] ? a[k][e] + x[l][k][e] : a[k][e];
  } else {
#pragma unroll
    for (int l = 0; l < L; ++l) {  // ascending level
      if (hit[l]) {
#pragma unroll
        for (int k = 0; k < kChunks<D>; ++k) {
          float x[8];
          Vec8<T>::load(og + (int64_t)slot[l] * D + 8 * kLanesPerRow * k, x);
#pragma unroll
          for (int e = 0; e < 8; ++e) a[k][e] += x[e];
        }
      }
    }
  }
  T* dst = O + (bh * g.N + t) * D + c * 8;
#pragma unroll
  for (int k = 0; k < kChunks<D>; ++k) store_stream<T>(dst + 8 * kLanesPerRow * k, a[k]);
}

constexpr int kBwdLanes = 4;  // lanes per slot row in the scatter backward (8 and 2 measured slower)
template <int D>
constexpr int kBwdChunks = D / 8 / kBwdLanes;
constexpr int kRowsPerBlockB = kThreads / kBwdLanes;

// Position, within its block, of the slot row that slot group `grp` handles
// when the block's rows are taken level by level: the rows of one level share
// one range length, so a warp's row sums mostly share one trip count.  Rows
// past S sort last.  Which group takes which row varies from run to run; each
// row's result does not.
template <int L>
__device__ __forceinline__ int slot_by_level(const Geo& g, const int32_t* __restrict__ sel_row,
                                             int first, int grp, int c) {
  __shared__ int s_level[kRowsPerBlockB];
  __shared__ int s_start[L + 1];
  __shared__ int s_order[kRowsPerBlockB];
  if (threadIdx.x <= L) s_start[threadIdx.x] = 0;
  __syncthreads();
  if (c == 0) {
    int lv = L;
    if (first + grp < (int)g.S) {
      int f = sel_row[first + grp];
      if (f < 0 || f >= (int)g.Ntot) f = (int)g.Ntot - 1;  // unreachable for a valid selection
      lv = 0;
#pragma unroll
      for (int q = 1; q < L; ++q)
        if (f >= (int)g.flat_off[q]) lv = q;
    }
    s_level[grp] = lv;
    atomicAdd(&s_start[lv], 1);
  }
  __syncthreads();
  if (threadIdx.x == 0) {  // counts -> exclusive prefix
    int run = 0;
    for (int q = 0; q <= L; ++q) {
      const int n = s_start[q];
      s_start[q] = run;
      run += n;
    }
  }
  __syncthreads();
  if (c == 0) s_order[atomicAdd(&s_start[s_level[grp]], 1)] = grp;
  __syncthreads();
  return s_order[grp];
}

template <typename T, int D, int LOGP, int L, bool kByLevel>
__global__ void __launch_bounds__(kThreads)
scatter_bwd_kernel(Geo g, const T* __restrict__ dO, const T* __restrict__ Og,
                   const int32_t* __restrict__ sel_idx, T* __restrict__ dOg, float* __restrict__ Drow) {
  const int64_t bh = blockIdx.y;
  const int first = blockIdx.x * kRowsPerBlockB;
  const int grp = (int)(threadIdx.x / kBwdLanes);
  const int c = threadIdx.x % kBwdLanes;
  int jj = grp;
  if constexpr (kByLevel) jj = slot_by_level<L>(g, sel_idx + bh * g.S, first, grp, c);
  const int j = first + jj;
  const int S = (int)g.S, N = (int)g.N;
  const bool live = j < S;
  const int64_t r = bh * g.S + (live ? j : 0);
  int f = sel_idx[r];
  if (f < 0 || f >= (int)g.Ntot) f = (int)g.Ntot - 1;  // unreachable for a valid selection
  int l = 0;
#pragma unroll
  for (int q = 1; q < L; ++q)
    if (f >= (int)g.flat_off[q]) l = q;
  const int i = f - (int)g.flat_off[l];
  const int sh = LOGP * l;
  const int lo = ((i + 1) << sh) - 1;
  const int hi = min(lo + (1 << sh) - 1, N - 1);
  const T* src = dO + bh * g.N * D + c * 8;
  float acc[kBwdChunks<D>][8];
#pragma unroll
  for (int k = 0; k < kBwdChunks<D>; ++k)
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[k][e] = 0.f;
  int t = lo;
  for (; t + 3 <= hi; t += 4) {  // four independent row loads in flight
#pragma unroll
    for (int k = 0; k < kBwdChunks<D>; ++k) {
      float x0[8], x1[8], x2[8], x3[8];
      const T* p = src + 8 * kBwdLanes * k;
      Vec8<T>::load(p + (int64_t)t * D, x0);
      Vec8<T>::load(p + (int64_t)(t + 1) * D, x1);
      Vec8<T>::load(p + (int64_t)(t + 2) * D, x2);
      Vec8<T>::load(p + (int64_t)(t + 3) * D, x3);
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[k][e] += ((x0[e] + x1[e]) + (x2[e] + x3[e]));
    }
  }
  for (; t <= hi; ++t) {
#pragma unroll
    for (int k = 0; k < kBwdChunks<D>; ++k) {
      float x[8];
      Vec8<T>::load(src + 8 * kBwdLanes * k + (int64_t)t * D, x);
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[k][e] += x[e];
    }
  }
  float dsum = 0.f;
#pragma unroll
  for (int k = 0; k < kBwdChunks<D>; ++k) {
    float o[8];
    Vec8<T>::load(Og + r * D + c * 8 + 8 * kBwdLanes * k, o);
#pragma unroll
    for (int e = 0; e < 8; ++e) dsum = fmaf(Vec8<T>::rounded(acc[k][e]), o[e], dsum);
  }
#pragma unroll
  for (int m = 1; m < kBwdLanes; m <<= 1) dsum += __shfl_xor_sync(0xffffffffu, dsum, m);
  if (!live) return;
#pragma unroll
  for (int k = 0; k < kBwdChunks<D>; ++k) Vec8<T>::store(dOg + r * D + c * 8 + 8 * kBwdLanes * k, acc[k]);
  if (c == 0) Drow[r] = dsum;
}

template <typename T, int D, int LOGP, int L, bool kAll>
__global__ void __launch_bounds__(kThreads)
gather_bwd_kernel(Geo g, const T* __restrict__ dQg, const T* __restrict__ dKg,
                  const T* __restrict__ dVg, const int32_t* __restrict__ slot_of,
                  T* __restrict__ dQ, T* __restrict__ dK, T* __restrict__ dV) {
  const int t = blockIdx.x * kRowsPerBlock4 + (int)(threadIdx.x / kLanesPerRow);
  const int c = threadIdx.x % kLanesPerRow;
  if (t >= (int)g.N) return;
  const int64_t bh = blockIdx.y;
  const int32_t* inv = slot_of + bh * g.Ntot;
  const int64_t base = bh * g.S * D + c * 8;
  const int S = (int)g.S;
  int32_t slot[L];
  bool hit[L];
#pragma unroll
  for (int l = 0; l < L; ++l) {
    const int32_t sl = __ldg(inv + (int)g.flat_off[l] + (t >> (LOGP * l)));
    hit[l] = (unsigned)sl < (unsigned)S;
    slot[l] = hit[l] ? sl : 0;
  }
  const int64_t out = (bh * g.N + t) * D + c * 8;
  const T* src[3] = {dQg, dKg, dVg};
  T* dst[3] = {dQ, dK, dV};
#pragma unroll
  for (int w = 0; w < 3; ++w) {
    float a[kChunks<D>][8];
#pragma unroll
    for (int k = 0; k < kChunks<D>; ++k)
#pragma unroll
      for (int e = 0; e < 8; ++e) a[k][e] = 0.f;
    if constexpr (kAll) {
      float x[L][kChunks<D>][8];
#pragma unroll
      for (int l = 0; l < L; ++l)
#pragma unroll
        for (int k = 0; k < kChunks<D>; ++k)
          Vec8<T>::load(src[w] + base + (int64_t)slot[l] * D + 8 * kLanesPerRow * k, x[l][k]);
#pragma unroll
      for (int l = 0; l < L; ++l) {  // ascending level; 1/p^l is a power of two: exact
        const float wgt = 1.f / (float)(1 << (LOGP * l));
#pragma unroll
        for (int k = 0; k < kChunks<D>; ++k)
#pragma unroll
          for (int e = 0; e < 8; ++e) a[k][e] = hit[l] ? fmaf(x[l][k][e], wgt, a[k][e]) : a[k][e];
      }
    } else {
#pragma unroll
      for (int l = 0; l < L; ++l) {  // ascending level; 1/p^l is a power of two: exact
        if (hit[l]) {
          const float wgt = 1.f / (float)(1 << (LOGP * l));
#pragma unroll
          for (int k = 0; k < kChunks<D>; ++k) {
            float x[8];
            Vec8<T>::load(src[w] + base + (int64_t)slot[l] * D + 8 * kLanesPerRow * k, x);
#pragma unroll
            for (int e = 0; e < 8; ++e) a[k][e] = fmaf(x[e], wgt, a[k][e]);
          }
        }
      }
    }
#pragma unroll
    for (int k = 0; k < kChunks<D>; ++k) store_stream<T>(dst[w] + out + 8 * kLanesPerRow * k, a[k]);
  }
}

unsigned blocks_for(int64_t rows) { return (unsigned)((rows + kRowsPerBlock - 1) / kRowsPerBlock); }
unsigned blocks_for4(int64_t rows) { return (unsigned)((rows + kRowsPerBlock4 - 1) / kRowsPerBlock4); }

}  // namespace

cudaError_t launch_gather(const lh_plan& plan, const void* Q, const void* K, const void* V,
                          const void* pyrQ, const void* pyrK, const void* pyrV,
                          const int32_t* sel_idx, void* Qg, void* Kg, void* Vg, cudaStream_t st) {
  const Geo g = make_geo(plan);
  const unsigned b = blocks_for(g.BH * g.S);
  with_type_dim(plan, [&]<typename T, int D>() {
    gather_kernel<T, D><<<b, kThreads, 0, st>>>(g, (const T*)Q, (const T*)K, (const T*)V,
                                                (const T*)pyrQ, (const T*)pyrK, (const T*)pyrV,
                                                sel_idx, (T*)Qg, (T*)Kg, (T*)Vg);
  });
  return cudaGetLastError();
}

// Calls f.template operator()<LOGP, L>() for the plan's p in {2, 4} and L <= 5.
template <typename F>
void with_levels(const Geo& g, F&& f) {
  if (g.logp == 1) {
    switch (g.L) {
      case 1: f.template operator()<1, 1>(); break;
      case 2: f.template operator()<1, 2>(); break;
      case 3: f.template operator()<1, 3>(); break;
      case 4: f.template operator()<1, 4>(); break;
      default: f.template operator()<1, 5>(); break;
    }
  } else {
    switch (g.L) {
      case 1: f.template operator()<2, 1>(); break;
      case 2: f.template operator()<2, 2>(); break;
      case 3: f.template operator()<2, 3>(); break;
      case 4: f.template operator()<2, 4>(); break;
      default: f.template operator()<2, 5>(); break;
    }
  }
}

// The all-levels form for selections of at least one slot per 8 tokens.
bool dense_selection(const Geo& g) { return 8 * g.S >= g.N; }

template <typename T, int D>
void scatter_t(const Geo& g, const void* Og, const int32_t* slot_of, void* O, cudaStream_t st) {
  const dim3 grid(blocks_for4(g.N), (unsigned)g.BH);
  const bool all = dense_selection(g);
  with_levels(g, [&]<int LOGP, int L>() {
    if (all)
      scatter_kernel<T, D, LOGP, L, true><<<grid, kThreads, 0, st>>>(g, (const T*)Og, slot_of, (T*)O);
    else
      scatter_kernel<T, D, LOGP, L, false><<<grid, kThreads, 0, st>>>(g, (const T*)Og, slot_of, (T*)O);
  });
}

cudaError_t launch_scatter(const lh_plan& plan, const void* Og, const int32_t* slot_of, void* O,
                           cudaStream_t st) {
  const Geo g = make_geo(plan);
  with_type_dim(plan, [&]<typename T, int D>() { scatter_t<T, D>(g, Og, slot_of, O, st); });
  return cudaGetLastError();
}

template <typename T, int D>
void scatter_bwd_t(const Geo& g, const void* dO, const void* Og, const int32_t* sel_idx, void* dOg,
                   float* Drow, cudaStream_t st) {
  const dim3 grid((unsigned)((g.S + kRowsPerBlockB - 1) / kRowsPerBlockB), (unsigned)g.BH);
  // Sparse selections mix long coarse ranges with single tokens inside one
  // block; taking the rows level by level pays there (0.273 vs 0.296 ms at
  // 512K tokens, 4 heads) and not for dense ones (0.073 vs 0.071 ms at 98K).
  const bool by_level = !dense_selection(g);
  with_levels(g, [&]<int LOGP, int L>() {
    if (by_level)
      scatter_bwd_kernel<T, D, LOGP, L, true><<<grid, kThreads, 0, st>>>(
          g, (const T*)dO, (const T*)Og, sel_idx, (T*)dOg, Drow);
    else
      scatter_bwd_kernel<T, D, LOGP, L, false><<<grid, kThreads, 0, st>>>(
          g, (const T*)dO, (const T*)Og, sel_idx, (T*)dOg, Drow);
  });
}

cudaError_t launch_scatter_bwd(const lh_plan& plan, const void* dO, const void* Og,
                               const int32_t* sel_idx, void* dOg, float* Drow, cudaStream_t st) {
  const Geo g = make_geo(plan);
  with_type_dim(plan, [&]<typename T, int D>() {
    scatter_bwd_t<T, D>(g, dO, Og, sel_idx, dOg, Drow, st);
  });
  return cudaGetLastError();
}

template <typename T, int D>
void gather_bwd_t(const Geo& g, const void* dQg, const void* dKg, const void* dVg,
                  const int32_t* slot_of, void* dQ, void* dK, void* dV, cudaStream_t st) {
  const dim3 grid(blocks_for4(g.N), (unsigned)g.BH);
  const bool all = dense_selection(g);
  with_levels(g, [&]<int LOGP, int L>() {
    if (all)
      gather_bwd_kernel<T, D, LOGP, L, true><<<grid, kThreads, 0, st>>>(
          g, (const T*)dQg, (const T*)dKg, (const T*)dVg, slot_of, (T*)dQ, (T*)dK, (T*)dV);
    else
      gather_bwd_kernel<T, D, LOGP, L, false><<<grid, kThreads, 0, st>>>(
          g, (const T*)dQg, (const T*)dKg, (const T*)dVg, slot_of, (T*)dQ, (T*)dK, (T*)dV);
  });
}

cudaError_t launch_gather_bwd(const lh_plan& plan, const void* dQg, const void* dKg,
                              const void* dVg, const int32_t* slot_of, void* dQ, void* dK,
                              void* dV, cudaStream_t st) {
  const Geo g = make_geo(plan);
  with_type_dim(plan, [&]<typename T, int D>() {
    gather_bwd_t<T, D>(g, dQg, dKg, dVg, slot_of, dQ, dK, dV, st);
  });
  return cudaGetLastError();
}

}  // namespace lh
