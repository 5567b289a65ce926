// Stage 3 backward on the 5th-generation tensor cores: gradients of the
// causal attention on the gathered [S, 64] bf16 sub-sequence flow into
// dQg, dKg, dVg (skill card "lighthouse-attention", "梯度流").
//
// With P = exp(s - lse) from the forward's LSE, dP = dO V^T and
// dS = P (dP - D), D = rowsum(dO O):
//   dV = P^T dO,  dK = dS^T Q / sqrt(d),  dQ = dS K / sqrt(d).
// Two schedules:
//  - fused (default): one kernel.  A CTA per 128-key tile streams query
//    chunks of 128 rows from its diagonal on.  S^T = K Q^T and dP^T = V dO^T
//    land in TMEM (lane = key), with lse and D folded in by one extra MMA
//    step (see the K=16 slices below); the element-wise warps turn them into
//    P^T (bf16, TMEM: the A operand of dV += P^T dO) and dS^T (bf16, swizzled
//    K-major smem: the A operand of dK += dS^T Q and, read MN-major, of the
//    chunk's dQ share dS K, which lands in TMEM).  dV and dK accumulate in
//    TMEM; each dQ share is staged through shared memory and reduce-added by
//    TMA into an fp32 dQ accumulator in global memory, whose summation order
//    (and so the last bits of dQ) varies from run to run.  A small kernel
//    scales and rounds the accumulator into dQ.  P and dS are formed once
//    per (key, query) pair: exactly the five products of the gradient.
//  - deterministic: two kernels, no atomics.  The dk/dv kernel above without
//    the dQ share, then a dq kernel: one CTA per 128-query tile streams key
//    chunks up to its diagonal; S = Q K^T and dP = dO V^T in TMEM (lane =
//    query), dS to smem, dQ += dS K in TMEM.  P and dS are formed twice.
// Warp roles: four element-wise groups of four warps split each step's 128
// columns (no row reductions are needed here), then one load warp (TMA for
// tiles; it also writes the per-chunk lse and D slices) and one warp that
// owns TMEM and issues the MMAs (and, fused, the dQ reduce-adds) from one
// thread.
// Overlap inside a CTA: each element-wise thread copies its S/dP columns out
// of TMEM and releases them at once, so the next step's S and dP MMAs run
// while it computes; the P^T / dS^T buffers have their own "consumed"
// barrier that the element-wise warps wait on just before overwriting them,
// and the dQ share of one step is staged while the next step's dV/dK MMAs
// run.
// Operand layouts are those of the forward kernel: K-major A/B tiles with the
// 128-byte swizzle, tiles read as the MN-major B operand (dO, Q, K) with
// 8-row groups 1024 bytes apart.  Every wait is bounded (see tc.cuh).
#include <algorithm>

#include "host.h"
#include "tc.cuh"

namespace lh {

bool make_tile_map(CUtensorMap* map, const void* ptr, int64_t rows, int box_rows);
bool make_acc_map(CUtensorMap* map, const float* ptr, int64_t rows);

namespace {

using bf16 = __nv_bfloat16;
using namespace tc;

constexpr int kRows = 128;                   // resident tile rows = MMA M
constexpr uint32_t kTileR = kRows * kD * 2;  // 16 KB
constexpr uint32_t kKBlock = kRows * 128;    // one 64-column K-block of a 128-row tile
constexpr float kLog2e = 1.4426950408889634f;

constexpr uint32_t pow2_cols(uint32_t n) {
  return n <= 32 ? 32 : n <= 64 ? 64 : n <= 128 ? 128 : n <= 256 ? 256 : 512;
}

template <int C>
struct Cfg {
  static_assert(C == 64 || C == 128, "step width");
  static constexpr int kGroups = C / 32;        // element-wise warp groups
  static constexpr int kEw = kGroups * 128;     // element-wise threads
  static constexpr int kLoadWarp = 4 * kGroups, kMmaWarp = kLoadWarp + 1;
  static constexpr int kThreads = (kMmaWarp + 1) * 32;
  static constexpr int kCtas = C == 64 ? 2 : 1;  // CTAs per SM
  static constexpr int kStages = C == 64 ? 2 : 3;
  static constexpr uint32_t kTileC = C * kD * 2;         // streamed tile bytes
  static constexpr uint32_t kWide = (C / 64) * kKBlock;  // 128 x C bf16, K-major
};

__device__ __forceinline__ bool wait_drain(uint32_t bar, uint32_t parity) {
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity))
    if (clock64() - t0 > kWaitCycles) return false;
  return true;
}

__device__ __forceinline__ void st_shared_v4(uint32_t addr, const uint32_t* w) {
  asm volatile("st.shared.v4.b32 [%0], {%1,%2,%3,%4};\n" ::"r"(addr), "r"(w[0]), "r"(w[1]),
               "r"(w[2]), "r"(w[3])
               : "memory");
}

// Writes columns [32 c0, 32 c0 + 32) of row r of a 128-row, swizzled K-major
// tile (16-byte chunk ch of a row sits in K-block ch / 8).
__device__ __forceinline__ void store_row32(uint32_t tile, int r, int c0, const uint32_t (&w)[16]) {
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const int ch = 4 * c0 + q;
    st_shared_v4(tile + (ch >> 3) * kKBlock + r * 128 + (((ch & 7) ^ (r & 7)) << 4), &w[4 * q]);
  }
}

// 32 fp32 values of a TMEM lane as bf16 (scaled) into global memory.
__device__ __forceinline__ void store_out32(bf16* dst, const float (&v)[32], float scale) {
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    uint32_t w[4];
#pragma unroll
    for (int h = 0; h < 4; ++h) w[h] = pack_bf16x2(v[8 * c + 2 * h] * scale, v[8 * c + 2 * h + 1] * scale);
    reinterpret_cast<uint4*>(dst)[c] = make_uint4(w[0], w[1], w[2], w[3]);
  }
}

// D[tmem] = A(128 x 64, K-major tile) * B(N x 64, K-major tile)^T.  Descriptors
// are built once per tile and advanced by adds: the issuing thread is serial.
__device__ __forceinline__ void gemm_sq(uint32_t d, uint32_t a, uint32_t b, uint32_t idesc) {
  const uint64_t da = sw128_desc(a, 16, 1024), db = sw128_desc(b, 16, 1024);
#pragma unroll
  for (int ks = 0; ks < 4; ++ks) mma_bf16(d, desc_add(da, ks * 32), desc_add(db, ks * 32), idesc, ks > 0);
}
// D[tmem] (+)= A(128 x C, K-major wide tile) * B(C x 64 tile read MN-major)
template <int C>
__device__ __forceinline__ void gemm_acc(uint32_t d, uint32_t a, uint32_t b, bool acc) {
  constexpr uint32_t idesc = idesc_bf16(kRows, kD, true);
  const uint64_t da = sw128_desc(a, 16, 1024), db = sw128_desc(b, Cfg<C>::kTileC, 1024);
#pragma unroll
  for (int kk = 0; kk < C / 16; ++kk)
    mma_bf16(d, desc_add(da, (kk >> 2) * kKBlock + (kk & 3) * 32), desc_add(db, kk * 2048), idesc,
             (acc || kk > 0) ? 1u : 0u);
}

// D[tmem] = dS(128 queries x 128 keys) * K(128 keys x 64): A is the dS^T tile
// (K-major for the dK product) read MN-major, its two 64-query column blocks
// kKBlock apart; B is the resident K tile read MN-major.
__device__ __forceinline__ void gemm_dq(uint32_t d, uint32_t dst_tile, uint32_t k_tile) {
  constexpr uint32_t idesc = idesc_bf16(kRows, kD, true, true);
  const uint64_t da = sw128_desc(dst_tile, kKBlock, 1024), db = sw128_desc(k_tile, kTileR, 1024);
#pragma unroll
  for (int kk = 0; kk < kRows / 16; ++kk)
    mma_bf16(d, desc_add(da, kk * 2048), desc_add(db, kk * 2048), idesc, kk > 0 ? 1u : 0u);
}

// D[tmem] (+)= A(128 x C, bf16 in TMEM at a_tmem) * B(C x 64 tile read MN-major)
template <int C>
__device__ __forceinline__ void gemm_acc_ts(uint32_t d, uint32_t a_tmem, uint32_t b, bool acc) {
  constexpr uint32_t idesc = idesc_bf16(kRows, kD, true);
  const uint64_t db = sw128_desc(b, Cfg<C>::kTileC, 1024);
#pragma unroll
  for (int kk = 0; kk < C / 16; ++kk)
    mma_bf16_ts(d, a_tmem + 8 * kk, desc_add(db, kk * 2048), idesc, (acc || kk > 0) ? 1u : 0u);
}

// Byte offset of row r, column 0 of a K=16 slice (no swizzle).
__device__ __forceinline__ uint32_t slice_off(int r) { return (r >> 3) * 256 + (r & 7) * 16; }
// Descriptor of a K=16 slice: no swizzle, K-direction core matrices 128
// bytes apart, 8-row groups 256 bytes apart.
__device__ __forceinline__ uint64_t slice_desc(uint32_t saddr) {
  return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)(128 >> 4) << 16) | ((uint64_t)(256 >> 4) << 32) |
         (1ull << 46);
}
// v split into three bf16 parts a + b + c (each the rounding of what the
// previous ones leave), stored in columns 0-2 of a slice row.
__device__ __forceinline__ void store_split3(uint8_t* row, float v) {
  const float a = __bfloat162float(__float2bfloat16_rn(v));
  const float b = __bfloat162float(__float2bfloat16_rn(v - a));
  *reinterpret_cast<uint32_t*>(row) = pack_bf16x2(a, b);
  *reinterpret_cast<__nv_bfloat16*>(row + 4) = __float2bfloat16_rn((v - a) - b);
}

// ===========================================================================
// dK, dV (and, fused, the dQ shares)
// ===========================================================================
// TMEM columns: S^T [0,C), dP^T [C,2C), dV [2C,2C+64), dK [2C+64,2C+128),
// the chunk's dQ share [2C+128, 2C+192) (fused), P^T as bf16 pairs
// [2C+192, 2C+192+C/2) (the A operand of dV += P^T dO).
// Shared memory: K, V tiles; kStages x (Q chunk, dO chunk); dS^T (K-major,
// also read MN-major by the dQ product); the dQ staging area: four boxes of
// 128 rows x 16 fp32 (64-byte swizzle), one per element-wise group, each
// reduced into the fp32 accumulator by one TMA reduce-add; and the K=16
// slices that fold the per-query terms into the MMAs (below).
//
// The per-query terms lse and D enter through one extra K=16 step of the
// S^T and dP^T products instead of per-column loads in the element-wise
// loop: a constant slice with -1 in columns 0-2 for every key row times a
// per-chunk slice holding, for each query, a three-part bf16 split of
// lse * log2(e) / (scale * log2(e)) (for S^T) or of D (for dP^T), zeros
// elsewhere.  So S^T holds s - lse / scale and dP^T holds dP - D, to about
// 2^-25 of the folded term.  The slices are K-major without swizzle:
// element (r, k) at (r / 8) * 256 + (k / 8) * 128 + (r % 8) * 16 + (k % 8) * 2.
template <int C>
struct KV {
  using F = Cfg<C>;
  static constexpr uint32_t kOffK = 0, kOffV = kTileR;
  static constexpr uint32_t kOffQ = 2 * kTileR;                        // kStages tiles
  static constexpr uint32_t kOffG = kOffQ + F::kStages * F::kTileC;    // dO, kStages tiles
  static constexpr uint32_t kOffDST = kOffG + F::kStages * F::kTileC;  // dS^T (128 x C)
  static constexpr uint32_t kOffStage = kOffDST + F::kWide;            // 4 x 8 KB dQ boxes
  static constexpr uint32_t kStageBox = kRows * 16 * 4;
  static constexpr uint32_t kSlice = kRows * 16 * 2;                   // 4 KB K=16 slice
  static constexpr uint32_t kOffNeg = kOffStage + 4 * kStageBox;       // the -1 slice
  static constexpr uint32_t kOffLx = kOffNeg + kSlice;                 // kStages lse slices
  static constexpr uint32_t kOffDx = kOffLx + F::kStages * kSlice;     // kStages D slices
  static constexpr uint32_t kOffBar = kOffDx + F::kStages * kSlice;
  static constexpr uint32_t kBarKV = 0, kBarFull = 8, kBarEmpty = kBarFull + 8 * F::kStages,
                            kBarSP = kBarEmpty + 8 * F::kStages, kBarPDS = kBarSP + 8,
                            kBarAcc = kBarPDS + 8, kBarDrain = kBarAcc + 8, kBarTF = kBarDrain + 8,
                            kBarPF = kBarTF + 8, kBarQD = kBarPF + 8, kBarBF = kBarQD + 8,
                            kSlotTmem = kBarBF + 8, kSlotAbort = kSlotTmem + 4;
  static constexpr uint32_t kSmemBytes = kOffBar + 256 + 1024;
  static constexpr uint32_t kColDQ = 2 * C + 2 * kD;
  static constexpr uint32_t kColPT = 2 * C + 3 * kD;
  static constexpr uint32_t kTmemCols = pow2_cols(kColPT + C / 2);
  static_assert(kColPT + C / 2 <= 512, "TMEM columns");
  static_assert(kOffBar + 256 <= 227 * 1024, "shared memory");
};

// This thread's 16 columns of its query row (TMEM lane) of a chunk's dQ
// share into its group's staging box (64-byte swizzle: the 16-byte chunk c
// of row r sits at chunk c ^ ((r >> 1) & 3)).
__device__ __forceinline__ void stage_dq16(uint32_t taddr, uint32_t box, int rq) {
  float v[16];
  tmem_ld16(taddr, v);
  tmem_wait_ld();
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    const uint32_t w[4] = {__float_as_uint(v[4 * c]), __float_as_uint(v[4 * c + 1]),
                           __float_as_uint(v[4 * c + 2]), __float_as_uint(v[4 * c + 3])};
    st_shared_v4(box + rq * 64 + ((c ^ ((rq >> 1) & 3)) << 4), w);
  }
}

// 18 warps: five of them share one SM sub-partition's 16K registers, so 96
// registers per thread is the most a launch can have.
template <int C, bool kFused>
__global__ void __launch_bounds__(Cfg<C>::kThreads, 1)
attn_bwd_dkdv_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                        const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmG,
                        const __grid_constant__ CUtensorMap tmDQ, const float* __restrict__ lse,
                        const float* __restrict__ Dv, bf16* __restrict__ dK, bf16* __restrict__ dV,
                        int S, float sl2, float scale, int tiles_on_y,
                        unsigned int* __restrict__ status) {
  static_assert(C == kRows, "a dQ share has one TMEM lane per query of the chunk");
  using F = Cfg<C>;
  using L = KV<C>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_addr(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw);
  const uint32_t bars = base + L::kOffBar;
  volatile int* abort = reinterpret_cast<volatile int*>(gbase + L::kOffBar + L::kSlotAbort);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // key tile; tile 0 sees the most query chunks and is launched first
  const int kt = tiles_on_y ? blockIdx.y : blockIdx.x;
  const int bh = tiles_on_y ? blockIdx.x : blockIdx.y;
  const int k0 = kt * kRows;
  const int nq = (S - k0 + C - 1) / C;  // query chunks [k0 + C t, k0 + C t + C)
  const int row0 = bh * S;

  if (threadIdx.x == 0) {
    mbar_init(bars + L::kBarKV, 1);
    for (int s = 0; s < F::kStages; ++s) {
      mbar_init(bars + L::kBarFull + 8 * s, 33);  // TMA (expect_tx) + 32 vector lanes
      mbar_init(bars + L::kBarEmpty + 8 * s, 1);
    }
    mbar_init(bars + L::kBarSP, 1);
    mbar_init(bars + L::kBarPDS, F::kEw);
    mbar_init(bars + L::kBarAcc, 1);
    mbar_init(bars + L::kBarDrain, 1);
    mbar_init(bars + L::kBarTF, F::kEw);  // S^T/dP^T copied out of TMEM
    mbar_init(bars + L::kBarPF, 1);       // P^T/dS^T (and the dQ share) consumed / complete
    mbar_init(bars + L::kBarQD, F::kEw);  // a dQ share read out of TMEM and staged
    mbar_init(bars + L::kBarBF, 1);       // the staging boxes read by the last reduce
    *abort = 0;
    fence_mbar_init();
  }
  // the K=16 slices: zero, then -1 in columns 0-2 of the constant one
  for (uint32_t i = threadIdx.x; i < (1 + 2 * F::kStages) * L::kSlice / 16; i += blockDim.x)
    *reinterpret_cast<uint4*>(gbase + L::kOffNeg + 16 * i) = make_uint4(0u, 0u, 0u, 0u);
  __syncthreads();
  if (threadIdx.x < kRows) {
    *reinterpret_cast<uint32_t*>(gbase + L::kOffNeg + slice_off(threadIdx.x)) = 0xBF80BF80u;  // -1, -1
    *reinterpret_cast<uint16_t*>(gbase + L::kOffNeg + slice_off(threadIdx.x) + 4) = 0xBF80u;  // -1
  }
  fence_proxy_async();
  if (warp == F::kMmaWarp) tmem_alloc(bars + L::kSlotTmem, L::kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(gbase + L::kOffBar + L::kSlotTmem);

  if (warp == F::kLoadWarp) {
    // ---------------- loads ----------------
    int issued = 0;
    if (lane == 0) {
      mbar_expect_tx(bars + L::kBarKV, 2 * kTileR);
      tma_load_2d(base + L::kOffK, &tmK, 0, row0 + k0, bars + L::kBarKV);
      tma_load_2d(base + L::kOffV, &tmV, 0, row0 + k0, bars + L::kBarKV);
    }
    const float inv_scale = 1.f / scale;  // lse * log2(e) / (scale * log2(e))
    for (int t = 0; t < nq; ++t) {
      const int s = t % F::kStages, u = t / F::kStages;
      bool go = true;
      if (t >= F::kStages) go = mbar_wait(bars + L::kBarEmpty + 8 * s, (u - 1) & 1, abort, status);
      if (!__all_sync(0xffffffffu, go)) break;
      const int q0 = k0 + t * C;
      if (lane == 0) {
        mbar_expect_tx(bars + L::kBarFull + 8 * s, 2 * F::kTileC);
        tma_load_2d(base + L::kOffQ + s * F::kTileC, &tmQ, 0, row0 + q0, bars + L::kBarFull + 8 * s);
        tma_load_2d(base + L::kOffG + s * F::kTileC, &tmG, 0, row0 + q0, bars + L::kBarFull + 8 * s);
      }
#pragma unroll
      for (int e = 0; e < C / 32; ++e) {
        const int q = 32 * e + lane;
        const bool in = q0 + q < S;
        const uint32_t off = slice_off(q);
        store_split3(gbase + L::kOffLx + s * L::kSlice + off, in ? lse[row0 + q0 + q] * inv_scale : 0.f);
        store_split3(gbase + L::kOffDx + s * L::kSlice + off, in ? Dv[row0 + q0 + q] : 0.f);
      }
      fence_proxy_async();  // the slices are read by the tensor core
      mbar_arrive(bars + L::kBarFull + 8 * s);
      issued = t + 1;
    }
    if (lane == 0 && *abort) {
      wait_drain(bars + L::kBarKV, 0);
      for (int t = issued - F::kStages < 0 ? 0 : issued - F::kStages; t < issued; ++t)
        wait_drain(bars + L::kBarFull + 8 * (t % F::kStages), (t / F::kStages) & 1);
    }
  } else if (warp == F::kMmaWarp) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      constexpr uint32_t idS = idesc_bf16(kRows, C, false);
      bool ok = mbar_wait(bars + L::kBarKV, 0, abort, status) &&
                mbar_wait(bars + L::kBarFull, 0, abort, status);
      // S^T - lse / scale = K Q^T - lse slice, dP^T - D = V dO^T - D slice
      auto issue_sp = [&](int s1) {
        gemm_sq(tmem, base + L::kOffK, base + L::kOffQ + s1 * F::kTileC, idS);
        mma_bf16(tmem, slice_desc(base + L::kOffNeg), slice_desc(base + L::kOffLx + s1 * L::kSlice), idS, 1u);
        gemm_sq(tmem + C, base + L::kOffV, base + L::kOffG + s1 * F::kTileC, idS);
        mma_bf16(tmem + C, slice_desc(base + L::kOffNeg), slice_desc(base + L::kOffDx + s1 * L::kSlice), idS, 1u);
        mma_commit(bars + L::kBarSP);
      };
      if (ok) {
        tc_fence_after();
        issue_sp(0);
      }
      // dQ share j: issued as step j's last MMA, staged by the element-wise
      // warps after step j+1's P/dS hand-off (QD), reduced from here into
      // rows [k0 + C j, +C) of the accumulator; its boxes are released (BF)
      // one step later.
      auto reduce_share = [&](int j) {
        for (int g = 0; g < 4; ++g)
          tma_reduce_add_2d(&tmDQ, 16 * g, row0 + k0 + j * C, base + L::kOffStage + g * L::kStageBox);
      };
      for (int t = 0; ok && t < nq; ++t) {
        const int s = t % F::kStages;
        // S^T/dP^T of step t copied out: start step t+1's while step t computes
        if (t + 1 < nq) {
          const int s1 = (t + 1) % F::kStages, u1 = (t + 1) / F::kStages;
          if (!(ok = mbar_wait2(bars + L::kBarTF, t & 1, bars + L::kBarFull + 8 * s1, u1 & 1, abort, status)))
            break;
          tc_fence_after();
          issue_sp(s1);
        } else {
          if (!(ok = mbar_wait(bars + L::kBarTF, t & 1, abort, status))) break;
          tc_fence_after();
        }
        if constexpr (kFused) {
          if (t >= 2) {  // share t-2's reduce has read the boxes
            bulk_wait_read();
            mbar_arrive(bars + L::kBarBF);
          }
        }
        if (!(ok = mbar_wait(bars + L::kBarPDS, t & 1, abort, status))) break;
        tc_fence_after();
        gemm_acc_ts<C>(tmem + 2 * C, tmem + L::kColPT, base + L::kOffG + s * F::kTileC, t > 0);  // dV += P^T dO
        gemm_acc<C>(tmem + 2 * C + kD, base + L::kOffDST, base + L::kOffQ + s * F::kTileC, t > 0); // dK += dS^T Q
        if constexpr (kFused) {
          if (t >= 1) {  // share t-1 out of TMEM and staged
            if (!(ok = mbar_wait(bars + L::kBarQD, (t - 1) & 1, abort, status))) break;
            tc_fence_after();
            reduce_share(t - 1);
          }
          gemm_dq(tmem + L::kColDQ, base + L::kOffDST, base + L::kOffK);  // share t = dS K
        }
        mma_commit(bars + L::kBarPF);
        mma_commit(bars + L::kBarEmpty + 8 * s);
      }
      if (ok) mma_commit(bars + L::kBarAcc);
      if constexpr (kFused) {
        if (ok && nq >= 2) {
          bulk_wait_read();
          mbar_arrive(bars + L::kBarBF);
        }
        if (ok && mbar_wait(bars + L::kBarQD, (nq - 1) & 1, abort, status)) reduce_share(nq - 1);
        bulk_wait_all();  // the reduces are complete before the CTA exits
      }
      mma_commit(bars + L::kBarDrain);
      wait_drain(bars + L::kBarDrain, 0);
    }
  } else {
    // ---------------- element-wise: P^T, dS^T (and the dQ shares) ----------------
    const int grp = warp >> 2, wr = warp & 3;
    const int r = wr * 32 + lane;  // TMEM lane: key row of the tile, query row of a dQ share
    const int key = k0 + r;
    const int col0 = grp * 32;     // this group's 32 query columns of the step
    const uint32_t lane_base = tmem + ((uint32_t)(wr * 32) << 16);
    const uint32_t box = base + L::kOffStage + grp * L::kStageBox;
    // share j: wait until share j-1's reduce has read the boxes, stage, arrive
    auto stage_share = [&](int j) -> bool {
      if (j >= 1 && !mbar_wait(bars + L::kBarBF, (j - 1) & 1, abort, status)) return false;
      stage_dq16(lane_base + L::kColDQ + 16 * grp, box, r);
      fence_proxy_async();
      tc_fence_before();
      mbar_arrive(bars + L::kBarQD);
      return true;
    };
    const float2 sc2 = make_float2(sl2, sl2);
    bool ok = true;
    for (int t = 0; t < nq; ++t) {
      const int s = t % F::kStages;
      ok = mbar_wait2(bars + L::kBarSP, t & 1, bars + L::kBarFull + 8 * s, (t / F::kStages) & 1, abort,
                      status);
      if (!(ok = __all_sync(0xffffffffu, ok))) break;
      tc_fence_after();
      const int q0 = k0 + t * C;
      // visible: key <= query < S
      const bool edge = (q0 < k0 + kRows) || (q0 + C > S);
      float st[32], dp[32];
      tmem_ld32(lane_base + col0, st);
      tmem_ld32(lane_base + C + col0, dp);
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive(bars + L::kBarTF);  // TMEM columns free for the next step's MMAs
      uint32_t wp[16], wd[16];
#pragma unroll
      for (int e = 0; e < 32; e += 4) {
        const float2 x0 = fmul2(make_float2(st[e], st[e + 1]), sc2);
        const float2 x1 = fmul2(make_float2(st[e + 2], st[e + 3]), sc2);
        float p[4] = {ex2_approx(x0.x), ex2_approx(x0.y), ex2_approx(x1.x), ex2_approx(x1.y)};
        if (edge) {
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int qa = q0 + col0 + e + u;
            if (qa < key || qa >= S) p[u] = 0.f;
          }
        }
        wp[e >> 1] = pack_bf16x2(p[0], p[1]);
        wp[(e >> 1) + 1] = pack_bf16x2(p[2], p[3]);
        const float2 d0 = fmul2(make_float2(p[0], p[1]), make_float2(dp[e], dp[e + 1]));
        const float2 d1 = fmul2(make_float2(p[2], p[3]), make_float2(dp[e + 2], dp[e + 3]));
        wd[e >> 1] = pack_bf16x2(d0.x, d0.y);
        wd[(e >> 1) + 1] = pack_bf16x2(d1.x, d1.y);
      }
      // the previous step's P^T / dS^T (and dQ share) must be consumed before
      // they are overwritten
      if (t > 0) ok = mbar_wait(bars + L::kBarPF, (t - 1) & 1, abort, status);
      if (!(ok = __all_sync(0xffffffffu, ok))) break;
      tc_fence_after();
      tmem_st16(lane_base + L::kColPT + 16 * grp, wp);
      store_row32(base + L::kOffDST, r, grp, wd);
      fence_proxy_async();
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(bars + L::kBarPDS);
      if constexpr (kFused) {
        // share t-1 (complete: PF above) leaves TMEM while dV/dK of step t run
        if (t >= 1) ok = stage_share(t - 1);
        if (!(ok = __all_sync(0xffffffffu, ok))) break;
      }
    }
    if (ok) ok = mbar_wait(bars + L::kBarAcc, 0, abort, status);
    if (__all_sync(0xffffffffu, ok)) {
      tc_fence_after();
      if constexpr (kFused) {
        if (nq > 0) stage_share(nq - 1);
      }
      // TMEM [2C, 2C+64) = dV, [2C+64, 2C+128) = dK: 128 columns over the groups
#pragma unroll
      for (int piece = 0; piece < 4 / F::kGroups; ++piece) {
        const int c = (grp * (4 / F::kGroups) + piece) * 32;  // 0..127
        float v[32];
        tmem_ld32(lane_base + 2 * C + c, v);
        tmem_wait_ld();
        if (key < S) {
          const bool isk = c >= kD;
          store_out32((isk ? dK : dV) + ((int64_t)row0 + key) * kD + (c & (kD - 1)), v,
                      isk ? scale : 1.f);
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == F::kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, L::kTmemCols);
  }
}

// ===========================================================================
// dQ
// ===========================================================================
template <int C>
struct QQ {
  using F = Cfg<C>;
  static constexpr uint32_t kOffQ = 0, kOffG = kTileR;
  static constexpr uint32_t kOffK = 2 * kTileR;                       // kStages tiles
  static constexpr uint32_t kOffV = kOffK + F::kStages * F::kTileC;   // kStages tiles
  static constexpr uint32_t kOffDS = kOffV + F::kStages * F::kTileC;  // dS (128 x C)
  static constexpr uint32_t kOffBar = kOffDS + F::kWide;
  static constexpr uint32_t kBarQ = 0, kBarK = 8, kBarV = kBarK + 8 * F::kStages,
                            kBarE = kBarV + 8 * F::kStages, kBarSP = kBarE + 8 * F::kStages,
                            kBarDS = kBarSP + 8, kBarAcc = kBarDS + 8, kBarDrain = kBarAcc + 8,
                            kBarTF = kBarDrain + 8, kBarDF = kBarTF + 8, kSlotTmem = kBarDF + 8,
                            kSlotAbort = kSlotTmem + 4;
  static constexpr uint32_t kSmemBytes = kOffBar + 256 + 1024;
  static constexpr uint32_t kTmemCols = pow2_cols(2 * C + kD);
};

template <int C>
__global__ void __launch_bounds__(Cfg<C>::kThreads, Cfg<C>::kCtas)
attn_bwd_dq_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                      const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmG,
                      const float* __restrict__ lse, const float* __restrict__ Dv,
                      bf16* __restrict__ dQ, int S, int ntiles, float sl2, float scale,
                      int tiles_on_y, unsigned int* __restrict__ status) {
  using F = Cfg<C>;
  using L = QQ<C>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_addr(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw);
  const uint32_t bars = base + L::kOffBar;
  volatile int* abort = reinterpret_cast<volatile int*>(gbase + L::kOffBar + L::kSlotAbort);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int qt = ntiles - 1 - (int)(tiles_on_y ? blockIdx.y : blockIdx.x);  // longest rows first
  const int bh = tiles_on_y ? blockIdx.x : blockIdx.y;
  const int q0 = qt * kRows;
  const int kend = min(q0 + kRows, S);  // keys [0, kend) reach this tile
  const int nk = (kend + C - 1) / C;
  const int row0 = bh * S;

  if (threadIdx.x == 0) {
    mbar_init(bars + L::kBarQ, 1);
    for (int s = 0; s < F::kStages; ++s) {
      mbar_init(bars + L::kBarK + 8 * s, 1);
      mbar_init(bars + L::kBarV + 8 * s, 1);
      mbar_init(bars + L::kBarE + 8 * s, 1);
    }
    mbar_init(bars + L::kBarSP, 1);
    mbar_init(bars + L::kBarDS, F::kEw);
    mbar_init(bars + L::kBarAcc, 1);
    mbar_init(bars + L::kBarDrain, 1);
    mbar_init(bars + L::kBarTF, F::kEw);  // S/dP copied out of TMEM
    mbar_init(bars + L::kBarDF, 1);       // dS tile consumed by the MMA
    *abort = 0;
    fence_mbar_init();
  }
  if (warp == F::kMmaWarp) tmem_alloc(bars + L::kSlotTmem, L::kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(gbase + L::kOffBar + L::kSlotTmem);

  if (warp == F::kLoadWarp) {
    if (lane == 0) {
      int issued = 0;
      mbar_expect_tx(bars + L::kBarQ, 2 * kTileR);
      tma_load_2d(base + L::kOffQ, &tmQ, 0, row0 + q0, bars + L::kBarQ);
      tma_load_2d(base + L::kOffG, &tmG, 0, row0 + q0, bars + L::kBarQ);
      for (int j = 0; j < nk; ++j) {
        const int s = j % F::kStages, u = j / F::kStages;
        if (j >= F::kStages && !mbar_wait(bars + L::kBarE + 8 * s, (u - 1) & 1, abort, status)) break;
        mbar_expect_tx(bars + L::kBarK + 8 * s, F::kTileC);
        tma_load_2d(base + L::kOffK + s * F::kTileC, &tmK, 0, row0 + j * C, bars + L::kBarK + 8 * s);
        mbar_expect_tx(bars + L::kBarV + 8 * s, F::kTileC);
        tma_load_2d(base + L::kOffV + s * F::kTileC, &tmV, 0, row0 + j * C, bars + L::kBarV + 8 * s);
        issued = j + 1;
      }
      if (*abort) {
        wait_drain(bars + L::kBarQ, 0);
        for (int j = issued - F::kStages < 0 ? 0 : issued - F::kStages; j < issued; ++j) {
          wait_drain(bars + L::kBarK + 8 * (j % F::kStages), (j / F::kStages) & 1);
          wait_drain(bars + L::kBarV + 8 * (j % F::kStages), (j / F::kStages) & 1);
        }
      }
    }
  } else if (warp == F::kMmaWarp) {
    if (lane == 0) {
      constexpr uint32_t idS = idesc_bf16(kRows, C, false);
      bool ok = mbar_wait(bars + L::kBarQ, 0, abort, status) && mbar_wait(bars + L::kBarK, 0, abort, status) &&
                mbar_wait(bars + L::kBarV, 0, abort, status);
      if (ok) {
        tc_fence_after();
        gemm_sq(tmem, base + L::kOffQ, base + L::kOffK, idS);      // S = Q K^T
        gemm_sq(tmem + C, base + L::kOffG, base + L::kOffV, idS);  // dP = dO V^T
        mma_commit(bars + L::kBarSP);
      }
      for (int j = 0; ok && j < nk; ++j) {
        const int s = j % F::kStages;
        if (!(ok = mbar_wait(bars + L::kBarTF, j & 1, abort, status))) break;
        tc_fence_after();
        if (j + 1 < nk) {
          const int s1 = (j + 1) % F::kStages, u1 = (j + 1) / F::kStages;
          if (!(ok = mbar_wait2(bars + L::kBarK + 8 * s1, u1 & 1, bars + L::kBarV + 8 * s1, u1 & 1, abort, status)))
            break;
          gemm_sq(tmem, base + L::kOffQ, base + L::kOffK + s1 * F::kTileC, idS);
          gemm_sq(tmem + C, base + L::kOffG, base + L::kOffV + s1 * F::kTileC, idS);
          mma_commit(bars + L::kBarSP);
        }
        if (!(ok = mbar_wait(bars + L::kBarDS, j & 1, abort, status))) break;
        tc_fence_after();
        gemm_acc<C>(tmem + 2 * C, base + L::kOffDS, base + L::kOffK + s * F::kTileC, j > 0);  // dQ += dS K
        mma_commit(bars + L::kBarDF);
        mma_commit(bars + L::kBarE + 8 * s);
      }
      if (ok) mma_commit(bars + L::kBarAcc);
      mma_commit(bars + L::kBarDrain);
      wait_drain(bars + L::kBarDrain, 0);
    }
  } else {
    const int grp = warp >> 2, wr = warp & 3;
    const int r = wr * 32 + lane;
    const int qrow = q0 + r;
    const int col0 = grp * 32;  // this group's 32 key columns of the step
    const uint32_t lane_base = tmem + ((uint32_t)(wr * 32) << 16);
    const float l2 = qrow < S ? lse[row0 + qrow] * kLog2e : 0.f;
    const float Dr = qrow < S ? Dv[row0 + qrow] : 0.f;
    const float2 sc2 = make_float2(sl2, sl2), nl2 = make_float2(-l2, -l2);
    bool ok = true;
    for (int j = 0; j < nk; ++j) {
      ok = mbar_wait(bars + L::kBarSP, j & 1, abort, status);
      if (!(ok = __all_sync(0xffffffffu, ok))) break;
      tc_fence_after();
      const int kc = j * C + col0;     // first key of this group's columns
      const bool diag = kc + 31 > q0;  // some key may follow some query of the tile
      const int lim = qrow - kc;       // visible columns: e <= lim
      float sv[32], dp[32];
      tmem_ld32(lane_base + col0, sv);
      tmem_ld32(lane_base + C + col0, dp);
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive(bars + L::kBarTF);  // TMEM columns free for the next step's MMAs
      uint32_t w[16];
#pragma unroll
      for (int e = 0; e < 32; e += 2) {
        float2 x = ffma2(make_float2(sv[e], sv[e + 1]), sc2, nl2);
        float pa = ex2_approx(x.x), pb = ex2_approx(x.y);
        if (diag) {
          if (e > lim) pa = 0.f;
          if (e + 1 > lim) pb = 0.f;
        }
        w[e >> 1] = pack_bf16x2(pa * (dp[e] - Dr), pb * (dp[e + 1] - Dr));
      }
      if (j > 0) ok = mbar_wait(bars + L::kBarDF, (j - 1) & 1, abort, status);
      if (!(ok = __all_sync(0xffffffffu, ok))) break;
      store_row32(base + L::kOffDS, r, grp, w);
      fence_proxy_async();
      tc_fence_before();
      mbar_arrive(bars + L::kBarDS);
    }
    if (ok) ok = mbar_wait(bars + L::kBarAcc, 0, abort, status);
    if (__all_sync(0xffffffffu, ok) && grp < 2) {
      tc_fence_after();
      float v[32];
      tmem_ld32(lane_base + 2 * C + grp * 32, v);
      tmem_wait_ld();
      if (qrow < S) store_out32(dQ + ((int64_t)row0 + qrow) * kD + grp * 32, v, scale);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == F::kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, L::kTmemCols);
  }
}

// dQ = scale * accumulator, rounded to bf16; 8 elements per thread.
__global__ void __launch_bounds__(256) dq_round_kernel(const float4* __restrict__ acc,
                                                       uint4* __restrict__ dQ, int64_t n8,
                                                       float scale) {
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n8;
       i += (int64_t)gridDim.x * blockDim.x) {
    const float4 a = __ldcs(acc + 2 * i), b = __ldcs(acc + 2 * i + 1);
    __stcs(dQ + i, make_uint4(pack_bf16x2(a.x * scale, a.y * scale), pack_bf16x2(a.z * scale, a.w * scale),
                              pack_bf16x2(b.x * scale, b.y * scale), pack_bf16x2(b.z * scale, b.w * scale)));
  }
}

constexpr int kStep = 128;  // streamed rows per step (64 measured slower: N=64 MMAs run at ~65% rate)

}  // namespace

// dQ = scale * acc, n elements (a multiple of 8), rounded to bf16.
cudaError_t launch_dq_round(const float* acc, void* dQ, int64_t n, float scale, cudaStream_t st) {
  const int64_t n8 = n / 8;
  const int blocks = (int)std::min<int64_t>((n8 + 255) / 256, 148 * 8);
  dq_round_kernel<<<blocks, 256, 0, st>>>(reinterpret_cast<const float4*>(acc), static_cast<uint4*>(dQ),
                                          n8, scale);
  return cudaGetLastError();
}

cudaError_t launch_attn_bwd_tc(int64_t BH, int64_t S, const void* Q, const void* K, const void* V,
                               const float* lse, const void* dO, const float* D, void* dQ,
                               void* dK, void* dV, float* dq_acc, cudaStream_t st) {
  constexpr int C = kStep;
  using F = Cfg<C>;
  // Tiles that stay resident in a CTA have 128 rows; streamed chunks have C.
  CUtensorMap qR, gR, kR, vR, qC, gC, kC, vC;
  const int64_t rows = BH * S;
  if (!make_tile_map(&qR, Q, rows, kRows) || !make_tile_map(&gR, dO, rows, kRows) ||
      !make_tile_map(&kR, K, rows, kRows) || !make_tile_map(&vR, V, rows, kRows) ||
      !make_tile_map(&qC, Q, rows, C) || !make_tile_map(&gC, dO, rows, C) ||
      !make_tile_map(&kC, K, rows, C) || !make_tile_map(&vC, V, rows, C))
    return cudaErrorInvalidValue;
  unsigned int* status = device_status_ptr();
  // The opt-in to more than 48 KB of dynamic shared memory belongs to the
  // function in the current device's context, so it is applied on every
  // launch (a host-side call): right for any device, thread or context.
  {
    cudaError_t e = cudaFuncSetAttribute(attn_bwd_dkdv_tc_kernel<C, false>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, KV<C>::kSmemBytes);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(attn_bwd_dkdv_tc_kernel<C, true>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, KV<C>::kSmemBytes);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(attn_bwd_dq_tc_kernel<C>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             QQ<C>::kSmemBytes);
    if (e != cudaSuccess) return e;
  }
  const int ntiles = (int)((S + kRows - 1) / kRows);
  const float sl2 = 0.125f * kLog2e;
  // (tiles, problems): one problem's key tiles are launched together,
  // longest first, so the operands and fp32 dQ accumulator of one or two
  // problems at a time stay in L2 (faster than interleaving the problems)
  const int ty = BH > 65535 ? 1 : 0;
  if (ty && ntiles > 65535) return cudaErrorInvalidConfiguration;
  const dim3 grid = ty ? dim3((unsigned)BH, ntiles) : dim3(ntiles, (unsigned)BH);
  if (dq_acc != nullptr) {
    const int64_t n = BH * S * kD;
    CUtensorMap accM;
    if (!make_acc_map(&accM, dq_acc, rows)) return cudaErrorInvalidValue;
    cudaError_t e = cudaMemsetAsync(dq_acc, 0, (size_t)n * sizeof(float), st);
    if (e != cudaSuccess) return e;
    attn_bwd_dkdv_tc_kernel<C, true><<<grid, F::kThreads, KV<C>::kSmemBytes, st>>>(
        qC, kR, vR, gC, accM, lse, D, static_cast<bf16*>(dK), static_cast<bf16*>(dV), (int)S, sl2,
        0.125f, ty, status);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    return launch_dq_round(dq_acc, dQ, n, 0.125f, st);
  }
  attn_bwd_dkdv_tc_kernel<C, false><<<grid, F::kThreads, KV<C>::kSmemBytes, st>>>(
      qC, kR, vR, gC, qC /* no dQ shares */, lse, D, static_cast<bf16*>(dK), static_cast<bf16*>(dV),
      (int)S, sl2, 0.125f, ty, status);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  attn_bwd_dq_tc_kernel<C><<<grid, F::kThreads, QQ<C>::kSmemBytes, st>>>(
      qR, kC, vC, gR, lse, D, static_cast<bf16*>(dQ), (int)S, ntiles, sl2, 0.125f, ty, status);
  return cudaGetLastError();
}

}  // namespace lh
