// Stage 3 backward on the 5th-generation tensor cores: gradients of the
// causal attention on the gathered [S, 64] bf16 sub-sequence flow into
// dQg, dKg, dVg (skill card "lighthouse-attention", "梯度流").
//
// With P = exp(s - lse) from the forward's LSE, dP = dO V^T and
// dS = P (dP - D), D = rowsum(dO O):
//   dV = P^T dO,  dK = dS^T Q / sqrt(d),  dQ = dS K / sqrt(d).
// Two kernels, deterministic, no atomics:
//  - dk/dv: one CTA per 128-key tile walks the query tiles from its diagonal
//    on.  S^T = K Q^T and dP^T = V dO^T land in TMEM (lane = key); the
//    softmax warps turn them into P^T and dS^T (bf16, swizzled K-major smem);
//    dV += P^T dO and dK += dS^T Q accumulate in TMEM.
//  - dq: one CTA per 128-query tile walks the key tiles up to its diagonal.
//    S = Q K^T and dP = dO V^T in TMEM (lane = query), dS to smem,
//    dQ += dS K in TMEM.
// Warp roles (576 threads): warps 0-15 are four element-wise groups of four
// warps that split the 128 columns of each tile in quarters (no row
// reductions are needed here), warp 16 loads (TMA for tiles, plain loads for
// LSE/D), warp 17 owns TMEM and issues the MMAs from one thread.  TMEM columns: [0,128) S or
// S^T, [128,256) dP or dP^T, [256,320) dQ or dV, [320,384) dK.
// Overlap: each element-wise thread copies its S/dP columns out of TMEM and
// releases them at once, so the next tile's S and dP MMAs run while it
// computes; the single P/dS shared-memory tile has its own "consumed"
// barrier that the element-wise warps wait on just before overwriting it.
// Operand layouts are those of the forward kernel: K-major A/B tiles with the
// 128-byte swizzle, tiles read as the MN-major B operand (dO, Q, K) with
// 8-row groups 1024 bytes apart.  Every wait is bounded (see tc.cuh).
#include "host.h"
#include "tc.cuh"

namespace lh {

bool make_tile_map(CUtensorMap* map, const void* ptr, int64_t rows);

namespace {

using bf16 = __nv_bfloat16;
using namespace tc;

constexpr int kRows = 128;
constexpr int kStages = 3;
constexpr uint32_t kTile = kRows * kD * 2;      // 16 KB
constexpr uint32_t kKBlock = kRows * 128;       // one 64-column K-block of a 128-wide tile
constexpr uint32_t kWide = 2 * kKBlock;         // 32 KB: 128 x 128 bf16
constexpr int kGroups = 4;                      // element-wise warp groups
constexpr int kEw = kGroups * 128;              // element-wise threads
constexpr int kLoadWarp = 4 * kGroups, kMmaWarp = kLoadWarp + 1;
constexpr int kThreads = (kMmaWarp + 1) * 32;
constexpr float kLog2e = 1.4426950408889634f;

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

// Row r of a 128 x 128 bf16 tile in the swizzled K-major layout: 16-byte
// chunk ch (0..15) of the row.
__device__ __forceinline__ uint32_t wide_chunk(uint32_t tile, int r, int ch) {
  return tile + (ch >> 3) * kKBlock + r * 128 + (((ch & 7) ^ (r & 7)) << 4);
}

// Writes columns [32 c0, 32 c0 + 32) of this thread's rows as bf16.
__device__ __forceinline__ void store_row32(uint32_t tile, int r, int c0, const uint32_t (&w)[16]) {
#pragma unroll
  for (int q = 0; q < 4; ++q) st_shared_v4(wide_chunk(tile, r, 4 * c0 + q), &w[4 * q]);
}

// 64 columns of a TMEM lane as one bf16 row (scaled) into global memory.
__device__ __forceinline__ void store_out32(bf16* dst, const float (&v)[32], float scale) {
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    uint32_t w[4];
#pragma unroll
    for (int h = 0; h < 4; ++h) w[h] = pack_bf16x2(v[8 * c + 2 * h] * scale, v[8 * c + 2 * h + 1] * scale);
    reinterpret_cast<uint4*>(dst)[c] = make_uint4(w[0], w[1], w[2], w[3]);
  }
}

// ===========================================================================
// dK, dV
// ===========================================================================
namespace kv {
constexpr uint32_t kOffK = 0, kOffV = kTile;
constexpr uint32_t kOffQ = 2 * kTile;                    // kStages tiles
constexpr uint32_t kOffG = kOffQ + kStages * kTile;      // dO, kStages tiles
constexpr uint32_t kOffPT = kOffG + kStages * kTile;     // P^T  (128 x 128)
constexpr uint32_t kOffDST = kOffPT + kWide;             // dS^T (128 x 128)
constexpr uint32_t kOffVec = kOffDST + kWide;            // kStages x (128 lse2 + 128 D) fp32
constexpr uint32_t kOffBar = kOffVec + kStages * 1024;
constexpr uint32_t kBarKV = 0, kBarFull = 8, kBarEmpty = kBarFull + 8 * kStages,
                   kBarSP = kBarEmpty + 8 * kStages, kBarPDS = kBarSP + 8, kBarAcc = kBarPDS + 8,
                   kBarDrain = kBarAcc + 8, kBarTF = kBarDrain + 8, kBarPF = kBarTF + 8,
                   kSlotTmem = kBarPF + 8, kSlotAbort = kSlotTmem + 4;
constexpr uint32_t kSmemBytes = kOffBar + 256 + 1024;
}  // namespace kv

__global__ void __launch_bounds__(kThreads, 1)
attn_bwd_dkdv_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                        const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmG,
                        const float* __restrict__ lse, const float* __restrict__ Dv,
                        bf16* __restrict__ dK, bf16* __restrict__ dV, int S, int ntiles, float sl2,
                        float scale, unsigned int* __restrict__ status) {
  using namespace kv;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_addr(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw);
  const uint32_t bars = base + kOffBar;
  volatile int* abort = reinterpret_cast<volatile int*>(gbase + kOffBar + kSlotAbort);
  const float* vec = reinterpret_cast<const float*>(gbase + kOffVec);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int kt = blockIdx.x;  // key tile; tile 0 sees the most query tiles
  const int bh = blockIdx.y;
  const int k0 = kt * kRows;
  const int nq = ntiles - kt;  // query tiles kt .. ntiles-1
  const int row0 = bh * S;

  if (threadIdx.x == 0) {
    mbar_init(bars + kBarKV, 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(bars + kBarFull + 8 * s, 33);  // TMA (expect_tx) + 32 vector lanes
      mbar_init(bars + kBarEmpty + 8 * s, 1);
    }
    mbar_init(bars + kBarSP, 1);
    mbar_init(bars + kBarPDS, kEw);
    mbar_init(bars + kBarAcc, 1);
    mbar_init(bars + kBarDrain, 1);
    mbar_init(bars + kBarTF, kEw);  // S^T/dP^T copied out of TMEM
    mbar_init(bars + kBarPF, 1);    // P^T/dS^T tile consumed by the MMAs
    *abort = 0;
    fence_mbar_init();
  }
  if (warp == kMmaWarp) tmem_alloc(bars + kSlotTmem, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(gbase + kOffBar + kSlotTmem);

  if (warp == kLoadWarp) {
    // ---------------- loads ----------------
    int issued = 0;
    if (lane == 0) {
      mbar_expect_tx(bars + kBarKV, 2 * kTile);
      tma_load_2d(base + kOffK, &tmK, 0, row0 + k0, bars + kBarKV);
      tma_load_2d(base + kOffV, &tmV, 0, row0 + k0, bars + kBarKV);
    }
    for (int t = 0; t < nq; ++t) {
      const int s = t % kStages, u = t / kStages;
      bool go = true;
      if (t >= kStages) go = mbar_wait(bars + kBarEmpty + 8 * s, (u - 1) & 1, abort, status);
      if (!__all_sync(0xffffffffu, go)) break;
      const int q0 = (kt + t) * kRows;
      if (lane == 0) {
        mbar_expect_tx(bars + kBarFull + 8 * s, 2 * kTile);
        tma_load_2d(base + kOffQ + s * kTile, &tmQ, 0, row0 + q0, bars + kBarFull + 8 * s);
        tma_load_2d(base + kOffG + s * kTile, &tmG, 0, row0 + q0, bars + kBarFull + 8 * s);
      }
      float* dst = reinterpret_cast<float*>(gbase + kOffVec + s * 1024);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int q = 32 * e + lane;
        const bool in = q0 + q < S;
        dst[q] = in ? lse[row0 + q0 + q] * kLog2e : 0.f;
        dst[128 + q] = in ? Dv[row0 + q0 + q] : 0.f;
      }
      mbar_arrive(bars + kBarFull + 8 * s);
      issued = t + 1;
    }
    if (lane == 0 && *abort) {
      wait_drain(bars + kBarKV, 0);
      for (int t = issued - kStages < 0 ? 0 : issued - kStages; t < issued; ++t)
        wait_drain(bars + kBarFull + 8 * (t % kStages), (t / kStages) & 1);
    }
  } else if (warp == kMmaWarp) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      constexpr uint32_t idSq = idesc_bf16(kRows, kRows, false);
      constexpr uint32_t idAcc = idesc_bf16(kRows, kD, true);
      // D[tmem] = A(128 x 64, K-major tile) * B(128 x 64, K-major tile)^T
      auto gemm_sq = [&](uint32_t d, uint32_t a, uint32_t b) {
#pragma unroll
        for (int ks = 0; ks < 4; ++ks)
          mma_bf16(d, sw128_desc(a + ks * 32, 16, 1024), sw128_desc(b + ks * 32, 16, 1024), idSq, ks > 0);
      };
      // D[tmem] (+)= A(128 x 128, K-major wide tile) * B(128 x 64 tile, MN-major)
      auto gemm_acc = [&](uint32_t d, uint32_t a, uint32_t b, bool acc) {
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_bf16(d, sw128_desc(a + (kk >> 2) * kKBlock + (kk & 3) * 32, 16, 1024),
                   sw128_desc(b + kk * 2048, kTile, 1024), idAcc, (acc || kk > 0) ? 1u : 0u);
      };
      bool ok = mbar_wait(bars + kBarKV, 0, abort, status) && mbar_wait(bars + kBarFull, 0, abort, status);
      if (ok) {
        tc_fence_after();
        gemm_sq(tmem, base + kOffK, base + kOffQ);                // S^T = K Q^T
        gemm_sq(tmem + kRows, base + kOffV, base + kOffG);        // dP^T = V dO^T
        mma_commit(bars + kBarSP);
      }
      for (int t = 0; ok && t < nq; ++t) {
        const int s = t % kStages;
        // S^T/dP^T of tile t copied out: start tile t+1's while tile t computes
        if (!(ok = mbar_wait(bars + kBarTF, t & 1, abort, status))) break;
        tc_fence_after();
        if (t + 1 < nq) {
          const int s1 = (t + 1) % kStages, u1 = (t + 1) / kStages;
          if (!(ok = mbar_wait(bars + kBarFull + 8 * s1, u1 & 1, abort, status))) break;
          gemm_sq(tmem, base + kOffK, base + kOffQ + s1 * kTile);
          gemm_sq(tmem + kRows, base + kOffV, base + kOffG + s1 * kTile);
          mma_commit(bars + kBarSP);
        }
        if (!(ok = mbar_wait(bars + kBarPDS, t & 1, abort, status))) break;
        tc_fence_after();
        gemm_acc(tmem + 2 * kRows, base + kOffPT, base + kOffG + s * kTile, t > 0);       // dV += P^T dO
        gemm_acc(tmem + 2 * kRows + kD, base + kOffDST, base + kOffQ + s * kTile, t > 0); // dK += dS^T Q
        mma_commit(bars + kBarPF);
        mma_commit(bars + kBarEmpty + 8 * s);
      }
      if (ok) mma_commit(bars + kBarAcc);
      mma_commit(bars + kBarDrain);
      wait_drain(bars + kBarDrain, 0);
    }
  } else {
    // ---------------- element-wise: P^T, dS^T ----------------
    const int grp = warp >> 2, wr = warp & 3;
    const int r = wr * 32 + lane;  // key row of the tile = TMEM lane
    const int key = k0 + r;
    const int col0 = grp * 32;     // this group's 32 query columns
    const uint32_t lane_base = tmem + ((uint32_t)(wr * 32) << 16);
    const float2 sc2 = make_float2(sl2, sl2);
    bool ok = true;
    for (int t = 0; t < nq; ++t) {
      const int s = t % kStages;
      ok = mbar_wait(bars + kBarSP, t & 1, abort, status);
      if (ok) ok = mbar_wait(bars + kBarFull + 8 * s, (t / kStages) & 1, abort, status);
      if (!(ok = __all_sync(0xffffffffu, ok))) break;
      tc_fence_after();
      const int q0 = (kt + t) * kRows;
      // visible: key <= query < S
      const bool edge = (t == 0) || (q0 + kRows > S);
      const float* l2 = vec + s * 256 + col0;
      const float* dd = l2 + 128;
      float st[32], dp[32];
      tmem_ld32(lane_base + col0, st);
      tmem_ld32(lane_base + kRows + col0, dp);
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive(bars + kBarTF);  // TMEM columns free for the next tile's MMAs
      uint32_t wp[16], wd[16];
#pragma unroll
      for (int e = 0; e < 32; e += 4) {
        const float4 lv = *reinterpret_cast<const float4*>(l2 + e);
        const float4 dv = *reinterpret_cast<const float4*>(dd + e);
        float2 x0 = ffma2(make_float2(st[e], st[e + 1]), sc2, make_float2(-lv.x, -lv.y));
        float2 x1 = ffma2(make_float2(st[e + 2], st[e + 3]), sc2, make_float2(-lv.z, -lv.w));
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
        wd[e >> 1] = pack_bf16x2(p[0] * (dp[e] - dv.x), p[1] * (dp[e + 1] - dv.y));
        wd[(e >> 1) + 1] = pack_bf16x2(p[2] * (dp[e + 2] - dv.z), p[3] * (dp[e + 3] - dv.w));
      }
      // the previous tile's P^T / dS^T must be consumed before they are overwritten
      if (t > 0) ok = mbar_wait(bars + kBarPF, (t - 1) & 1, abort, status);
      if (!(ok = __all_sync(0xffffffffu, ok))) break;
      store_row32(base + kOffPT, r, grp, wp);
      store_row32(base + kOffDST, r, grp, wd);
      fence_proxy_async();
      tc_fence_before();
      mbar_arrive(bars + kBarPDS);
    }
    if (ok) ok = mbar_wait(bars + kBarAcc, 0, abort, status);
    if (__all_sync(0xffffffffu, ok)) {
      // groups 0,1: dV columns [32 grp, +32); groups 2,3: dK columns [32 (grp-2), +32)
      tc_fence_after();
      const bool isk = grp >= 2;
      const int c = (grp & 1) * 32;
      float v[32];
      tmem_ld32(lane_base + 2 * kRows + (isk ? kD : 0) + c, v);
      tmem_wait_ld();
      if (key < S)
        store_out32((isk ? dK : dV) + ((int64_t)row0 + key) * kD + c, v, isk ? scale : 1.f);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ===========================================================================
// dQ
// ===========================================================================
namespace qq {
constexpr uint32_t kOffQ = 0, kOffG = kTile;
constexpr uint32_t kOffK = 2 * kTile;                  // kStages tiles
constexpr uint32_t kOffV = kOffK + kStages * kTile;    // kStages tiles
constexpr uint32_t kOffDS = kOffV + kStages * kTile;   // dS (128 x 128)
constexpr uint32_t kOffBar = kOffDS + kWide;
constexpr uint32_t kBarQ = 0, kBarK = 8, kBarV = kBarK + 8 * kStages, kBarE = kBarV + 8 * kStages,
                   kBarSP = kBarE + 8 * kStages, kBarDS = kBarSP + 8, kBarAcc = kBarDS + 8,
                   kBarDrain = kBarAcc + 8, kBarTF = kBarDrain + 8, kBarDF = kBarTF + 8,
                   kSlotTmem = kBarDF + 8, kSlotAbort = kSlotTmem + 4;
constexpr uint32_t kSmemBytes = kOffBar + 256 + 1024;
}  // namespace qq

__global__ void __launch_bounds__(kThreads, 1)
attn_bwd_dq_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                      const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmG,
                      const float* __restrict__ lse, const float* __restrict__ Dv,
                      bf16* __restrict__ dQ, int S, int ntiles, float sl2, float scale,
                      unsigned int* __restrict__ status) {
  using namespace qq;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_addr(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw);
  const uint32_t bars = base + kOffBar;
  volatile int* abort = reinterpret_cast<volatile int*>(gbase + kOffBar + kSlotAbort);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int qt = ntiles - 1 - (int)blockIdx.x;  // longest rows first
  const int bh = blockIdx.y;
  const int q0 = qt * kRows;
  const int nk = qt + 1;
  const int row0 = bh * S;

  if (threadIdx.x == 0) {
    mbar_init(bars + kBarQ, 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(bars + kBarK + 8 * s, 1);
      mbar_init(bars + kBarV + 8 * s, 1);
      mbar_init(bars + kBarE + 8 * s, 1);
    }
    mbar_init(bars + kBarSP, 1);
    mbar_init(bars + kBarDS, kEw);
    mbar_init(bars + kBarAcc, 1);
    mbar_init(bars + kBarDrain, 1);
    mbar_init(bars + kBarTF, kEw);  // S/dP copied out of TMEM
    mbar_init(bars + kBarDF, 1);    // dS tile consumed by the MMA
    *abort = 0;
    fence_mbar_init();
  }
  if (warp == kMmaWarp) tmem_alloc(bars + kSlotTmem, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(gbase + kOffBar + kSlotTmem);

  if (warp == kLoadWarp) {
    if (lane == 0) {
      int issued = 0;
      mbar_expect_tx(bars + kBarQ, 2 * kTile);
      tma_load_2d(base + kOffQ, &tmQ, 0, row0 + q0, bars + kBarQ);
      tma_load_2d(base + kOffG, &tmG, 0, row0 + q0, bars + kBarQ);
      for (int j = 0; j < nk; ++j) {
        const int s = j % kStages, u = j / kStages;
        if (j >= kStages && !mbar_wait(bars + kBarE + 8 * s, (u - 1) & 1, abort, status)) break;
        mbar_expect_tx(bars + kBarK + 8 * s, kTile);
        tma_load_2d(base + kOffK + s * kTile, &tmK, 0, row0 + j * kRows, bars + kBarK + 8 * s);
        mbar_expect_tx(bars + kBarV + 8 * s, kTile);
        tma_load_2d(base + kOffV + s * kTile, &tmV, 0, row0 + j * kRows, bars + kBarV + 8 * s);
        issued = j + 1;
      }
      if (*abort) {
        wait_drain(bars + kBarQ, 0);
        for (int j = issued - kStages < 0 ? 0 : issued - kStages; j < issued; ++j) {
          wait_drain(bars + kBarK + 8 * (j % kStages), (j / kStages) & 1);
          wait_drain(bars + kBarV + 8 * (j % kStages), (j / kStages) & 1);
        }
      }
    }
  } else if (warp == kMmaWarp) {
    if (lane == 0) {
      constexpr uint32_t idSq = idesc_bf16(kRows, kRows, false);
      constexpr uint32_t idAcc = idesc_bf16(kRows, kD, true);
      auto gemm_sq = [&](uint32_t d, uint32_t a, uint32_t b) {
#pragma unroll
        for (int ks = 0; ks < 4; ++ks)
          mma_bf16(d, sw128_desc(a + ks * 32, 16, 1024), sw128_desc(b + ks * 32, 16, 1024), idSq, ks > 0);
      };
      bool ok = mbar_wait(bars + kBarQ, 0, abort, status) && mbar_wait(bars + kBarK, 0, abort, status) &&
                mbar_wait(bars + kBarV, 0, abort, status);
      if (ok) {
        tc_fence_after();
        gemm_sq(tmem, base + kOffQ, base + kOffK);           // S = Q K^T
        gemm_sq(tmem + kRows, base + kOffG, base + kOffV);   // dP = dO V^T
        mma_commit(bars + kBarSP);
      }
      for (int j = 0; ok && j < nk; ++j) {
        const int s = j % kStages;
        if (!(ok = mbar_wait(bars + kBarTF, j & 1, abort, status))) break;
        tc_fence_after();
        if (j + 1 < nk) {
          const int s1 = (j + 1) % kStages, u1 = (j + 1) / kStages;
          if (!(ok = mbar_wait(bars + kBarK + 8 * s1, u1 & 1, abort, status))) break;
          if (!(ok = mbar_wait(bars + kBarV + 8 * s1, u1 & 1, abort, status))) break;
          gemm_sq(tmem, base + kOffQ, base + kOffK + s1 * kTile);
          gemm_sq(tmem + kRows, base + kOffG, base + kOffV + s1 * kTile);
          mma_commit(bars + kBarSP);
        }
        if (!(ok = mbar_wait(bars + kBarDS, j & 1, abort, status))) break;
        tc_fence_after();
        const uint32_t kk_tile = base + kOffK + s * kTile;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)  // dQ += dS K
          mma_bf16(tmem + 2 * kRows, sw128_desc(base + kOffDS + (kk >> 2) * kKBlock + (kk & 3) * 32, 16, 1024),
                   sw128_desc(kk_tile + kk * 2048, kTile, 1024), idAcc, (j > 0 || kk > 0) ? 1u : 0u);
        mma_commit(bars + kBarDF);
        mma_commit(bars + kBarE + 8 * s);
      }
      if (ok) mma_commit(bars + kBarAcc);
      mma_commit(bars + kBarDrain);
      wait_drain(bars + kBarDrain, 0);
    }
  } else {
    const int grp = warp >> 2, wr = warp & 3;
    const int r = wr * 32 + lane;
    const int qrow = q0 + r;
    const int col0 = grp * 32;  // this group's 32 key columns
    const uint32_t lane_base = tmem + ((uint32_t)(wr * 32) << 16);
    const float l2 = qrow < S ? lse[row0 + qrow] * kLog2e : 0.f;
    const float Dr = qrow < S ? Dv[row0 + qrow] : 0.f;
    const float2 sc2 = make_float2(sl2, sl2), nl2 = make_float2(-l2, -l2);
    bool ok = true;
    for (int j = 0; j < nk; ++j) {
      ok = mbar_wait(bars + kBarSP, j & 1, abort, status);
      if (!(ok = __all_sync(0xffffffffu, ok))) break;
      tc_fence_after();
      const bool diag = j == nk - 1;
      const int lim = qrow - j * kRows - col0;  // visible columns of this group: c <= lim
      float sv[32], dp[32];
      tmem_ld32(lane_base + col0, sv);
      tmem_ld32(lane_base + kRows + col0, dp);
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive(bars + kBarTF);  // TMEM columns free for the next tile's MMAs
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
      if (j > 0) ok = mbar_wait(bars + kBarDF, (j - 1) & 1, abort, status);
      if (!(ok = __all_sync(0xffffffffu, ok))) break;
      store_row32(base + kOffDS, r, grp, w);
      fence_proxy_async();
      tc_fence_before();
      mbar_arrive(bars + kBarDS);
    }
    if (ok) ok = mbar_wait(bars + kBarAcc, 0, abort, status);
    if (__all_sync(0xffffffffu, ok) && grp < 2) {
      tc_fence_after();
      float v[32];
      tmem_ld32(lane_base + 2 * kRows + grp * 32, v);
      tmem_wait_ld();
      if (qrow < S) store_out32(dQ + ((int64_t)row0 + qrow) * kD + grp * 32, v, scale);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace

cudaError_t launch_attn_bwd_tc(int64_t BH, int64_t S, const void* Q, const void* K, const void* V,
                               const float* lse, const void* dO, const float* D, void* dQ,
                               void* dK, void* dV, cudaStream_t st) {
  CUtensorMap mq, mk, mv, mg;
  if (!make_tile_map(&mq, Q, BH * S) || !make_tile_map(&mk, K, BH * S) ||
      !make_tile_map(&mv, V, BH * S) || !make_tile_map(&mg, dO, BH * S))
    return cudaErrorInvalidValue;
  unsigned int* status = device_status_ptr();
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(attn_bwd_dkdv_tc_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, kv::kSmemBytes);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(attn_bwd_dq_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             qq::kSmemBytes);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  const int ntiles = (int)((S + kRows - 1) / kRows);
  const float sl2 = 0.125f * kLog2e;
  const dim3 grid(ntiles, (unsigned)BH);
  attn_bwd_dkdv_tc_kernel<<<grid, kThreads, kv::kSmemBytes, st>>>(
      mq, mk, mv, mg, lse, D, static_cast<bf16*>(dK), static_cast<bf16*>(dV), (int)S, ntiles, sl2,
      0.125f, status);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  attn_bwd_dq_tc_kernel<<<grid, kThreads, qq::kSmemBytes, st>>>(
      mq, mk, mv, mg, lse, D, static_cast<bf16*>(dQ), (int)S, ntiles, sl2, 0.125f, status);
  return cudaGetLastError();
}

}  // namespace lh
