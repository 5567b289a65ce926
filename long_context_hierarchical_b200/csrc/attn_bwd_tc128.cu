// Stage 3 backward for head dimension 128 on the 5th-generation tensor
// cores: gradients of the causal attention on the gathered [S, 128] bf16
// sub-sequence flow into dQg, dKg, dVg (skill card "lighthouse-attention",
// "梯度流").  With P = exp(s - lse), dP = dO V^T, dS = P (dP - D),
// D = rowsum(dO O):  dV = P^T dO,  dK = dS^T Q / sqrt(d),  dQ = dS K / sqrt(d).
//
// dk/dv kernel: a CTA per 128-key tile streams 64-query chunks from its
// diagonal on.  TMEM: S^T [0,64) and dP^T [64,128) (lane = key), dV
// [128,256), dK [256,384), and P^T as bf16 pairs [448,480), the TMEM A
// operand of dV += P^T dO.  dS^T goes to swizzled K-major shared memory,
// the A operand of dK += dS^T Q.  With d = 128 the two accumulators take 256
// columns, so a step streams 64 queries: S^T and dP^T are N = 64 products,
// dV and dK N = 128 ones.  Two schedules:
//  - fused (default): the same kernel also forms each chunk's dQ share, and
//    forms it transposed, dQ^T = K^T dS^T (M = 128 channels, N = 64 queries:
//    TMEM [384,448), lane = channel), with both operands read MN-major from
//    the resident K tile and the dS^T tile.  The element-wise threads stage
//    it into four 64-query x 32-channel fp32 boxes and the MMA thread
//    reduce-adds them with TMA into an fp32 dQ accumulator (run-to-run
//    order, so the last bits of dQ vary); a rounding kernel scales it into
//    dQ.  P and dS are formed once;
//  - deterministic: no dQ share; a dq kernel, one CTA per 128-query tile
//    streaming 64-key chunks up to its diagonal: S = Q K^T and dP = dO V^T
//    (lane = query) in TMEM [0,64) and [64,128), dS to shared memory,
//    dQ += dS K in TMEM [128,256).
// The element-wise threads copy their S/dP columns out of TMEM and release
// them at once, so the next step's S and dP products run while they compute
// P and dS.  lse (times log2 e) and D of the streamed queries are staged in
// shared memory by the load warp with each chunk.
// Tiles are 128-byte-swizzled K-major in two 64-column halves (a 256-byte
// row is two TMA boxes); a tile read as the MN-major B operand has its two
// 64-column halves as the two MN atoms (LBO = the distance between them) and
// 8-row groups 1024 bytes apart.  Every wait is bounded (see tc.cuh).
#include <algorithm>

#include "host.h"
#include "tc.cuh"

namespace lh {

bool make_tile_map_d(CUtensorMap* map, const void* ptr, int64_t rows, int box_rows, int d);
bool make_acc_map_d(CUtensorMap* map, const float* ptr, int64_t rows, int d, int box_rows);
cudaError_t launch_dq_round(const float* acc, void* dQ, int64_t n, float scale, cudaStream_t st);

namespace {

using bf16 = __nv_bfloat16;
using namespace tc;

constexpr int kD128 = 128;
constexpr int kRows = 128;                    // resident tile rows = MMA M
constexpr int kC = 64;                        // streamed rows per step
constexpr uint32_t kHalfR = kRows * 128;      // 16 KB: 128 rows x 64 columns
constexpr uint32_t kTileR = 2 * kHalfR;       // 32 KB: a resident tile
constexpr uint32_t kHalfC = kC * 128;         // 8 KB: 64 rows x 64 columns
constexpr uint32_t kTileC = 2 * kHalfC;       // 16 KB: a streamed chunk
constexpr uint32_t kWide = kRows * kC * 2;    // 16 KB: 128 x 64 bf16 (dS^T or dS)
constexpr int kStages = 3;
constexpr int kEw = 256;                      // element-wise threads: 2 groups of 4 warps
constexpr int kLoadWarp = 8, kMmaWarp = 9;
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

// Columns [32 g, 32 g + 32) of row r of a 128-row x 64-column swizzled
// K-major bf16 tile.
__device__ __forceinline__ void store_row32(uint32_t tile, int r, int g, const uint32_t (&w)[16]) {
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const int ch = 4 * g + q;  // 16-byte chunk of the 128-byte row
    st_shared_v4(tile + r * 128 + ((ch ^ (r & 7)) << 4), &w[4 * q]);
  }
}

__device__ __forceinline__ void store_out32(bf16* dst, const float (&v)[32], float scale) {
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    uint32_t w[4];
#pragma unroll
    for (int h = 0; h < 4; ++h) w[h] = pack_bf16x2(v[8 * c + 2 * h] * scale, v[8 * c + 2 * h + 1] * scale);
    reinterpret_cast<uint4*>(dst)[c] = make_uint4(w[0], w[1], w[2], w[3]);
  }
}

// D[tmem] = A(128 x 128) B(64 x 128)^T over d: A a resident tile (halves
// kHalfR apart), B a streamed chunk (halves kHalfC apart), both K-major.
__device__ __forceinline__ void gemm_rc(uint32_t d, uint32_t a, uint32_t b) {
  constexpr uint32_t idesc = idesc_bf16(kRows, kC, false);
  const uint64_t da = sw128_desc(a, 16, 1024), db = sw128_desc(b, 16, 1024);
#pragma unroll
  for (int ks = 0; ks < 8; ++ks)
    mma_bf16(d, desc_add(da, (ks >> 2) * kHalfR + (ks & 3) * 32),
             desc_add(db, (ks >> 2) * kHalfC + (ks & 3) * 32), idesc, ks > 0);
}

// D[tmem] (+)= A(128 x 64, K-major smem) * B(64 x 128): B a streamed chunk
// read MN-major (its halves are the two 64-column MN atoms).
__device__ __forceinline__ void gemm_acc(uint32_t d, uint32_t a, uint32_t b, bool acc) {
  constexpr uint32_t idesc = idesc_bf16(kRows, kD128, true);
  const uint64_t da = sw128_desc(a, 16, 1024), db = sw128_desc(b, kHalfC, 1024);
#pragma unroll
  for (int kk = 0; kk < kC / 16; ++kk)
    mma_bf16(d, desc_add(da, kk * 32), desc_add(db, kk * 2048), idesc, (acc || kk > 0) ? 1u : 0u);
}

// The same with A (128 x 64 bf16) in TMEM.
__device__ __forceinline__ void gemm_acc_ts(uint32_t d, uint32_t a_tmem, uint32_t b, bool acc) {
  constexpr uint32_t idesc = idesc_bf16(kRows, kD128, true);
  const uint64_t db = sw128_desc(b, kHalfC, 1024);
#pragma unroll
  for (int kk = 0; kk < kC / 16; ++kk)
    mma_bf16_ts(d, a_tmem + 8 * kk, desc_add(db, kk * 2048), idesc, (acc || kk > 0) ? 1u : 0u);
}

// D[tmem] = K^T (128 channels x 128 keys) * dS^T (128 keys x 64 queries): the
// transposed dQ share.  A is the resident K tile read MN-major (its two
// 64-channel halves are the two M atoms, kHalfR apart); B is the dS^T tile
// read MN-major (one 64-query atom).  K = keys: 16 key rows = 2048 bytes.
__device__ __forceinline__ void gemm_dqt(uint32_t d, uint32_t k_tile, uint32_t dst_tile) {
  constexpr uint32_t idesc = idesc_bf16(kRows, kC, true, true);
  const uint64_t da = sw128_desc(k_tile, kHalfR, 1024), db = sw128_desc(dst_tile, kWide, 1024);
#pragma unroll
  for (int kk = 0; kk < kRows / 16; ++kk)
    mma_bf16(d, desc_add(da, kk * 2048), desc_add(db, kk * 2048), idesc, kk > 0 ? 1u : 0u);
}

// Both 64-column halves of a box_rows-row tile, completing on one barrier.
__device__ __forceinline__ void load_tile(uint32_t dst, uint32_t half, const CUtensorMap* map, int row,
                                          uint32_t bar) {
  tma_load_2d(dst, map, 0, row, bar);
  tma_load_2d(dst + half, map, 64, row, bar);
}

// ===========================================================================
// dK, dV
// ===========================================================================
struct KV {
  static constexpr uint32_t kOffK = 0, kOffV = kTileR;
  static constexpr uint32_t kOffQ = 2 * kTileR;                   // kStages chunks
  static constexpr uint32_t kOffG = kOffQ + kStages * kTileC;     // dO, kStages chunks
  static constexpr uint32_t kOffDST = kOffG + kStages * kTileC;   // dS^T (128 keys x 64 queries)
  static constexpr uint32_t kStageBox = kC * 32 * 4;              // 8 KB: 64 queries x 32 channels fp32
  static constexpr uint32_t kOffStage = kOffDST + kWide;          // 4 dQ share boxes (fused)
  static constexpr uint32_t kOffL = kOffStage + 4 * kStageBox;    // kStages x 64 lse * log2 e
  static constexpr uint32_t kOffDv = kOffL + kStages * kC * 4;    // kStages x 64 D
  static constexpr uint32_t kOffBar = kOffDv + kStages * kC * 4;
  static constexpr uint32_t kBarKV = 0, kBarFull = 8, kBarEmpty = kBarFull + 8 * kStages,
                            kBarSP = kBarEmpty + 8 * kStages, kBarPDS = kBarSP + 8,
                            kBarAcc = kBarPDS + 8, kBarDrain = kBarAcc + 8, kBarTF = kBarDrain + 8,
                            kBarPF = kBarTF + 8, kBarQD = kBarPF + 8, kBarBF = kBarQD + 8,
                            kSlotTmem = kBarBF + 8, kSlotAbort = kSlotTmem + 4;
  static constexpr uint32_t kSmemBytes = kOffBar + 256 + 1024;
  static constexpr uint32_t kColDV = 2 * kC, kColDK = kColDV + kD128, kColDQT = kColDK + kD128,
                            kColPT = kColDQT + kC;
  static_assert(kColPT + kC / 2 <= 512, "TMEM columns");
  static_assert(kSlotAbort + 4 <= 256, "barrier area");
  static_assert(kSmemBytes <= 227 * 1024, "shared memory");
};

// This thread's channel (TMEM lane) of 32 queries of a dQ^T share into
// the staging box of its 32-channel block: query q is row q of the box
// (128 bytes, 128-byte swizzle: 16-byte chunk j of row q at j ^ (q % 8)).
__device__ __forceinline__ void stage_dqt32(uint32_t taddr, uint32_t box, int q0, int ch) {
  float v[32];
  tmem_ld32(taddr, v);
  tmem_wait_ld();
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    const int q = q0 + i;
    const uint32_t addr = box + q * 128 + ((((ch >> 2) ^ (q & 7))) << 4) + (ch & 3) * 4;
    asm volatile("st.shared.f32 [%0], %1;\n" ::"r"(addr), "f"(v[i]) : "memory");
  }
}

template <bool kFused>
__global__ void __maxnreg__(168)
attn_bwd_dkdv_tc128_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                           const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmG,
                           const __grid_constant__ CUtensorMap tmDQ,
                           const float* __restrict__ lse, const float* __restrict__ Dv,
                           bf16* __restrict__ dK, bf16* __restrict__ dV, int S, float sl2, float scale,
                           int tiles_on_y, unsigned int* __restrict__ status) {
  using L = KV;
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
  const int nq = (S - k0 + kC - 1) / kC;  // query chunks [k0 + kC t, k0 + kC t + kC)
  const int row0 = bh * S;

  if (threadIdx.x == 0) {
    mbar_init(bars + L::kBarKV, 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(bars + L::kBarFull + 8 * s, 33);  // TMA (expect_tx) + 32 lanes writing lse / D
      mbar_init(bars + L::kBarEmpty + 8 * s, 1);
    }
    mbar_init(bars + L::kBarSP, 1);
    mbar_init(bars + L::kBarPDS, kEw);
    mbar_init(bars + L::kBarAcc, 1);
    mbar_init(bars + L::kBarDrain, 1);
    mbar_init(bars + L::kBarTF, kEw);  // S^T/dP^T copied out of TMEM
    mbar_init(bars + L::kBarPF, 1);    // P^T/dS^T consumed (and the dQ share complete)
    mbar_init(bars + L::kBarQD, kEw);  // a dQ share read out of TMEM and staged
    mbar_init(bars + L::kBarBF, 1);    // the staging boxes read by the last reduce
    *abort = 0;
    fence_mbar_init();
  }
  if (warp == kMmaWarp) tmem_alloc(bars + L::kSlotTmem, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(gbase + L::kOffBar + L::kSlotTmem);

  if (warp == kLoadWarp) {
    // ---------------- loads ----------------
    int issued = 0;
    if (lane == 0) {
      mbar_expect_tx(bars + L::kBarKV, 2 * kTileR);
      load_tile(base + L::kOffK, kHalfR, &tmK, row0 + k0, bars + L::kBarKV);
      load_tile(base + L::kOffV, kHalfR, &tmV, row0 + k0, bars + L::kBarKV);
    }
    for (int t = 0; t < nq; ++t) {
      const int s = t % kStages, u = t / kStages;
      bool go = true;
      if (t >= kStages) go = mbar_wait(bars + L::kBarEmpty + 8 * s, (u - 1) & 1, abort, status);
      if (!__all_sync(0xffffffffu, go)) break;
      const int q0 = k0 + t * kC;
      if (lane == 0) {
        mbar_expect_tx(bars + L::kBarFull + 8 * s, 2 * kTileC);
        load_tile(base + L::kOffQ + s * kTileC, kHalfC, &tmQ, row0 + q0, bars + L::kBarFull + 8 * s);
        load_tile(base + L::kOffG + s * kTileC, kHalfC, &tmG, row0 + q0, bars + L::kBarFull + 8 * s);
      }
      float* lx = reinterpret_cast<float*>(gbase + L::kOffL + s * kC * 4);
      float* dx = reinterpret_cast<float*>(gbase + L::kOffDv + s * kC * 4);
#pragma unroll
      for (int e = 0; e < kC / 32; ++e) {
        const int q = 32 * e + lane;
        const bool in = q0 + q < S;
        lx[q] = in ? lse[row0 + q0 + q] * kLog2e : 0.f;
        dx[q] = in ? Dv[row0 + q0 + q] : 0.f;
      }
      mbar_arrive(bars + L::kBarFull + 8 * s);
      issued = t + 1;
    }
    if (lane == 0 && *abort) {
      wait_drain(bars + L::kBarKV, 0);
      for (int t = issued - kStages < 0 ? 0 : issued - kStages; t < issued; ++t)
        wait_drain(bars + L::kBarFull + 8 * (t % kStages), (t / kStages) & 1);
    }
  } else if (warp == kMmaWarp) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      bool ok = mbar_wait(bars + L::kBarKV, 0, abort, status) &&
                mbar_wait(bars + L::kBarFull, 0, abort, status);
      auto issue_sp = [&](int s1) {
        gemm_rc(tmem, base + L::kOffK, base + L::kOffQ + s1 * kTileC);       // S^T = K Q^T
        gemm_rc(tmem + kC, base + L::kOffV, base + L::kOffG + s1 * kTileC);  // dP^T = V dO^T
        mma_commit(bars + L::kBarSP);
      };
      if (ok) {
        tc_fence_after();
        issue_sp(0);
      }
      // dQ share j: issued as step j's last MMA, staged by the element-wise
      // warps after step j+1's P/dS hand-off (QD), reduced from here into
      // rows [k0 + kC j, +kC) of the accumulator; its boxes are released
      // (BF) one step later.
      auto reduce_share = [&](int j) {
        for (int b = 0; b < 4; ++b)
          tma_reduce_add_2d(&tmDQ, 32 * b, row0 + k0 + j * kC, base + L::kOffStage + b * L::kStageBox);
      };
      for (int t = 0; ok && t < nq; ++t) {
        const int s = t % kStages;
        // S^T/dP^T of step t copied out: start step t+1's while step t computes
        if (t + 1 < nq) {
          const int s1 = (t + 1) % kStages, u1 = (t + 1) / kStages;
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
        gemm_acc_ts(tmem + L::kColDV, tmem + L::kColPT, base + L::kOffG + s * kTileC, t > 0);  // dV += P^T dO
        gemm_acc(tmem + L::kColDK, base + L::kOffDST, base + L::kOffQ + s * kTileC, t > 0);    // dK += dS^T Q
        if constexpr (kFused) {
          if (t >= 1) {  // share t-1 out of TMEM and staged
            if (!(ok = mbar_wait(bars + L::kBarQD, (t - 1) & 1, abort, status))) break;
            tc_fence_after();
            reduce_share(t - 1);
          }
          gemm_dqt(tmem + L::kColDQT, base + L::kOffK, base + L::kOffDST);  // share t = K^T dS^T
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
    // ---------------- element-wise: P^T and dS^T ----------------
    const int grp = warp >> 2, wr = warp & 3;
    const int r = wr * 32 + lane;  // TMEM lane: key row of the tile
    const int key = k0 + r;
    const int col0 = grp * 32;     // this group's 32 query columns of the step
    const uint32_t lane_base = tmem + ((uint32_t)(wr * 32) << 16);
    // share j: wait until share j-1's reduce has read the boxes, stage this
    // thread's channel (lane r) for the group's 32 queries, arrive
    auto stage_share = [&](int j) -> bool {
      if (j >= 1 && !mbar_wait(bars + L::kBarBF, (j - 1) & 1, abort, status)) return false;
      stage_dqt32(lane_base + L::kColDQT + col0, base + L::kOffStage + wr * L::kStageBox, col0, lane);
      fence_proxy_async();
      tc_fence_before();
      mbar_arrive(bars + L::kBarQD);
      return true;
    };
    const float2 sc2 = make_float2(sl2, sl2);
    bool ok = true;
    for (int t = 0; t < nq; ++t) {
      const int s = t % kStages;
      ok = mbar_wait2(bars + L::kBarSP, t & 1, bars + L::kBarFull + 8 * s, (t / kStages) & 1, abort, status);
      if (!(ok = __all_sync(0xffffffffu, ok))) break;
      tc_fence_after();
      const int q0 = k0 + t * kC;
      const bool edge = (q0 < k0 + kRows) || (q0 + kC > S);  // visible: key <= query < S
      float st[32], dp[32];
      tmem_ld32(lane_base + col0, st);
      tmem_ld32(lane_base + kC + col0, dp);
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive(bars + L::kBarTF);  // TMEM columns free for the next step's products
      const float* lx = reinterpret_cast<const float*>(gbase + L::kOffL + s * kC * 4) + col0;
      const float* dx = reinterpret_cast<const float*>(gbase + L::kOffDv + s * kC * 4) + col0;
      uint32_t wp[16], wd[16];
#pragma unroll
      for (int e = 0; e < 32; e += 4) {
        const float4 l4 = *reinterpret_cast<const float4*>(lx + e);
        const float4 d4 = *reinterpret_cast<const float4*>(dx + e);
        const float2 x0 = ffma2(make_float2(st[e], st[e + 1]), sc2, make_float2(-l4.x, -l4.y));
        const float2 x1 = ffma2(make_float2(st[e + 2], st[e + 3]), sc2, make_float2(-l4.z, -l4.w));
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
        wd[e >> 1] = pack_bf16x2(p[0] * (dp[e] - d4.x), p[1] * (dp[e + 1] - d4.y));
        wd[(e >> 1) + 1] = pack_bf16x2(p[2] * (dp[e + 2] - d4.z), p[3] * (dp[e + 3] - d4.w));
      }
      // the previous step's P^T / dS^T must be consumed before they are overwritten
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
      // group 0 writes dV, group 1 dK: 128 columns each, 32 at a time
#pragma unroll
      for (int piece = 0; piece < 4; ++piece) {
        float v[32];
        tmem_ld32(lane_base + (grp ? L::kColDK : L::kColDV) + 32 * piece, v);
        tmem_wait_ld();
        if (key < S)
          store_out32((grp ? dK : dV) + ((int64_t)row0 + key) * kD128 + 32 * piece, v, grp ? scale : 1.f);
      }
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
struct QQ {
  static constexpr uint32_t kOffQ = 0, kOffG = kTileR;
  static constexpr uint32_t kOffK = 2 * kTileR;                   // kStages chunks
  static constexpr uint32_t kOffV = kOffK + kStages * kTileC;     // kStages chunks
  static constexpr uint32_t kOffDS = kOffV + kStages * kTileC;    // dS (128 queries x 64 keys)
  static constexpr uint32_t kOffBar = kOffDS + kWide;
  static constexpr uint32_t kBarQ = 0, kBarK = 8, kBarV = kBarK + 8 * kStages,
                            kBarE = kBarV + 8 * kStages, kBarSP = kBarE + 8 * kStages,
                            kBarDS = kBarSP + 8, kBarAcc = kBarDS + 8, kBarDrain = kBarAcc + 8,
                            kBarTF = kBarDrain + 8, kBarDF = kBarTF + 8, kSlotTmem = kBarDF + 8,
                            kSlotAbort = kSlotTmem + 4;
  static constexpr uint32_t kSmemBytes = kOffBar + 256 + 1024;
  static constexpr uint32_t kColDQ = 2 * kC;
  static_assert(kSlotAbort + 4 <= 256, "barrier area");
  static_assert(kSmemBytes <= 227 * 1024, "shared memory");
};

__global__ void __maxnreg__(168)
attn_bwd_dq_tc128_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                         const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmG,
                         const float* __restrict__ lse, const float* __restrict__ Dv,
                         bf16* __restrict__ dQ, int S, int ntiles, float sl2, float scale,
                         int tiles_on_y, unsigned int* __restrict__ status) {
  using L = QQ;
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
  const int nk = (kend + kC - 1) / kC;
  const int row0 = bh * S;

  if (threadIdx.x == 0) {
    mbar_init(bars + L::kBarQ, 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(bars + L::kBarK + 8 * s, 1);
      mbar_init(bars + L::kBarV + 8 * s, 1);
      mbar_init(bars + L::kBarE + 8 * s, 1);
    }
    mbar_init(bars + L::kBarSP, 1);
    mbar_init(bars + L::kBarDS, kEw);
    mbar_init(bars + L::kBarAcc, 1);
    mbar_init(bars + L::kBarDrain, 1);
    mbar_init(bars + L::kBarTF, kEw);  // S/dP copied out of TMEM
    mbar_init(bars + L::kBarDF, 1);    // dS tile consumed by the MMA
    *abort = 0;
    fence_mbar_init();
  }
  if (warp == kMmaWarp) tmem_alloc(bars + L::kSlotTmem, 256);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(gbase + L::kOffBar + L::kSlotTmem);

  if (warp == kLoadWarp) {
    if (lane == 0) {
      int issued = 0;
      mbar_expect_tx(bars + L::kBarQ, 2 * kTileR);
      load_tile(base + L::kOffQ, kHalfR, &tmQ, row0 + q0, bars + L::kBarQ);
      load_tile(base + L::kOffG, kHalfR, &tmG, row0 + q0, bars + L::kBarQ);
      for (int j = 0; j < nk; ++j) {
        const int s = j % kStages, u = j / kStages;
        if (j >= kStages && !mbar_wait(bars + L::kBarE + 8 * s, (u - 1) & 1, abort, status)) break;
        mbar_expect_tx(bars + L::kBarK + 8 * s, kTileC);
        load_tile(base + L::kOffK + s * kTileC, kHalfC, &tmK, row0 + j * kC, bars + L::kBarK + 8 * s);
        mbar_expect_tx(bars + L::kBarV + 8 * s, kTileC);
        load_tile(base + L::kOffV + s * kTileC, kHalfC, &tmV, row0 + j * kC, bars + L::kBarV + 8 * s);
        issued = j + 1;
      }
      if (*abort) {
        wait_drain(bars + L::kBarQ, 0);
        for (int j = issued - kStages < 0 ? 0 : issued - kStages; j < issued; ++j) {
          wait_drain(bars + L::kBarK + 8 * (j % kStages), (j / kStages) & 1);
          wait_drain(bars + L::kBarV + 8 * (j % kStages), (j / kStages) & 1);
        }
      }
    }
  } else if (warp == kMmaWarp) {
    if (lane == 0) {
      bool ok = mbar_wait(bars + L::kBarQ, 0, abort, status) && mbar_wait(bars + L::kBarK, 0, abort, status) &&
                mbar_wait(bars + L::kBarV, 0, abort, status);
      if (ok) {
        tc_fence_after();
        gemm_rc(tmem, base + L::kOffQ, base + L::kOffK);       // S = Q K^T
        gemm_rc(tmem + kC, base + L::kOffG, base + L::kOffV);  // dP = dO V^T
        mma_commit(bars + L::kBarSP);
      }
      for (int j = 0; ok && j < nk; ++j) {
        const int s = j % kStages;
        if (!(ok = mbar_wait(bars + L::kBarTF, j & 1, abort, status))) break;
        tc_fence_after();
        if (j + 1 < nk) {
          const int s1 = (j + 1) % kStages, u1 = (j + 1) / kStages;
          if (!(ok = mbar_wait2(bars + L::kBarK + 8 * s1, u1 & 1, bars + L::kBarV + 8 * s1, u1 & 1, abort, status)))
            break;
          gemm_rc(tmem, base + L::kOffQ, base + L::kOffK + s1 * kTileC);
          gemm_rc(tmem + kC, base + L::kOffG, base + L::kOffV + s1 * kTileC);
          mma_commit(bars + L::kBarSP);
        }
        if (!(ok = mbar_wait(bars + L::kBarDS, j & 1, abort, status))) break;
        tc_fence_after();
        gemm_acc(tmem + L::kColDQ, base + L::kOffDS, base + L::kOffK + s * kTileC, j > 0);  // dQ += dS K
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
      const int kc = j * kC + col0;    // first key of this group's columns
      const bool diag = kc + 31 > q0;  // some key may follow some query of the tile
      const int lim = qrow - kc;       // visible columns: e <= lim
      float sv[32], dp[32];
      tmem_ld32(lane_base + col0, sv);
      tmem_ld32(lane_base + kC + col0, dp);
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive(bars + L::kBarTF);  // TMEM columns free for the next step's products
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
    if (__all_sync(0xffffffffu, ok)) {
      tc_fence_after();
      // dQ: 128 columns, 64 per group
#pragma unroll
      for (int piece = 0; piece < 2; ++piece) {
        const int c = 64 * grp + 32 * piece;
        float v[32];
        tmem_ld32(lane_base + L::kColDQ + c, v);
        tmem_wait_ld();
        if (qrow < S) store_out32(dQ + ((int64_t)row0 + qrow) * kD128 + c, v, scale);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

}  // namespace

cudaError_t launch_attn_bwd_tc128(int64_t BH, int64_t S, const void* Q, const void* K, const void* V,
                                  const float* lse, const void* dO, const float* D, void* dQ,
                                  void* dK, void* dV, float* dq_acc, cudaStream_t st) {
  // Tiles that stay resident in a CTA have 128 rows; streamed chunks 64.
  CUtensorMap qR, gR, kR, vR, qC, gC, kC_, vC;
  const int64_t rows = BH * S;
  if (!make_tile_map_d(&qR, Q, rows, kRows, kD128) || !make_tile_map_d(&gR, dO, rows, kRows, kD128) ||
      !make_tile_map_d(&kR, K, rows, kRows, kD128) || !make_tile_map_d(&vR, V, rows, kRows, kD128) ||
      !make_tile_map_d(&qC, Q, rows, kC, kD128) || !make_tile_map_d(&gC, dO, rows, kC, kD128) ||
      !make_tile_map_d(&kC_, K, rows, kC, kD128) || !make_tile_map_d(&vC, V, rows, kC, kD128))
    return cudaErrorInvalidValue;
  unsigned int* status = device_status_ptr();
  // The opt-in to more than 48 KB of dynamic shared memory belongs to the
  // function in the current device's context, so it is applied on every
  // launch (a host-side call): right for any device, thread or context.
  {
    cudaError_t e = cudaFuncSetAttribute(attn_bwd_dkdv_tc128_kernel<false>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, KV::kSmemBytes);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(attn_bwd_dkdv_tc128_kernel<true>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, KV::kSmemBytes);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(attn_bwd_dq_tc128_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             QQ::kSmemBytes);
    if (e != cudaSuccess) return e;
  }
  const int ntiles = (int)((S + kRows - 1) / kRows);
  const float scale = (float)0.08838834764831845;  // 1/sqrt(128)
  const float sl2 = (float)(0.08838834764831845 * 1.4426950408889634);
  // (tiles, problems): one problem's key tiles are launched together,
  // longest first, so the operands and fp32 dQ accumulator of one or two
  // problems at a time stay in L2 (faster than interleaving the problems)
  const int ty = BH > 65535 ? 1 : 0;
  if (ty && ntiles > 65535) return cudaErrorInvalidConfiguration;
  const dim3 grid = ty ? dim3((unsigned)BH, ntiles) : dim3(ntiles, (unsigned)BH);
  if (dq_acc != nullptr) {
    const int64_t n = rows * kD128;
    CUtensorMap accM;
    if (!make_acc_map_d(&accM, dq_acc, rows, kD128, kC)) return cudaErrorInvalidValue;
    cudaError_t e = cudaMemsetAsync(dq_acc, 0, (size_t)n * sizeof(float), st);
    if (e != cudaSuccess) return e;
    attn_bwd_dkdv_tc128_kernel<true><<<grid, kThreads, KV::kSmemBytes, st>>>(
        qC, kR, vR, gC, accM, lse, D, static_cast<bf16*>(dK), static_cast<bf16*>(dV), (int)S, sl2,
        scale, ty, status);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    return launch_dq_round(dq_acc, dQ, n, scale, st);
  }
  attn_bwd_dkdv_tc128_kernel<false><<<grid, kThreads, KV::kSmemBytes, st>>>(
      qC, kR, vR, gC, qC /* no dQ shares */, lse, D, static_cast<bf16*>(dK), static_cast<bf16*>(dV),
      (int)S, sl2, scale, ty, status);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  attn_bwd_dq_tc128_kernel<<<grid, kThreads, QQ::kSmemBytes, st>>>(
      qR, kC_, vC, gR, lse, D, static_cast<bf16*>(dQ), (int)S, ntiles, sl2, scale, ty, status);
  return cudaGetLastError();
}

}  // namespace lh
