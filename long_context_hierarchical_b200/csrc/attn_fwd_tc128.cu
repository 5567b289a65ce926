// Stage 3 forward for head dimension 128 on the 5th-generation tensor cores:
// causal attention on the gathered [S, 128] bf16 sub-sequence (skill card
// "lighthouse-attention", stage 3: a standard S x S causal mask; gist.science
// 2.C).
//
// Same CTA shape as the d = 64 kernel: 256 query rows as two 128-row tiles A
// and B walking the 128-key tiles up to the diagonal, softmax warps 0-3 (A)
// and 4-7 (B) with one query row per thread, warp 8 the TMA producer, warp 9
// the MMA issuer.  What d = 128 changes:
//  - a tile row is 256 bytes, loaded as two 64-column boxes (128-byte
//    swizzle), each a [128 x 64] K-major half 16 KB apart; S = Q K^T takes
//    8 K-steps, the first four in half 0;
//  - O is 128 fp32 columns per tile, so TMEM (512 columns) holds
//    S_A [0,128), S_B [128,256), O_A [256,384), O_B [384,512) and P_X
//    (bf16 pairs, 64 columns) overwrites the first half of S_X once the
//    softmax threads have loaded S_X into registers;
//  - so S_X(j+1) cannot be computed before P_X(j) V_j has read P_X: the MMA
//    thread issues, per key tile, P_A V, S_A(next), P_B V, S_B(next), and a
//    tile's exponentials overlap the other tile's MMAs.  Because the MMAs of
//    one thread complete in issue order, S_X(j) being ready also means
//    P_X(j-1) V_{j-1} is complete, so O_X may be rescaled right away;
//  - P V is an N = 128 MMA reading V MN-major across both halves (LBO = the
//    16 KB between them);
//  - K/V tiles are 32 KB each: two ring stages (192 KB of tiles in all).
// Every wait is bounded, as in the d = 64 kernel.
#include <cudaTypedefs.h>

#include "host.h"
#include "tc.cuh"

namespace lh {

bool make_tile_map_d(CUtensorMap* map, const void* ptr, int64_t rows, int box_rows, int d);

namespace {

using bf16 = __nv_bfloat16;
using namespace tc;

constexpr int kD128 = 128;
constexpr int kRows = 128;                       // query rows per tile, keys per tile
constexpr int kStages = 2;
constexpr uint32_t kHalf = kRows * 64 * 2;       // 16 KB: 128 rows x 64 columns
constexpr uint32_t kTile = 2 * kHalf;            // 32 KB: 128 rows x 128 columns
constexpr int kLoadWarp = 8, kMmaWarp = 9;
constexpr int kThreads = (kMmaWarp + 1) * 32;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kRescale = 8.0f;                 // log2 units
constexpr uint32_t kColO = 2 * kRows;            // O_A at 256, O_B at 384

// Shared-memory map (offsets from a 1024-byte aligned base).
constexpr uint32_t kOffQ = 0;                          // 2 tiles
constexpr uint32_t kOffK = kOffQ + 2 * kTile;          // kStages tiles
constexpr uint32_t kOffV = kOffK + kStages * kTile;    // kStages tiles
constexpr uint32_t kOffBar = kOffV + kStages * kTile;
// per tile x (8 bytes apart): S ready, P written, last P V done
constexpr uint32_t kBarQ = 0, kBarK = 8, kBarV = kBarK + 8 * kStages, kBarE = kBarV + 8 * kStages,
                   kBarS = kBarE + 8 * kStages, kBarP = kBarS + 16, kBarPV = kBarP + 16,
                   kBarDrain = kBarPV + 16, kSlotTmem = kBarDrain + 8, kSlotAbort = kSlotTmem + 4;
constexpr uint32_t kSmemBytes = kOffBar + 256 + 1024;  // + alignment slack
static_assert(kSlotAbort + 4 <= 256, "barrier area");
static_assert(kSmemBytes <= 227 * 1024, "shared memory per CTA");

__device__ __forceinline__ float row_max(const float (&v)[4][32]) {
  float pm[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
  for (int c = 0; c < 4; ++c)
#pragma unroll
    for (int e = 0; e < 32; e += 2) pm[c] = fmax3f(pm[c], v[c][e], v[c][e + 1]);
  return fmaxf(fmaxf(pm[0], pm[1]), fmaxf(pm[2], pm[3]));
}

__device__ __forceinline__ bool wait_drain(uint32_t bar, uint32_t parity) {
  // Bounded wait that ignores the abort flag (used to drain own copies).
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity))
    if (clock64() - t0 > kWaitCycles) return false;
  return true;
}

// Both 64-column halves of a 128-row tile, completing on one barrier.
__device__ __forceinline__ void load_tile(uint32_t dst, const CUtensorMap* map, int row, uint32_t bar) {
  tma_load_2d(dst, map, 0, row, bar);
  tma_load_2d(dst + kHalf, map, 64, row, bar);
}

__global__ void __maxnreg__(168)
attn_fwd_tc128_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                      const __grid_constant__ CUtensorMap tmV, bf16* __restrict__ O,
                      float* __restrict__ lse, int S, int npairs, float sl2, int tiles_on_y,
                      unsigned int* __restrict__ status) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_addr(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw);
  const uint32_t bars = base + kOffBar;
  volatile int* abort = reinterpret_cast<volatile int*>(gbase + kOffBar + kSlotAbort);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int pair = npairs - 1 - (int)(tiles_on_y ? blockIdx.y : blockIdx.x);  // longest rows first
  const int bh = tiles_on_y ? blockIdx.x : blockIdx.y;
  const int q0 = pair * 2 * kRows;
  const int nA = 2 * pair + 1, nB = 2 * pair + 2;  // key tiles of tile A / tile B
  const int row0 = bh * S;                          // first row of this head in the maps

  if (threadIdx.x == 0) {
    mbar_init(bars + kBarQ, 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(bars + kBarK + 8 * s, 1);
      mbar_init(bars + kBarV + 8 * s, 1);
      mbar_init(bars + kBarE + 8 * s, 1);
    }
    for (int x = 0; x < 2; ++x) {
      mbar_init(bars + kBarS + 8 * x, 1);
      mbar_init(bars + kBarP + 8 * x, 128);
      mbar_init(bars + kBarPV + 8 * x, 1);
    }
    mbar_init(bars + kBarDrain, 1);
    *abort = 0;
    fence_mbar_init();
  }
  if (warp == kMmaWarp) tmem_alloc(bars + kSlotTmem, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(gbase + kOffBar + kSlotTmem);

  if (warp == kLoadWarp) {
    // ---------------- TMA producer ----------------
    if (lane == 0) {
      int issued = 0;
      mbar_expect_tx(bars + kBarQ, 2 * kTile);
      load_tile(base + kOffQ, &tmQ, row0 + q0, bars + kBarQ);
      load_tile(base + kOffQ + kTile, &tmQ, row0 + q0 + kRows, bars + kBarQ);
      for (int j = 0; j < nB; ++j) {
        const int s = j % kStages, u = j / kStages;
        if (j >= kStages && !mbar_wait(bars + kBarE + 8 * s, (u - 1) & 1, abort, status)) break;
        mbar_expect_tx(bars + kBarK + 8 * s, kTile);
        load_tile(base + kOffK + s * kTile, &tmK, row0 + j * kRows, bars + kBarK + 8 * s);
        mbar_expect_tx(bars + kBarV + 8 * s, kTile);
        load_tile(base + kOffV + s * kTile, &tmV, row0 + j * kRows, bars + kBarV + 8 * s);
        issued = j + 1;
      }
      if (*abort) {  // let this CTA's own copies land before its smem is released
        wait_drain(bars + kBarQ, 0);
        for (int j = issued - kStages < 0 ? 0 : issued - kStages; j < issued; ++j) {
          const int s = j % kStages, u = j / kStages;
          wait_drain(bars + kBarK + 8 * s, u & 1);
          wait_drain(bars + kBarV + 8 * s, u & 1);
        }
      }
    }
  } else if (warp == kMmaWarp) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      constexpr uint32_t idS = idesc_bf16(kRows, kRows, false);
      constexpr uint32_t idPV = idesc_bf16(kRows, kD128, true);
      auto issue_S = [&](int x, int j) {
        const uint64_t dq = sw128_desc(base + kOffQ + x * kTile, 16, 1024);
        const uint64_t dk = sw128_desc(base + kOffK + (j % kStages) * kTile, 16, 1024);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
          const uint32_t off = (ks >> 2) * kHalf + (ks & 3) * 32;
          mma_bf16(tmem + x * kRows, desc_add(dq, off), desc_add(dk, off), idS, ks > 0);
        }
        mma_commit(bars + kBarS + 8 * x);
      };
      // O_x += P_x V_j: P_x (bf16) in the first 64 columns of S_x; V read
      // MN-major, its two 64-column halves kHalf apart.
      auto issue_PV = [&](int x, int j) {
        const uint64_t dv = sw128_desc(base + kOffV + (j % kStages) * kTile, kHalf, 1024);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_bf16_ts(tmem + kColO + x * kD128, tmem + x * kRows + 8 * kk, desc_add(dv, kk * 2048),
                      idPV, (j > 0 || kk > 0) ? 1u : 0u);
      };
      // tile x at key tile j: P_x(j) V_j, then S_x(j+1) over the same columns
      auto step = [&](int x, int j, int n) -> bool {
        if (!mbar_wait2(bars + kBarP + 8 * x, j & 1, bars + kBarV + 8 * (j % kStages), (j / kStages) & 1,
                        abort, status))
          return false;
        tc_fence_after();
        issue_PV(x, j);
        if (j + 1 < n) {
          const int s1 = (j + 1) % kStages, u1 = (j + 1) / kStages;
          if (!mbar_wait(bars + kBarK + 8 * s1, u1 & 1, abort, status)) return false;
          tc_fence_after();
          issue_S(x, j + 1);
        } else {
          mma_commit(bars + kBarPV + 8 * x);  // this tile's last P V
        }
        return true;
      };
      bool ok = mbar_wait(bars + kBarQ, 0, abort, status) && mbar_wait(bars + kBarK, 0, abort, status);
      if (ok) {
        tc_fence_after();
        issue_S(0, 0);
        issue_S(1, 0);
      }
      for (int j = 0; ok && j < nB; ++j) {
        if (j < nA && !(ok = step(0, j, nA))) break;
        if (!(ok = step(1, j, nB))) break;
        mma_commit(bars + kBarE + 8 * (j % kStages));  // K_j and V_j free once these MMAs are done
      }
      // Every MMA issued here has finished before TMEM is released.
      mma_commit(bars + kBarDrain);
      wait_drain(bars + kBarDrain, 0);
    }
  } else {
    // ---------------- softmax, one query row (128 columns) per thread ----------------
    const int x = warp >> 2, wr = warp & 3;
    const int r = wr * 32 + lane;
    const uint32_t lane_base = tmem + ((uint32_t)(wr * 32) << 16);
    const uint32_t tS = lane_base + x * kRows, tO = lane_base + kColO + x * kD128;
    const int n = x ? nB : nA;
    const int qrow = q0 + x * kRows + r;
    const float2 sc2 = make_float2(sl2, sl2);
    float m_ref = -INFINITY;
    float2 l2 = make_float2(0.f, 0.f);  // row sum, two partial sums
    bool ok = true;
    for (int j = 0; j < n; ++j) {
      // S_x(j) ready: P_x(j-1) V_{j-1} (issued before it) is complete too
      ok = mbar_wait(bars + kBarS + 8 * x, j & 1, abort, status);
      if (!(ok = __all_sync(0xffffffffu, ok))) break;  // warp-uniform before TMEM access
      tc_fence_after();
      float v[4][32];
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_ld32(tS + 32 * c, v[c]);
      tmem_wait_ld();
      if (j == n - 1) {  // diagonal tile: keys after this query are masked
        const int lim = qrow - j * kRows;
#pragma unroll
        for (int c = 0; c < 4; ++c)
#pragma unroll
          for (int e = 0; e < 32; ++e)
            if (32 * c + e > lim) v[c][e] = -INFINITY;
      }
      const float mx = row_max(v) * sl2;
      const float m_new = mx > m_ref + kRescale ? mx : m_ref;
      const float alpha = exp2f(m_ref - m_new);  // 1 when unchanged, 0 on the first tile
      // P = 2^(s*sl2 - m_new): row sum, bf16 P over the first 64 columns of S_x
      const float2 nm2 = make_float2(-m_new, -m_new);
      float2 part[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t w[16];
#pragma unroll
        for (int e = 0; e < 32; e += 2) {
          float2 t = ffma2(make_float2(v[c][e], v[c][e + 1]), sc2, nm2);
          t.x = ex2_approx(t.x);
          t.y = ex2_approx(t.y);
          part[(e >> 1) & 1] = fadd2(part[(e >> 1) & 1], t);
          w[e >> 1] = pack_bf16x2(t.x, t.y);
        }
        tmem_st16(tS + 16 * c, w);
      }
      // O_x follows a grown reference maximum (no MMA writes O_x until this
      // tile's P is released below)
      if (j > 0 && __any_sync(0xffffffffu, m_new != m_ref)) {
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          float o[32];
          tmem_ld32(tO + 32 * c, o);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) o[e] *= alpha;
          tmem_st32(tO + 32 * c, o);
        }
      }
      m_ref = m_new;
      l2 = ffma2(l2, make_float2(alpha, alpha), fadd2(part[0], part[1]));
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(bars + kBarP + 8 * x);
    }
    if (ok) ok = mbar_wait(bars + kBarPV + 8 * x, 0, abort, status);
    if (__all_sync(0xffffffffu, ok)) {
      const float l = l2.x + l2.y;
      tc_fence_after();
#pragma unroll
      for (int h = 0; h < 4; ++h) {
        float o[32];
        tmem_ld32(tO + 32 * h, o);
        tmem_wait_ld();
        if (qrow < S) {
          const float inv = 1.f / l;
          bf16* dst = O + ((int64_t)row0 + qrow) * kD128 + 32 * h;
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            uint32_t w[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) w[q] = pack_bf16x2(o[8 * c + 2 * q] * inv, o[8 * c + 2 * q + 1] * inv);
            reinterpret_cast<uint4*>(dst)[c] = make_uint4(w[0], w[1], w[2], w[3]);
          }
        }
      }
      if (qrow < S) lse[(int64_t)row0 + qrow] = (m_ref + log2f(l)) * kLn2;
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

cudaError_t launch_attn_fwd_tc128(int64_t BH, int64_t S, const void* Q, const void* K,
                                  const void* V, void* O, float* lse, cudaStream_t st) {
  CUtensorMap mq, mk, mv;
  if (!make_tile_map_d(&mq, Q, BH * S, kRows, kD128) || !make_tile_map_d(&mk, K, BH * S, kRows, kD128) ||
      !make_tile_map_d(&mv, V, BH * S, kRows, kD128))
    return cudaErrorInvalidValue;
  unsigned int* status = device_status_ptr();
  // The opt-in to more than 48 KB of dynamic shared memory belongs to the
  // function in the current device's context, so it is applied on every
  // launch (a host-side call): right for any device, thread or context.
  {
    cudaError_t e = cudaFuncSetAttribute(attn_fwd_tc128_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (e != cudaSuccess) return e;
  }
  const int npairs = (int)((S + 2 * kRows - 1) / (2 * kRows));
  // 1/sqrt(128) * log2(e), rounded once
  const float sl2 = (float)(0.08838834764831845 * 1.4426950408889634);
  const int ty = npairs <= 65535 ? 1 : 0;
  if (!ty && BH > 65535) return cudaErrorInvalidConfiguration;
  const dim3 grid = ty ? dim3((unsigned)BH, npairs) : dim3(npairs, (unsigned)BH);
  attn_fwd_tc128_kernel<<<grid, kThreads, kSmemBytes, st>>>(mq, mk, mv, static_cast<bf16*>(O), lse,
                                                           (int)S, npairs, sl2, ty, status);
  return cudaGetLastError();
}

}  // namespace lh
