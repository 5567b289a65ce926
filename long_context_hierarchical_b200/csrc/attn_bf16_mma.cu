// Backward of the dense causal attention on the gathered sub-sequence, bf16
// storage, on the warp-level tensor-core path (mma.sync m16n8k16, fp32
// accumulate).  Gradients flow through attention into the gathered rows
// (skill card "lighthouse-attention", "梯度流").
//
// Tiles are 64 x 64 (queries x keys), d = 64, 4 warps per CTA, each warp
// owning 16 rows of the CTA's tile.  K/V (or Q/dO) tiles are double-buffered
// in shared memory with cp.async; rows are 128 bytes and their 16-byte chunks
// are XOR-swizzled by (row % 8), so ldmatrix reads are conflict-free.
// Causality: key tiles above the diagonal are never visited; the diagonal
// tile is masked element-wise.  Softmax runs in the log2 domain.
//
// Backward (FlashAttention-2 style, deterministic): one kernel per key tile
// accumulates dK and dV over query tiles, one kernel per query tile
// accumulates dQ over key tiles; no atomics.
#include "host.h"

namespace lh {
namespace {

using bf16 = __nv_bfloat16;
constexpr int kT = 64;       // tile rows / cols
constexpr int kNT = 128;     // threads per CTA
constexpr int kTileBytes = kT * kD * 2;
constexpr float kLog2e = 1.4426950408889634f;

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ uint32_t tile_off(int row, int chunk) {
  return row * 128 + ((chunk ^ (row & 7)) << 4);
}
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, bool valid) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(dst), "l"(src),
               "r"(valid ? 16 : 0));
}
__device__ __forceinline__ void cp_commit() { asm volatile("cp.async.commit_group;\n" ::); }
template <int N>
__device__ __forceinline__ void cp_wait() { asm volatile("cp.async.wait_group %0;\n" ::"n"(N)); }

// Copy rows [r0, r0 + 64) of a [S, 64] bf16 matrix into a swizzled tile;
// rows at or past S are zero-filled.
__device__ __forceinline__ void load_tile(uint32_t dst, const bf16* src, int64_t r0, int64_t S) {
  for (int idx = threadIdx.x; idx < kT * 8; idx += kNT) {
    const int row = idx >> 3, ch = idx & 7;
    const int64_t gr = r0 + row;
    const bool ok = gr < S;
    cp_async16(dst + tile_off(row, ch), src + (ok ? gr : 0) * kD + ch * 8, ok);
  }
}
// 64 fp32 values (one per row) into shared memory, zero past S.
__device__ __forceinline__ void load_vec(float* dst, const float* src, int64_t r0, int64_t S) {
  if (threadIdx.x < kT) {
    const int64_t gr = r0 + threadIdx.x;
    dst[threadIdx.x] = gr < S ? __ldg(src + gr) : 0.f;
  }
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                        uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                          uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                         uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

// A fragments (16 rows x 64 channels) of rows [r0, r0+16) of a tile.
__device__ __forceinline__ void load_a_frags(uint32_t tile, int r0, uint32_t (&a)[4][4]) {
  const int i = threadIdx.x & 31;
  const int row = r0 + (i & 7) + ((i >> 3) & 1) * 8;
#pragma unroll
  for (int ks = 0; ks < 4; ++ks)
    ldsm_x4(tile + tile_off(row, ks * 2 + (i >> 4)), a[ks][0], a[ks][1], a[ks][2], a[ks][3]);
}

// acc[nb] += A(16 x 64) * B^T where B's rows are the tile's 64 rows (the n
// dimension) and its columns the 64 channels (the k dimension).
__device__ __forceinline__ void mma_abt(float (&acc)[8][4], const uint32_t (&a)[4][4], uint32_t tile) {
  const int i = threadIdx.x & 31;
#pragma unroll
  for (int ks = 0; ks < 4; ++ks)
#pragma unroll
    for (int nbp = 0; nbp < 4; ++nbp) {
      uint32_t b0, b1, b2, b3;
      const int row = nbp * 16 + (i & 7) + (i >> 4) * 8;
      ldsm_x4(tile + tile_off(row, ks * 2 + ((i >> 3) & 1)), b0, b1, b2, b3);
      mma16816(acc[2 * nbp], a[ks], b0, b1);
      mma16816(acc[2 * nbp + 1], a[ks], b2, b3);
    }
}

// acc[nb] += P(16 x 64, C-fragment layout, k = tile rows) * tile(64 x 64).
__device__ __forceinline__ void mma_pb(float (&acc)[8][4], const float (&p)[8][4], uint32_t tile) {
  const int i = threadIdx.x & 31;
#pragma unroll
  for (int kk = 0; kk < 4; ++kk) {
    uint32_t a[4];
    a[0] = pack_bf16(p[2 * kk][0], p[2 * kk][1]);
    a[1] = pack_bf16(p[2 * kk][2], p[2 * kk][3]);
    a[2] = pack_bf16(p[2 * kk + 1][0], p[2 * kk + 1][1]);
    a[3] = pack_bf16(p[2 * kk + 1][2], p[2 * kk + 1][3]);
    const int row = kk * 16 + (i & 7) + ((i >> 3) & 1) * 8;
#pragma unroll
    for (int nbp = 0; nbp < 4; ++nbp) {
      uint32_t b0, b1, b2, b3;
      ldsm_x4_t(tile + tile_off(row, 2 * nbp + (i >> 4)), b0, b1, b2, b3);
      mma16816(acc[2 * nbp], a, b0, b1);
      mma16816(acc[2 * nbp + 1], a, b2, b3);
    }
  }
}

__device__ __forceinline__ void zero(float (&a)[8][4]) {
#pragma unroll
  for (int n = 0; n < 8; ++n)
#pragma unroll
    for (int e = 0; e < 4; ++e) a[n][e] = 0.f;
}

// Store a 16 x 64 C-fragment block (rows r0.., scaled) as bf16 rows.
__device__ __forceinline__ void store_rows(bf16* dst, int64_t r0, int64_t S, const float (&a)[8][4],
                                           float sa, float sb) {
  const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
#pragma unroll
  for (int nb = 0; nb < 8; ++nb) {
    const int col = nb * 8 + 2 * t;
    if (r0 + g < S)
      *reinterpret_cast<uint32_t*>(dst + (r0 + g) * kD + col) = pack_bf16(a[nb][0] * sa, a[nb][1] * sa);
    if (r0 + g + 8 < S)
      *reinterpret_cast<uint32_t*>(dst + (r0 + g + 8) * kD + col) =
          pack_bf16(a[nb][2] * sb, a[nb][3] * sb);
  }
}

// ---------------------------------------------------------------------------
// backward: dK, dV per key tile
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(kNT)
attn_bwd_dkdv_mma_kernel(const bf16* __restrict__ Q, const bf16* __restrict__ K,
                         const bf16* __restrict__ V, const float* __restrict__ lse,
                         const bf16* __restrict__ dO, const float* __restrict__ D,
                         bf16* __restrict__ dK, bf16* __restrict__ dV, int64_t S, int ntiles,
                         float sl2, float scale) {
  extern __shared__ __align__(128) uint8_t smem[];  // 6 tiles + 4 x 64 floats
  const uint32_t sK = smem_u32(smem), sV = sK + kTileBytes;
  const uint32_t sQ = sK + 2 * kTileBytes, sG = sK + 4 * kTileBytes;  // [2] each
  float* fL = reinterpret_cast<float*>(smem + 6 * kTileBytes);  // [2][64] lse
  float* fD = fL + 2 * kT;                                      // [2][64] D
  const int kt = blockIdx.x;  // tile 0 sees the most query tiles
  const int64_t bh = blockIdx.y;
  const int64_t k0 = (int64_t)kt * kT;
  const bf16* Qb = Q + bh * S * kD;
  const bf16* Gb = dO + bh * S * kD;
  const float* Lb = lse + bh * S;
  const float* Db = D + bh * S;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;

  load_tile(sK, K + bh * S * kD, k0, S);
  load_tile(sV, V + bh * S * kD, k0, S);
  load_tile(sQ, Qb, k0, S);
  load_tile(sG, Gb, k0, S);
  load_vec(fL, Lb, k0, S);
  load_vec(fD, Db, k0, S);
  cp_commit();

  uint32_t ka[4][4], va[4][4];
  float dk[8][4], dv[8][4];
  zero(dk);
  zero(dv);
  for (int i = kt; i < ntiles; ++i) {
    const int buf = (i - kt) & 1;
    if (i + 1 < ntiles) {
      const int64_t r = (int64_t)(i + 1) * kT;
      load_tile(sQ + (buf ^ 1) * kTileBytes, Qb, r, S);
      load_tile(sG + (buf ^ 1) * kTileBytes, Gb, r, S);
      load_vec(fL + (buf ^ 1) * kT, Lb, r, S);
      load_vec(fD + (buf ^ 1) * kT, Db, r, S);
    }
    cp_commit();
    cp_wait<1>();
    __syncthreads();
    if (i == kt) {
      load_a_frags(sK, warp * 16, ka);
      load_a_frags(sV, warp * 16, va);
    }
    const uint32_t q = sQ + buf * kTileBytes, gq = sG + buf * kTileBytes;
    const float* l2 = fL + buf * kT;
    const float* dd = fD + buf * kT;
    float p[8][4], dp[8][4];
    zero(p);
    zero(dp);
    mma_abt(p, ka, q);   // S^T: rows = keys, cols = queries
    mma_abt(dp, va, gq); // dP^T
    const int64_t q0 = (int64_t)i * kT;
#pragma unroll
    for (int nb = 0; nb < 8; ++nb)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int col = nb * 8 + 2 * t + (e & 1);  // query within tile
        const int row = warp * 16 + g + (e < 2 ? 0 : 8);  // key within tile
        const int64_t qi = q0 + col, kj = k0 + row;
        float pv = 0.f;
        if (qi >= kj && qi < S) pv = exp2f(p[nb][e] * sl2 - l2[col] * kLog2e);
        p[nb][e] = pv;
        dp[nb][e] = pv * (dp[nb][e] - dd[col]);  // dS^T
      }
    mma_pb(dv, p, gq);
    mma_pb(dk, dp, q);
    __syncthreads();
  }
  const int64_t r0 = k0 + warp * 16;
  store_rows(dK + bh * S * kD, r0, S, dk, scale, scale);
  store_rows(dV + bh * S * kD, r0, S, dv, 1.f, 1.f);
}

// ---------------------------------------------------------------------------
// backward: dQ per query tile
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(kNT)
attn_bwd_dq_mma_kernel(const bf16* __restrict__ Q, const bf16* __restrict__ K,
                       const bf16* __restrict__ V, const float* __restrict__ lse,
                       const bf16* __restrict__ dO, const float* __restrict__ D,
                       bf16* __restrict__ dQ, int64_t S, int ntiles, float sl2, float scale) {
  __shared__ __align__(128) uint8_t smem[6 * kTileBytes];
  const uint32_t sQ = smem_u32(smem), sG = sQ + kTileBytes;
  const uint32_t sK = sQ + 2 * kTileBytes, sV = sQ + 4 * kTileBytes;  // [2] each
  const int qt = ntiles - 1 - blockIdx.x;
  const int64_t bh = blockIdx.y;
  const int64_t q0 = (int64_t)qt * kT;
  const bf16* Kb = K + bh * S * kD;
  const bf16* Vb = V + bh * S * kD;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;

  load_tile(sQ, Q + bh * S * kD, q0, S);
  load_tile(sG, dO + bh * S * kD, q0, S);
  load_tile(sK, Kb, 0, S);
  load_tile(sV, Vb, 0, S);
  cp_commit();

  const int64_t ra = q0 + warp * 16 + g, rb = ra + 8;
  const float l2a = ra < S ? lse[bh * S + ra] * kLog2e : 0.f;
  const float l2b = rb < S ? lse[bh * S + rb] * kLog2e : 0.f;
  const float Da = ra < S ? D[bh * S + ra] : 0.f;
  const float Db = rb < S ? D[bh * S + rb] : 0.f;

  uint32_t qa[4][4], ga[4][4];
  float dq[8][4];
  zero(dq);
  for (int j = 0; j <= qt; ++j) {
    const int buf = j & 1;
    if (j + 1 <= qt) {
      load_tile(sK + (buf ^ 1) * kTileBytes, Kb, (int64_t)(j + 1) * kT, S);
      load_tile(sV + (buf ^ 1) * kTileBytes, Vb, (int64_t)(j + 1) * kT, S);
    }
    cp_commit();
    cp_wait<1>();
    __syncthreads();
    if (j == 0) {
      load_a_frags(sQ, warp * 16, qa);
      load_a_frags(sG, warp * 16, ga);
    }
    const uint32_t kk = sK + buf * kTileBytes, vv = sV + buf * kTileBytes;
    float p[8][4], dp[8][4];
    zero(p);
    zero(dp);
    mma_abt(p, qa, kk);
    mma_abt(dp, ga, vv);
    const int64_t k0 = (int64_t)j * kT;
#pragma unroll
    for (int nb = 0; nb < 8; ++nb)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int64_t kj = k0 + nb * 8 + 2 * t + (e & 1);
        const int64_t qi = e < 2 ? ra : rb;
        float pv = 0.f;
        if (kj <= qi && qi < S) pv = exp2f(p[nb][e] * sl2 - (e < 2 ? l2a : l2b));
        dp[nb][e] = pv * (dp[nb][e] - (e < 2 ? Da : Db));
      }
    mma_pb(dq, dp, kk);
    __syncthreads();
  }
  store_rows(dQ + bh * S * kD, q0 + warp * 16, S, dq, scale, scale);
}

}  // namespace

cudaError_t launch_attn_bwd_mma(int64_t BH, int64_t S, const void* Q, const void* K, const void* V,
                                const float* lse, const void* dO, const float* D, void* dQ,
                                void* dK, void* dV, cudaStream_t st) {
  const int ntiles = (int)((S + kT - 1) / kT);
  const float sl2 = 0.125f * kLog2e;
  const dim3 grid(ntiles, (unsigned)BH);
  constexpr int dkdv_smem = 6 * kTileBytes + 4 * kT * 4;
  cudaError_t e = cudaFuncSetAttribute(attn_bwd_dkdv_mma_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, dkdv_smem);
  if (e != cudaSuccess) return e;
  attn_bwd_dkdv_mma_kernel<<<grid, kNT, dkdv_smem, st>>>((const bf16*)Q, (const bf16*)K, (const bf16*)V, lse,
                                                 (const bf16*)dO, D, (bf16*)dK, (bf16*)dV, S,
                                                 ntiles, sl2, 0.125f);
  attn_bwd_dq_mma_kernel<<<grid, kNT, 0, st>>>((const bf16*)Q, (const bf16*)K, (const bf16*)V, lse,
                                               (const bf16*)dO, D, (bf16*)dQ, S, ntiles, sl2, 0.125f);
  return cudaGetLastError();
}

}  // namespace lh
