// Stage 2b: joint top-K over the candidate levels and the causal order of the
// gathered sub-sequence.
//
// Selection (skill card "lighthouse-attention", stage 2 "打分与选择";
// gist.science Technical Summary 2.B): per (batch, head), the Ksel candidates
// with the largest scores are kept, ties going to the lower level-major flat
// index, and every coarsest-level entry is kept.  The pages' kernel splits the
// score stream into 2048-entry chunks with per-CTA register top-128 buffers
// (skill card, "Kernel Design"); here the selection is an exact radix select
// on a unique 64-bit key, because only the threshold is needed:
//
//   key(f) = orderable(score_f) << 32 | (0xffffffff - f)
//
// Larger keys are better and no two are equal, so "f is selected" is exactly
// key(f) >= kappa where kappa is the Ksel-th largest key.  kappa is found with
// two 12-bit histogram passes over the score bits, a compaction of the few
// candidates left in the threshold bucket, and an 8-bit radix select on those.
//
// Order (stage 3 "密集子序列注意力"; gist.science 2.C asks for a topological order):
// selected entries are laid out by (last token of the span, level), which is
// a walk over tokens t with, at each t, the levels l whose spans end at t
// ((t + 1) % p^l == 0).  A count per token block, a scan of the block counts
// and a rewrite give each selected entry its slot with no sort.
//
// Hierarchical descent (lh_select LH_SELECT_DESCENT, the other reading of
// the (L-1)*p*k budget): one block per (batch, head) walks from the coarsest
// level down; at each level it finds the k-th largest key among the level's
// kept entries by an exact 8-bit radix select over the 64-bit keys, keeps
// the p children of the entries at or above it (a byte mask over the
// candidates) and continues with those children.  A coarsest entry's score
// is the maximum of its p children's, the same max-pool as the candidates'.
// The ordering kernels then read the mask instead of a threshold.
//
// Regional rule (lh_select LH_SELECT_REGIONAL, the pages' chunked top-K with
// every region contributing): one block per region of LH_REGION candidates
// holds the region's keys in shared memory, finds the key of rank quota =
// floor(Ksel * |region| / M) by the same radix select and marks the entries
// at or above it; with R = Ksel - (sum of quotas) > 0 it also writes its R
// best entries below that line to a list, and one block per (batch, head)
// then keeps the R best keys of all regions' lists.
//
// Grid-wide phases are separate launches, and the reduction that closes a
// phase runs in the last block to finish (an atomic ticket); no block ever
// waits for another.
#include <algorithm>

#include "host.h"

namespace lh {
namespace {

constexpr int kHistBins = 4096;
constexpr int kSelThreads = 512;
constexpr int kChunk = 8192;       // candidates per block in the histogram passes
constexpr int kOrdThreads = 256;
constexpr int kTokPerThread = 8;
constexpr int kTokBlock = kOrdThreads * kTokPerThread;  // tokens per order block

struct HeadState {
  uint32_t b1, need1;      // bucket of the top 12 score bits, rank left inside it
  uint32_t b2, need2;      // bucket of the next 12 bits, rank left inside it
  uint32_t list_count;     // candidates compacted for the final select
  uint32_t ticket1, ticket2, ticket3, ticket_count;
  uint32_t pad[3];
  unsigned long long kappa;
  unsigned long long pad2;
};
static_assert(sizeof(HeadState) == 64, "HeadState is 64 bytes");

constexpr int kDescThreads = 1024;
constexpr int kRegThreads = 512;

struct Layout {
  int64_t hist1, hist2, state, blockcnt, list, mask, keys, zero_bytes, total;
  int64_t cap;   // descent: keys per level list
  int64_t nreg;  // regional: regions of LH_REGION candidates
  int64_t rest;  // regional: budget left after the regions' quotas
};

// Regional rule: Ksel minus the sum over regions of floor(Ksel * |region| / M).
int64_t regional_rest(const lh_plan& p) {
  int64_t q = 0;
  for (int64_t a = 0; a < p.M; a += LH_REGION)
    q += p.Ksel * (std::min<int64_t>(p.M, a + LH_REGION) - a) / p.M;
  return p.Ksel - q;
}

int64_t align256(int64_t x) { return (x + 255) & ~int64_t(255); }

Layout layout(const lh_plan& p) {
  const int64_t BH = (int64_t)p.c.B * p.c.H;
  const int64_t nblk = (p.c.N + kTokBlock - 1) / kTokBlock;
  Layout l{};
  int64_t o = 0;
  l.hist1 = o; o += BH * kHistBins * 4;
  l.hist2 = o; o += BH * kHistBins * 4;
  l.state = o; o += BH * (int64_t)sizeof(HeadState);
  l.zero_bytes = o;
  o = align256(o);
  l.blockcnt = o; o = align256(o + BH * nblk * 4);
  l.list = o; o = align256(o + BH * p.M * 8);
  l.cap = l.nreg = l.rest = 0;
  l.mask = l.keys = o;
  if (p.c.select == LH_SELECT_DESCENT && p.c.L >= 2) {
    l.cap = std::max<int64_t>(p.n[p.c.L - 1], (int64_t)p.c.p * p.c.k);
    l.mask = o; o = align256(o + BH * p.M);
    l.keys = o; o = align256(o + BH * 2 * l.cap * 8);
  }
  if (p.c.select == LH_SELECT_REGIONAL && p.M > 0) {
    l.nreg = (p.M + LH_REGION - 1) / LH_REGION;
    l.rest = regional_rest(p);
    l.mask = o; o = align256(o + BH * p.M);
    l.keys = o; o = align256(o + BH * l.nreg * l.rest * 8);
  }
  l.total = o;
  return l;
}

__device__ __forceinline__ uint32_t orderable(float s) {
  if (s == 0.f) s = 0.f;  // -0 and +0 are the same score
  const uint32_t u = __float_as_uint(s);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ unsigned long long full_key(float s, int64_t f) {
  return ((unsigned long long)orderable(s) << 32) | (0xffffffffull - (unsigned long long)f);
}

// Exclusive scan of one value per thread over a block of NT threads.
template <int NT>
__device__ __forceinline__ uint32_t block_excl_scan(uint32_t v, uint32_t* warp_sums, uint32_t* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) warp_sums[warp] = x;
  __syncthreads();
  if (warp == 0) {
    constexpr int NW = NT / 32;
    uint32_t w = lane < NW ? warp_sums[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += y;
    }
    if (lane < NW) warp_sums[lane] = w;  // inclusive
  }
  __syncthreads();
  const uint32_t before = warp == 0 ? 0 : warp_sums[warp - 1];
  if (total) *total = warp_sums[NT / 32 - 1];
  const uint32_t r = before + x - v;
  __syncthreads();
  return r;
}

// Takes a ticket after this block's global writes; true in the last block.
__device__ __forceinline__ bool last_block(uint32_t* ticket, uint32_t nblocks) {
  __shared__ bool s_last;
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) s_last = atomicAdd(ticket, 1u) == nblocks - 1;
  __syncthreads();
  if (s_last) __threadfence();
  return s_last;
}

// In the last block: find the bucket where the rank `need` (1-based, from the
// top) falls in hist[0..4095]; returns bucket and the rank left inside it.
__device__ void find_bucket(const uint32_t* hist, uint32_t need, uint32_t* out_b, uint32_t* out_need) {
  __shared__ uint32_t warp_sums[kSelThreads / 32];
  constexpr int PER = kHistBins / kSelThreads;  // 8 bins per thread, descending
  const int t = threadIdx.x;
  // thread t owns bins [4096 - 8(t+1), 4096 - 8t), i.e. thread 0 the top bins
  const int hi = kHistBins - PER * t;
  uint32_t h[PER];
  uint32_t sum = 0;
#pragma unroll
  for (int i = 0; i < PER; ++i) {
    h[i] = __ldcg(hist + hi - 1 - i);
    sum += h[i];
  }
  const uint32_t above = block_excl_scan<kSelThreads>(sum, warp_sums, nullptr);
  if (above < need && need <= above + sum) {
    uint32_t cum = above;
#pragma unroll
    for (int i = 0; i < PER; ++i) {
      if (cum + h[i] >= need) {
        *out_b = hi - 1 - i;
        *out_need = need - cum;
        break;
      }
      cum += h[i];
    }
  }
}

__global__ void __launch_bounds__(kSelThreads)
hist1_kernel(Geo g, const float* __restrict__ scores, uint32_t* hist1, HeadState* state) {
  __shared__ uint32_t h[kHistBins];
  const int64_t bh = blockIdx.y;
  for (int i = threadIdx.x; i < kHistBins; i += kSelThreads) h[i] = 0;
  __syncthreads();
  const float* s = scores + bh * g.M;
  const int64_t f0 = (int64_t)blockIdx.x * kChunk;
  const int64_t f1 = min(g.M, f0 + kChunk);
  for (int64_t f = f0 + threadIdx.x; f < f1; f += kSelThreads) atomicAdd(&h[orderable(s[f]) >> 20], 1u);
  __syncthreads();
  uint32_t* gh = hist1 + bh * kHistBins;
  for (int i = threadIdx.x; i < kHistBins; i += kSelThreads)
    if (h[i]) atomicAdd(gh + i, h[i]);
  if (last_block(&state[bh].ticket1, gridDim.x))
    find_bucket(gh, (uint32_t)g.Ksel, &state[bh].b1, &state[bh].need1);
}

__global__ void __launch_bounds__(kSelThreads)
hist2_kernel(Geo g, const float* __restrict__ scores, uint32_t* hist2, HeadState* state) {
  __shared__ uint32_t h[kHistBins];
  const int64_t bh = blockIdx.y;
  for (int i = threadIdx.x; i < kHistBins; i += kSelThreads) h[i] = 0;
  __syncthreads();
  const uint32_t b1 = __ldcg(&state[bh].b1);
  const float* s = scores + bh * g.M;
  const int64_t f0 = (int64_t)blockIdx.x * kChunk;
  const int64_t f1 = min(g.M, f0 + kChunk);
  for (int64_t f = f0 + threadIdx.x; f < f1; f += kSelThreads) {
    const uint32_t k = orderable(s[f]);
    if ((k >> 20) == b1) atomicAdd(&h[(k >> 8) & 0xfffu], 1u);
  }
  __syncthreads();
  uint32_t* gh = hist2 + bh * kHistBins;
  for (int i = threadIdx.x; i < kHistBins; i += kSelThreads)
    if (h[i]) atomicAdd(gh + i, h[i]);
  if (last_block(&state[bh].ticket2, gridDim.x))
    find_bucket(gh, __ldcg(&state[bh].need1), &state[bh].b2, &state[bh].need2);
}

// Compacts the candidates of the threshold bucket (top 24 key bits fixed);
// the last block then resolves the remaining 8 score bits and the index by a
// radix select over 5 digits of 8 bits.
__global__ void __launch_bounds__(kSelThreads)
collect_kernel(Geo g, const float* __restrict__ scores, unsigned long long* list, HeadState* state) {
  const int64_t bh = blockIdx.y;
  HeadState* st = &state[bh];
  const uint32_t prefix = (__ldcg(&st->b1) << 12) | __ldcg(&st->b2);
  const float* s = scores + bh * g.M;
  unsigned long long* lst = list + bh * g.M;
  const int64_t f0 = (int64_t)blockIdx.x * kChunk;
  const int64_t f1 = min(g.M, f0 + kChunk);
  const int lane = threadIdx.x & 31;
  for (int64_t base = f0; base < f1; base += kSelThreads) {
    const int64_t f = base + threadIdx.x;
    bool hit = false;
    unsigned long long key = 0;
    if (f < f1) {
      key = full_key(s[f], f);
      hit = (uint32_t)(key >> 40) == prefix;
    }
    const uint32_t m = __ballot_sync(0xffffffffu, hit);
    if (m) {
      uint32_t pos = 0;
      if (lane == 0) pos = atomicAdd(&st->list_count, (uint32_t)__popc(m));
      pos = __shfl_sync(0xffffffffu, pos, 0);
      if (hit) lst[pos + __popc(m & ((1u << lane) - 1))] = key;
    }
  }
  if (!last_block(&st->ticket3, gridDim.x)) return;

  __shared__ uint32_t h[256];
  __shared__ uint32_t s_digit, s_need;
  __shared__ uint32_t warp_sums[kSelThreads / 32];
  const uint32_t cnt = __ldcg(&st->list_count);
  uint32_t need = __ldcg(&st->need2);
  unsigned long long rem = 0;        // resolved low 40 bits so far
  unsigned long long rem_mask = 0;   // which of them are resolved
  for (int shift = 32; shift >= 0; shift -= 8) {
    for (int i = threadIdx.x; i < 256; i += kSelThreads) h[i] = 0;
    __syncthreads();
    for (uint32_t i = threadIdx.x; i < cnt; i += kSelThreads) {
      const unsigned long long k = __ldcg(lst + i) & 0xffffffffffull;
      if ((k & rem_mask) == rem) atomicAdd(&h[(k >> shift) & 0xffu], 1u);
    }
    __syncthreads();
    // descending scan over 256 bins: thread t < 256 takes bin 255 - t
    const int t = threadIdx.x;
    const uint32_t v = t < 256 ? h[255 - t] : 0;
    const uint32_t above = block_excl_scan<kSelThreads>(v, warp_sums, nullptr);
    if (t < 256 && above < need && need <= above + v) {
      s_digit = 255 - t;
      s_need = need - above;
    }
    __syncthreads();
    rem |= (unsigned long long)s_digit << shift;
    rem_mask |= 0xffull << shift;
    need = s_need;
    __syncthreads();
  }
  if (threadIdx.x == 0) st->kappa = ((unsigned long long)prefix << 40) | rem;
}

// --- hierarchical descent ----------------------------------------------------

// The k-th largest of n unique keys (1 <= k <= n), by eight 8-bit radix passes
// over the keys from the most significant digit.  Whole block of NT threads.
template <int NT>
__device__ unsigned long long block_kth_largest(const unsigned long long* keys, int64_t n, uint32_t k,
                                                uint32_t* h, uint32_t* warp_sums, uint32_t* s_digit,
                                                uint32_t* s_need) {
  static_assert(NT >= 256, "one thread per digit bin");
  unsigned long long prefix = 0, pmask = 0;
  uint32_t need = k;
  for (int shift = 56; shift >= 0; shift -= 8) {
    for (int i = threadIdx.x; i < 256; i += NT) h[i] = 0;
    __syncthreads();
    for (int64_t j = threadIdx.x; j < n; j += NT) {
      const unsigned long long key = keys[j];
      if ((key & pmask) == prefix) atomicAdd(&h[(key >> shift) & 0xffu], 1u);
    }
    __syncthreads();
    const int t = threadIdx.x;
    const uint32_t v = t < 256 ? h[255 - t] : 0;  // descending digits
    const uint32_t above = block_excl_scan<NT>(v, warp_sums, nullptr);
    if (t < 256 && above < need && need <= above + v) {
      *s_digit = 255 - t;
      *s_need = need - above;
    }
    __syncthreads();
    prefix |= (unsigned long long)*s_digit << shift;
    pmask |= 0xffull << shift;
    need = *s_need;
    __syncthreads();
  }
  return prefix;
}

__global__ void __launch_bounds__(kDescThreads)
descent_kernel(Geo g, const float* __restrict__ scores, uint8_t* __restrict__ mask,
               unsigned long long* __restrict__ keys, int64_t cap) {
  __shared__ uint32_t h[256];
  __shared__ uint32_t warp_sums[kDescThreads / 32];
  __shared__ uint32_t s_digit, s_need;
  const int64_t bh = blockIdx.x;
  const float* s = scores + bh * g.M;
  uint8_t* msk = mask + bh * g.M;
  unsigned long long* cur = keys + bh * 2 * cap;
  unsigned long long* nxt = cur + cap;
  const int L = g.L, p = g.p;
  const uint32_t k = (uint32_t)g.k;
  // the coarsest level: score = max over the p children (level L-2)
  int64_t n = g.n[L - 1];
  for (int64_t i = threadIdx.x; i < n; i += kDescThreads) {
    const float* c = s + g.flat_off[L - 2] + i * p;
    float m = c[0];
    for (int j = 1; j < p; ++j) m = fmaxf(m, c[j]);
    cur[i] = full_key(m, g.flat_off[L - 1] + i);
  }
  __syncthreads();
  for (int l = L - 1; l >= 1; --l) {
    const unsigned long long kappa =
        block_kth_largest<kDescThreads>(cur, n, k, h, warp_sums, &s_digit, &s_need);
    // keep the p children of every entry at or above kappa (exactly k of them)
    uint32_t base = 0;
    for (int64_t j0 = 0; j0 < n; j0 += kDescThreads) {
      const int64_t j = j0 + threadIdx.x;
      const unsigned long long key = j < n ? cur[j] : 0ull;
      const bool keep = j < n && key >= kappa;
      uint32_t total;
      const uint32_t pos = base + block_excl_scan<kDescThreads>(keep ? 1u : 0u, warp_sums, &total);
      if (keep) {
        const int64_t f = 0xffffffffll - (int64_t)(key & 0xffffffffull);  // flat index at level l
        const int64_t i = f - g.flat_off[l];
        for (int c = 0; c < p; ++c) {
          const int64_t child = g.flat_off[l - 1] + i * p + c;
          msk[child] = 1;
          if (l - 1 >= 1 && pos < k) nxt[(int64_t)pos * p + c] = full_key(s[child], child);
        }
      }
      base += total;
    }
    __syncthreads();
    unsigned long long* t = cur;
    cur = nxt;
    nxt = t;
    n = (int64_t)p * k;
  }
}

// --- regional rule -----------------------------------------------------------

// One block per (region, head): the region's quota of best entries into the
// mask (every candidate byte of the region is written), and with rest > 0
// the region's `rest` best entries below the quota line into its list slot
// (zero keys pad a short list; every real key is larger).
__global__ void __launch_bounds__(kRegThreads)
regional_kernel(Geo g, const float* __restrict__ scores, uint8_t* __restrict__ mask,
                unsigned long long* __restrict__ rest_list, int64_t rest) {
  __shared__ unsigned long long keys[LH_REGION];
  __shared__ uint32_t h[256];
  __shared__ uint32_t warp_sums[kRegThreads / 32];
  __shared__ uint32_t s_digit, s_need;
  const int64_t bh = blockIdx.y;
  const int64_t a = (int64_t)blockIdx.x * LH_REGION;
  const int64_t b = min(g.M, a + (int64_t)LH_REGION);
  const int n = (int)(b - a);
  const float* s = scores + bh * g.M;
  for (int i = threadIdx.x; i < n; i += kRegThreads) keys[i] = full_key(s[a + i], a + i);
  __syncthreads();
  const uint32_t quota = (uint32_t)(g.Ksel * (b - a) / g.M);
  unsigned long long kappa = 0;
  if (quota > 0) kappa = block_kth_largest<kRegThreads>(keys, n, quota, h, warp_sums, &s_digit, &s_need);
  uint8_t* msk = mask + bh * g.M + a;
  for (int i = threadIdx.x; i < n; i += kRegThreads) msk[i] = (quota > 0 && keys[i] >= kappa) ? 1 : 0;
  if (rest <= 0) return;
  unsigned long long* out = rest_list + (bh * gridDim.x + blockIdx.x) * rest;
  const uint32_t extra = (uint32_t)(rest < (int64_t)n - quota ? rest : (int64_t)n - quota);
  if (extra > 0) {
    const unsigned long long kappa2 =
        block_kth_largest<kRegThreads>(keys, n, quota + extra, h, warp_sums, &s_digit, &s_need);
    uint32_t base = 0;
    for (int i0 = 0; i0 < n; i0 += kRegThreads) {
      const int i = i0 + threadIdx.x;
      const unsigned long long key = i < n ? keys[i] : 0ull;
      const bool left = i < n && key >= kappa2 && !(quota > 0 && key >= kappa);
      uint32_t total;
      const uint32_t pos = base + block_excl_scan<kRegThreads>(left ? 1u : 0u, warp_sums, &total);
      if (left && pos < extra) out[pos] = key;
      base += total;
    }
  }
  for (int64_t i = extra + threadIdx.x; i < rest; i += kRegThreads) out[i] = 0ull;
}

// One block per (batch, head): the `rest` best keys of all regions' lists
// join the mask.
__global__ void __launch_bounds__(kDescThreads)
regional_rest_kernel(Geo g, uint8_t* __restrict__ mask, const unsigned long long* __restrict__ rest_list,
                     int64_t nreg, int64_t rest) {
  __shared__ uint32_t h[256];
  __shared__ uint32_t warp_sums[kDescThreads / 32];
  __shared__ uint32_t s_digit, s_need;
  const int64_t bh = blockIdx.x;
  const int64_t n = nreg * rest;
  const unsigned long long* lst = rest_list + bh * n;
  const unsigned long long kth =
      block_kth_largest<kDescThreads>(lst, n, (uint32_t)rest, h, warp_sums, &s_digit, &s_need);
  uint8_t* msk = mask + bh * g.M;
  for (int64_t i = threadIdx.x; i < n; i += kDescThreads) {
    const unsigned long long key = lst[i];
    if (key != 0ull && key >= kth) {
      const int64_t f = 0xffffffffll - (int64_t)(key & 0xffffffffull);
      if (f >= 0 && f < g.M) msk[f] = 1;
    }
  }
}

// --- ordering -------------------------------------------------------------

struct SelCtx {
  const float* s;      // this head's candidate scores
  const uint8_t* msk;  // descent: this head's candidate mask (else null)
  unsigned long long kappa;
  bool any;            // Ksel > 0
};

__device__ __forceinline__ bool is_selected(const Geo& g, const SelCtx& c, int l, int64_t i) {
  if (l == g.L - 1) return true;
  if (!c.any) return false;
  const int64_t f = g.flat_off[l] + i;
  if (c.msk) return c.msk[f] != 0;
  return full_key(c.s[f], f) >= c.kappa;
}

// Number of selected entries whose span ends at tokens [t0, t1).
__device__ __forceinline__ uint32_t count_range(const Geo& g, const SelCtx& c, int64_t t0, int64_t t1) {
  uint32_t n = 0;
  for (int64_t t = t0; t < t1; ++t) {
    for (int l = 0; l < g.L; ++l) {
      const int sh = g.logp * l;  // p^l = 2^sh
      if (((t + 1) & ((int64_t(1) << sh) - 1)) != 0) break;  // coarser levels fail too
      n += is_selected(g, c, l, ((t + 1) >> sh) - 1);
    }
  }
  return n;
}

__global__ void __launch_bounds__(kOrdThreads)
order_count_kernel(Geo g, const float* __restrict__ scores, const uint8_t* __restrict__ mask,
                   const HeadState* state, uint32_t* blockcnt, HeadState* wstate, int64_t nblk) {
  __shared__ uint32_t warp_sums[kOrdThreads / 32];
  const int64_t bh = blockIdx.y;
  SelCtx c{scores + bh * g.M, mask ? mask + bh * g.M : nullptr, state[bh].kappa, g.Ksel > 0};
  const int64_t t0 = (int64_t)blockIdx.x * kTokBlock + threadIdx.x * kTokPerThread;
  const int64_t t1 = min(g.N, t0 + kTokPerThread);
  const uint32_t mine = t0 < g.N ? count_range(g, c, t0, t1) : 0;
  uint32_t total;
  block_excl_scan<kOrdThreads>(mine, warp_sums, &total);
  uint32_t* bc = blockcnt + bh * nblk;
  if (threadIdx.x == 0) bc[blockIdx.x] = total;
  if (!last_block(&wstate[bh].ticket_count, gridDim.x)) return;
  // Exclusive scan of the block counts, in place.
  uint32_t carry = 0;
  for (int64_t base = 0; base < nblk; base += kOrdThreads) {
    const int64_t i = base + threadIdx.x;
    const uint32_t v = i < nblk ? __ldcg(bc + i) : 0;
    uint32_t tot;
    const uint32_t ex = block_excl_scan<kOrdThreads>(v, warp_sums, &tot);
    if (i < nblk) bc[i] = carry + ex;
    carry += tot;
  }
}

__global__ void __launch_bounds__(kOrdThreads)
order_write_kernel(Geo g, const float* __restrict__ scores, const uint8_t* __restrict__ mask,
                   const HeadState* state, const uint32_t* blockoff, int32_t* __restrict__ sel_idx,
                   int32_t* __restrict__ slot_of, int64_t nblk) {
  __shared__ uint32_t warp_sums[kOrdThreads / 32];
  const int64_t bh = blockIdx.y;
  SelCtx c{scores + bh * g.M, mask ? mask + bh * g.M : nullptr, state[bh].kappa, g.Ksel > 0};
  const int64_t t0 = (int64_t)blockIdx.x * kTokBlock + threadIdx.x * kTokPerThread;
  const int64_t t1 = min(g.N, t0 + kTokPerThread);
  const uint32_t mine = t0 < g.N ? count_range(g, c, t0, t1) : 0;
  uint32_t slot = blockoff[bh * nblk + blockIdx.x] +
                  block_excl_scan<kOrdThreads>(mine, warp_sums, nullptr);
  int32_t* sel = sel_idx + bh * g.S;
  int32_t* inv = slot_of + bh * g.Ntot;
  for (int64_t t = t0; t < t1; ++t) {
    for (int l = 0; l < g.L; ++l) {
      const int sh = g.logp * l;
      if (((t + 1) & ((int64_t(1) << sh) - 1)) != 0) break;
      const int64_t i = ((t + 1) >> sh) - 1;
      const int64_t f = g.flat_off[l] + i;
      if (is_selected(g, c, l, i)) {
        // slot < S holds whenever exactly Ksel candidates pass; the guard
        // keeps a wrong threshold from writing past the buffer.
        if (slot < g.S) sel[slot] = (int32_t)f;
        inv[f] = slot < g.S ? (int32_t)slot : -1;
        ++slot;
      } else {
        inv[f] = -1;
      }
    }
  }
}

}  // namespace

int64_t topk_ws_bytes(const lh_plan& plan) { return layout(plan).total; }

cudaError_t launch_topk(const lh_plan& plan, const float* scores, int32_t* sel_idx,
                        int32_t* slot_of, void* ws, cudaStream_t st) {
  const Geo g = make_geo(plan);
  const Layout lay = layout(plan);
  char* w = static_cast<char*>(ws);
  uint32_t* hist1 = reinterpret_cast<uint32_t*>(w + lay.hist1);
  uint32_t* hist2 = reinterpret_cast<uint32_t*>(w + lay.hist2);
  HeadState* state = reinterpret_cast<HeadState*>(w + lay.state);
  uint32_t* blockcnt = reinterpret_cast<uint32_t*>(w + lay.blockcnt);
  unsigned long long* list = reinterpret_cast<unsigned long long*>(w + lay.list);
  const int64_t nblk = (g.N + kTokBlock - 1) / kTokBlock;

  cudaError_t e = cudaMemsetAsync(w, 0, lay.zero_bytes, st);
  if (e != cudaSuccess) return e;
  const bool descent = g.select == LH_SELECT_DESCENT && g.Ksel > 0;
  const bool regional = g.select == LH_SELECT_REGIONAL && g.Ksel > 0;
  uint8_t* mask = (descent || regional) ? reinterpret_cast<uint8_t*>(w + lay.mask) : nullptr;
  if (regional) {
    // every candidate's mask byte is written by its region's block
    unsigned long long* rl = reinterpret_cast<unsigned long long*>(w + lay.keys);
    regional_kernel<<<dim3((unsigned)lay.nreg, (unsigned)g.BH), kRegThreads, 0, st>>>(g, scores, mask, rl,
                                                                                     lay.rest);
    if (lay.rest > 0)
      regional_rest_kernel<<<(unsigned)g.BH, kDescThreads, 0, st>>>(g, mask, rl, lay.nreg, lay.rest);
  } else if (descent) {
    e = cudaMemsetAsync(mask, 0, (size_t)(g.BH * g.M), st);
    if (e != cudaSuccess) return e;
    descent_kernel<<<(unsigned)g.BH, kDescThreads, 0, st>>>(
        g, scores, mask, reinterpret_cast<unsigned long long*>(w + lay.keys), lay.cap);
  } else if (g.Ksel > 0) {
    const dim3 grid((unsigned)((g.M + kChunk - 1) / kChunk), (unsigned)g.BH);
    hist1_kernel<<<grid, kSelThreads, 0, st>>>(g, scores, hist1, state);
    hist2_kernel<<<grid, kSelThreads, 0, st>>>(g, scores, hist2, state);
    collect_kernel<<<grid, kSelThreads, 0, st>>>(g, scores, list, state);
  }
  const dim3 ogrid((unsigned)nblk, (unsigned)g.BH);
  order_count_kernel<<<ogrid, kOrdThreads, 0, st>>>(g, scores, mask, state, blockcnt, state, nblk);
  order_write_kernel<<<ogrid, kOrdThreads, 0, st>>>(g, scores, mask, state, blockcnt, sel_idx, slot_of,
                                                    nblk);
  return cudaGetLastError();
}

}  // namespace lh
