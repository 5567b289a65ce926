/*
 * lh.h -- C ABI of the Lighthouse Attention layer for NVIDIA B200 (sm_100a).
 *
 * Lighthouse Attention is a training-time wrapper around causal scaled
 * dot-product attention for one layer's Q, K, V of shape [B, H, N, d]
 * (skill card "lighthouse-attention", skillsmp.com, "四阶段 Pipeline";
 * gist.science "Long Context Pre-Training with Lighthouse Attention",
 * Technical Summary section 2).  Its four stages are
 *   1. a symmetric average-pool pyramid of Q, K and V       (lh_pyramid),
 *   2. parameter-free l2-norm scores and a top-K selection  (lh_score, lh_topk),
 *   3. a gather into a causally ordered sub-sequence of length
 *      S = N/p^(L-1) + (L-1)*p*k and dense S x S causal attention
 *                                                            (lh_gather, lh_attn_fwd),
 *   4. a scatter-back of each level-l output to R(l, i) = [i p^l + p^l - 1,
 *      i p^l + 2 p^l - 2], summed over levels                (lh_scatter),
 * and gradients flow back through scatter, attention and gather
 * (skill card, "梯度流"; lh_scatter_bwd, lh_attn_bwd, lh_gather_bwd).
 * lh_forward / lh_backward run the whole layer.
 *
 * Conventions for every call:
 *  - All tensors are dense row-major ("BHND": batch, head, token, channel),
 *    live in device memory, and are allocated and owned by the caller.  The
 *    library allocates no device memory and never synchronises the stream.
 *  - Device pointers must be 16-byte aligned.
 *  - dtype: LH_F32 or LH_BF16; d = 64.  Gradients and outputs have the input
 *    dtype.  Scores and LSE are fp32; indices are int32.
 *  - Every call validates its arguments before enqueuing anything.  On a
 *    validation failure it returns LH_ERR_INVALID_ARG / LH_ERR_UNSUPPORTED /
 *    LH_ERR_WORKSPACE and enqueues nothing.  If a launch fails it returns
 *    LH_ERR_CUDA.  lh_last_error() gives a one-line reason (thread-local).
 *  - Work is enqueued on `stream` (a cudaStream_t; 0 = the legacy default
 *    stream) and is asynchronous.  Calls are re-entrant given distinct
 *    output, ctx and workspace buffers.
 *  - Inputs must be finite; non-finite scores give an unspecified selection.
 *
 * Readings of points the pages leave open (fixed by this library):
 *  - score of level-0 token t: ||Q_t||_2 + ||K_t||_2, computed in fp64 and
 *    rounded to fp32; coarser levels take the max over their span
 *    (gist.science Technical Summary 2.B: a coarse entry takes the largest
    score of the tokens it pools).
 *  - the budget: (L-1)*p*k entries chosen jointly from levels 0..L-2 by
 *    score, ties to the lower level-major flat index; the coarsest level is
 *    always kept in full (skill card, "阶段 2").
 *  - gathered order: by the last token of the span, then by level (finer
 *    first); the sub-sequence runs under a plain S x S causal mask.
 *  - scatter ranges are clipped to N-1; positions no entry reaches are 0.
 *  - selection is independent per (batch, head).
 */
#ifndef LH_H_
#define LH_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define LH_MAX_LEVELS 8

typedef struct CUstream_st* lh_stream_t; /* = cudaStream_t */

typedef enum {
  LH_OK = 0,
  LH_ERR_INVALID_ARG = 1,  /* bad size, null or misaligned pointer */
  LH_ERR_UNSUPPORTED = 2,  /* valid for the method, not built here (d, p, L, dtype) */
  LH_ERR_WORKSPACE = 3,    /* ctx or workspace smaller than the plan needs */
  LH_ERR_CUDA = 4,         /* a CUDA runtime call or launch failed */
  LH_ERR_TIMEOUT = 5       /* a device-side wait gave up (see lh_device_status) */
} lh_status;

typedef enum { LH_F32 = 0, LH_BF16 = 1 } lh_dtype;

/* Layer shape and hyperparameters.  p: pooling factor, L: pyramid levels
 * (level 0 = tokens), k: per-level budget unit, so (L-1)*p*k entries are
 * selected (skill card, "阶段 3").  The method needs N to be a multiple of
 * p^(L-1).  Built here: d in {64, 128}, p in {2, 4}, 1 <= L <= 5,
 * p^(L-1) <= 256. */
/* Selection rule for the (L-1)*p*k budget (lh_config.select):
 *  LH_SELECT_JOINT   one top-K of (L-1)*p*k over all candidate levels
 *                    0..L-2 (the default reading);
 *  LH_SELECT_DESCENT hierarchical descent: from the coarsest level down, the
 *                    k best entries of a level keep their p children one
 *                    level down (p*k per finer level); needs k <= n[L-1];
 *  LH_SELECT_REGIONAL every region contributes (skill card "Kernel Design",
 *                    chunked top-K): the M candidates, level-major, in
 *                    regions of LH_REGION consecutive entries (the last one
 *                    shorter); region c keeps its floor(Ksel*|c|/M) best and
 *                    the remaining budget goes to the best entries left.
 * All keep every coarsest-level entry and break ties to the lower
 * level-major flat index (skill card "阶段 2", "阶段 3"). */
typedef enum { LH_SELECT_JOINT = 0, LH_SELECT_DESCENT = 1, LH_SELECT_REGIONAL = 2 } lh_select;
#define LH_REGION 2048

typedef struct {
  int32_t B, H, N, d, p, L, k;
  int32_t dtype;  /* lh_dtype */
  int32_t select; /* lh_select */
} lh_config;

/* Sizes and buffer layout derived from a config by lh_plan_init.
 * P[l] = p^l tokens per level-l entry, n[l] = N / P[l] entries.
 * Flat index: level-major over all L levels, f = flat_off[l] + i.
 * Candidates are levels 0..L-2 (M = flat_off[L-1] of them); Ksel of them are
 * selected; S = n[L-1] + Ksel.  pyr_off[l] is the row offset of level l
 * (l >= 1) inside the per-head pyramid buffer of Npyr = Ntot - N rows. */
typedef struct {
  lh_config c;
  int64_t P[LH_MAX_LEVELS];
  int64_t n[LH_MAX_LEVELS];
  int64_t flat_off[LH_MAX_LEVELS + 1];
  int64_t pyr_off[LH_MAX_LEVELS];
  int64_t Ntot, Npyr, M, Ksel, S;
  int64_t elem_bytes;
  /* Bytes of the caller-owned buffers: ctx (written by lh_forward, read by
   * lh_backward), ws (scratch of lh_forward and lh_backward), topk_ws
   * (scratch of lh_topk), attn_bwd_ws (scratch of lh_attn_bwd at this S). */
  int64_t ctx_bytes, ws_bytes, topk_ws_bytes, attn_bwd_ws_bytes;
  /* Byte offsets inside ctx. */
  int64_t ctx_sel_idx, ctx_slot_of, ctx_Qg, ctx_Kg, ctx_Vg, ctx_Og, ctx_lse;
  /* Byte offsets inside ws (forward use). */
  int64_t ws_pyrQ, ws_pyrK, ws_pyrV, ws_scores, ws_topk;
  /* Byte offsets inside ws (backward use; overlaps the forward part). */
  int64_t ws_dOg, ws_D, ws_dQg, ws_dKg, ws_dVg, ws_attn;
} lh_plan;

/* Fill *out from *cfg.  Host only, enqueues nothing.  Returns
 * LH_ERR_INVALID_ARG when the method itself is undefined for the config
 * (N % p^(L-1) != 0, L < 1, p < 2, k < 0, (L-1)*p*k > M, S >= 2^31, an
 * unknown select, descent with k > n[L-1]) and LH_ERR_UNSUPPORTED for
 * shapes this build does not implement (d != 64, p not in {2, 4}, L > 5,
 * p^(L-1) > 256, B*H > 65535, bf16 with B*H*S >= 2^31). */
lh_status lh_plan_init(const lh_config* cfg, lh_plan* out);

/* Stage 1 (skill card "阶段 1"; gist.science 2.A).  Writes pyramid levels
 * 1..L-1 of Q, K and V: level l entry i = mean of tokens [i p^l, (i+1) p^l),
 * accumulated in fp32 and rounded once.  Q, K, V: [B,H,N,d].  pyrQ, pyrK,
 * pyrV: [B,H,Npyr,d], level l at row offset pyr_off[l]. */
lh_status lh_pyramid(const lh_plan* plan, const void* Q, const void* K, const void* V,
                     void* pyrQ, void* pyrK, void* pyrV, lh_stream_t stream);

/* Stage 2, scores (skill card "阶段 2"; gist.science 2.B).  scores:
 * [B,H,M] fp32, level-major over levels 0..L-2: level 0 holds
 * fp32(||Q_t|| + ||K_t||) (fp64 arithmetic), level l the max over its span. */
lh_status lh_score(const lh_plan* plan, const void* Q, const void* K, float* scores,
                   lh_stream_t stream);

/* Stages 1 and 2 fused: one pass over Q, K and V writes the pyramid and the
 * scores (same outputs as lh_pyramid followed by lh_score). */
lh_status lh_pyramid_score(const lh_plan* plan, const void* Q, const void* K, const void* V,
                           void* pyrQ, void* pyrK, void* pyrV, float* scores,
                           lh_stream_t stream);

/* Stage 2, selection and order (skill card "阶段 2", "阶段 3"; gist.science
 * 2.B-C).  From scores [B,H,M] selects, per (b,h), Ksel candidates by the
 * plan's rule -- LH_SELECT_JOINT: the Ksel largest by (score desc, flat index
 * asc); LH_SELECT_DESCENT: the p children of the k best entries of each
 * level, from the coarsest down, a coarsest entry scoring the max of its p
 * children; LH_SELECT_REGIONAL: each region's quota of its best entries,
 * then the best of the rest -- adds every level-(L-1) entry, and orders them by (span end,
 * level).  sel_idx: [B,H,S] int32 flat indices in gathered order.  slot_of:
 * [B,H,Ntot] int32, the slot of each pyramid entry or -1.  ws:
 * plan->topk_ws_bytes of scratch (contents on entry are ignored). */
lh_status lh_topk(const lh_plan* plan, const float* scores, int32_t* sel_idx, int32_t* slot_of,
                  void* ws, size_t ws_bytes, lh_stream_t stream);

/* Stage 3, gather: Xg[b,h,j] = level l_j entry i_j of X (X in Q, K, V), where
 * sel_idx[b,h,j] = flat_off[l_j] + i_j.  Level 0 is read from Q/K/V, levels
 * >= 1 from the pyramid buffers.  Qg, Kg, Vg: [B,H,S,d]. */
lh_status lh_gather(const lh_plan* plan, const void* Q, const void* K, const void* V,
                    const void* pyrQ, const void* pyrK, const void* pyrV,
                    const int32_t* sel_idx, void* Qg, void* Kg, void* Vg, lh_stream_t stream);

/* Stage 3, dense causal attention on the gathered sub-sequence (skill card
 * "阶段 3": a standard S x S causal mask).  BH independent problems of
 * [S, d]: Og = softmax(Qg Kg^T / sqrt(d) + causal) Vg, lse = natural-log
 * row log-sum-exp [BH, S] fp32.  With S = N and ungathered inputs this is
 * dense causal attention, the layer's L = 1 fixed point. */
lh_status lh_attn_fwd(int64_t BH, int64_t S, int32_t d, int32_t dtype, const void* Qg,
                      const void* Kg, const void* Vg, void* Og, float* lse, lh_stream_t stream);

/* Bytes of scratch lh_attn_bwd needs for BH problems of length S: the row
 * term D (BH * S floats) and, for bf16, an fp32 dQ accumulator (BH * S * d
 * floats), each rounded up to 256 bytes. */
int64_t lh_attn_bwd_ws_bytes(int64_t BH, int64_t S, int32_t d, int32_t dtype);

/* Gradients of lh_attn_fwd.  D: [BH, S] fp32 rowsum(dOg * Og), or NULL, in
 * which case it is computed into ws from Og and dOg.  Writes dQg, dKg, dVg
 * [BH, S, d].  ws: lh_attn_bwd_ws_bytes() bytes.
 * bf16 runs one fused kernel by default: each key tile's share of dQg is
 * added into an fp32 accumulator in ws with TMA bulk reduce-adds, whose order
 * varies, so the last bits of dQg may differ between runs (dKg and dVg are
 * bit-reproducible).  lh_set_deterministic(1) selects a two-kernel schedule
 * without reductions (dK/dV, then dQ per query tile; bit-reproducible and
 * slower: 1.5-1.6x the fused time at BH * S = 16 * 18432), as does
 * lh_attn_bwd_static. */
lh_status lh_attn_bwd(int64_t BH, int64_t S, int32_t d, int32_t dtype, const void* Qg,
                      const void* Kg, const void* Vg, const void* Og, const float* lse,
                      const void* dOg, const float* D, void* dQg, void* dKg, void* dVg,
                      void* ws, size_t ws_bytes, lh_stream_t stream);

/* Allocation-free variant of lh_attn_bwd (the paper has no counterpart; it
 * exists for callers, not for the method).  Some callers hold only their
 * input and output buffers and cannot allocate device memory: a kernel
 * plug-in running inside another framework's engine with no allocator
 * handle, or code on a path where a device allocation is not permitted.
 * This entry point needs no workspace: the row term D = rowsum(dOg * Og) goes
 * to a scratch array of LH_ATTN_BWD_STATIC_MAX_ROWS floats (4 MiB) compiled
 * into the library, which every GPU that loads the library keeps until the
 * process exits.  Same arguments and results as lh_attn_bwd with D = NULL.
 *  - BH * S above LH_ATTN_BWD_STATIC_MAX_ROWS returns LH_ERR_WORKSPACE and
 *    enqueues nothing.
 *  - Every call looks up the array's device address in the current context
 *    (a host-side call that enqueues nothing).
 *  - All calls share the one array and it keeps the last call's contents:
 *    calls whose work overlaps on the GPU (other streams, other threads) race
 *    on it and must be serialised by the caller.
 *  - Allocates nothing: no cudaMalloc, no cudaFree, no allocating library
 *    call. */
#define LH_ATTN_BWD_STATIC_MAX_ROWS (1 << 20)
/* Process-wide switch for lh_attn_bwd and lh_backward: on != 0 makes every
 * later bf16 attention backward bit-reproducible (two kernels, no atomics);
 * 0 (the default) restores the fused kernel.  Affects work enqueued after
 * the call only; thread-safe. */
void lh_set_deterministic(int on);

lh_status lh_attn_bwd_static(int64_t BH, int64_t S, int32_t d, int32_t dtype, const void* Qg,
                             const void* Kg, const void* Vg, const void* Og, const float* lse,
                             const void* dOg, void* dQg, void* dKg, void* dVg, lh_stream_t stream);

/* Stage 4 (skill card "阶段 4"; gist.science 2.C: a deterministic scatter).
 * O[t] = sum over levels l (ascending) of Og[slot_of(l, floor((t+1)/p^l) - 1)]
 * where that index is >= 0 and selected; fp32 sum rounded once; 0 where no
 * entry reaches t.  O: [B,H,N,d].  No atomics. */
lh_status lh_scatter(const lh_plan* plan, const void* Og, const int32_t* slot_of, void* O,
                     lh_stream_t stream);

/* Backward of stage 4: dOg[j] = sum of dO over R(l_j, i_j) clipped to N-1,
 * rounded to the dtype; D[j] = sum_c dOg[j,c] * Og[j,c] in fp32 (the
 * softmax-backward row term).  dOg: [B,H,S,d], D: [B,H,S]. */
lh_status lh_scatter_bwd(const lh_plan* plan, const void* dO, const void* Og,
                         const int32_t* sel_idx, void* dOg, float* D, lh_stream_t stream);

/* Backward of stages 1 and 3 (gather of the pooled pyramid):
 * dX[t] = sum over levels l (ascending) of dXg[slot_of(l, t / p^l)] / p^l over
 * selected entries, fp32, rounded once.  Scores and top-K get no gradient
 * (skill card, "梯度流"). */
lh_status lh_gather_bwd(const lh_plan* plan, const void* dQg, const void* dKg, const void* dVg,
                        const int32_t* slot_of, void* dQ, void* dK, void* dV, lh_stream_t stream);

/* Whole forward: O = layer(Q, K, V).  ctx (kept for lh_backward) and ws
 * (scratch) are caller-owned device buffers of ctx_bytes and ws_bytes bytes;
 * fewer than plan->ctx_bytes or plan->ws_bytes returns LH_ERR_WORKSPACE and
 * enqueues nothing. */
lh_status lh_forward(const lh_plan* plan, const void* Q, const void* K, const void* V, void* O,
                     void* ctx, size_t ctx_bytes, void* ws, size_t ws_bytes, lh_stream_t stream);

/* Whole backward from the ctx of the matching lh_forward: dQ, dK, dV
 * [B,H,N,d] from dO.  ctx_bytes, ws_bytes: the buffers' sizes, checked as in
 * lh_forward. */
lh_status lh_backward(const lh_plan* plan, const void* dO, const void* ctx, size_t ctx_bytes,
                      void* dQ, void* dK, void* dV, void* ws, size_t ws_bytes,
                      lh_stream_t stream);

/* Device-side status word: LH_OK, or LH_ERR_TIMEOUT if a bounded wait inside
 * a kernel gave up since the last reset.  Synchronises the current device;
 * reset != 0 clears the word. */
lh_status lh_device_status(int reset);

/* Self-test of that failure path: enqueues one CTA that waits, through the
 * same bounded mbarrier wait as the attention kernels, on a barrier nothing
 * signals.  The wait gives up after its budget (about 2 s at full SM clock),
 * the kernel returns normally and the next lh_device_status reports
 * LH_ERR_TIMEOUT; the CUDA context stays usable.  Returns LH_ERR_CUDA only if
 * the launch fails. */
lh_status lh_selftest_wait_timeout(lh_stream_t stream);

const char* lh_status_string(lh_status s);
const char* lh_last_error(void);

/* sizeof(lh_plan) as compiled into the library, for bindings to check their
 * mirror of the struct. */
int64_t lh_plan_bytes(void);

#ifdef __cplusplus
}
#endif

#endif /* LH_H_ */
