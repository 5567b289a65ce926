// C-ABI entry points of the Lighthouse layer: validation, buffer layout and
// the stage order of the whole forward and backward pass.
#include <cuda_runtime.h>
#include <stdio.h>

#include <string>

#include "host.h"

namespace lh {

// Device status word (LH_OK or LH_ERR_TIMEOUT); kernels with bounded waits
// receive its address from device_status_ptr().
static __device__ unsigned int g_device_status = 0;

unsigned int* device_status_ptr() {
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_device_status) != cudaSuccess) return nullptr;
  return static_cast<unsigned int*>(p);
}

static thread_local std::string t_last_error;

lh_status fail(lh_status s, const std::string& why) {
  t_last_error = why;
  return s;
}
lh_status ok() {
  t_last_error.clear();
  return LH_OK;
}
lh_status cuda_status(cudaError_t e, const char* where) {
  if (e == cudaSuccess) return LH_OK;
  return fail(LH_ERR_CUDA, std::string(where) + ": " + cudaGetErrorString(e));
}

bool aligned16(const void* ptr) {
  return ptr != nullptr && (reinterpret_cast<uintptr_t>(ptr) & 15u) == 0;
}

Geo make_geo(const lh_plan& p) {
  Geo g{};
  g.BH = (int64_t)p.c.B * p.c.H;
  g.N = p.c.N;
  g.S = p.S;
  g.Ntot = p.Ntot;
  g.Npyr = p.Npyr;
  g.M = p.M;
  g.Ksel = p.Ksel;
  g.L = p.c.L;
  g.p = p.c.p;
  g.logp = p.c.p == 2 ? 1 : 2;
  g.k = p.c.k;
  g.select = p.c.select;
  for (int l = 0; l < LH_MAX_LEVELS; ++l) {
    g.n[l] = p.n[l];
    g.pyr_off[l] = p.pyr_off[l];
  }
  for (int l = 0; l <= LH_MAX_LEVELS; ++l) g.flat_off[l] = p.flat_off[l];
  return g;
}

static int64_t align256(int64_t x) { return (x + 255) & ~int64_t(255); }

int64_t attn_bwd_ws_bytes(int64_t BH, int64_t S, int d, int dtype);

}  // namespace lh

using namespace lh;

lh_status lh::check_attn(int64_t BH, int64_t S, int32_t d, int32_t dtype) {
  if (BH < 1 || S < 1) return fail(LH_ERR_INVALID_ARG, "BH and S must be >= 1");
  if (S >= (int64_t(1) << 31)) return fail(LH_ERR_INVALID_ARG, "S must stay below 2^31");
  if (dtype != LH_F32 && dtype != LH_BF16) return fail(LH_ERR_UNSUPPORTED, "dtype must be LH_F32 or LH_BF16");
  if (d != 64 && d != 128) return fail(LH_ERR_UNSUPPORTED, "only d in {64, 128} is built");
  if (dtype == LH_BF16 && BH > ((int64_t(1) << 31) - 1) / S)
    return fail(LH_ERR_UNSUPPORTED, "bf16 attention needs BH * S < 2^31 (TMA row coordinates)");
  return LH_OK;
}

extern "C" {

const char* lh_status_string(lh_status s) {
  switch (s) {
    case LH_OK: return "ok";
    case LH_ERR_INVALID_ARG: return "invalid argument";
    case LH_ERR_UNSUPPORTED: return "unsupported configuration";
    case LH_ERR_WORKSPACE: return "workspace too small";
    case LH_ERR_CUDA: return "CUDA error";
    case LH_ERR_TIMEOUT: return "device-side wait timed out";
  }
  return "unknown status";
}

const char* lh_last_error(void) { return t_last_error.c_str(); }

int64_t lh_plan_bytes(void) { return (int64_t)sizeof(lh_plan); }

lh_status lh_plan_init(const lh_config* cfg, lh_plan* out) {
  if (!cfg || !out) return fail(LH_ERR_INVALID_ARG, "null config or plan");
  const lh_config c = *cfg;
  if (c.B < 1 || c.H < 1 || c.N < 1 || c.d < 1)
    return fail(LH_ERR_INVALID_ARG, "B, H, N and d must be >= 1");
  if (c.p < 2) return fail(LH_ERR_INVALID_ARG, "pooling factor p must be >= 2");
  if (c.L < 1) return fail(LH_ERR_INVALID_ARG, "levels L must be >= 1");
  if (c.k < 0) return fail(LH_ERR_INVALID_ARG, "k must be >= 0");
  if (c.L > LH_MAX_LEVELS) return fail(LH_ERR_UNSUPPORTED, "L above LH_MAX_LEVELS");
  int64_t P[LH_MAX_LEVELS];
  P[0] = 1;
  for (int l = 1; l < c.L; ++l) {
    P[l] = P[l - 1] * c.p;
    if (P[l] > c.N) return fail(LH_ERR_INVALID_ARG, "p^(L-1) exceeds N");
  }
  if (c.N % P[c.L - 1] != 0) return fail(LH_ERR_INVALID_ARG, "N must be a multiple of p^(L-1)");
  if (c.dtype != LH_F32 && c.dtype != LH_BF16) return fail(LH_ERR_UNSUPPORTED, "dtype must be LH_F32 or LH_BF16");
  if (c.d != 64 && c.d != 128) return fail(LH_ERR_UNSUPPORTED, "only d in {64, 128} is built");
  if (c.p != 2 && c.p != 4) return fail(LH_ERR_UNSUPPORTED, "only p in {2, 4} is built");
  if (c.L > 5) return fail(LH_ERR_UNSUPPORTED, "only L <= 5 is built");
  if (P[c.L - 1] > 256) return fail(LH_ERR_UNSUPPORTED, "only p^(L-1) <= 256 is built");

  lh_plan p{};
  p.c = c;
  int64_t off = 0;
  for (int l = 0; l < LH_MAX_LEVELS; ++l) {
    p.P[l] = l < c.L ? P[l] : 0;
    p.n[l] = l < c.L ? c.N / P[l] : 0;
  }
  for (int l = 0; l <= LH_MAX_LEVELS; ++l) {
    p.flat_off[l] = off;
    if (l < c.L) off += p.n[l];
  }
  p.Ntot = p.flat_off[c.L];
  p.Npyr = p.Ntot - c.N;
  int64_t po = 0;
  for (int l = 0; l < LH_MAX_LEVELS; ++l) {
    p.pyr_off[l] = (l >= 1 && l < c.L) ? po : 0;
    if (l >= 1 && l < c.L) po += p.n[l];
  }
  p.M = p.flat_off[c.L - 1];
  p.Ksel = (int64_t)(c.L - 1) * c.p * c.k;
  if (p.Ksel > p.M) return fail(LH_ERR_INVALID_ARG, "(L-1)*p*k exceeds the candidate count");
  p.S = p.n[c.L - 1] + p.Ksel;
  if (c.select != LH_SELECT_JOINT && c.select != LH_SELECT_DESCENT && c.select != LH_SELECT_REGIONAL)
    return fail(LH_ERR_INVALID_ARG,
                "select must be LH_SELECT_JOINT, LH_SELECT_DESCENT or LH_SELECT_REGIONAL");
  if (c.select == LH_SELECT_DESCENT && c.L >= 2 && c.k > p.n[c.L - 1])
    return fail(LH_ERR_INVALID_ARG, "descent selection needs k <= N / p^(L-1)");
  if (p.S >= (int64_t(1) << 31) || p.Ntot >= (int64_t(1) << 31))
    return fail(LH_ERR_INVALID_ARG, "S and the pyramid size must stay below 2^31");
  // The per-head stage kernels put the head on the grid's y dimension.
  if ((int64_t)c.B * c.H > 65535) return fail(LH_ERR_UNSUPPORTED, "B * H above 65535 is not built");
  // The bf16 attention addresses rows of [B*H*S, d] with 32-bit TMA coordinates.
  if (c.dtype == LH_BF16 && (int64_t)c.B * c.H * p.S >= (int64_t(1) << 31))
    return fail(LH_ERR_UNSUPPORTED, "bf16 attention needs B * H * S < 2^31 (TMA row coordinates)");
  p.elem_bytes = c.dtype == LH_BF16 ? 2 : 4;

  const int64_t BH = (int64_t)c.B * c.H;
  const int64_t row = (int64_t)c.d * p.elem_bytes;
  // ctx: kept from forward to backward.
  int64_t o = 0;
  p.ctx_sel_idx = o; o = align256(o + BH * p.S * 4);
  p.ctx_slot_of = o; o = align256(o + BH * p.Ntot * 4);
  p.ctx_Qg = o; o = align256(o + BH * p.S * row);
  p.ctx_Kg = o; o = align256(o + BH * p.S * row);
  p.ctx_Vg = o; o = align256(o + BH * p.S * row);
  p.ctx_Og = o; o = align256(o + BH * p.S * row);
  p.ctx_lse = o; o = align256(o + BH * p.S * 4);
  p.ctx_bytes = o;
  // ws, forward part.
  o = 0;
  p.ws_pyrQ = o; o = align256(o + BH * p.Npyr * row);
  p.ws_pyrK = o; o = align256(o + BH * p.Npyr * row);
  p.ws_pyrV = o; o = align256(o + BH * p.Npyr * row);
  p.ws_scores = o; o = align256(o + BH * p.M * 4);
  p.topk_ws_bytes = topk_ws_bytes(p);
  p.ws_topk = o; o = align256(o + p.topk_ws_bytes);
  const int64_t fwd = o;
  // ws, backward part (reuses the same bytes).
  o = 0;
  p.ws_dOg = o; o = align256(o + BH * p.S * row);
  p.ws_D = o; o = align256(o + BH * p.S * 4);
  p.ws_dQg = o; o = align256(o + BH * p.S * row);
  p.ws_dKg = o; o = align256(o + BH * p.S * row);
  p.ws_dVg = o; o = align256(o + BH * p.S * row);
  p.attn_bwd_ws_bytes = attn_bwd_ws_bytes(BH, p.S, c.d, c.dtype);
  p.ws_attn = o; o = align256(o + p.attn_bwd_ws_bytes);
  const int64_t bwd = o;
  p.ws_bytes = fwd > bwd ? fwd : bwd;
  *out = p;
  return ok();
}

static lh_status check_plan(const lh_plan* plan) {
  if (!plan) return fail(LH_ERR_INVALID_ARG, "null plan");
  lh_plan again;
  lh_status s = lh_plan_init(&plan->c, &again);
  if (s != LH_OK) return s;
  if (again.S != plan->S || again.Ntot != plan->Ntot || again.M != plan->M ||
      again.ws_bytes != plan->ws_bytes || again.ctx_bytes != plan->ctx_bytes)
    return fail(LH_ERR_INVALID_ARG, "plan does not match its config (not from lh_plan_init?)");
  return LH_OK;
}

#define LH_CHECK_PTR(ptr)                                                      \
  do {                                                                         \
    if (!aligned16(ptr)) return fail(LH_ERR_INVALID_ARG, #ptr " is null or not 16-byte aligned"); \
  } while (0)

#define LH_TRY(expr)                    \
  do {                                  \
    lh_status s_ = (expr);              \
    if (s_ != LH_OK) return s_;         \
  } while (0)

lh_status lh_pyramid(const lh_plan* plan, const void* Q, const void* K, const void* V,
                     void* pyrQ, void* pyrK, void* pyrV, lh_stream_t stream) {
  Range range("lh_pyramid");
  LH_TRY(check_plan(plan));
  LH_CHECK_PTR(Q); LH_CHECK_PTR(K); LH_CHECK_PTR(V);
  if (plan->Npyr > 0) { LH_CHECK_PTR(pyrQ); LH_CHECK_PTR(pyrK); LH_CHECK_PTR(pyrV); }
  if (plan->Npyr == 0) return ok();
  LH_TRY(cuda_status(launch_pyramid_score(*plan, Q, K, V, pyrQ, pyrK, pyrV, nullptr, true, false,
                                          as_cuda(stream)), "lh_pyramid"));
  return ok();
}

lh_status lh_score(const lh_plan* plan, const void* Q, const void* K, float* scores,
                   lh_stream_t stream) {
  Range range("lh_score");
  LH_TRY(check_plan(plan));
  LH_CHECK_PTR(Q); LH_CHECK_PTR(K);
  if (plan->M == 0) return ok();
  LH_CHECK_PTR(scores);
  LH_TRY(cuda_status(launch_pyramid_score(*plan, Q, K, nullptr, nullptr, nullptr, nullptr, scores,
                                          false, true, as_cuda(stream)), "lh_score"));
  return ok();
}

lh_status lh_pyramid_score(const lh_plan* plan, const void* Q, const void* K, const void* V,
                           void* pyrQ, void* pyrK, void* pyrV, float* scores,
                           lh_stream_t stream) {
  Range range("lh_pyramid_score");
  LH_TRY(check_plan(plan));
  LH_CHECK_PTR(Q); LH_CHECK_PTR(K); LH_CHECK_PTR(V);
  if (plan->Npyr > 0) { LH_CHECK_PTR(pyrQ); LH_CHECK_PTR(pyrK); LH_CHECK_PTR(pyrV); }
  if (plan->M > 0) LH_CHECK_PTR(scores);
  if (plan->Npyr == 0 && plan->M == 0) return ok();
  LH_TRY(cuda_status(launch_pyramid_score(*plan, Q, K, V, pyrQ, pyrK, pyrV, scores,
                                          plan->Npyr > 0, plan->M > 0, as_cuda(stream)),
                     "lh_pyramid_score"));
  return ok();
}

lh_status lh_topk(const lh_plan* plan, const float* scores, int32_t* sel_idx, int32_t* slot_of,
                  void* ws, size_t ws_bytes, lh_stream_t stream) {
  Range range("lh_topk");
  LH_TRY(check_plan(plan));
  if (plan->M > 0) LH_CHECK_PTR(scores);
  LH_CHECK_PTR(sel_idx); LH_CHECK_PTR(slot_of);
  if (plan->topk_ws_bytes > 0) {
    LH_CHECK_PTR(ws);
    if ((int64_t)ws_bytes < plan->topk_ws_bytes)
      return fail(LH_ERR_WORKSPACE, "lh_topk workspace smaller than plan->topk_ws_bytes");
  }
  LH_TRY(cuda_status(launch_topk(*plan, scores, sel_idx, slot_of, ws, as_cuda(stream)), "lh_topk"));
  return ok();
}

lh_status lh_gather(const lh_plan* plan, const void* Q, const void* K, const void* V,
                    const void* pyrQ, const void* pyrK, const void* pyrV,
                    const int32_t* sel_idx, void* Qg, void* Kg, void* Vg, lh_stream_t stream) {
  Range range("lh_gather");
  LH_TRY(check_plan(plan));
  LH_CHECK_PTR(Q); LH_CHECK_PTR(K); LH_CHECK_PTR(V); LH_CHECK_PTR(sel_idx);
  if (plan->Npyr > 0) { LH_CHECK_PTR(pyrQ); LH_CHECK_PTR(pyrK); LH_CHECK_PTR(pyrV); }
  LH_CHECK_PTR(Qg); LH_CHECK_PTR(Kg); LH_CHECK_PTR(Vg);
  LH_TRY(cuda_status(launch_gather(*plan, Q, K, V, pyrQ, pyrK, pyrV, sel_idx, Qg, Kg, Vg,
                                   as_cuda(stream)), "lh_gather"));
  return ok();
}


lh_status lh_attn_fwd(int64_t BH, int64_t S, int32_t d, int32_t dtype, const void* Qg,
                      const void* Kg, const void* Vg, void* Og, float* lse, lh_stream_t stream) {
  Range range("lh_attn_fwd");
  LH_TRY(check_attn(BH, S, d, dtype));
  LH_CHECK_PTR(Qg); LH_CHECK_PTR(Kg); LH_CHECK_PTR(Vg); LH_CHECK_PTR(Og); LH_CHECK_PTR(lse);
  LH_TRY(cuda_status(launch_attn_fwd(BH, S, d, dtype, Qg, Kg, Vg, Og, lse, as_cuda(stream)),
                     "lh_attn_fwd"));
  return ok();
}

void lh_set_deterministic(int on) { set_deterministic(on); }

int64_t lh_attn_bwd_ws_bytes(int64_t BH, int64_t S, int32_t d, int32_t dtype) {
  if (check_attn(BH, S, d, dtype) != LH_OK) return -1;
  return attn_bwd_ws_bytes(BH, S, d, dtype);
}

lh_status lh_attn_bwd(int64_t BH, int64_t S, int32_t d, int32_t dtype, const void* Qg,
                      const void* Kg, const void* Vg, const void* Og, const float* lse,
                      const void* dOg, const float* D, void* dQg, void* dKg, void* dVg,
                      void* ws, size_t ws_bytes, lh_stream_t stream) {
  Range range("lh_attn_bwd");
  LH_TRY(check_attn(BH, S, d, dtype));
  LH_CHECK_PTR(Qg); LH_CHECK_PTR(Kg); LH_CHECK_PTR(Vg); LH_CHECK_PTR(lse); LH_CHECK_PTR(dOg);
  LH_CHECK_PTR(dQg); LH_CHECK_PTR(dKg); LH_CHECK_PTR(dVg);
  if (D == nullptr) LH_CHECK_PTR(Og);
  else LH_CHECK_PTR(D);
  const int64_t need = attn_bwd_ws_bytes(BH, S, d, dtype);
  if (need > 0) {
    LH_CHECK_PTR(ws);
    if ((int64_t)ws_bytes < need)
      return fail(LH_ERR_WORKSPACE, "lh_attn_bwd workspace smaller than lh_attn_bwd_ws_bytes()");
  }
  LH_TRY(cuda_status(launch_attn_bwd(BH, S, d, dtype, Qg, Kg, Vg, Og, lse, dOg, D, dQg, dKg, dVg, ws,
                                     as_cuda(stream)), "lh_attn_bwd"));
  return ok();
}

lh_status lh_scatter(const lh_plan* plan, const void* Og, const int32_t* slot_of, void* O,
                     lh_stream_t stream) {
  Range range("lh_scatter");
  LH_TRY(check_plan(plan));
  LH_CHECK_PTR(Og); LH_CHECK_PTR(slot_of); LH_CHECK_PTR(O);
  LH_TRY(cuda_status(launch_scatter(*plan, Og, slot_of, O, as_cuda(stream)), "lh_scatter"));
  return ok();
}

lh_status lh_scatter_bwd(const lh_plan* plan, const void* dO, const void* Og,
                         const int32_t* sel_idx, void* dOg, float* D, lh_stream_t stream) {
  Range range("lh_scatter_bwd");
  LH_TRY(check_plan(plan));
  LH_CHECK_PTR(dO); LH_CHECK_PTR(Og); LH_CHECK_PTR(sel_idx); LH_CHECK_PTR(dOg); LH_CHECK_PTR(D);
  LH_TRY(cuda_status(launch_scatter_bwd(*plan, dO, Og, sel_idx, dOg, D, as_cuda(stream)),
                     "lh_scatter_bwd"));
  return ok();
}

lh_status lh_gather_bwd(const lh_plan* plan, const void* dQg, const void* dKg, const void* dVg,
                        const int32_t* slot_of, void* dQ, void* dK, void* dV, lh_stream_t stream) {
  Range range("lh_gather_bwd");
  LH_TRY(check_plan(plan));
  LH_CHECK_PTR(dQg); LH_CHECK_PTR(dKg); LH_CHECK_PTR(dVg); LH_CHECK_PTR(slot_of);
  LH_CHECK_PTR(dQ); LH_CHECK_PTR(dK); LH_CHECK_PTR(dV);
  LH_TRY(cuda_status(launch_gather_bwd(*plan, dQg, dKg, dVg, slot_of, dQ, dK, dV, as_cuda(stream)),
                     "lh_gather_bwd"));
  return ok();
}

lh_status lh_forward(const lh_plan* plan, const void* Q, const void* K, const void* V, void* O,
                     void* ctx, size_t ctx_bytes, void* ws, size_t ws_bytes, lh_stream_t stream) {
  Range range("lh_forward");
  LH_TRY(check_plan(plan));
  LH_CHECK_PTR(Q); LH_CHECK_PTR(K); LH_CHECK_PTR(V); LH_CHECK_PTR(O);
  LH_CHECK_PTR(ctx); LH_CHECK_PTR(ws);
  if ((int64_t)ctx_bytes < plan->ctx_bytes)
    return fail(LH_ERR_WORKSPACE, "lh_forward: ctx_bytes is below plan->ctx_bytes");
  if ((int64_t)ws_bytes < plan->ws_bytes)
    return fail(LH_ERR_WORKSPACE, "lh_forward: ws_bytes is below plan->ws_bytes");
  cudaStream_t st = as_cuda(stream);
  char* c = static_cast<char*>(ctx);
  char* w = static_cast<char*>(ws);
  int32_t* sel_idx = reinterpret_cast<int32_t*>(c + plan->ctx_sel_idx);
  int32_t* slot_of = reinterpret_cast<int32_t*>(c + plan->ctx_slot_of);
  void* Qg = c + plan->ctx_Qg;
  void* Kg = c + plan->ctx_Kg;
  void* Vg = c + plan->ctx_Vg;
  void* Og = c + plan->ctx_Og;
  float* lse = reinterpret_cast<float*>(c + plan->ctx_lse);
  void* pyrQ = w + plan->ws_pyrQ;
  void* pyrK = w + plan->ws_pyrK;
  void* pyrV = w + plan->ws_pyrV;
  float* scores = reinterpret_cast<float*>(w + plan->ws_scores);
  void* tws = w + plan->ws_topk;
  const int64_t BH = (int64_t)plan->c.B * plan->c.H;

  if (plan->Npyr > 0 || plan->M > 0) {
    Range r("pyramid_score");
    LH_TRY(cuda_status(launch_pyramid_score(*plan, Q, K, V, pyrQ, pyrK, pyrV, scores,
                                            plan->Npyr > 0, plan->M > 0, st), "lh_forward/pyramid"));
  }
  {
    Range r("topk");
    LH_TRY(cuda_status(launch_topk(*plan, scores, sel_idx, slot_of, tws, st), "lh_forward/topk"));
  }
  {
    Range r("gather");
    LH_TRY(cuda_status(launch_gather(*plan, Q, K, V, pyrQ, pyrK, pyrV, sel_idx, Qg, Kg, Vg, st),
                       "lh_forward/gather"));
  }
  {
    Range r("attn_fwd");
    LH_TRY(cuda_status(launch_attn_fwd(BH, plan->S, plan->c.d, plan->c.dtype, Qg, Kg, Vg, Og, lse, st),
                       "lh_forward/attention"));
  }
  {
    Range r("scatter");
    LH_TRY(cuda_status(launch_scatter(*plan, Og, slot_of, O, st), "lh_forward/scatter"));
  }
  return ok();
}

lh_status lh_backward(const lh_plan* plan, const void* dO, const void* ctx, size_t ctx_bytes,
                      void* dQ, void* dK, void* dV, void* ws, size_t ws_bytes, lh_stream_t stream) {
  Range range("lh_backward");
  LH_TRY(check_plan(plan));
  LH_CHECK_PTR(dO); LH_CHECK_PTR(ctx); LH_CHECK_PTR(dQ); LH_CHECK_PTR(dK); LH_CHECK_PTR(dV);
  LH_CHECK_PTR(ws);
  if ((int64_t)ctx_bytes < plan->ctx_bytes)
    return fail(LH_ERR_WORKSPACE, "lh_backward: ctx_bytes is below plan->ctx_bytes");
  if ((int64_t)ws_bytes < plan->ws_bytes)
    return fail(LH_ERR_WORKSPACE, "lh_backward: ws_bytes is below plan->ws_bytes");
  cudaStream_t st = as_cuda(stream);
  const char* c = static_cast<const char*>(ctx);
  char* w = static_cast<char*>(ws);
  const int32_t* sel_idx = reinterpret_cast<const int32_t*>(c + plan->ctx_sel_idx);
  const int32_t* slot_of = reinterpret_cast<const int32_t*>(c + plan->ctx_slot_of);
  const void* Qg = c + plan->ctx_Qg;
  const void* Kg = c + plan->ctx_Kg;
  const void* Vg = c + plan->ctx_Vg;
  const void* Og = c + plan->ctx_Og;
  const float* lse = reinterpret_cast<const float*>(c + plan->ctx_lse);
  void* dOg = w + plan->ws_dOg;
  float* D = reinterpret_cast<float*>(w + plan->ws_D);
  void* dQg = w + plan->ws_dQg;
  void* dKg = w + plan->ws_dKg;
  void* dVg = w + plan->ws_dVg;
  void* aws = w + plan->ws_attn;
  const int64_t BH = (int64_t)plan->c.B * plan->c.H;

  {
    Range r("scatter_bwd");
    LH_TRY(cuda_status(launch_scatter_bwd(*plan, dO, Og, sel_idx, dOg, D, st), "lh_backward/scatter"));
  }
  {
    Range r("attn_bwd");
    LH_TRY(cuda_status(launch_attn_bwd(BH, plan->S, plan->c.d, plan->c.dtype, Qg, Kg, Vg, Og, lse, dOg, D, dQg,
                                       dKg, dVg, aws, st), "lh_backward/attention"));
  }
  {
    Range r("gather_bwd");
    LH_TRY(cuda_status(launch_gather_bwd(*plan, dQg, dKg, dVg, slot_of, dQ, dK, dV, st),
                       "lh_backward/gather"));
  }
  return ok();
}

lh_status lh_selftest_wait_timeout(lh_stream_t stream) {
  LH_TRY(cuda_status(launch_wait_timeout_selftest(as_cuda(stream)), "lh_selftest_wait_timeout"));
  return ok();
}

lh_status lh_device_status(int reset) {
  cudaError_t e = cudaDeviceSynchronize();
  if (e != cudaSuccess) return cuda_status(e, "lh_device_status");
  unsigned int v = 0;
  e = cudaMemcpyFromSymbol(&v, g_device_status, sizeof(v));
  if (e != cudaSuccess) return cuda_status(e, "lh_device_status");
  if (reset) {
    unsigned int z = 0;
    e = cudaMemcpyToSymbol(g_device_status, &z, sizeof(z));
    if (e != cudaSuccess) return cuda_status(e, "lh_device_status");
  }
  if (v != 0) return fail(LH_ERR_TIMEOUT, "a bounded device-side wait gave up");
  return ok();
}

}  // extern "C"
