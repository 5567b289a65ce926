"""Parity at the full benchmark sizes (98K and 512K tokens, 16 heads, bf16).

The layer runs on the GPU exactly as the benchmark runs it (lh_forward /
lh_backward on the whole [1, H, N, d] problem).  The oracle then checks
sampled heads: pyramid levels, scores and the selection in full; the
attention output at sampled tokens (through the oracle's attention rows of
the slots that reach them); and dQ/dK/dV on a 4096-token prefix (oracle
backward restricted to the slots that reach the prefix, with the full
forward's LSE and D), for every workload: 98K with k = 1536 and k = 6144,
512K, 98K with p = 2, 98K with the descent selection, and 98K with d = 128
(8 heads).
"""
import numpy as np
import pytest
import torch

from oracle import lighthouse as oracle
from long_context_hierarchical_b200.synth import WORKLOADS, make_workload_inputs
from tests.helpers import Bound, assert_grad_close, assert_pyr_close, grad_term_bounds_rows, np64

pytestmark = pytest.mark.gpu

HEADS = (0, 11)           # sampled (b=0) heads
N_TOKENS = 192            # sampled output tokens per head
PREFIX = 4096             # gradient prefix


def _bf16(x):
    return oracle.round_bf16(x)


def _attention_rows_with_bounds(Qg, Kg, Vg, rows):
    """Oracle output rows plus the term bounds of Og_i = sum_j P_ij Vg_j:
    sum_j P_ij |Vg_j| and (sum_j (P_ij Vg_j)^2)^(1/2)."""
    O, lse = oracle.attention_rows(Qg, Kg, Vg, rows)
    d = Qg.shape[1]
    T = np.empty_like(O)
    R = np.empty_like(O)
    for a, r in enumerate(rows):
        s = (Kg[: r + 1] @ Qg[r]) / np.sqrt(d)
        P = np.exp(s - lse[a])
        T[a] = P @ np.abs(Vg[: r + 1])
        R[a] = np.sqrt((P * P) @ Vg[: r + 1] ** 2)
    return O, lse, T, R


@pytest.fixture(scope="module", params=["98k_k1536", "98k_k6144", "512k_k2048", "98k_p2_k1536",
                                        "98k_descent_k1536", "98k_regional_k1536", "98k_d128_k1536"])
def run(request):
    from long_context_hierarchical_b200 import lh
    w = WORKLOADS[request.param]
    Q, K, V, dO = make_workload_inputs(w, seed=0, device="cuda")
    pl = lh.plan(w.B, w.H, w.N, w.d, w.p, w.L, w.k, w.dtype, select=w.select)
    O, ctx = lh.forward(pl, Q, K, V)
    grads = lh.backward(pl, dO, ctx)
    pyr, scores = lh.pyramid_score(pl, Q, K, V)
    torch.cuda.synchronize()
    lh.device_status()
    yield dict(w=w, lh=lh, pl=pl, Q=Q, K=K, V=V, dO=dO, O=O, ctx=ctx, grads=grads, pyr=pyr,
               scores=scores)
    del Q, K, V, dO, O, ctx, grads, pyr, scores
    torch.cuda.empty_cache()


@pytest.mark.parametrize("h", HEADS)
def test_fullsize_selection_and_output(run, h):
    w, pl, ctx = run["w"], run["pl"], run["ctx"]
    h = min(h, w.H - 1)  # the d = 128 workload has 8 heads
    sz = oracle.sizes(w.N, w.p, w.L, w.k)
    Qh, Kh, Vh = (np64(run[x][0, h]) for x in ("Q", "K", "V"))
    # scores and selection, in full
    cand, sel_idx, slot_of = oracle.head_select(Qh, Kh, sz, w.select)
    got_scores = np64(run["scores"][0, h])
    assert np.max(np.abs(got_scores - cand) / np.maximum(cand, 1e-30)) <= 1e-6
    assert np.array_equal(ctx.sel_idx[0, h].cpu().numpy(), sel_idx)
    assert np.array_equal(ctx.slot_of[0, h].cpu().numpy(), slot_of)
    # pyramid levels, in full (one rounding step plus the fp32 summation bound)
    levels = [oracle.pyramid(X, sz, "bf16") for X in (Qh, Kh, Vh)]
    for t, X in enumerate((Qh, Kh, Vh)):
        exp = np.concatenate(levels[t][1:], axis=0)
        absmean = np.concatenate(oracle.pyramid(np.abs(X), sz, "f64")[1:], axis=0)
        span = np.concatenate([np.full(sz.n[l], sz.P[l]) for l in range(1, sz.L)])
        assert_pyr_close(np64(run["pyr"][t][0, h]), exp, torch.bfloat16, f"pyramid[{t}]", absmean, span)
    # the gathered rows are the selected pyramid entries
    Qg, Kg, Vg = (oracle.gather(levels[t], sel_idx, sz) for t in range(3))
    for name, exp in (("Qg", Qg), ("Kg", Kg), ("Vg", Vg)):
        got = np64(ctx.gathered(name)[0, h])
        assert np.all(np.abs(got - exp) <= 2.0 ** -7 * np.abs(exp) + 1e-4), name
    # output at sampled tokens (first, last and spread), via the slots reaching them
    rng = np.random.default_rng(h)
    tokens = np.unique(np.concatenate([[0, 1, sz.P[-1] - 1, w.N - 1],
                                       rng.integers(0, w.N, N_TOKENS)]))
    need = set()
    for t in tokens:
        for l in range(sz.L):
            i = (t + 1) // sz.P[l] - 1
            if i >= 0 and slot_of[sz.flat_off[l] + i] >= 0:
                need.add(int(slot_of[sz.flat_off[l] + i]))
    need = sorted(need)
    Orows, lse_rows, Trows, Rrows = _attention_rows_with_bounds(Qg, Kg, Vg, need)
    Og = {j: _bf16(Orows[a]) for a, j in enumerate(need)}
    Tg = {j: Trows[a] for a, j in enumerate(need)}
    Rg = {j: Rrows[a] for a, j in enumerate(need)}
    got_lse = np64(ctx.lse[0, h])[need]
    assert np.max(np.abs(got_lse - lse_rows)) <= 1e-3
    exp_O = np.zeros((tokens.size, w.d))
    term = np.zeros((tokens.size, w.d))
    spread = np.zeros((tokens.size, w.d))
    for a, t in enumerate(tokens):
        for l in range(sz.L):
            i = (t + 1) // sz.P[l] - 1
            if i >= 0 and slot_of[sz.flat_off[l] + i] >= 0:
                j = int(slot_of[sz.flat_off[l] + i])
                exp_O[a] += Og[j]
                term[a] += Tg[j]
                spread[a] += Rg[j]
    assert_grad_close(np64(run["O"][0, h])[tokens], _bf16(exp_O), Bound(term, spread, spread, spread),
                      torch.bfloat16, f"{w.name}:O sampled (head {h})")


def test_fullsize_gradient_prefix(run):
    """dQ, dK, dV on tokens t < 4096 of one head, every full-size workload.

    The oracle's restricted backward (``attention_bwd_rows``) forms the
    gathered gradients of the slots whose spans start before the prefix end,
    with the full forward's LSE and D; the pool backward then gives the
    prefix tokens' gradients."""
    w, ctx = run["w"], run["ctx"]
    h = min(HEADS[1], w.H - 1)
    sz = oracle.sizes(w.N, w.p, w.L, w.k)
    Qh, Kh, Vh, dOh = (np64(run[x][0, h]) for x in ("Q", "K", "V", "dO"))
    _, sel_idx, slot_of = oracle.head_select(Qh, Kh, sz, w.select)
    levels = [oracle.pyramid(X, sz, "bf16") for X in (Qh, Kh, Vh)]
    Qg, Kg, Vg = (oracle.gather(levels[t], sel_idx, sz) for t in range(3))
    Og_exact, lse = oracle.causal_attention(Qg, Kg, Vg)
    Og = _bf16(Og_exact)
    dOg = oracle.scatter_bwd(dOh, sel_idx, sz, "bf16")
    D = np.sum(dOg * Og, axis=1)
    # slots whose span starts before the prefix end
    lev, idx = oracle.entry_level_index(sel_idx, sz)
    J = np.nonzero(idx * np.asarray(sz.P)[lev] < PREFIX)[0]
    rows = oracle.attention_bwd_rows(Qg, Kg, Vg, dOg, lse, D, J, J)
    bounds = grad_term_bounds_rows(Qg, Kg, Vg, Og, lse, dOg, J, J)
    got = [np64(g[0, h][:PREFIX]) for g in run["grads"]]
    for g, part, key in zip(got, rows, ("dQg", "dKg", "dVg")):
        dXg = np.zeros_like(Qg)
        dXg[J] = part
        exp = oracle.gather_bwd(_bf16(dXg), slot_of, sz, "bf16")[:PREFIX]
        parts = []
        for b in bounds[key]:
            full = np.zeros_like(Qg)
            full[J] = b
            parts.append(oracle.gather_bwd(full, slot_of, sz, "f64")[:PREFIX])
        assert_grad_close(g, exp, Bound(*parts), torch.bfloat16, f"{w.name}:{key[:2]} prefix (head {h})")
