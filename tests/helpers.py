"""Shared helpers of the parity tests: tolerances and oracle runs on tensors."""
from typing import NamedTuple

import numpy as np
import torch

from oracle import lighthouse as oracle

# Output/gradient tolerance: |gpu - oracle| <= TOL[dtype] * max(1, |oracle|).
# bf16 keeps 8 significant bits, so past |x| = 1 a bound in absolute terms
# would be tighter than one rounding step of the stored value; the bound is
# relative above 1 and absolute below.
TOL = {torch.bfloat16: 2e-2, torch.float32: 1e-4}
# A stored pyramid mean may differ from the oracle's by one rounding step
# (fp32 sum then round vs fp64 sum then round).
PYR_REL = {torch.bfloat16: 2.0 ** -7, torch.float32: 1e-6}
MODE = {torch.bfloat16: "bf16", torch.float32: "f32"}
# One rounding step of an MMA operand: bf16 keeps 8 significant bits, so a
# rounded operand is within 2^-8 of its value relative to its leading power
# of two (half an ulp of 2^-7); fp32 operands (the fp32 path) 2^-24.
OPERAND_STEP = {torch.bfloat16: 2.0 ** -8, torch.float32: 2.0 ** -24}
# Row and head checks of cancelling sums (see ``cancelling_sum_errors``).
# A rounding to the nearest value is off by at most half a step, evenly
# spread over that interval, so its standard deviation is the bound over
# sqrt(3): 2^-8 / sqrt(3) relative for a bf16 operand.
SPREAD = {torch.bfloat16: 2.0 ** -8 / np.sqrt(3.0), torch.float32: 2.0 ** -24 / np.sqrt(3.0)}
# fp32 error of forming a term before it is rounded (the dot products dP and
# D accumulate in fp32, the exponent and the folded lse and D carry a few fp32
# steps), relative to the sum of the magnitudes that enter it: 16 fp32 steps.
FORM = 2.0 ** -20
ROW_REL = {torch.bfloat16: 2e-2, torch.float32: 1e-4}
HEAD_REL = {torch.bfloat16: 1e-2, torch.float32: 1e-5}
RSS_SIGMAS = 4.0

# Error statistics of every cancelling-sum check of the session, printed in
# pytest's terminal summary (tests/conftest.py).
STATS = []


class Bound(NamedTuple):
    """Term bounds of a cancelling sum, element by element.

    l1:    sum over the terms of |term| (worst case: every rounding adds up);
    rss:   square root of the sum of squared rounded terms (the spread of
           independent roundings of the terms), given the oracle's Og;
    rss_d: the same where the GPU formed its own Og, which shifts D;
    rss_f: square root of the sum of squared magnitudes that enter each term
           before its rounding (the spread of its fp32 formation errors).
    """
    l1: np.ndarray
    rss: np.ndarray
    rss_d: np.ndarray
    rss_f: np.ndarray


def np64(t):
    return t.detach().to("cpu", torch.float64).numpy()


def bf16_ulp(x):
    """Spacing of bf16 values at |x|: 2^(floor(log2 |x|) - 7) (normal range)."""
    a = np.maximum(np.abs(np.asarray(x, dtype=np.float64)), 2.0 ** -126)
    return np.exp2(np.floor(np.log2(a)) - 7)


def assert_close(got, exp, dtype, what):
    got = np.asarray(got, dtype=np.float64)
    exp = np.asarray(exp, dtype=np.float64)
    assert got.shape == exp.shape, (what, got.shape, exp.shape)
    err = np.abs(got - exp)
    tol = TOL[dtype] * np.maximum(1.0, np.abs(exp))
    bad = err > tol
    assert np.all(np.isfinite(got)), f"{what}: non-finite values"
    assert not bad.any(), (
        f"{what}: {int(bad.sum())} of {bad.size} outside tolerance; max abs err {err.max():.3e}; "
        f"first at {np.argwhere(bad)[0].tolist()} got {got[bad][0]!r} want {exp[bad][0]!r}")
    return float(err.max()) if err.size else 0.0


def assert_pyr_close(got, exp, dtype, what, abs_mean=None, span=None):
    """One rounding step of the stored mean, plus the fp32 summation bound.

    The GPU sums the span in fp32 (error <= (P-1) 2^-24 sum|x|, i.e. at most
    P 2^-24 mean|x| after the exact scaling by 1/P) and rounds once; the
    oracle sums in fp64 and rounds once.  ``abs_mean`` is the span mean of
    |x| and ``span`` the number of tokens P per entry, row by row.
    """
    got = np.asarray(got, dtype=np.float64)
    exp = np.asarray(exp, dtype=np.float64)
    err = np.abs(got - exp)
    tol = PYR_REL[dtype] * np.abs(exp) + 1e-30
    if abs_mean is not None:
        tol = tol + (1 + PYR_REL[dtype]) * np.asarray(span)[..., None] * 2.0 ** -24 * abs_mean
    bad = err > tol
    assert not bad.any(), (
        f"{what}: {int(bad.sum())} of {bad.size} differ by more than one rounding step; "
        f"max abs err {err.max():.3e}")


def _term_block(Qg, Kg, Vg, Og, lse, dOg, r0, r1, c1):
    """For query rows r0..r1-1 against keys < c1: P, the worst-case term
    factor P (|dP| + A) and the rounded operand dS = P (dP - D), where
    A_i = sum_c |dOg_ic Og_ic|, D_i = sum_c dOg_ic Og_ic, the root-sum-square
    A2_i = (sum_c (dOg_ic Og_ic)^2)^(1/2), and the magnitudes that enter dS
    in fp32, F_ij = P_ij (sum_c |dOg_ic| |Vg_jc| + A_i)."""
    scale = 1.0 / np.sqrt(Qg.shape[1])
    s = (Qg[r0:r1] @ Kg[:c1].T) * scale
    rows = np.arange(r0, r1)[:, None]
    cols = np.arange(c1)[None, :]
    P = np.where(cols <= rows, np.exp(s - lse[r0:r1, None]), 0.0)
    dP = dOg[r0:r1] @ Vg[:c1].T
    A = np.sum(np.abs(dOg[r0:r1] * Og[r0:r1]), axis=1)
    A2 = np.sqrt(np.sum((dOg[r0:r1] * Og[r0:r1]) ** 2, axis=1))
    D = np.sum(dOg[r0:r1] * Og[r0:r1], axis=1)
    F = P * (np.abs(dOg[r0:r1]) @ np.abs(Vg[:c1]).T + A[:, None])
    return P, P * (np.abs(dP) + A[:, None]), P * (dP - D[:, None]), A2, F


def grad_term_bounds(Qg, Kg, Vg, Og, lse, dOg):
    """Term bounds (``Bound``) of each gathered gradient element and of Og.

    dQg_i = s sum_j dS_ij Kg_j and dKg_j = s sum_i dS_ij Qg_i with
    dS_ij = P_ij (dP_ij - D_i) sum terms that cancel (sum_j dS_ij = 0), so
    their rounding error scales with the terms, not with the result.

    l1 (worst case, element by element): two roundings reach the terms on
    the GPU, the bf16 operand dS of the MMA and the bf16 storage of Og,
    which enters D_i = sum_c dOg_ic Og_ic; per term the bound used is
    P_ij (|dP_ij| + A_i) |Kg_j| (or |Qg_i|), A_i = sum_c |dOg_ic Og_ic|;
    dVg_j = sum_i P_ij dOg_i gets P_ij |dOg_i|; the forward output Og_i =
    sum_j P_ij Vg_j (P rounded to bf16 for the MMA) gets P_ij |Vg_j|.

    rss (spread): the values the GPU rounds are dS_ij (for dQg, dKg) and P_ij
    (for dVg, Og), each independently, so the error of a sum spreads like
    the root of the sum of the squared rounded terms: |dS_ij Kg_j| s,
    |dS_ij Qg_i| s, |P_ij dOg_i|, |P_ij Vg_j|.  Where the GPU forms its own
    Og (a whole layer) some of its elements round to the neighbouring bf16
    value, one step (2^-7) away, which shifts D_i by a spread of about
    2 A2_i rounding spreads and moves every term of row i alike: one more
    term 2 A2_i s |sum_j P_ij Kg_j| for dQg_i, and 2 P_ij A2_i |Qg_i| s per
    term of dKg_j.

    rss_f: dS_ij is formed in fp32 from dP_ij and D_i, whose own sums cancel,
    so its formation error scales with F_ij (``_term_block``): terms
    F_ij |Kg_j| s and F_ij |Qg_i| s; for dVg and Og (P formed by the
    exponential alone) the rss terms.  Returns a dict of ``Bound`` for dQg,
    dKg, dVg and Og.
    """
    S, d = Qg.shape
    scale = 1.0 / np.sqrt(d)
    aK, aQ, aG, aV = np.abs(Kg), np.abs(Qg), np.abs(dOg), np.abs(Vg)
    acc = {k: [np.zeros((S, d)) for _ in range(4)] for k in ("dQg", "dKg", "dVg", "Og")}
    for r0 in range(0, S, 512):
        r1 = min(S, r0 + 512)
        P, T, dS, A2, F = _term_block(Qg, Kg, Vg, Og, lse, dOg, r0, r1, r1)
        acc["dQg"][0][r0:r1] = (T @ aK[:r1]) * scale
        acc["dQg"][1][r0:r1] = ((dS * dS) @ Kg[:r1] ** 2) * scale ** 2
        acc["dQg"][2][r0:r1] = ((2 * A2[:, None] * (P @ Kg[:r1])) ** 2) * scale ** 2
        acc["dQg"][3][r0:r1] = ((F * F) @ Kg[:r1] ** 2) * scale ** 2
        acc["Og"][0][r0:r1] = P @ aV[:r1]
        acc["Og"][1][r0:r1] = (P * P) @ Vg[:r1] ** 2
        acc["dKg"][0][:r1] += (T.T @ aQ[r0:r1]) * scale
        acc["dKg"][1][:r1] += ((dS * dS).T @ Qg[r0:r1] ** 2) * scale ** 2
        acc["dKg"][2][:r1] += ((P * P).T @ (2 * A2[:, None] * Qg[r0:r1]) ** 2) * scale ** 2
        acc["dKg"][3][:r1] += ((F * F).T @ Qg[r0:r1] ** 2) * scale ** 2
        acc["dVg"][0][:r1] += P.T @ aG[r0:r1]
        acc["dVg"][1][:r1] += (P * P).T @ dOg[r0:r1] ** 2
    for k in ("dVg", "Og"):
        acc[k][3] = acc[k][1]
    return {k: Bound(v[0], np.sqrt(v[1]), np.sqrt(v[1] + v[2]), np.sqrt(v[3])) for k, v in acc.items()}


def grad_term_bounds_rows(Qg, Kg, Vg, Og, lse, dOg, q_rows, k_cols):
    """``grad_term_bounds`` restricted to dQg rows ``q_rows`` and dKg / dVg
    rows ``k_cols`` (full-size checks; the forward's LSE of every row)."""
    S, d = Qg.shape
    scale = 1.0 / np.sqrt(d)
    q_rows = np.asarray(q_rows, dtype=np.int64)
    k_cols = np.asarray(k_cols, dtype=np.int64)
    out = {}
    qq = [np.zeros((q_rows.size, d)) for _ in range(4)]
    for a, r in enumerate(q_rows):
        P, T, dS, A2, F = _term_block(Qg, Kg, Vg, Og, lse, dOg, r, r + 1, r + 1)
        qq[0][a] = (T @ np.abs(Kg[: r + 1]))[0] * scale
        qq[1][a] = ((dS * dS) @ Kg[: r + 1] ** 2)[0] * scale ** 2
        qq[2][a] = ((2 * A2[:, None] * (P @ Kg[: r + 1])) ** 2)[0] * scale ** 2
        qq[3][a] = ((F * F) @ Kg[: r + 1] ** 2)[0] * scale ** 2
    out["dQg"] = Bound(qq[0], np.sqrt(qq[1]), np.sqrt(qq[1] + qq[2]), np.sqrt(qq[3]))
    kk = [np.zeros((k_cols.size, d)) for _ in range(6)]
    for a, c in enumerate(k_cols):
        P = np.exp((Qg[c:] @ Kg[c]) * scale - lse[c:])
        A = np.sum(np.abs(dOg[c:] * Og[c:]), axis=1)
        A2 = np.sqrt(np.sum((dOg[c:] * Og[c:]) ** 2, axis=1))
        D = np.sum(dOg[c:] * Og[c:], axis=1)
        dP = dOg[c:] @ Vg[c]
        T = P * (np.abs(dP) + A)
        dS = P * (dP - D)
        F = P * (np.abs(dOg[c:]) @ np.abs(Vg[c]) + A)
        kk[0][a] = (T @ np.abs(Qg[c:])) * scale
        kk[1][a] = ((dS * dS) @ Qg[c:] ** 2) * scale ** 2
        kk[4][a] = ((P * P * 4 * A2 * A2) @ Qg[c:] ** 2) * scale ** 2
        kk[5][a] = ((F * F) @ Qg[c:] ** 2) * scale ** 2
        kk[2][a] = P @ np.abs(dOg[c:])
        kk[3][a] = (P * P) @ dOg[c:] ** 2
    out["dKg"] = Bound(kk[0], np.sqrt(kk[1]), np.sqrt(kk[1] + kk[4]), np.sqrt(kk[5]))
    out["dVg"] = Bound(kk[2], np.sqrt(kk[3]), np.sqrt(kk[3]), np.sqrt(kk[3]))
    return out


def grad_tolerance_terms(ctxs, grads, sz):
    """Term bounds of dQ/dK/dV and O (gathered and per token), all heads.

    A token's gradient sums at most L gathered rows, each scaled by 1/p^l,
    and a token's output at most L; both bounds add up over those rows
    (for the root-sum-square bound that is the triangle inequality)."""
    keys = ("dQg", "dKg", "dVg", "dQ", "dK", "dV", "Og", "O")
    out = {k: ([], [], [], []) for k in keys}
    for crow, grow in zip(ctxs, grads[3]):
        r = {k: ([], [], [], []) for k in keys}
        for ctx, g in zip(crow, grow):
            b = grad_term_bounds(ctx["Qg"], ctx["Kg"], ctx["Vg"], ctx["Og"], ctx["lse"], g["dOg"])
            for key in ("dQ", "dK", "dV"):
                for i in range(4):
                    r[key + "g"][i].append(b[key + "g"][i])
                    r[key][i].append(oracle.gather_bwd(b[key + "g"][i], ctx["slot_of"], sz, "f64"))
            for i in range(4):
                r["Og"][i].append(b["Og"][i])
                r["O"][i].append(oracle.scatter(b["Og"][i], ctx["slot_of"], sz, "f64"))
        for k in keys:
            for i in range(4):
                out[k][i].append(np.stack(r[k][i]))
    return {k: Bound(*(np.stack(x) for x in v)) for k, v in out.items()}


def cancelling_sum_errors(got, exp, terms, dtype, own_og=True):
    """Error statistics of a cancelling sum and the three checks' margins.

    Checks (each must be <= 1 to pass):
      elem: |g - o| / (TOL max(1, |o|) + 2 step |terms|_1)  per element, with
            step = 2^-8 (bf16 operands; two roundings reach each term, so
            2 step = 2^-7) -- the worst case;
      row:  ||g_r - o_r|| / (ROW_REL ||o_r|| + RSS_SIGMAS ||sigma_r||) per
            row r over the channels, where an element's spread sigma is
            ((SPREAD rss)^2 + (FORM rss_f)^2)^(1/2): independent roundings of
            the terms add up like a random walk; ROW_REL covers the
            roundings of the stored result (the gathered and the final
            gradient);
      head: ||g - o|| / (HEAD_REL ||o|| + RSS_SIGMAS ||sigma||) per head.
    ``own_og``: the GPU formed Og itself (a whole layer), so D may shift
    (``Bound.rss_d``); False where the stage was fed the oracle's Og.
    """
    got = np.asarray(got, dtype=np.float64)
    exp = np.asarray(exp, dtype=np.float64)
    if isinstance(terms, Bound):
        l1 = terms.l1
        rss = np.sqrt((SPREAD[dtype] * (terms.rss_d if own_og else terms.rss)) ** 2
                      + (FORM * terms.rss_f) ** 2)
    else:
        l1, rss = terms, np.zeros_like(exp)
    step = OPERAND_STEP[dtype]
    err = np.abs(got - exp)
    base = TOL[dtype] * np.maximum(1.0, np.abs(exp))
    elem = err / (base + 2 * step * l1)
    e_r = np.sqrt(np.sum(err ** 2, axis=-1))
    row = e_r / (ROW_REL[dtype] * np.sqrt(np.sum(exp ** 2, axis=-1))
                 + RSS_SIGMAS * np.sqrt(np.sum(rss ** 2, axis=-1)) + 1e-30)
    hx = lambda a: np.sqrt(np.sum(a.reshape(-1, a.shape[-2] * a.shape[-1]) ** 2, axis=1)) \
        if a.ndim >= 2 else np.sqrt(np.sum(a ** 2))[None]
    e_h, o_h, s_h = hx(err), hx(exp), hx(rss)
    head = e_h / (HEAD_REL[dtype] * o_h + RSS_SIGMAS * s_h + 1e-30)
    nz = np.abs(exp) > 0
    ulp = err[nz] / bf16_ulp(exp[nz]) if nz.any() else np.zeros(1)
    return {
        "elements": int(err.size), "max_abs_err": float(err.max()) if err.size else 0.0,
        "max_bf16_ulp_err": float(ulp.max()) if ulp.size else 0.0,
        "median_bf16_ulp_err": float(np.median(ulp)) if ulp.size else 0.0,
        "n_term_allowance": int((err > base).sum()),
        "head_rel_l2": float(np.max(e_h / np.maximum(o_h, 1e-30))),
        "elem_margin": float(elem.max()) if elem.size else 0.0,
        "row_margin": float(row.max()) if row.size else 0.0,
        "head_margin": float(head.max()),
        "_elem": elem, "_row": row, "_head": head,
    }


def assert_grad_close(got, exp, terms, dtype, what, own_og=True):
    """Check of a cancelling sum (attention output or gradient): element by
    element within TOL max(1, |exp|) plus one bf16 rounding step (2^-7) of
    the sum of |terms|; per row and per head within a relative bound plus
    RSS_SIGMAS rounding steps of the root-sum-square of the terms
    (``cancelling_sum_errors``).  Records the error statistics in STATS and
    returns them."""
    got = np.asarray(got, dtype=np.float64)
    assert got.shape == np.shape(exp), (what, got.shape, np.shape(exp))
    assert np.all(np.isfinite(got)), f"{what}: non-finite values"
    st = cancelling_sum_errors(got, exp, terms, dtype, own_og)
    STATS.append({"what": what, **{k: v for k, v in st.items() if not k.startswith("_")}})
    elem, row, head = st["_elem"], st["_row"], st["_head"]
    if (elem > 1).any():
        i = tuple(np.argwhere(elem > 1)[0])
        raise AssertionError(
            f"{what}: {int((elem > 1).sum())} of {elem.size} elements outside tolerance; max abs err "
            f"{st['max_abs_err']:.3e}; first at {list(i)} got {got[i]!r} want {np.asarray(exp)[i]!r}")
    assert not (row > 1).any(), (
        f"{what}: {int((row > 1).sum())} of {row.size} rows outside the row bound "
        f"(worst margin {row.max():.3f} at {np.argwhere(row > 1)[0].tolist()})")
    assert not (head > 1).any(), f"{what}: head error outside the head bound (margin {head.max():.3f})"
    return st


def oracle_layer(Q, K, V, dO, p, L, k, dtype, rule="joint"):
    """Oracle forward (and backward when dO is given) of [B,H,N,d] tensors."""
    mode = MODE[dtype]
    Qn, Kn, Vn = np64(Q), np64(K), np64(V)
    O, ctxs, sz = oracle.forward(Qn, Kn, Vn, p, L, k, mode, rule=rule)
    grads = None
    if dO is not None:
        grads = oracle.backward(ctxs, np64(dO), sz, mode)
    return O, ctxs, sz, grads


def stack(ctxs, key):
    return np.stack([np.stack([c[key] for c in row]) for row in ctxs])
