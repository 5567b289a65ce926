"""Shared helpers of the parity tests: tolerances and oracle runs on tensors."""
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


def np64(t):
    return t.detach().to("cpu", torch.float64).numpy()


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


def grad_term_bounds(Qg, Kg, Vg, Og, lse, dOg):
    """Sum of |terms| of each gathered gradient element, in fp64.

    dQg_i = s sum_j dS_ij Kg_j and dKg_j = s sum_i dS_ij Qg_i with
    dS_ij = P_ij (dP_ij - D_i) sum terms that cancel (sum_j dS_ij = 0), so
    their rounding error scales with sum |terms|, not with the result.  Two
    roundings reach the terms on the GPU: the bf16 operand dS of the MMA and
    the bf16 storage of Og, which enters D_i = sum_c dOg_ic Og_ic.  Per term
    the bound used is P_ij (|dP_ij| + sum_c |dOg_ic Og_ic|) times |Kg_j| (or
    |Qg_i|); dVg_j = sum_i P_ij dOg_i gets P_ij |dOg_i|.  The forward output
    Og_i = sum_j P_ij Vg_j (P rounded to bf16 for the MMA on the GPU) gets
    sum_j P_ij |Vg_j|.
    """
    S, d = Qg.shape
    scale = 1.0 / np.sqrt(d)
    A = np.sum(np.abs(dOg * Og), axis=1)
    mq = np.zeros_like(Qg)
    mk = np.zeros_like(Kg)
    mv = np.zeros_like(Vg)
    mo = np.zeros_like(Vg)
    aK, aQ, aG, aV = np.abs(Kg), np.abs(Qg), np.abs(dOg), np.abs(Vg)
    for r0 in range(0, S, 512):
        r1 = min(S, r0 + 512)
        s = (Qg[r0:r1] @ Kg[:r1].T) * scale
        rows = np.arange(r0, r1)[:, None]
        cols = np.arange(r1)[None, :]
        P = np.where(cols <= rows, np.exp(s - lse[r0:r1, None]), 0.0)
        dP = dOg[r0:r1] @ Vg[:r1].T
        T = P * (np.abs(dP) + A[r0:r1, None])
        mq[r0:r1] = (T @ aK[:r1]) * scale
        mk[:r1] += (T.T @ aQ[r0:r1]) * scale
        mv[:r1] += P.T @ aG[r0:r1]
        mo[r0:r1] = P @ aV[:r1]
    return mq, mk, mv, mo


def grad_tolerance_terms(ctxs, grads, sz):
    """Per-element term bounds of dQ/dK/dV (gathered and per token), all heads."""
    out = {k: [] for k in ("dQg", "dKg", "dVg", "dQ", "dK", "dV", "Og", "O")}
    for crow, grow in zip(ctxs, grads[3]):
        r = {k: [] for k in out}
        for ctx, g in zip(crow, grow):
            mq, mk, mv, mo = grad_term_bounds(ctx["Qg"], ctx["Kg"], ctx["Vg"], ctx["Og"], ctx["lse"],
                                              g["dOg"])
            for key, m in (("dQ", mq), ("dK", mk), ("dV", mv)):
                r[key + "g"].append(m)
                r[key].append(oracle.gather_bwd(m, ctx["slot_of"], sz, "f64"))
            r["Og"].append(mo)
            r["O"].append(oracle.scatter(mo, ctx["slot_of"], sz, "f64"))
        for k in out:
            out[k].append(np.stack(r[k]))
    return {k: np.stack(v) for k, v in out.items()}


def assert_grad_close(got, exp, terms, dtype, what):
    """Check of a cancelling sum (attention output or gradient): TOL * max(1,
    |exp|) plus one bf16 rounding step (2^-7) of the sum of |terms|
    (``grad_term_bounds``); fp32 uses 2^-23."""
    got = np.asarray(got, dtype=np.float64)
    exp = np.asarray(exp, dtype=np.float64)
    step = 2.0 ** -7 if dtype == torch.bfloat16 else 2.0 ** -23
    err = np.abs(got - exp)
    base = TOL[dtype] * np.maximum(1.0, np.abs(exp))
    tol = base + step * terms
    bad = err > tol
    assert np.all(np.isfinite(got)), f"{what}: non-finite values"
    assert not bad.any(), (
        f"{what}: {int(bad.sum())} of {bad.size} outside tolerance; max abs err {err.max():.3e}; "
        f"first at {np.argwhere(bad)[0].tolist()} got {got[bad][0]!r} want {exp[bad][0]!r} "
        f"term bound {terms[bad][0]!r}")
    return int((err > base).sum())


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
