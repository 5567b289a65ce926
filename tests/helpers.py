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


def assert_pyr_close(got, exp, dtype, what):
    got = np.asarray(got, dtype=np.float64)
    exp = np.asarray(exp, dtype=np.float64)
    err = np.abs(got - exp)
    tol = PYR_REL[dtype] * np.abs(exp) + 1e-30
    bad = err > tol
    assert not bad.any(), (
        f"{what}: {int(bad.sum())} of {bad.size} differ by more than one rounding step; "
        f"max abs err {err.max():.3e}")


def oracle_layer(Q, K, V, dO, p, L, k, dtype):
    """Oracle forward (and backward when dO is given) of [B,H,N,d] tensors."""
    mode = MODE[dtype]
    Qn, Kn, Vn = np64(Q), np64(K), np64(V)
    O, ctxs, sz = oracle.forward(Qn, Kn, Vn, p, L, k, mode)
    grads = None
    if dO is not None:
        grads = oracle.backward(ctxs, np64(dO), sz, mode)
    return O, ctxs, sz, grads


def stack(ctxs, key):
    return np.stack([np.stack([c[key] for c in row]) for row in ctxs])
