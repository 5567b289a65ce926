"""The parity checks of cancelling sums, checked on the CPU (no GPU).

``assert_grad_close`` checks attention outputs and gradients element by
element (worst case), per row and per head (spread of independent bf16
roundings).  Here it must accept an emulation of the GPU's bf16 arithmetic
(the oracle's attention backward with its MMA operands dS and P rounded to
bf16, as the tensor-core kernels round them) and reject mistakes planted in
the oracle's backward that stay small element by element: a dropped
diagonal term, a few per cent of scale on one gradient, and a shifted LSE on
one 128-row tile.
"""
import numpy as np
import pytest
import torch

from oracle import lighthouse as oracle
from long_context_hierarchical_b200.synth import make_inputs
from tests.helpers import Bound, assert_grad_close, cancelling_sum_errors, grad_term_bounds, np64

BF16 = torch.bfloat16


def _head(seed=0, N=2048, p=4, L=3, k=48):
    Q, K, V, dO = make_inputs(1, 1, N, 64, "bf16", seed=seed)
    sz = oracle.sizes(N, p, L, k)
    ctx = oracle.head_forward(np64(Q[0, 0]), np64(K[0, 0]), np64(V[0, 0]), sz, "bf16")
    g = oracle.head_backward(ctx, np64(dO[0, 0]), sz, "bf16")
    return ctx, g, sz


def _planted_bwd(Qg, Kg, Vg, dOg, lse, D, round_ops=False, drop_diag=False, tile_lse_shift=None):
    """The oracle's attention backward with optional roundings and plants."""
    S, d = Qg.shape
    scale = 1.0 / np.sqrt(d)
    s = (Qg @ Kg.T) * scale
    lse = lse.copy()
    if tile_lse_shift is not None:
        lse[128:256] += tile_lse_shift
    keep = np.tril(np.ones((S, S), dtype=bool), 0 if not drop_diag else -1)
    P = np.where(keep, np.exp(s - lse[:, None]), 0.0)
    dP = dOg @ Vg.T
    dS = P * (dP - D[:, None])
    if round_ops:
        P, dS = oracle.round_bf16(P), oracle.round_bf16(dS)
    return (dS @ Kg) * scale, (dS.T @ Qg) * scale, P.T @ dOg


@pytest.fixture(scope="module")
def head():
    ctx, g, sz = _head()
    tb = grad_term_bounds(ctx["Qg"], ctx["Kg"], ctx["Vg"], ctx["Og"], ctx["lse"], g["dOg"])
    return ctx, g, sz, tb


def _run(head, **plant):
    ctx, g, _, _ = head
    return _planted_bwd(ctx["Qg"], ctx["Kg"], ctx["Vg"], g["dOg"], ctx["lse"], g["D"], **plant)


def test_bf16_emulation_passes(head):
    """Rounded MMA operands and rounded results stay inside every check."""
    ctx, g, _, tb = head
    for got, key in zip(_run(head, round_ops=True), ("dQg", "dKg", "dVg")):
        st = assert_grad_close(oracle.round_bf16(got), g[key], tb[key], BF16, f"emulation:{key}",
                               own_og=False)
        # and with room to spare: well inside the row and head bounds
        assert st["row_margin"] < 0.6 and st["head_margin"] < 0.6, (key, st)


@pytest.mark.parametrize("plant", ["drop_diag", "scale_dK", "tile_lse"])
def test_planted_mistakes_fail(head, plant):
    ctx, g, _, tb = head
    if plant == "drop_diag":
        got = _run(head, drop_diag=True)
    elif plant == "tile_lse":
        got = _run(head, tile_lse_shift=0.05)
    else:
        dQ, dK, dV = _run(head)
        got = (dQ, dK * 0.96, dV)
    failed = []
    for x, key in zip(got, ("dQg", "dKg", "dVg")):
        try:
            assert_grad_close(oracle.round_bf16(x), g[key], tb[key], BF16, f"planted {plant}:{key}",
                              own_og=False)
        except AssertionError:
            failed.append(key)
    assert failed, f"planted mistake {plant} passed every check"


def test_row_and_head_checks_catch_what_elements_miss(head):
    """A 2.5 % scale error on dK stays inside the element-wise bound (the
    term allowance is wide where terms cancel) but not inside the head bound."""
    ctx, g, _, tb = head
    _, dK, _ = _run(head)
    st = cancelling_sum_errors(oracle.round_bf16(dK * 0.975), g["dKg"], tb["dKg"], BF16, own_og=False)
    assert st["elem_margin"] <= 1.0
    assert st["head_margin"] > 1.0 or st["row_margin"] > 1.0


def test_bound_without_spread_terms_is_elementwise_only():
    """A plain array of term bounds (no spread) gives the element-wise check
    only; its row and head bounds reduce to the relative parts."""
    exp = np.ones((2, 3, 4))
    st = cancelling_sum_errors(exp * (1 + 1e-3), exp, np.zeros_like(exp), BF16)
    assert st["elem_margin"] < 1 and st["row_margin"] < 1 and st["head_margin"] < 1
    b = Bound(*(np.zeros_like(exp),) * 4)
    st = cancelling_sum_errors(exp * 1.03, exp, b, BF16)
    assert st["row_margin"] > 1 and st["head_margin"] > 1
