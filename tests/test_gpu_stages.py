"""Per-stage and whole-layer parity of the CUDA path against the oracle.

Each stage is fed the oracle's own inputs for that stage (seeded inputs,
never values from the CUDA path) and compared element by element:
selection and order bit-exact, scores within 1e-6 relative, pyramid means
within one rounding step, outputs and gradients within 2e-2 (bf16) or 1e-4
(fp32) of max(1, |oracle|).
"""
import numpy as np
import pytest
import torch

from oracle import lighthouse as oracle
from long_context_hierarchical_b200.synth import make_inputs, make_scores
from tests.helpers import (TOL, assert_close, assert_grad_close, assert_pyr_close,
                           grad_term_bounds, grad_tolerance_terms, np64, oracle_layer, stack)

pytestmark = pytest.mark.gpu

# name: (B, H, N, dtype, p, L, k[, d]); d is 64 unless given
CASES = {
    "tiny_f32": (1, 2, 1024, "f32", 4, 3, 32),          # S = 320
    "8k_bf16": (1, 8, 8192, "bf16", 4, 4, 256),         # S = 3200
    "p2_ragged": (2, 3, 96, "bf16", 2, 3, 5),           # S = 44: partial tiles
    "L2": (1, 2, 512, "bf16", 4, 2, 16),                # S = 192
    "L5": (1, 2, 2048, "bf16", 4, 5, 8),                # p^(L-1) = 256, S = 136
    "L1_dense": (1, 2, 256, "bf16", 4, 1, 0),           # selection off: S = N
    "k0": (1, 2, 1024, "bf16", 4, 3, 0),                # coarsest level only: S = 64
    "kmax": (1, 2, 64, "bf16", 2, 2, 32),               # every candidate: S = 96
    "f32_p2_L5": (1, 1, 256, "f32", 2, 5, 3),           # S = 40
    "p2_L4_odd": (1, 2, 200, "bf16", 2, 4, 7),          # N = 25 * 8, S = 67
    # S = 1792 < N / 8: the token kernels' sparse forms (a branch per level;
    # scatter backward rows taken level by level) over 28 slot blocks
    "sparse_64k": (1, 2, 65536, "bf16", 4, 4, 64),
    # head dimension 128
    "d128_f32": (1, 2, 512, "f32", 4, 3, 16, 128),      # S = 160
    "d128_ragged": (2, 3, 200, "bf16", 2, 4, 7, 128),   # S = 67: partial tiles and chunks
    "d128_4k": (1, 4, 4096, "bf16", 4, 3, 64, 128),     # S = 768: six key tiles
    "d128_L1_dense": (1, 2, 384, "bf16", 4, 1, 0, 128), # S = 384: a half-empty tile pair
}

DT = {"f32": torch.float32, "bf16": torch.bfloat16}


@pytest.fixture(scope="module", params=list(CASES))
def case(request):
    from long_context_hierarchical_b200 import lh
    B, H, N, dtype, p, L, k, *rest = CASES[request.param]
    d = rest[0] if rest else 64
    Q, K, V, dO = make_inputs(B, H, N, d, dtype, seed=0)
    O, ctxs, sz, grads = oracle_layer(Q, K, V, dO, p, L, k, DT[dtype])
    pl = lh.plan(B, H, N, d, p, L, k, dtype)
    dev = torch.device("cuda")
    terms = grad_tolerance_terms(ctxs, grads, sz)
    return dict(name=request.param, B=B, H=H, N=N, d=d, dt=DT[dtype], p=p, L=L, k=k, lh=lh, pl=pl,
                Q=Q.to(dev), K=K.to(dev), V=V.to(dev), dO=dO.to(dev), O=O, ctxs=ctxs, sz=sz,
                grads=grads, terms=terms)


def _t(a, dtype, dev="cuda"):
    return torch.from_numpy(np.ascontiguousarray(a)).to(dev).to(dtype)


def _oracle_pyr(c, which):
    """Levels 1..L-1 of tensor `which` (0,1,2) as one [B,H,Npyr,d] array."""
    rows = []
    for row in c["ctxs"]:
        hs = []
        for ctx in row:
            lv = ctx["levels"][which]
            hs.append(np.concatenate(lv[1:], axis=0) if len(lv) > 1 else np.zeros((1, c["d"])))
        rows.append(np.stack(hs))
    return np.stack(rows)


def _abs_means(c, which):
    """Span means of |X| over levels 1..L-1 and the span length of each row."""
    X = np64((c["Q"], c["K"], c["V"])[which])
    sz = c["sz"]
    means, spans = [], []
    for l in range(1, sz.L):
        P = sz.P[l]
        means.append(np.abs(X).reshape(X.shape[0], X.shape[1], sz.n[l], P, X.shape[3]).mean(axis=3))
        spans.append(np.full(sz.n[l], P))
    return np.concatenate(means, axis=2), np.concatenate(spans)


def test_pyramid_and_scores(case):
    c = case
    lh, pl = c["lh"], c["pl"]
    pyr, scores = lh.pyramid_score(pl, c["Q"], c["K"], c["V"])
    torch.cuda.synchronize()
    if pl.Npyr > 0:
        for w in range(3):
            am, span = _abs_means(c, w)
            assert_pyr_close(np64(pyr[w]), _oracle_pyr(c, w), c["dt"], f"pyramid[{w}]", am, span)
    if pl.M > 0:
        got = np64(scores)
        exp = stack(c["ctxs"], "cand")
        rel = np.abs(got - exp) / np.maximum(np.abs(exp), 1e-30)
        assert rel.max() <= 1e-6, rel.max()
        # the separate entry points give the fused kernel's bytes
        assert torch.equal(lh.score(pl, c["Q"], c["K"]), scores)
    if pl.Npyr > 0:
        sep = lh.pyramid(pl, c["Q"], c["K"], c["V"])
        for w in range(3):
            assert torch.equal(sep[w], pyr[w])


def test_topk_on_oracle_scores(case):
    c = case
    lh, pl = c["lh"], c["pl"]
    cand = stack(c["ctxs"], "cand") if pl.M > 0 else np.zeros((c["B"], c["H"], 1))
    sel, inv = lh.topk(pl, _t(cand, torch.float32))
    assert np.array_equal(sel.cpu().numpy(), stack(c["ctxs"], "sel_idx"))
    assert np.array_equal(inv.cpu().numpy(), stack(c["ctxs"], "slot_of"))


@pytest.mark.parametrize("distinct", [None, 3, 1])
def test_topk_ties_and_random_scores(distinct):
    """Selection on seeded score arrays, including exact ties everywhere."""
    from long_context_hierarchical_b200 import lh
    B, H, N, p, L, k = 1, 3, 4096, 4, 4, 40
    sz = oracle.sizes(N, p, L, k)
    scores = make_scores(B, H, sz.M, seed=5, distinct=distinct)
    pl = lh.plan(B, H, N, 64, p, L, k, "bf16")
    sel, inv = lh.topk(pl, scores.cuda())
    for h in range(H):
        mask = oracle.select(scores[0, h].double().numpy(), sz)
        es, ei = oracle.order_selection(mask, sz)
        assert np.array_equal(sel[0, h].cpu().numpy(), es)
        assert np.array_equal(inv[0, h].cpu().numpy(), ei)


# (B, H, N, p, L, k, distinct score levels or None)
DESCENT_CASES = {
    "p4_L3": (1, 3, 4096, 4, 3, 40, None),
    "p2_L4_ties": (1, 2, 1024, 2, 4, 16, 3),
    "p2_L5": (1, 2, 2048, 2, 5, 8, None),
    "p4_L2_ties": (1, 2, 512, 4, 2, 30, 2),
    "k_is_n_coarsest": (1, 2, 1024, 4, 3, 64, None),
    "all_equal": (1, 1, 1024, 2, 3, 20, 1),
}


@pytest.mark.parametrize("case", list(DESCENT_CASES))
def test_descent_selection_on_seeded_scores(case):
    """Hierarchical-descent selection (lh_select LH_SELECT_DESCENT) against
    the oracle's rule, bit for bit, including ties everywhere."""
    from long_context_hierarchical_b200 import lh
    B, H, N, p, L, k, distinct = DESCENT_CASES[case]
    sz = oracle.sizes(N, p, L, k)
    scores = make_scores(B, H, sz.M, seed=9, distinct=distinct)
    pl = lh.plan(B, H, N, 64, p, L, k, "bf16", select="descent")
    sel, inv = lh.topk(pl, scores.cuda())
    for h in range(H):
        mask = oracle.select_descent(scores[0, h].double().numpy(), sz)
        es, ei = oracle.order_selection(mask, sz)
        assert np.array_equal(sel[0, h].cpu().numpy(), es)
        assert np.array_equal(inv[0, h].cpu().numpy(), ei)
    lh.device_status()


# (B, H, N, p, L, k, distinct score levels or None): M spans several
# 2048-candidate regions, a region straddling a level boundary, a ragged
# last region, and a budget of every candidate
REGIONAL_CASES = {
    "p4_L3_3reg": (1, 3, 4096, 4, 3, 40, None),          # M = 5120: 2048, 2048, 1024
    "p2_L3_straddle": (1, 2, 2400, 2, 3, 100, None),     # M = 3600: level 0 ends at 2400
    "p4_L4_ties": (1, 2, 8192, 4, 4, 256, 3),            # M = 10752, three score values
    "all_equal": (1, 1, 8192, 4, 4, 100, 1),
    "everything": (1, 2, 4096, 2, 2, 2048, None),        # Ksel = M = 4096
    "one_region": (1, 2, 1024, 4, 3, 16, None),          # M = 1280: the joint rule
}


@pytest.mark.parametrize("case", list(REGIONAL_CASES))
def test_regional_selection_on_seeded_scores(case):
    """Regional selection (LH_SELECT_REGIONAL) against the oracle's rule, bit
    for bit, including ties everywhere and the budget of every candidate."""
    from long_context_hierarchical_b200 import lh
    B, H, N, p, L, k, distinct = REGIONAL_CASES[case]
    sz = oracle.sizes(N, p, L, k)
    scores = make_scores(B, H, sz.M, seed=11, distinct=distinct)
    pl = lh.plan(B, H, N, 64, p, L, k, "bf16", select="regional")
    sel, inv = lh.topk(pl, scores.cuda())
    for h in range(H):
        mask = oracle.select_regional(scores[0, h].double().numpy(), sz)
        es, ei = oracle.order_selection(mask, sz)
        assert np.array_equal(sel[0, h].cpu().numpy(), es)
        assert np.array_equal(inv[0, h].cpu().numpy(), ei)
    lh.device_status()


def test_regional_whole_layer():
    """The whole layer with regional selection: selection bit-exact, output
    and gradients within the attention tolerances."""
    from long_context_hierarchical_b200 import lh
    B, H, N, p, L, k = 1, 2, 4096, 4, 3, 48
    Q, K, V, dO = make_inputs(B, H, N, 64, "bf16", seed=6)
    O_e, ctxs, sz, grads = oracle_layer(Q, K, V, dO, p, L, k, torch.bfloat16, rule="regional")
    terms = grad_tolerance_terms(ctxs, grads, sz)
    pl = lh.plan(B, H, N, 64, p, L, k, "bf16", select="regional")
    dev = [x.cuda() for x in (Q, K, V, dO)]
    O, ctx = lh.forward(pl, *dev[:3])
    g = lh.backward(pl, dev[3], ctx)
    torch.cuda.synchronize()
    assert np.array_equal(ctx.sel_idx.cpu().numpy(), stack(ctxs, "sel_idx"))
    assert np.array_equal(ctx.slot_of.cpu().numpy(), stack(ctxs, "slot_of"))
    assert_grad_close(np64(O), O_e, terms["O"], torch.bfloat16, "regional:O")
    for got, i, key in ((g[0], 0, "dQ"), (g[1], 1, "dK"), (g[2], 2, "dV")):
        assert_grad_close(np64(got), grads[i], terms[key], torch.bfloat16, f"regional:{key}")
    lh.device_status()


def test_descent_whole_layer():
    """The whole layer with descent selection: selection bit-exact, output
    and gradients within the attention tolerances."""
    from long_context_hierarchical_b200 import lh
    B, H, N, p, L, k = 1, 2, 2048, 4, 3, 24
    Q, K, V, dO = make_inputs(B, H, N, 64, "bf16", seed=4)
    O_e, ctxs, sz, grads = oracle_layer(Q, K, V, dO, p, L, k, torch.bfloat16, rule="descent")
    terms = grad_tolerance_terms(ctxs, grads, sz)
    pl = lh.plan(B, H, N, 64, p, L, k, "bf16", select="descent")
    dev = [x.cuda() for x in (Q, K, V, dO)]
    O, ctx = lh.forward(pl, *dev[:3])
    g = lh.backward(pl, dev[3], ctx)
    torch.cuda.synchronize()
    assert np.array_equal(ctx.sel_idx.cpu().numpy(), stack(ctxs, "sel_idx"))
    assert np.array_equal(ctx.slot_of.cpu().numpy(), stack(ctxs, "slot_of"))
    assert_grad_close(np64(O), O_e, terms["O"], torch.bfloat16, "descent:O")
    for got, i, key in ((g[0], 0, "dQ"), (g[1], 1, "dK"), (g[2], 2, "dV")):
        assert_grad_close(np64(got), grads[i], terms[key], torch.bfloat16, f"descent:{key}")
    lh.device_status()


def test_gather(case):
    c = case
    lh, pl, dt = c["lh"], c["pl"], c["dt"]
    pyr = [_t(_oracle_pyr(c, w), dt) for w in range(3)]
    sel = _t(stack(c["ctxs"], "sel_idx"), torch.int32)
    out = lh.gather(pl, c["Q"], c["K"], c["V"], pyr, sel)
    for w, key in enumerate(("Qg", "Kg", "Vg")):
        assert np.array_equal(np64(out[w]), stack(c["ctxs"], key)), key


def test_attention_forward(case):
    c = case
    lh, dt = c["lh"], c["dt"]
    Qg, Kg, Vg = (_t(stack(c["ctxs"], k), dt) for k in ("Qg", "Kg", "Vg"))
    Og, lse = lh.attn_fwd(Qg, Kg, Vg)
    assert_grad_close(np64(Og), stack(c["ctxs"], "Og"), c["terms"]["Og"], dt, f"{c['name']}:attn_fwd:Og",
                      own_og=False)
    lt = 1e-3 if dt == torch.bfloat16 else 1e-5
    assert np.max(np.abs(np64(lse) - stack(c["ctxs"], "lse"))) <= lt


def test_scatter(case):
    c = case
    lh, pl, dt = c["lh"], c["pl"], c["dt"]
    Og = _t(stack(c["ctxs"], "Og"), dt)
    inv = _t(stack(c["ctxs"], "slot_of"), torch.int32)
    O = lh.scatter(pl, Og, inv)
    assert_close(np64(O), c["O"], dt, "O")


def _grad_stack(c, key):
    return np.stack([np.stack([g[key] for g in row]) for row in c["grads"][3]])


def test_scatter_backward(case):
    c = case
    lh, pl, dt = c["lh"], c["pl"], c["dt"]
    Og = _t(stack(c["ctxs"], "Og"), dt)
    sel = _t(stack(c["ctxs"], "sel_idx"), torch.int32)
    dOg, D = lh.scatter_bwd(pl, c["dO"], Og, sel)
    assert_close(np64(dOg), _grad_stack(c, "dOg"), dt, "dOg")
    assert_close(np64(D), _grad_stack(c, "D"), dt, "D")


@pytest.mark.parametrize("deterministic", [False, True])
def test_attention_backward(case, deterministic):
    c = case
    lh, dt = c["lh"], c["dt"]
    Qg, Kg, Vg, Og = (_t(stack(c["ctxs"], k), dt) for k in ("Qg", "Kg", "Vg", "Og"))
    lse = _t(stack(c["ctxs"], "lse"), torch.float32)
    dOg = _t(_grad_stack(c, "dOg"), dt)
    D = _t(_grad_stack(c, "D"), torch.float32)
    lh.set_deterministic(deterministic)
    try:
        for Din in (D, None):
            dQg, dKg, dVg = lh.attn_bwd(Qg, Kg, Vg, Og, lse, dOg, Din)
            for got, key in ((dQg, "dQg"), (dKg, "dKg"), (dVg, "dVg")):
                assert_grad_close(np64(got), _grad_stack(c, key), c["terms"][key], dt,
                                  f"{c['name']}:attn_bwd{'_det' if deterministic else ''}:{key}",
                                  own_og=False)
    finally:
        lh.set_deterministic(False)
    lh.device_status()


def test_attention_backward_schedules_agree(case):
    """The fused schedule (dQ shares reduce-added in fp32) and the
    deterministic two-kernel one: dK, dV from the same kernel code are
    bit-identical; dQ agrees to the rounding of its terms (the fused kernel
    forms dS with lse and D folded into its MMAs, the dq kernel subtracts
    them in fp32, so a dS element may round to the neighbouring bf16 value,
    and the fp32 sums run in different orders); the deterministic schedule
    repeats bit for bit."""
    c = case
    lh, dt = c["lh"], c["dt"]
    Qg, Kg, Vg, Og = (_t(stack(c["ctxs"], k), dt) for k in ("Qg", "Kg", "Vg", "Og"))
    lse = _t(stack(c["ctxs"], "lse"), torch.float32)
    dOg = _t(_grad_stack(c, "dOg"), dt)
    fused = lh.attn_bwd(Qg, Kg, Vg, Og, lse, dOg, None)
    lh.set_deterministic(True)
    try:
        det = [lh.attn_bwd(Qg, Kg, Vg, Og, lse, dOg, None) for _ in range(2)]
    finally:
        lh.set_deterministic(False)
    for a, b in zip(det[0], det[1]):
        assert torch.equal(a, b)
    assert torch.equal(fused[1], det[0][1]) and torch.equal(fused[2], det[0][2])
    a, b = np64(fused[0]), np64(det[0][0])
    # one rounding step of the output, plus one bf16 rounding of each term
    # (dS differently rounded) within the term bound tq = sum |dS| |K| (and more)
    step = 2.0 ** -7 if dt == torch.bfloat16 else 2.0 ** -22
    tq = c["terms"]["dQg"].l1
    err = np.abs(a - b)
    bad = err > step * np.abs(b) + step / 2 * tq + 1e-30
    assert not bad.any(), f"dQg fused vs deterministic: {int(bad.sum())} elements, max {err.max():.3e}"


def test_gather_backward(case):
    c = case
    lh, pl, dt = c["lh"], c["pl"], c["dt"]
    dXg = [_t(_grad_stack(c, k), dt) for k in ("dQg", "dKg", "dVg")]
    inv = _t(stack(c["ctxs"], "slot_of"), torch.int32)
    dQ, dK, dV = lh.gather_bwd(pl, *dXg, inv)
    for got, exp, name in ((dQ, c["grads"][0], "dQ"), (dK, c["grads"][1], "dK"), (dV, c["grads"][2], "dV")):
        assert_close(np64(got), exp, dt, name)


def test_whole_layer(case):
    c = case
    lh, pl, dt = c["lh"], c["pl"], c["dt"]
    O, ctx = lh.forward(pl, c["Q"], c["K"], c["V"])
    dQ, dK, dV = lh.backward(pl, c["dO"], ctx)
    torch.cuda.synchronize()
    assert np.array_equal(ctx.sel_idx.cpu().numpy(), stack(c["ctxs"], "sel_idx"))
    assert np.array_equal(ctx.slot_of.cpu().numpy(), stack(c["ctxs"], "slot_of"))
    assert_grad_close(np64(O), c["O"], c["terms"]["O"], dt, f"{c['name']}:layer:O")
    for got, i, key in ((dQ, 0, "dQ"), (dK, 1, "dK"), (dV, 2, "dV")):
        assert_grad_close(np64(got), c["grads"][i], c["terms"][key], dt, f"{c['name']}:layer:{key}")
    # run to run: the forward, dK and dV bit-identical (the default fused
    # backward sums dQ with TMA reduce-adds in varying order); everything in
    # deterministic mode
    O2, ctx2 = lh.forward(pl, c["Q"], c["K"], c["V"])
    g2 = lh.backward(pl, c["dO"], ctx2)
    assert torch.equal(O, O2)
    assert torch.equal(dK, g2[1]) and torch.equal(dV, g2[2])
    lh.set_deterministic(True)
    try:
        g3 = lh.backward(pl, c["dO"], ctx2)
        g4 = lh.backward(pl, c["dO"], ctx2)
    finally:
        lh.set_deterministic(False)
    for got, i, key in ((g3[0], 0, "dQ"), (g3[1], 1, "dK"), (g3[2], 2, "dV")):
        assert_grad_close(np64(got), c["grads"][i], c["terms"][key], dt, f"{c['name']}:layer_det:{key}")
    for a, b in zip(g3, g4):
        assert torch.equal(a, b)
    lh.device_status()


@pytest.mark.parametrize("S", [1000, 2304])
def test_attention_with_growing_row_maxima(S):
    """Keys whose scale grows along the sequence make each query's running
    maximum rise by many powers of two across key tiles, so the forward's
    lazy rescaling of O (only when the maximum grows by more than 2^8) runs
    repeatedly; forward and backward against the oracle in fp64."""
    from long_context_hierarchical_b200 import lh
    BH = 2
    g = np.random.default_rng(7)
    ramp = (1.0 + 5.0 * np.arange(S) / S)[None, :, None]
    Q = oracle.round_bf16(g.standard_normal((BH, S, 64)))
    K = oracle.round_bf16(g.standard_normal((BH, S, 64)) * ramp)
    V = oracle.round_bf16(g.standard_normal((BH, S, 64)))
    dO = oracle.round_bf16(g.standard_normal((BH, S, 64)))
    dev = [_t(x, torch.bfloat16) for x in (Q, K, V, dO)]
    O, lse = lh.attn_fwd(*dev[:3])
    grads = lh.attn_bwd(*dev[:3], O, lse, dev[3], None)
    torch.cuda.synchronize()
    for b in range(BH):
        Oe, lse_e = oracle.causal_attention(Q[b], K[b], V[b])
        Ob = oracle.round_bf16(Oe)
        D = np.sum(dO[b] * Ob, axis=1)
        ge = oracle.causal_attention_bwd(Q[b], K[b], V[b], dO[b], lse_e, D)
        tb = grad_term_bounds(Q[b], K[b], V[b], Ob, lse_e, dO[b])
        assert np.max(np.abs(np64(lse[b]) - lse_e)) <= 1e-3
        assert_grad_close(np64(O[b]), Oe, tb["Og"], torch.bfloat16, f"ramp{S}:O (head {b})",
                          own_og=False)
        for got, exp, key in zip(grads, ge, ("dQg", "dKg", "dVg")):
            assert_grad_close(np64(got[b]), exp, tb[key], torch.bfloat16, f"ramp{S}:{key} (head {b})")
    lh.device_status()


def test_host_pipeline_matches_device_calls():
    """lh.HostPipeline (host tensors, copies overlapping the kernels, two device
    buffer sets) returns what lh.forward / lh.backward return on the device, for
    every step of a sequence with different inputs (deterministic mode: bit for bit)."""
    from long_context_hierarchical_b200 import lh
    B, H, N, p, L, k = 1, 4, 2048, 4, 3, 32
    pl = lh.plan(B, H, N, 64, p, L, k, "bf16")
    steps = [make_inputs(B, H, N, 64, "bf16", seed=20 + i) for i in range(3)]
    lh.set_deterministic(True)
    try:
        pipe = lh.HostPipeline(pl, "cuda")
        host_in = [tuple(x.pin_memory() for x in s) for s in steps]
        host_out = [tuple(torch.empty_like(x).pin_memory() for x in s) for s in steps]
        for hi, ho in zip(host_in, host_out):
            pipe.step(hi, ho)
        pipe.synchronize()
        for (Q, K, V, dO), ho in zip(steps, host_out):
            Qd, Kd, Vd, dOd = (x.cuda() for x in (Q, K, V, dO))
            O, ctx = lh.forward(pl, Qd, Kd, Vd)
            grads = lh.backward(pl, dOd, ctx)
            torch.cuda.synchronize()
            for got, exp in zip(ho, (O, *grads)):
                assert torch.equal(got, exp.cpu())
    finally:
        lh.set_deterministic(False)
    lh.device_status()


def test_dense_fixed_point_matches_attention():
    """L = 1: the layer is plain causal attention on Q, K, V (skill card, 选择-注意力解耦)."""
    from long_context_hierarchical_b200 import lh
    Q, K, V, _ = make_inputs(1, 4, 1024, 64, "bf16", seed=3, device="cuda", with_grad=False)
    pl = lh.plan(1, 4, 1024, 64, 4, 1, 0, "bf16")
    O, _ = lh.forward(pl, Q, K, V)
    Oa, _ = lh.attn_fwd(Q, K, V)
    assert torch.equal(O, Oa)
    ref = torch.nn.functional.scaled_dot_product_attention(Q.float(), K.float(), V.float(), is_causal=True)
    assert_close(np64(O), np64(ref), torch.bfloat16, "O vs SDPA")
