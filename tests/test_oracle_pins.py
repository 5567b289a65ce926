"""Pins of the CPU oracle to facts other than itself (CPU only).

Each check rests on something the pages or the mathematics fix: hand-worked
cases (tests/golden/hand_worked.json), brute force on tiny inputs, closed
forms, library routines for special cases, invariants the pages state, and
finite differences.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import lighthouse as lh

GOLDEN = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "hand_worked.json")))


def rng(seed=0):
    return np.random.default_rng(seed)


def rand_head(N, d, seed, scale=True):
    r = rng(seed)
    x = r.standard_normal((N, d))
    if scale:
        x *= np.exp(0.5 * r.standard_normal((N, 1)))
    return x


# --------------------------------------------------------------------------
# rounding
# --------------------------------------------------------------------------


def test_round_bf16_matches_torch_on_fp32_values():
    r = rng(1)
    x = (r.standard_normal(100000) * np.exp(3 * r.standard_normal(100000))).astype(np.float32)
    ref = torch.from_numpy(x).to(torch.bfloat16).to(torch.float64).numpy()
    got = lh.round_bf16(x.astype(np.float64))
    assert np.array_equal(got, ref)


def test_round_bf16_halfway_and_direct_rounding():
    # 1 + 2^-8 is halfway between 1 and 1 + 2^-7: ties to even -> 1.
    assert lh.round_bf16(np.array([1 + 2.0 ** -8]))[0] == 1.0
    # 1 + 3*2^-8 is halfway between 1 + 2^-7 (odd) and 1 + 2^-6 (even).
    assert lh.round_bf16(np.array([1 + 3 * 2.0 ** -8]))[0] == 1 + 2.0 ** -6
    # Just above halfway must round up, which a detour through fp32 would miss.
    assert lh.round_bf16(np.array([1 + 2.0 ** -8 + 2.0 ** -40]))[0] == 1 + 2.0 ** -7
    # Negative values round symmetrically; exact values are kept.
    assert lh.round_bf16(np.array([-(1 + 3 * 2.0 ** -8)]))[0] == -(1 + 2.0 ** -6)
    assert lh.round_bf16(np.array([0.15625]))[0] == 0.15625


# --------------------------------------------------------------------------
# sizes
# --------------------------------------------------------------------------


@pytest.mark.parametrize("N,p,L,k,S", [
    (1024, 4, 3, 32, 320),
    (8192, 4, 4, 256, 3200),
    (98304, 4, 3, 1536, 18432),
    (98304, 4, 3, 6144, 55296),
    (524288, 4, 4, 2048, 32768),
])
def test_sizes_of_the_workloads(N, p, L, k, S):
    sz = lh.sizes(N, p, L, k)
    assert sz.S == N // p ** (L - 1) + (L - 1) * p * k == S
    # total pyramid entries <= N p / (p - 1)  (skill card, stage 1)
    assert sz.Ntot * (p - 1) <= N * p
    assert sz.Ksel <= sz.M


def test_sizes_reject_bad_configs():
    with pytest.raises(ValueError):
        lh.sizes(1000, 4, 3, 1)        # N not a multiple of p^(L-1)
    with pytest.raises(ValueError):
        lh.sizes(64, 4, 3, 100)        # budget above the candidate count
    with pytest.raises(ValueError):
        lh.sizes(64, 1, 2, 1)


# --------------------------------------------------------------------------
# stage 1: pyramid
# --------------------------------------------------------------------------


def test_pyramid_hand_worked():
    g = GOLDEN["pyramid_means"]
    sz = lh.sizes(g["N"], g["p"], g["L"], 0)
    levels = lh.pyramid(np.array(g["X"], float), sz, "f64")
    for got, exp in zip(levels, g["levels"]):
        assert np.array_equal(got, np.array(exp, float))


@pytest.mark.parametrize("p,L", [(2, 4), (4, 3), (3, 3)])
def test_pyramid_brute_force_means(p, L):
    N, d = p ** (L - 1) * 3, 5
    X = rand_head(N, d, 7)
    sz = lh.sizes(N, p, L, 0)
    levels = lh.pyramid(X, sz, "f64")
    for l in range(L):
        P = p ** l
        for i in range(N // P):
            for c in range(d):
                ref = math.fsum(X[t, c] for t in range(i * P, (i + 1) * P)) / P
                assert abs(levels[l][i, c] - ref) <= 1e-14 * max(1.0, abs(ref))


def test_pyramid_levels_nest():
    # level l entry = mean of p level-(l-1) entries, in exact arithmetic
    # (integer inputs make every mean an exact dyadic value).
    p, L, N, d = 4, 4, 256, 8
    X = rng(3).integers(-50, 50, size=(N, d)).astype(float)
    sz = lh.sizes(N, p, L, 0)
    levels = lh.pyramid(X, sz, "f64")
    for l in range(1, L):
        prev = levels[l - 1].reshape(-1, p, d).mean(axis=1)
        assert np.array_equal(levels[l], prev)


def test_pyramid_rounds_once_to_bf16():
    p, L, N, d = 4, 3, 64, 8
    X = lh.round_bf16(rand_head(N, d, 9))
    sz = lh.sizes(N, p, L, 0)
    lv = lh.pyramid(X, sz, "bf16")
    ex = lh.pyramid(X, sz, "f64")
    for l in range(1, L):
        assert np.array_equal(lv[l], lh.round_bf16(ex[l]))
        assert np.all(np.abs(lv[l] - ex[l]) <= np.abs(ex[l]) * 2.0 ** -8 + 1e-300)


# --------------------------------------------------------------------------
# stage 2: scores and selection
# --------------------------------------------------------------------------


def test_norm_sum_closed_form():
    g = GOLDEN["norm_sum"]
    s = lh.level0_scores(np.array([g["q"]], float), np.array([g["k"]], float))
    assert s[0] == g["score"]


def test_scores_brute_force_and_max_inheritance():
    p, L, N, d = 2, 4, 32, 6
    Q, K = rand_head(N, d, 1), rand_head(N, d, 2)
    sz = lh.sizes(N, p, L, 1)
    s0 = lh.level0_scores(Q, K)
    for t in range(N):
        ref = math.sqrt(math.fsum(q * q for q in Q[t])) + math.sqrt(math.fsum(k * k for k in K[t]))
        assert s0[t] == float(np.float32(ref))
    cand = lh.candidate_scores(s0, sz)
    assert cand.size == sz.M
    for l in range(L - 1):
        for i in range(sz.n[l]):
            span = s0[i * p ** l:(i + 1) * p ** l]
            assert cand[sz.flat_off[l] + i] == max(span)


def test_select_order_scatter_hand_worked():
    g = GOLDEN["select_order_scatter"]
    sz = lh.sizes(g["N"], g["p"], g["L"], g["k"])
    assert sz.S == g["S"]
    s0 = np.array(g["s0"], float)
    # Q_t = (s0[t], 0, ...), K_t = 0 gives exactly these level-0 scores.
    Q = np.zeros((g["N"], 4)); Q[:, 0] = s0
    assert np.array_equal(lh.level0_scores(Q, np.zeros_like(Q)), s0)
    cand = lh.candidate_scores(s0, sz)
    assert cand.tolist() == g["cand"]
    sel_idx, slot_of = lh.order_selection(lh.select(cand, sz), sz)
    assert sel_idx.tolist() == g["sel_idx"]
    assert slot_of.tolist() == g["slot_of"]
    # scatter: slot j carries the one-hot value e_j
    Og = np.eye(sz.S)
    O = lh.scatter(Og, slot_of, sz, "f64")
    for t, slots in enumerate(g["scatter_slots"]):
        exp = np.zeros(sz.S); exp[slots] = 1
        assert np.array_equal(O[t], exp)
    # scatter backward: token t carries e_t
    dOg = lh.scatter_bwd(np.eye(sz.N), sel_idx, sz, "f64")
    for j, (lo, hi) in enumerate(g["scatter_bwd_ranges"]):
        exp = np.zeros(sz.N); exp[lo:hi + 1] = 1
        assert np.array_equal(dOg[j], exp)
    # gather backward: slot j carries e_j
    dX = lh.gather_bwd(np.eye(sz.S), slot_of, sz, "f64")
    for t, terms in enumerate(g["gather_bwd_terms"]):
        exp = np.zeros(sz.S)
        for j, w in terms:
            exp[j] += w
        assert np.array_equal(dX[t], exp)


@pytest.mark.parametrize("case", ["all_equal_ties", "structural_ties"])
def test_tie_rule_hand_worked(case):
    g = GOLDEN[case]
    sz = lh.sizes(g["N"], g["p"], g["L"], g["k"])
    cand = lh.candidate_scores(np.array(g["s0"], float), sz)
    sel_idx, _ = lh.order_selection(lh.select(cand, sz), sz)
    assert sel_idx.tolist() == g["sel_idx"]


@pytest.mark.parametrize("seed,distinct", [(0, None), (1, 5), (2, 2)])
def test_select_full_sort_brute_force(seed, distinct):
    p, L, N, k = 2, 4, 64, 3
    sz = lh.sizes(N, p, L, k)
    r = rng(seed)
    if distinct is None:
        s0 = r.random(N).astype(np.float32).astype(float)
    else:
        s0 = r.integers(0, distinct, N).astype(float)
    cand = lh.candidate_scores(s0, sz)
    mask = lh.select(cand, sz)
    ranked = sorted(range(sz.M), key=lambda f: (-cand[f], f))
    exp = set(ranked[:sz.Ksel]) | set(range(sz.flat_off[L - 1], sz.Ntot))
    assert set(np.nonzero(mask)[0].tolist()) == exp
    assert mask.sum() == sz.S


def test_selection_invariants_random():
    p, L, N, k = 4, 4, 1024, 8
    sz = lh.sizes(N, p, L, k)
    Q, K = rand_head(N, 8, 4), rand_head(N, 8, 5)
    cand, sel_idx, slot_of = lh.head_select(Q, K, sz)
    assert sel_idx.size == sz.S
    # coarsest level always present
    assert set(range(sz.flat_off[L - 1], sz.Ntot)) <= set(sel_idx.tolist())
    # strictly increasing (end, level)
    lev, idx = lh.entry_level_index(sel_idx, sz)
    end = (idx + 1) * np.array(sz.P)[lev] - 1
    keys = list(zip(end.tolist(), lev.tolist()))
    assert all(a < b for a, b in zip(keys, keys[1:]))
    # upward closure: a parent's score is the max over its span, so the parent
    # of every selected candidate scores at least the selection threshold.
    chosen = set(sel_idx.tolist())
    thr = min(cand[f] for f in chosen if f < sz.M)
    for f in chosen:
        if f >= sz.flat_off[L - 2]:
            continue
        l, i = sz.level_of(f)
        parent = sz.flat_off[l + 1] + i // p
        assert cand[parent] >= thr


def test_descent_hand_worked():
    """Hierarchical descent (reading R8) on a hand-worked case, which the joint
    rule selects differently."""
    g = GOLDEN["descent"]
    sz = lh.sizes(g["N"], g["p"], g["L"], g["k"])
    cand = lh.candidate_scores(np.array(g["s0"], float), sz)
    sel_idx, _ = lh.order_selection(lh.select_descent(cand, sz), sz)
    assert sel_idx.tolist() == g["sel_idx"]
    joint, _ = lh.order_selection(lh.select(cand, sz), sz)
    assert joint.tolist() == g["joint_sel_idx"]
    t = GOLDEN["descent_ties"]
    sz = lh.sizes(t["N"], t["p"], t["L"], t["k"])
    cand = lh.candidate_scores(np.array(t["s0"], float), sz)
    sel_idx, _ = lh.order_selection(lh.select_descent(cand, sz), sz)
    assert sel_idx.tolist() == t["sel_idx"]


@pytest.mark.parametrize("p", [2, 4])
def test_descent_two_levels_is_best_blocks(p):
    """L = 2: the level-0 tokens kept are exactly the spans of the k blocks
    with the largest maximum token score (ties to the lower block)."""
    N, k = 64 * p, 5
    sz = lh.sizes(N, p, 2, k)
    s0 = rng(3).integers(0, 6, N).astype(float)
    mask = lh.select_descent(lh.candidate_scores(s0, sz), sz)
    blocks = sorted(range(N // p), key=lambda b: (-max(s0[b * p:(b + 1) * p]), b))[:k]
    exp = {b * p + c for b in blocks for c in range(p)} | set(range(sz.flat_off[1], sz.Ntot))
    assert set(np.nonzero(mask)[0].tolist()) == exp


@pytest.mark.parametrize("p,L,k,distinct", [(2, 4, 3, None), (4, 3, 4, 3), (2, 5, 2, 2), (4, 4, 2, None)])
def test_descent_invariants_random(p, L, k, distinct):
    """Per finer level exactly p*k entries; each is a child of an entry one
    level up that is kept; those parents are the k best of their level's
    kept entries under (score desc, index asc)."""
    N = 64 * p ** (L - 1)
    sz = lh.sizes(N, p, L, k)
    r = rng(11)
    s0 = r.random(N) if distinct is None else r.integers(0, distinct, N).astype(float)
    cand = lh.candidate_scores(s0, sz)
    mask = lh.select_descent(cand, sz)
    assert mask.sum() == sz.S
    assert mask[sz.flat_off[L - 1]:].all()
    # scores of every level, by max-pooling level 0 directly
    score = [s0.reshape(sz.n[l], sz.P[l]).max(axis=1) for l in range(L)]
    for l in range(L - 1):
        kept = np.nonzero(mask[sz.flat_off[l]:sz.flat_off[l + 1]])[0]
        assert kept.size == p * k
        parents = np.unique(kept // p)
        assert parents.size == k and np.array_equal(np.sort(kept), np.sort((parents[:, None] * p + np.arange(p)).ravel()))
        up = np.nonzero(mask[sz.flat_off[l + 1]:sz.flat_off[l + 2]])[0]  # kept entries one level up
        assert set(parents.tolist()) <= set(up.tolist())
        ranked = sorted(up.tolist(), key=lambda i: (-score[l + 1][i], i))
        assert set(ranked[:k]) == set(parents.tolist())


@pytest.mark.parametrize("p", [2, 4])
def test_descent_and_joint_agree_when_everything_is_kept(p):
    """L = 2 with k = N/p: both rules keep every entry of both levels, so the
    gathered sub-sequence is the whole pyramid in (end, level) order."""
    N = 16 * p
    sz = lh.sizes(N, p, 2, N // p)
    s0 = rng(5).random(N)
    cand = lh.candidate_scores(s0, sz)
    a, _ = lh.order_selection(lh.select(cand, sz), sz)
    b, _ = lh.order_selection(lh.select_descent(cand, sz), sz)
    assert np.array_equal(a, b) and a.size == sz.Ntot == sz.S


def test_descent_needs_k_within_the_coarsest_level():
    sz = lh.sizes(64, 2, 4, 9)  # n_3 = 8 < k
    with pytest.raises(ValueError):
        lh.select_descent(np.zeros(sz.M), sz)


def test_regional_hand_worked():
    """The regional rule on the hand-worked scores, regions of 4 entries:
    quotas 1, 1, 1 and one more entry from the best leftovers (a tie at 6
    goes to the lower flat index 7)."""
    g = GOLDEN["regional_select"]
    sz = lh.sizes(g["N"], g["p"], g["L"], g["k"])
    cand = np.array(g["cand"], float)
    mask = lh.select_regional(cand, sz, region=g["region"])
    kept = sorted(g["kept_by_region"] + g["kept_by_remainder"])
    assert np.nonzero(mask[: sz.M])[0].tolist() == kept
    assert lh.order_selection(mask, sz)[0].tolist() == g["sel_idx"]
    # the joint rule keeps entry 11 instead of entry 1 on the same scores
    assert not np.array_equal(lh.select(cand, sz), mask)


@pytest.mark.parametrize("region", [1 << 20, 2048])
def test_regional_is_joint_with_one_region(region):
    """With a single region the quota is the whole budget: the joint rule."""
    N, p, L, k = 1024, 4, 3, 16     # M = 1280 <= 2048
    sz = lh.sizes(N, p, L, k)
    cand = lh.candidate_scores(lh.level0_scores(rand_head(N, 8, 1), rand_head(N, 8, 2)), sz)
    assert np.array_equal(lh.select_regional(cand, sz, region=region), lh.select(cand, sz))


@pytest.mark.parametrize("N,p,L,k,region,distinct", [
    (4096, 4, 3, 40, 512, None), (2400, 2, 3, 100, 2048, None), (4096, 4, 4, 30, 700, 3),
    (2048, 2, 2, 1024, 300, None), (8192, 4, 4, 256, 2048, 1)])
def test_regional_invariants(N, p, L, k, region, distinct):
    """Exactly Ksel candidates; every region keeps at least its quota, and
    its quota best entries (by score, then lower index) are among them; the
    entries kept beyond the quotas beat every entry left out."""
    sz = lh.sizes(N, p, L, k)
    r = rng(N + region)
    cand = r.standard_normal(sz.M)
    if distinct:
        cand = np.floor(r.random(sz.M) * distinct)
    mask = lh.select_regional(cand, sz, region=region)
    kept = mask[: sz.M]
    assert kept.sum() == sz.Ksel and mask[sz.M:].all()
    key = lambda f: (-cand[f], f)
    extra_kept, left_out = [], []
    for a in range(0, sz.M, region):
        b = min(sz.M, a + region)
        quota = sz.Ksel * (b - a) // sz.M
        order = sorted(range(a, b), key=key)
        assert kept[order[:quota]].all()
        extra_kept += [f for f in order[quota:] if kept[f]]
        left_out += [f for f in order[quota:] if not kept[f]]
    if extra_kept and left_out:
        assert max(key(f) for f in extra_kept) < min(key(f) for f in left_out)


# --------------------------------------------------------------------------
# stage 3: attention
# --------------------------------------------------------------------------


def test_attention_matches_torch_sdpa_fp64():
    S, d = 77, 16
    Q, K, V = rand_head(S, d, 1), rand_head(S, d, 2), rand_head(S, d, 3)
    O, lse = lh.causal_attention(Q, K, V)
    t = lambda a: torch.from_numpy(a)[None, None]
    ref = torch.nn.functional.scaled_dot_product_attention(t(Q), t(K), t(V), is_causal=True)[0, 0]
    assert np.allclose(O, ref.numpy(), rtol=1e-12, atol=1e-12)
    # LSE from its definition on a few rows
    for r in (0, 5, 76):
        s = Q[r] @ K[: r + 1].T / math.sqrt(d)
        assert abs(lse[r] - math.log(math.fsum(math.exp(x) for x in s))) < 1e-10
    rows = [0, 3, 40, 76]
    Or, lr = lh.attention_rows(Q, K, V, rows)
    assert np.allclose(Or, O[rows], rtol=1e-12, atol=1e-12)
    assert np.allclose(lr, lse[rows], rtol=1e-12, atol=1e-12)


def test_attention_rows_sum_to_one():
    S, d = 50, 8
    Q, K = rand_head(S, d, 4), rand_head(S, d, 5)
    O, _ = lh.causal_attention(Q, K, np.ones((S, 3)))
    assert np.allclose(O, 1.0, atol=1e-13)


def test_L1_is_dense_causal_sdpa():
    """Disabling selection recovers the dense baseline (skill card, 选择-注意力解耦)."""
    N, d = 96, 16
    Q, K, V = rand_head(N, d, 1), rand_head(N, d, 2), rand_head(N, d, 3)
    sz = lh.sizes(N, 4, 1, 0)
    assert sz.S == N
    ctx = lh.head_forward(Q, K, V, sz, "f64")
    assert np.array_equal(ctx["sel_idx"], np.arange(N))
    t = lambda a: torch.from_numpy(a)[None, None].requires_grad_(True)
    q, k, v = t(Q), t(K), t(V)
    ref = torch.nn.functional.scaled_dot_product_attention(q, k, v, is_causal=True)
    assert np.allclose(ctx["O"], ref[0, 0].detach().numpy(), rtol=1e-12, atol=1e-12)
    dO = rand_head(N, d, 4, scale=False)
    ref.backward(torch.from_numpy(dO)[None, None])
    g = lh.head_backward(ctx, dO, sz, "f64")
    assert np.allclose(g["dQ"], q.grad[0, 0].numpy(), rtol=1e-10, atol=1e-10)
    assert np.allclose(g["dK"], k.grad[0, 0].numpy(), rtol=1e-10, atol=1e-10)
    assert np.allclose(g["dV"], v.grad[0, 0].numpy(), rtol=1e-10, atol=1e-10)


# --------------------------------------------------------------------------
# stage 4: scatter invariants
# --------------------------------------------------------------------------


def test_fan_in_and_coverage():
    p, L, N, k = 4, 4, 1024, 8
    sz = lh.sizes(N, p, L, k)
    _, sel_idx, slot_of = lh.head_select(rand_head(N, 8, 1), rand_head(N, 8, 2), sz)
    cover = lh.scatter(np.ones((sz.S, 1)), slot_of, sz, "f64")[:, 0]
    assert cover.max() <= L
    P = p ** (L - 1)
    assert np.all(cover[P - 1:] >= 1)           # coarsest level reaches every t >= p^(L-1) - 1
    # uncovered positions can only be t < p^(L-1) - 1
    assert np.all(np.nonzero(cover == 0)[0] < P - 1)


def test_offset_causality_frozen_selection():
    """Perturbing tokens after t leaves O[0..t] bit-identical (skill card, stage 4)."""
    p, L, N, k, d = 2, 4, 128, 4, 8
    sz = lh.sizes(N, p, L, k)
    Q, K, V = rand_head(N, d, 1), rand_head(N, d, 2), rand_head(N, d, 3)
    base = lh.head_forward(Q, K, V, sz, "bf16")
    sel = (base["sel_idx"], base["slot_of"])
    for t in (0, 7, 50, 100):
        Q2, K2, V2 = Q.copy(), K.copy(), V.copy()
        r = rng(t)
        Q2[t + 1:] += r.standard_normal(Q2[t + 1:].shape)
        K2[t + 1:] += r.standard_normal(K2[t + 1:].shape)
        V2[t + 1:] += r.standard_normal(V2[t + 1:].shape)
        out = lh.head_forward(Q2, K2, V2, sz, "bf16", selection=sel)
        assert np.array_equal(out["O"][: t + 1], base["O"][: t + 1])
        assert not np.array_equal(out["O"][t + 1:], base["O"][t + 1:])


# --------------------------------------------------------------------------
# backward
# --------------------------------------------------------------------------


def test_adjoint_identities():
    p, L, N, k, d = 2, 4, 64, 2, 3
    sz = lh.sizes(N, p, L, k)
    _, sel_idx, slot_of = lh.head_select(rand_head(N, 4, 1), rand_head(N, 4, 2), sz)
    x = rand_head(sz.S, d, 3, scale=False)
    y = rand_head(N, d, 4, scale=False)
    lhs = np.sum(lh.scatter(x, slot_of, sz, "f64") * y)
    rhs = np.sum(x * lh.scatter_bwd(y, sel_idx, sz, "f64"))
    assert abs(lhs - rhs) < 1e-12 * max(1, abs(lhs))
    # pyramid + gather vs gather_bwd
    X = rand_head(N, d, 5, scale=False)
    Yg = rand_head(sz.S, d, 6, scale=False)
    Xg = lh.gather(lh.pyramid(X, sz, "f64"), sel_idx, sz)
    lhs = np.sum(Xg * Yg)
    rhs = np.sum(X * lh.gather_bwd(Yg, slot_of, sz, "f64"))
    assert abs(lhs - rhs) < 1e-12 * max(1, abs(lhs))


def test_finite_difference_gradients():
    p, L, N, k, d = 2, 3, 16, 1, 4
    sz = lh.sizes(N, p, L, k)
    Q, K, V = rand_head(N, d, 1), rand_head(N, d, 2), rand_head(N, d, 3)
    dO = rand_head(N, d, 4, scale=False)
    ctx = lh.head_forward(Q, K, V, sz, "f64")
    sel = (ctx["sel_idx"], ctx["slot_of"])
    g = lh.head_backward(ctx, dO, sz, "f64")
    loss = lambda q, kk, v: np.sum(lh.head_forward(q, kk, v, sz, "f64", selection=sel)["O"] * dO)
    h = 1e-6
    for name, X, grad in (("Q", Q, g["dQ"]), ("K", K, g["dK"]), ("V", V, g["dV"])):
        for (t, c) in itertools.product(range(0, N, 3), range(d)):
            Xp, Xm = X.copy(), X.copy()
            Xp[t, c] += h
            Xm[t, c] -= h
            args_p = [Q, K, V]; args_m = [Q, K, V]
            i = "QKV".index(name)
            args_p[i] = Xp; args_m[i] = Xm
            fd = (loss(*args_p) - loss(*args_m)) / (2 * h)
            assert abs(fd - grad[t, c]) <= 1e-6 * max(1.0, abs(fd)), (name, t, c, fd, grad[t, c])


def test_attention_bwd_rows_equals_the_full_backward():
    """The restricted backward (some dQg rows, some dKg / dVg rows) equals the
    same rows of the full one, which finite differences and torch autograd
    pin (test_finite_difference_gradients, test_L1_is_dense_causal_sdpa)."""
    S, d = 600, 16
    Q, K, V = rand_head(S, d, 11), rand_head(S, d, 12), rand_head(S, d, 13)
    dO = rand_head(S, d, 14, scale=False)
    O, lse = lh.causal_attention(Q, K, V)
    D = np.sum(dO * O, axis=1)
    fq, fk, fv = lh.causal_attention_bwd(Q, K, V, dO, lse, D)
    rows, cols = [0, 1, 127, 128, 300, 511, 512, 599], [0, 5, 127, 128, 450, 598, 599]
    q, k, v = lh.attention_bwd_rows(Q, K, V, dO, lse, D, rows, cols)
    for got, full, idx in ((q, fq, rows), (k, fk, cols), (v, fv, cols)):
        ref = full[idx]
        assert np.allclose(got, ref, rtol=1e-12, atol=1e-12 * np.abs(ref).max())


def _rounding_case(d=8, seed=3):
    """The hand-worked selection case (N=8, p=2, L=3, k=1) with inputs that
    give exactly its level-0 scores: K_t has norm 5/8 (a 3-4-5 direction that
    changes from token to token) and Q_t = (s0[t] - 5/8) e_0, all values exact
    in bf16; V and dO are seeded bf16 values."""
    g = GOLDEN["select_order_scatter"]
    N = g["N"]
    s0 = np.array(g["s0"], float)
    dirs = [(3, 4), (4, 3), (-3, 4), (4, -3), (-4, -3), (-3, -4), (3, -4), (-4, 3)]
    K = np.zeros((N, d))
    K[:, :2] = np.array(dirs, float) / 8
    Q = np.zeros((N, d))
    Q[:, 0] = s0 - 0.625
    r = rng(seed)
    V = lh.round_bf16(r.standard_normal((N, d)))
    dO = lh.round_bf16(r.standard_normal((N, d)))
    sz = lh.sizes(N, g["p"], g["L"], g["k"])
    ctx = lh.head_forward(Q, K, V, sz, "bf16")
    assert ctx["sel_idx"].tolist() == g["sel_idx"]
    return g, sz, ctx, dO, lh.head_backward(ctx, dO, sz, "bf16")


def test_backward_rounds_dOg_once_from_the_range_sums():
    """dOg (the MMA operand dO~) is the exact sum of dO over R(l, i), rounded
    once to bf16; the ranges are the hand-worked ones."""
    g, sz, ctx, dO, b = _rounding_case()
    exact = np.array([[math.fsum(dO[lo:hi + 1, c]) for c in range(dO.shape[1])]
                      for lo, hi in g["scatter_bwd_ranges"]])
    assert np.array_equal(b["dOg"], lh.round_bf16(exact))
    assert not np.array_equal(lh.round_bf16(exact), exact)  # the rounding matters here


def test_backward_forms_D_from_the_stored_operands():
    """D_j = sum_c dOg_jc Og_jc with both factors as stored (bf16), not from the
    unrounded range sums."""
    g, sz, ctx, dO, b = _rounding_case()
    assert np.array_equal(ctx["Og"], lh.round_bf16(ctx["Og"]))
    D = [math.fsum(b["dOg"][j] * ctx["Og"][j]) for j in range(sz.S)]
    assert np.allclose(b["D"], D, rtol=1e-15, atol=1e-15)
    exact = np.array([[math.fsum(dO[lo:hi + 1, c]) for c in range(dO.shape[1])]
                      for lo, hi in g["scatter_bwd_ranges"]])
    D_unrounded = [math.fsum(exact[j] * ctx["Og"][j]) for j in range(sz.S)]
    assert np.max(np.abs(np.array(D_unrounded) - b["D"])) > 1e-6


def test_backward_rounds_gathered_gradients_before_the_pool_backward():
    """dQg, dKg, dVg are stored in bf16 and the per-token gradient sums the
    stored values with the hand-worked weights 1/p^l, rounding once at the
    end; summing the unrounded values first gives different bits."""
    g, sz, ctx, dO, b = _rounding_case()
    exact = lh.causal_attention_bwd(ctx["Qg"], ctx["Kg"], ctx["Vg"], b["dOg"], ctx["lse"], b["D"])
    differs = False
    for key, full in zip(("dQ", "dK", "dV"), exact):
        stored = b[key + "g"]
        assert np.array_equal(stored, lh.round_bf16(full))
        want = np.zeros_like(b[key])
        alt = np.zeros_like(b[key])
        for t, terms in enumerate(g["gather_bwd_terms"]):
            for c in range(stored.shape[1]):
                want[t, c] = math.fsum(w * stored[j, c] for j, w in terms)
                alt[t, c] = math.fsum(w * full[j, c] for j, w in terms)
        assert np.array_equal(b[key], lh.round_bf16(want))
        differs |= not np.array_equal(lh.round_bf16(alt), b[key])
    assert differs, "the case does not tell the two rounding orders apart"


def test_planted_mistakes_are_caught():
    """A transposed operand or a dropped term in the oracle fails a pin."""
    p, L, N, k, d = 2, 3, 16, 1, 4
    sz = lh.sizes(N, p, L, k)
    _, sel_idx, slot_of = lh.head_select(rand_head(N, 4, 1), rand_head(N, 4, 2), sz)
    x = rand_head(sz.S, d, 3, scale=False)
    y = rand_head(N, d, 4, scale=False)
    # planted: scatter without the p^l - 1 offset (R(l,i) starting at i*p^l)
    def bad_scatter(Og):
        O = np.zeros((N, d))
        for l in range(L):
            t = np.arange(N)
            s = slot_of[sz.flat_off[l] + t // sz.P[l]]
            O[s >= 0] += Og[s[s >= 0]]
        return O
    lhs = np.sum(bad_scatter(x) * y)
    rhs = np.sum(x * lh.scatter_bwd(y, sel_idx, sz, "f64"))
    assert abs(lhs - rhs) > 1e-6
