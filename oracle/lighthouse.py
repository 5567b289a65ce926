"""Lighthouse Attention oracle: a plain, slow fp64 CPU restatement of the layer.

TEST INFRASTRUCTURE.  Only the tests, the package smoke check and the CPU
baseline leg of the benchmark may import this module.  It shares no code with
the CUDA path (it never imports the package); both sides only receive the same
seeded inputs.

What it follows (page title, section):
  [card]  skill card "lighthouse-attention" (skillsmp.com): stages 1-4
          ("阶段 1 金字塔构建" ... "阶段 4 Scatter-back 重建"), "梯度流",
          "Complexity Analysis".
  [gist]  gist.science, "Long Context Pre-Training with Lighthouse Attention",
          Technical Summary section 2 (A. Symmetric Pyramid Construction,
          B. Parameter-Free Scoring and Selection, C. Dense Sub-Sequence
          Attention).
  [it]    gist.science/it, "Riepilogo Tecnico", section 2 A-C (same content).

Every step runs in fp64.  ``mode`` names the storage type of the layer
("bf16", "f32" or "f64"); values are rounded to it exactly where the layer
stores a tensor (pyramid levels, the attention output, the scattered output,
the gathered gradients and the final gradients), and nowhere else.  "f64"
disables all rounding; the finite-difference pins use it.

Readings of points the pages leave open (each marked READING below):
  R1 score combination: s = ||Q_t||_2 + ||K_t||_2 per level-0 token, rounded
     to fp32, then max-pooled to coarser levels.
  R2 the budget: a joint top-K of (L-1)*p*k entries over levels 0..L-2, plus
     every coarsest-level entry.
  R3 ties: equal scores go to the lower level-major flat index.
  R4 gathered order: by span end, then by level (finer first).
  R5 uncovered output positions are 0; R(l, i) is clipped to N-1.
  R6 selection is per (batch, head).
  R7 scatter sums levels in ascending order, without atomics.
  R8 (alternative selection, rule "descent") hierarchical descent: keep
     every coarsest entry; at the coarsest level pick the k best entries,
     keep their p children one level down, pick the k best of those, and so
     on to level 0.  Another reading of the budget (L-1)*p*k: p*k entries per
     finer level.  Needs k <= N/p^(L-1).  Coarse scores are the same
     max-pools as in R1; ties as in R3.
  R9 (alternative selection, rule "regional") every region contributes: the
     candidate score stream (level-major flat order) is cut into regions of
     2048 entries (the pages' chunk size, the last one ragged); region c
     keeps its floor(Ksel * |c| / M) best entries, and the Ksel - sum of
     those go to the best of all entries not yet kept.  Ties as in R3.  The
     budget and S stay those of R2.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

# ---------------------------------------------------------------------------
# Rounding to the storage type
# ---------------------------------------------------------------------------


def round_bf16(x):
    """Round fp64 values to the nearest bfloat16 value, ties to even.

    bfloat16 keeps 8 significant bits; an fp64 value keeps 53, so 45 low bits
    of the fp64 significand are dropped with round-to-nearest-even.  The
    result is returned as fp64.  (Finite values in the normal bf16 range;
    bf16 subnormals and overflow are outside what the layer produces.)
    """
    a = np.ascontiguousarray(np.asarray(x, dtype=np.float64))
    u = a.view(np.uint64).copy()
    drop = np.uint64(45)
    lsb = (u >> drop) & np.uint64(1)
    u = u + (np.uint64((1 << 44) - 1) + lsb)
    u = u & ~np.uint64((1 << 45) - 1)
    return u.view(np.float64).reshape(a.shape)


def round_f32(x):
    return np.asarray(x, dtype=np.float64).astype(np.float32).astype(np.float64)


def round_to(x, mode: str):
    if mode == "bf16":
        return round_bf16(x)
    if mode == "f32":
        return round_f32(x)
    if mode == "f64":
        return np.asarray(x, dtype=np.float64)
    raise ValueError(f"unknown mode {mode!r}")


# ---------------------------------------------------------------------------
# Sizes
# ---------------------------------------------------------------------------


@dataclass
class Sizes:
    N: int
    p: int
    L: int
    k: int
    P: list = field(default_factory=list)      # P[l] = p**l tokens per level-l entry
    n: list = field(default_factory=list)      # n[l] = N / p**l entries at level l
    flat_off: list = field(default_factory=list)  # level-major flat offsets, len L+1
    Ntot: int = 0   # all pyramid entries
    M: int = 0      # candidates: levels 0..L-2
    Ksel: int = 0   # jointly selected candidates
    S: int = 0      # gathered length

    def level_of(self, f: int):
        """Level and in-level index of a level-major flat index."""
        for l in range(self.L):
            if f < self.flat_off[l + 1]:
                return l, f - self.flat_off[l]
        raise IndexError(f)


def sizes(N: int, p: int, L: int, k: int) -> Sizes:
    """Pyramid and selection sizes.

    Levels 0..L-1, level l averages p**l tokens [card, 阶段 1].  The gathered
    length is S = N/p^(L-1) + (L-1)*p*k [card, 阶段 3]; the coarsest level is
    always kept and the rest of the budget is chosen from finer levels
    [card, 阶段 2] (READING R2).
    """
    if L < 1 or p < 2 or N < 1 or k < 0:
        raise ValueError("need L >= 1, p >= 2, N >= 1, k >= 0")
    if N % (p ** (L - 1)) != 0:
        raise ValueError("N must be a multiple of p^(L-1)")
    sz = Sizes(N, p, L, k)
    sz.P = [p ** l for l in range(L)]
    sz.n = [N // P for P in sz.P]
    sz.flat_off = [0]
    for l in range(L):
        sz.flat_off.append(sz.flat_off[-1] + sz.n[l])
    sz.Ntot = sz.flat_off[L]
    sz.M = sz.flat_off[L - 1]
    sz.Ksel = (L - 1) * p * k
    if sz.Ksel > sz.M:
        raise ValueError("selection budget (L-1)*p*k exceeds the candidate count")
    sz.S = sz.n[L - 1] + sz.Ksel
    return sz


# ---------------------------------------------------------------------------
# Stage 1: symmetric average-pool pyramid  [card 阶段 1; gist 2.A]
# ---------------------------------------------------------------------------


def pyramid(X, sz: Sizes, mode: str):
    """Levels of one head's [N, d] tensor.

    Level 0 is X itself; level l entry i is the mean of the p**l tokens
    X[i*p**l : (i+1)*p**l], taken directly from level 0 in fp64 and rounded
    once to the storage type.
    """
    X = np.asarray(X, dtype=np.float64)
    levels = [X]
    for l in range(1, sz.L):
        P = sz.P[l]
        mean = X.reshape(sz.n[l], P, X.shape[1]).mean(axis=1)
        levels.append(round_to(mean, mode))
    return levels


# ---------------------------------------------------------------------------
# Stage 2: parameter-free scores and joint top-K  [card 阶段 2; gist 2.B]
# ---------------------------------------------------------------------------


def level0_scores(Qh, Kh):
    """s[t] = ||Q_t||_2 + ||K_t||_2 in fp64, rounded to fp32 (READING R1).

    The pages give the two l2 norms s_QK = ||Q|| and s_KQ = ||K|| as the
    scores and no rule to combine them; the sum is used.
    """
    Qh = np.asarray(Qh, dtype=np.float64)
    Kh = np.asarray(Kh, dtype=np.float64)
    nq = np.sqrt(np.sum(Qh * Qh, axis=1))
    nk = np.sqrt(np.sum(Kh * Kh, axis=1))
    return round_f32(nq + nk)


def candidate_scores(s0, sz: Sizes):
    """Scores of the candidates, levels 0..L-2, level-major.

    A coarse entry inherits the maximum level-0 score of its span, so a
    coarse span keeps the importance of its strongest token [gist 2.B].
    """
    out = []
    for l in range(sz.L - 1):
        out.append(np.asarray(s0).reshape(sz.n[l], sz.P[l]).max(axis=1))
    if not out:
        return np.zeros(0, dtype=np.float64)
    return np.concatenate(out)


def select(cand, sz: Sizes):
    """Boolean mask over all Ntot pyramid entries (level-major flat index).

    The Ksel best candidates by score, ties to the lower flat index
    (READING R3), plus every coarsest-level entry, which is always kept
    [card 阶段 2].  No gradient flows through this step [card 梯度流].
    """
    order = np.argsort(-np.asarray(cand, dtype=np.float64), kind="stable")
    mask = np.zeros(sz.Ntot, dtype=bool)
    mask[order[: sz.Ksel]] = True
    mask[sz.flat_off[sz.L - 1]:] = True
    return mask


def select_descent(cand, sz: Sizes):
    """Boolean mask over all Ntot entries for the hierarchical descent (READING R8).

    ``cand`` holds the scores of levels 0..L-2 (level-major, as from
    ``candidate_scores``); a level-(L-1) entry's score is the maximum of its p
    children's, i.e. of its span's level-0 scores, the same max-pool.  From
    the coarsest level down: the k best of the current entries (ties to the
    lower flat index) pass their p children to the next level down, which
    are all kept; at level 0 the descent stops.
    """
    L, p, k = sz.L, sz.p, sz.k
    mask = np.zeros(sz.Ntot, dtype=bool)
    mask[sz.flat_off[L - 1]:] = True
    if L < 2 or k == 0:
        return mask
    if k > sz.n[L - 1]:
        raise ValueError("descent needs k <= N/p^(L-1)")
    cand = np.asarray(cand, dtype=np.float64)
    top = cand[sz.flat_off[L - 2]: sz.flat_off[L - 1]].reshape(sz.n[L - 1], p).max(axis=1)
    current = np.arange(sz.n[L - 1], dtype=np.int64)  # entries of level l, ascending
    cur_scores = top
    for l in range(L - 1, 0, -1):
        best = current[np.argsort(-cur_scores, kind="stable")[:k]]
        children = np.sort((best[:, None] * p + np.arange(p)[None, :]).ravel())
        mask[sz.flat_off[l - 1] + children] = True
        current = children
        cur_scores = cand[sz.flat_off[l - 1] + children]
    return mask


REGION = 2048  # candidates per region of the regional rule (the pages' chunk size)


def select_regional(cand, sz: Sizes, region: int = REGION):
    """Boolean mask over all Ntot entries for the regional rule (READING R9).

    The M candidate scores (levels 0..L-2, level-major) are cut into regions
    of ``region`` consecutive entries; region c keeps its floor(Ksel * |c| /
    M) best entries (ties to the lower flat index), so every part of the
    sequence contributes; the rest of the budget goes to the best entries
    not yet kept, over all regions.  Every coarsest-level entry is kept.
    """
    cand = np.asarray(cand, dtype=np.float64)
    mask = np.zeros(sz.Ntot, dtype=bool)
    mask[sz.flat_off[sz.L - 1]:] = True
    if sz.Ksel == 0:
        return mask
    kept = np.zeros(sz.M, dtype=bool)
    for a in range(0, sz.M, region):
        b = min(sz.M, a + region)
        quota = sz.Ksel * (b - a) // sz.M
        best = np.argsort(-cand[a:b], kind="stable")[:quota]
        kept[a + best] = True
    rest = np.nonzero(~kept)[0]
    extra = sz.Ksel - int(kept.sum())
    kept[rest[np.argsort(-cand[rest], kind="stable")[:extra]]] = True
    mask[: sz.M] = kept
    return mask


def entry_level_index(f, sz: Sizes):
    f = np.asarray(f, dtype=np.int64)
    lev = np.searchsorted(np.asarray(sz.flat_off[1:]), f, side="right")
    idx = f - np.asarray(sz.flat_off)[lev]
    return lev, idx


def order_selection(mask, sz: Sizes):
    """Gathered order and its inverse.

    Selected entries are arranged by the last token of their span,
    end(l, i) = (i+1)*p**l - 1, then by level, finer first (READING R4); the
    result is causally coherent, so a plain S x S causal mask applies
    [card 阶段 3; gist 2.C].  Returns (sel_idx [S], slot_of [Ntot]).
    """
    f = np.nonzero(mask)[0].astype(np.int64)
    lev, idx = entry_level_index(f, sz)
    P = np.asarray(sz.P, dtype=np.int64)[lev]
    end = (idx + 1) * P - 1
    perm = np.lexsort((lev, end))
    sel_idx = f[perm]
    slot_of = np.full(sz.Ntot, -1, dtype=np.int64)
    slot_of[sel_idx] = np.arange(sel_idx.size)
    return sel_idx, slot_of


# ---------------------------------------------------------------------------
# Stage 3: gather and dense causal attention  [card 阶段 3; gist 2.C]
# ---------------------------------------------------------------------------


def gather(levels, sel_idx, sz: Sizes):
    lev, idx = entry_level_index(sel_idx, sz)
    d = levels[0].shape[1]
    out = np.empty((sel_idx.size, d), dtype=np.float64)
    for j in range(sel_idx.size):
        out[j] = levels[lev[j]][idx[j]]
    return out


ROW_BLOCK = 512


def causal_attention(Qg, Kg, Vg):
    """softmax(Qg Kg^T / sqrt(d) + causal mask) Vg and the natural-log LSE.

    Processed in blocks of query rows only to bound memory; each row is the
    textbook formula.
    """
    S, d = Qg.shape
    scale = 1.0 / np.sqrt(d)
    O = np.empty((S, Vg.shape[1]), dtype=np.float64)
    lse = np.empty(S, dtype=np.float64)
    for r0 in range(0, S, ROW_BLOCK):
        r1 = min(S, r0 + ROW_BLOCK)
        s = (Qg[r0:r1] @ Kg[:r1].T) * scale
        rows = np.arange(r0, r1)[:, None]
        cols = np.arange(r1)[None, :]
        s = np.where(cols <= rows, s, -np.inf)
        m = s.max(axis=1, keepdims=True)
        e = np.exp(s - m)
        l = e.sum(axis=1, keepdims=True)
        O[r0:r1] = (e @ Vg[:r1]) / l
        lse[r0:r1] = (m + np.log(l))[:, 0]
    return O, lse


def attention_rows(Qg, Kg, Vg, rows):
    """The same attention for selected query rows only."""
    d = Qg.shape[1]
    scale = 1.0 / np.sqrt(d)
    rows = np.asarray(rows, dtype=np.int64)
    O = np.empty((rows.size, Vg.shape[1]), dtype=np.float64)
    lse = np.empty(rows.size, dtype=np.float64)
    for a, r in enumerate(rows):
        s = (Kg[: r + 1] @ Qg[r]) * scale
        m = s.max()
        e = np.exp(s - m)
        l = e.sum()
        O[a] = (e @ Vg[: r + 1]) / l
        lse[a] = m + np.log(l)
    return O, lse


# ---------------------------------------------------------------------------
# Stage 4: scatter-back  [card 阶段 4; gist 2.C]
# ---------------------------------------------------------------------------


def scatter(Og, slot_of, sz: Sizes, mode: str):
    """O[t] = sum over levels l of Og[slot(l, i)] for t in R(l, i).

    R(l, i) = [i*p^l + p^l - 1, i*p^l + 2p^l - 2], i.e. t in R(l, i) exactly
    when i = floor((t+1)/p^l) - 1; the p^l - 1 offset keeps the layer causal
    and at most L levels reach any t [card 阶段 4].  Levels are summed in
    ascending order (READING R7); positions no entry reaches stay 0 and the
    last range is clipped to N-1 (READING R5).
    """
    N = sz.N
    O = np.zeros((N, Og.shape[1]), dtype=np.float64)
    t = np.arange(N)
    for l in range(sz.L):
        i = (t + 1) // sz.P[l] - 1
        ok = i >= 0
        slots = np.full(N, -1, dtype=np.int64)
        slots[ok] = slot_of[sz.flat_off[l] + i[ok]]
        hit = slots >= 0
        O[hit] += Og[slots[hit]]
    return round_to(O, mode)


# ---------------------------------------------------------------------------
# Backward  [card 梯度流: dL -> scatter -> attention -> gather -> W_Q,W_K,W_V]
# ---------------------------------------------------------------------------


def scatter_bwd(dO, sel_idx, sz: Sizes, mode: str):
    """Adjoint of ``scatter``: dOg[slot(l,i)] = sum of dO over R(l,i) clipped to N-1."""
    lev, idx = entry_level_index(sel_idx, sz)
    dOg = np.zeros((sel_idx.size, dO.shape[1]), dtype=np.float64)
    for j in range(sel_idx.size):
        P = sz.P[lev[j]]
        lo = (idx[j] + 1) * P - 1
        hi = min((idx[j] + 2) * P - 2, sz.N - 1)
        dOg[j] = dO[lo: hi + 1].sum(axis=0)
    return round_to(dOg, mode)


def causal_attention_bwd(Qg, Kg, Vg, dOg, lse, D):
    """Gradients of causal attention given the forward LSE and D = rowsum(dOg*Og).

    P = exp(s - lse); dVg = P^T dOg; dP = dOg Vg^T; dS = P (dP - D);
    dQg = dS Kg / sqrt(d); dKg = dS^T Qg / sqrt(d).
    """
    S, d = Qg.shape
    scale = 1.0 / np.sqrt(d)
    dQ = np.zeros_like(Qg)
    dK = np.zeros_like(Kg)
    dV = np.zeros_like(Vg)
    for r0 in range(0, S, ROW_BLOCK):
        r1 = min(S, r0 + ROW_BLOCK)
        s = (Qg[r0:r1] @ Kg[:r1].T) * scale
        rows = np.arange(r0, r1)[:, None]
        cols = np.arange(r1)[None, :]
        P = np.where(cols <= rows, np.exp(s - lse[r0:r1, None]), 0.0)
        dV[:r1] += P.T @ dOg[r0:r1]
        dP = dOg[r0:r1] @ Vg[:r1].T
        dS = P * (dP - D[r0:r1, None])
        dQ[r0:r1] = (dS @ Kg[:r1]) * scale
        dK[:r1] += (dS.T @ Qg[r0:r1]) * scale
    return dQ, dK, dV


def attention_bwd_rows(Qg, Kg, Vg, dOg, lse, D, q_rows, k_cols):
    """The gradients of ``causal_attention_bwd`` for some rows only.

    dQg of query row r needs the keys j <= r only; dKg and dVg of key
    column c need every query row i >= c, with that row's forward LSE and
    D_i, which the caller passes for all S rows.  Each row and column is
    formed on its own, straight from the definitions: P_ij = exp(s_ij -
    lse_i), dP_ij = dOg_i . Vg_j, dS_ij = P_ij (dP_ij - D_i), dQg_r =
    sum_j dS_rj Kg_j / sqrt(d), dKg_c = sum_i dS_ic Qg_i / sqrt(d), dVg_c =
    sum_i P_ic dOg_i.  Returns (dQg[q_rows], dKg[k_cols], dVg[k_cols]).
    """
    S, d = Qg.shape
    scale = 1.0 / np.sqrt(d)
    q_rows = np.asarray(q_rows, dtype=np.int64)
    k_cols = np.asarray(k_cols, dtype=np.int64)
    dQ = np.empty((q_rows.size, d), dtype=np.float64)
    for a, r in enumerate(q_rows):
        P = np.exp((Kg[: r + 1] @ Qg[r]) * scale - lse[r])
        dS = P * (Vg[: r + 1] @ dOg[r] - D[r])
        dQ[a] = (dS @ Kg[: r + 1]) * scale
    dK = np.empty((k_cols.size, d), dtype=np.float64)
    dV = np.empty((k_cols.size, Vg.shape[1]), dtype=np.float64)
    for a, c in enumerate(k_cols):
        P = np.exp((Qg[c:] @ Kg[c]) * scale - lse[c:])
        dS = P * (dOg[c:] @ Vg[c] - D[c:])
        dK[a] = (dS @ Qg[c:]) * scale
        dV[a] = P @ dOg[c:]
    return dQ, dK, dV


def gather_bwd(dXg, slot_of, sz: Sizes, mode: str):
    """Adjoint of pyramid + gather: dX[t] = sum_l dXg[slot(l, t // p^l)] / p^l.

    Only selected entries contribute; levels are summed in ascending order.
    """
    N = sz.N
    dX = np.zeros((N, dXg.shape[1]), dtype=np.float64)
    t = np.arange(N)
    for l in range(sz.L):
        slots = slot_of[sz.flat_off[l] + t // sz.P[l]]
        hit = slots >= 0
        dX[hit] += dXg[slots[hit]] / sz.P[l]
    return round_to(dX, mode)


# ---------------------------------------------------------------------------
# Whole layer, one head
# ---------------------------------------------------------------------------


def head_select(Qh, Kh, sz: Sizes, rule: str = "joint"):
    """Scores, mask and order of one head (stages 2 and the ordering of 3).

    rule: "joint" (READING R2), "descent" (READING R8) or "regional"
    (READING R9)."""
    s0 = level0_scores(Qh, Kh)
    cand = candidate_scores(s0, sz)
    rules = {"joint": select, "descent": select_descent, "regional": select_regional}
    mask = rules[rule](cand, sz)
    sel_idx, slot_of = order_selection(mask, sz)
    return cand, sel_idx, slot_of


def head_forward(Qh, Kh, Vh, sz: Sizes, mode: str, selection=None, rule: str = "joint"):
    """One head's forward.  ``selection`` = (sel_idx, slot_of) freezes stage 2."""
    Qh = np.asarray(Qh, dtype=np.float64)
    Kh = np.asarray(Kh, dtype=np.float64)
    Vh = np.asarray(Vh, dtype=np.float64)
    pq, pk, pv = pyramid(Qh, sz, mode), pyramid(Kh, sz, mode), pyramid(Vh, sz, mode)
    if selection is None:
        cand, sel_idx, slot_of = head_select(Qh, Kh, sz, rule)
    else:
        cand = None
        sel_idx, slot_of = selection
    Qg, Kg, Vg = gather(pq, sel_idx, sz), gather(pk, sel_idx, sz), gather(pv, sel_idx, sz)
    Og_exact, lse = causal_attention(Qg, Kg, Vg)
    Og = round_to(Og_exact, mode)
    O = scatter(Og, slot_of, sz, mode)
    return dict(levels=(pq, pk, pv), cand=cand, sel_idx=sel_idx, slot_of=slot_of,
                Qg=Qg, Kg=Kg, Vg=Vg, Og=Og, lse=lse, O=O)


def head_backward(ctx, dOh, sz: Sizes, mode: str):
    dOh = np.asarray(dOh, dtype=np.float64)
    dOg = scatter_bwd(dOh, ctx["sel_idx"], sz, mode)
    D = np.sum(dOg * ctx["Og"], axis=1)
    dQg, dKg, dVg = causal_attention_bwd(ctx["Qg"], ctx["Kg"], ctx["Vg"], dOg, ctx["lse"], D)
    dQg, dKg, dVg = round_to(dQg, mode), round_to(dKg, mode), round_to(dVg, mode)
    dQ = gather_bwd(dQg, ctx["slot_of"], sz, mode)
    dK = gather_bwd(dKg, ctx["slot_of"], sz, mode)
    dV = gather_bwd(dVg, ctx["slot_of"], sz, mode)
    return dict(dOg=dOg, D=D, dQg=dQg, dKg=dKg, dVg=dVg, dQ=dQ, dK=dK, dV=dV)


def forward(Q, K, V, p: int, L: int, k: int, mode: str, rule: str = "joint"):
    """Whole layer forward over [B, H, N, d] arrays; returns per-head contexts."""
    Q = np.asarray(Q, dtype=np.float64)
    B, H, N, d = Q.shape
    sz = sizes(N, p, L, k)
    ctxs = [[head_forward(Q[b, h], K[b, h], V[b, h], sz, mode, rule=rule) for h in range(H)]
            for b in range(B)]
    O = np.stack([np.stack([c["O"] for c in row]) for row in ctxs])
    return O, ctxs, sz


def backward(ctxs, dO, sz: Sizes, mode: str):
    dO = np.asarray(dO, dtype=np.float64)
    outs = [[head_backward(ctxs[b][h], dO[b, h], sz, mode) for h in range(len(ctxs[b]))]
            for b in range(len(ctxs))]
    stack = lambda key: np.stack([np.stack([o[key] for o in row]) for row in outs])
    return stack("dQ"), stack("dK"), stack("dV"), outs
