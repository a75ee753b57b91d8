"""CPU oracle for block-sparse global attention with ReSS / SparseVGGT block selection.

TEST INFRASTRUCTURE.  Only the tests, `__graft_entry__.smoke()` and the CPU-baseline
leg of `bench.py` may import this module.  The product path (the CUDA library and its
Python binding) never imports, links or calls it, and this module imports nothing from
the product.

It is a plain, slow restatement of what the pages define, in float32 unless a caller
passes dtype=np.float64 (the identity pins do).  Sources, cited by page title and
section / equation:
    [ReSS]       "ReSS: Residual-Restoring Sparse Attention for 3D Vision Transformers"
    [SparseVGGT] "Block-Sparse Global Attention for Efficient Multi-View Geometry
                 Transformers" (abstract page)

Readings of points the pages leave open:
    pooled map      P = softmax over ALL key blocks of tau * mean(Q_blk) . mean(K_blk),
                    tau = 1/sqrt(d_h): pool first, then softmax ([ReSS] §3 step (1), §4.1).
    special tokens  key blocks flagged always-kept are never candidates; query blocks
                    flagged dense keep every key block ([ReSS] §3, §4.1, Supp. F).
    ties            every top-k orders by (score descending, block index ascending).
    swap count      m_r = max(1, round-half-up(rho * c * 2^-(r+1))), capped at |D| and c.
    K guard         every K and K + u in Eq. 16 is guarded as max(., eps), the same eps as
                    Eq. 7.
    swaps           restores and drops of one round are both chosen from the gains of the
                    start-of-round state (one gain evaluation per round, Supp. E).
    updates         g and K follow Eq. 13 (and its mirror for a drop) block by block,
                    restores in ascending block order, then drops; G = g^T M g is
                    recomputed from the new g.
    random control  key(b,h,i,j) = SplitMix64 output number (linear index + 1) of a
                    generator seeded with `seed`; keep the c largest keys.
    sign flip       the drift-maximising control of [ReSS] Fig. 8: "swap only" negates
                    the Eq. 16 gains (each round restores and drops the moves that raise J
                    most) and keeps the selection of largest J seen; "full" also keeps the
                    c candidates with the SMALLEST rank key kappa in the initial selection.
    realized drift  J of a returned selection = Eq. 12 on its drop set (Eq. 10), for any
                    method ([ReSS] §6.1, Figs. 7 and 9); 0 for a dense query block.
    CDF threshold   SparseVGGT's top-p rule ([ReSS] §2 related work, §4.4, Table 2
                    "+CDF threshold", Supp. F): candidates in (P descending, block index
                    ascending) order are kept until the kept mass, always-kept blocks
                    included, reaches top_p (partial sums in float64), never more than the
                    budget c and never fewer than one candidate when c >= 1.
Parity status: every function below is pinned by tests/test_oracle_*.py.  The
restoration rounds (select_row with rounds > 0) are pinned move by move: each round's
restored and dropped blocks are checked against the top-m moves recomputed by a masked
softmax from the start-of-round drop set, and every J after a round against the
masked-softmax J of the drop set it leaves; the brute-force bounds (J_opt <= J_ress <=
J_init, |S| = c, swaps = sum of m_r) hold as well.  What the pages leave open in a round
(simultaneous choice, rounding of m_r, the K guard) is fixed by the readings above.
"""
from __future__ import annotations

import math
from typing import Optional, Sequence

import numpy as np

MASS, DRIFT, RANDOM, CDF = 0, 1, 2, 3
MINIMISE, MAXIMISE_SWAPS, MAXIMISE_FULL = 0, 1, 2   # drift objective ([ReSS] Fig. 8)
MASK64 = (1 << 64) - 1
SPLITMIX_GAMMA = 0x9E3779B97F4A7C15


# ----------------------------------------------------------------------------------------
# Counter-based random keys for the random-selection control ([ReSS] §6.1, Fig. 8).
# SplitMix64 as published by Steele, Lea and Flood, "Fast Splittable Pseudorandom Number
# Generators" (OOPSLA 2014): state advances by the golden gamma, output = mix(state).
# ----------------------------------------------------------------------------------------
def splitmix64_mix(z: int) -> int:
    z &= MASK64
    z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & MASK64
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & MASK64
    return z ^ (z >> 31)


def splitmix64_stream(seed: int, count: int) -> list[int]:
    """The first `count` outputs of a SplitMix64 generator seeded with `seed`."""
    out, state = [], seed & MASK64
    for _ in range(count):
        state = (state + SPLITMIX_GAMMA) & MASK64
        out.append(splitmix64_mix(state))
    return out


def random_key(seed: int, linear_index: int) -> int:
    """Output number linear_index + 1 of the SplitMix64 stream seeded with `seed`."""
    return splitmix64_mix((seed + (linear_index + 1) * SPLITMIX_GAMMA) & MASK64)


# ----------------------------------------------------------------------------------------
# Step (1): block partition and mean pooling.  [ReSS] §3 "Block-Sparse Attention for 3D
# ViTs", step (1); pooled values V_j of §4.1.
# ----------------------------------------------------------------------------------------
def pool_blocks(x, block: int = 128, dtype=np.float32) -> np.ndarray:
    """x: [B, H, N, D] -> [B, H, nb, D]; each block's mean, the last (partial) block
    divided by its true token count.  Tokens are summed one after another."""
    x = np.asarray(x, dtype=dtype)
    B, H, N, D = x.shape
    nb = -(-N // block)
    out = np.zeros((B, H, nb, D), dtype=dtype)
    for j in range(nb):
        t0, t1 = j * block, min(N, (j + 1) * block)
        acc = np.zeros((B, H, D), dtype=dtype)
        for t in range(t0, t1):
            acc += x[:, :, t, :]
        out[:, :, j, :] = acc / dtype(t1 - t0)
    return out


# ----------------------------------------------------------------------------------------
# Pooled block map and dense pooled output.  [ReSS] §4.1, Eq. 1.
# ----------------------------------------------------------------------------------------
def block_scores(q_pool, k_pool, v_pool, scale: float, dtype=np.float32):
    """P[b,h,i,j] = softmax over all key blocks j of scale * Qbar_i . Kbar_j;
    vbar[b,h,i] = sum_j P_ij Vbar_j (Eq. 1)."""
    qp = np.asarray(q_pool, dtype=dtype)
    kp = np.asarray(k_pool, dtype=dtype)
    vp = np.asarray(v_pool, dtype=dtype)
    logits = np.matmul(qp, np.swapaxes(kp, -1, -2)) * dtype(scale)
    m = logits.max(axis=-1, keepdims=True)
    e = np.exp(logits - m)
    P = e / e.sum(axis=-1, keepdims=True)
    vbar = np.matmul(P, vp)
    return P.astype(dtype), vbar.astype(dtype)


# ----------------------------------------------------------------------------------------
# Head Gram matrix.  [ReSS] §4.2, Eq. 8: M_h = (W_O^h)^T W_O^h, W_O^h the d x d_h slice of
# the output projection that multiplies head h.
# ----------------------------------------------------------------------------------------
def head_gram(w_o, heads: int, head_dim: int = 64) -> np.ndarray:
    w = np.asarray(w_o, dtype=np.float64)
    out = np.empty((heads, head_dim, head_dim), dtype=np.float64)
    for h in range(heads):
        wh = w[:, h * head_dim:(h + 1) * head_dim]
        out[h] = wh.T @ wh
    return out.astype(np.float32)


# ----------------------------------------------------------------------------------------
# Block drift score.  [ReSS] §4.2, Eqs. 4-7 and the first line of Eq. 9.
# ----------------------------------------------------------------------------------------
def drift_row(P_row, vbar_row, v_pool_head, M, dtype=np.float32) -> np.ndarray:
    """s_ij = P_ij * sqrt(e_ij^T M e_ij), e_ij = vbar_i - V_j (Eqs. 5, 6, 9), for one row.
    The quadratic form is evaluated directly; a value below zero from rounding is
    clamped to zero before the square root."""
    P_row = np.asarray(P_row, dtype=dtype)
    e = np.asarray(vbar_row, dtype=dtype)[None, :] - np.asarray(v_pool_head, dtype=dtype)
    q = np.einsum("jd,de,je->j", e, np.asarray(M, dtype=dtype), e)
    return (P_row * np.sqrt(np.maximum(q, dtype(0)))).astype(dtype)


def drift_scores(P, v_pool, vbar, gram, dtype=np.float32) -> np.ndarray:
    B, H, nq, nk = np.shape(P)
    s = np.empty((B, H, nq, nk), dtype=dtype)
    for b in range(B):
        for h in range(H):
            for i in range(nq):
                s[b, h, i] = drift_row(P[b, h, i], vbar[b, h, i], v_pool[b, h], gram[h], dtype)
    return s


def rank_key(P_row, s_row, eps: float, dtype=np.float32) -> np.ndarray:
    """Eq. 7: exact single-block drift magnitude s_ij / max(1 - P_ij, eps)."""
    P_row = np.asarray(P_row, dtype=dtype)
    return (np.asarray(s_row, dtype=dtype) / np.maximum(dtype(1) - P_row, dtype(eps))).astype(dtype)


# ----------------------------------------------------------------------------------------
# Selection.  [ReSS] §4.1 (Eq. 2), §4.2 (Eq. 7), §4.3 (Eqs. 10-17), §4.4; SparseVGGT / HeSS
# attention-mass top-k ([ReSS] §1, §3; [SparseVGGT] abstract).
# ----------------------------------------------------------------------------------------
def _rel_gap(a: float, b: float, scale: float = 0.0) -> float:
    den = max(abs(a), abs(b), abs(scale), 1e-30)
    return abs(a - b) / den


def top_by_score(cands: Sequence[int], score, k: int, scale: float = 0.0):
    """The k candidates with the largest score, ties to the lower block index, and the
    relative gap between the k-th and (k+1)-th sorted scores (inf if no cut)."""
    order = sorted(cands, key=lambda j: (-score[j], j))
    chosen = order[:k]
    if 0 < k < len(order):
        margin = _rel_gap(float(score[order[k - 1]]), float(score[order[k]]), scale)
    else:
        margin = math.inf
    return chosen, margin


def swap_count(r: int, c: int, rho: float, n_drop: int) -> int:
    """Eq. 17, m_r = rho * 2^-(r+1) * c, rounded half up, at least one swap, and no more
    than the drop set or the kept set can give."""
    m = max(1, int(math.floor(rho * c * 2.0 ** (-(r + 1)) + 0.5)))
    return min(m, n_drop, c)


def net_drift(D: Sequence[int], P_row, v_pool_head, vbar_row, dtype=np.float32):
    """Eq. 10: g = sum_{j in D} P_ij (vbar_i - V_j), K = 1 - sum_{j in D} P_ij, summed in
    ascending block order."""
    g = np.zeros(np.shape(vbar_row)[-1], dtype=dtype)
    Psum = dtype(0)
    for j in sorted(D):
        g = g + dtype(P_row[j]) * (np.asarray(vbar_row, dtype=dtype) - np.asarray(v_pool_head[j], dtype=dtype))
        Psum = dtype(Psum + dtype(P_row[j]))
    return g.astype(dtype), dtype(dtype(1) - Psum)


def objective(g, K, M, eps: float, dtype=np.float32):
    """Eq. 12: J = g^T M g / K^2 with K guarded by eps; returns (J, G, h = M g)."""
    h = (np.asarray(M, dtype=dtype) @ np.asarray(g, dtype=dtype)).astype(dtype)
    G = dtype(np.dot(np.asarray(g, dtype=dtype), h))
    Kg = max(dtype(K), dtype(eps))
    return dtype(G / (Kg * Kg)), G, h


def swap_gains(D, S, P_row, s_sq, v_pool_head, vbar_row, h, G, K, eps: float,
               dtype=np.float32):
    """Eq. 16 objective decrease for restoring each k in D (Eq. 14, u = +P_k) and for
    dropping each kept candidate k in S (Eq. 15, u = -P_k), all from one state (g, G, K),
    h = M g.  Returns ({k: gain}, G / K^2)."""
    Kh = max(dtype(K), dtype(eps))
    base = dtype(G / (Kh * Kh))
    vbar_row = np.asarray(vbar_row, dtype=dtype)
    gain = {}
    for k in set(D) | set(S):
        t = dtype(P_row[k]) * dtype(np.dot(vbar_row - v_pool_head[k], h))   # d_k^T M g
        if k in D:
            dG = dtype(dtype(-2) * t + dtype(s_sq[k]))
            Kn = max(dtype(K + P_row[k]), dtype(eps))
        else:
            dG = dtype(dtype(2) * t + dtype(s_sq[k]))
            Kn = max(dtype(K - P_row[k]), dtype(eps))
        gain[k] = float(dtype(base - dtype(G + dG) / (Kn * Kn)))
    return gain, float(base)


def realized_drift(selected: Sequence[int], cand: Sequence[int], P_row, v_pool_head, vbar_row,
                   M, eps: float, dtype=np.float32) -> float:
    """Eq. 12 objective of a selection: J of its drop set D = candidates not selected
    (Eq. 10), as [ReSS] §6.1 reports it per selection."""
    D = set(cand) - set(selected)
    g, K = net_drift(D, P_row, v_pool_head, vbar_row, dtype)
    return float(objective(g, K, M, eps, dtype)[0])


def cdf_keep(P_row, cand: Sequence[int], budget: int, top_p: float, fixed_mass: float):
    """Top-p selection (reading above): the kept candidates and the smallest relative gap
    of the decisions (the cumulative mass against top_p where the count was cut, and the
    probability gap at the cut)."""
    order = sorted(cand, key=lambda j: (-float(P_row[j]), j))
    c = max(0, min(budget, len(order)))
    if c == 0:
        return [], math.inf
    cum = float(fixed_mass)
    n = c
    sums = []
    for q, j in enumerate(order[:c]):
        cum += float(P_row[j])      # python floats: float64
        sums.append(cum)
        if cum >= top_p:
            n = q + 1
            break
    n = max(1, n)
    margin = math.inf
    if n < c:    # cut by the threshold: how close the sums before and at the cut came
        before = float(fixed_mass) if n == 1 else sums[n - 2]
        margin = min(abs(sums[n - 1] - top_p), abs(before - top_p)) / max(top_p, 1e-30)
    if n < len(order):   # the order itself at the cut
        margin = min(margin, _rel_gap(float(P_row[order[n - 1]]), float(P_row[order[n]])))
    return order[:n], margin


def select_row(method: int, P_row, cand: Sequence[int], budget: int, *, s_row=None,
               v_pool_head=None, vbar_row=None, M=None, rounds: int = 0, rho: float = 0.5,
               eps: float = 1e-4, rand_keys=None, sign: int = MINIMISE, top_p: float = 1.0,
               fixed_mass: float = 0.0, dtype=np.float32) -> dict:
    """Block selection for one (query block, head) row.

    `sign` selects the drift objective (drift only): MINIMISE ([ReSS] §4), or the
    maximising controls of Fig. 8, MAXIMISE_SWAPS (restoration rounds only) and
    MAXIMISE_FULL (initial selection too).

    Returns dict(selected = sorted kept candidates, margin = smallest relative decision
    gap met on the way, J_init / J_best = Eq. 12 objective of the initial and returned drop
    sets (drift with rounds only), J = realized drift of the returned selection (when M,
    the pooled values and vbar are given), swaps = blocks restored over all rounds,
    J_trace = J after each round, moves = the blocks each round restored and dropped)."""
    cand = list(cand)
    c = max(0, min(budget, len(cand)))
    out = dict(margin=math.inf, J_init=None, J_best=None, J=None, swaps=0, J_trace=[], moves=[])
    have_state = M is not None and v_pool_head is not None and vbar_row is not None

    def finish(selected, margin, J=None):
        out.update(selected=sorted(selected), margin=margin)
        if J is None and have_state:
            J = realized_drift(selected, cand, P_row, v_pool_head, vbar_row, M, eps, dtype)
        out["J"] = None if J is None else float(J)
        return out

    assert sign == MINIMISE or method == DRIFT, "the sign flip is defined for drift selection"
    if method == MASS:
        sel, mg = top_by_score(cand, {j: float(dtype(P_row[j])) for j in cand}, c)
        return finish(sel, mg)
    if method == RANDOM:
        sel, _ = top_by_score(cand, {j: rand_keys[j] for j in cand}, c)
        return finish(sel, math.inf)
    if method == CDF:
        sel, mg = cdf_keep(P_row, cand, c, top_p, fixed_mass)
        return finish(sel, mg)
    assert method == DRIFT
    maximise = sign != MINIMISE
    P_row = np.asarray(P_row, dtype=dtype)
    kap = rank_key(P_row, s_row, eps, dtype)
    flip0 = -1.0 if sign == MAXIMISE_FULL else 1.0
    S0, margin = top_by_score(cand, {j: flip0 * float(kap[j]) for j in cand}, c)
    S = set(S0)
    D = set(cand) - S
    if rounds <= 0 or not D or c == 0:
        return finish(S, margin)
    vbar_row = np.asarray(vbar_row, dtype=dtype)
    Vp = np.asarray(v_pool_head, dtype=dtype)
    s_sq = {j: float(dtype(dtype(s_row[j]) * dtype(s_row[j]))) for j in cand}
    g, K = net_drift(D, P_row, Vp, vbar_row, dtype)
    J, G, h = objective(g, K, M, eps, dtype)
    best_D, best_J = set(D), J
    out["J_init"] = float(J)
    for r in range(rounds):
        m = swap_count(r, c, rho, len(D))
        gain, base = swap_gains(D, S, P_row, s_sq, Vp, vbar_row, h, G, K, eps, dtype)
        if maximise:       # the moves that raise J most ([ReSS] Fig. 8)
            gain = {k: -v for k, v in gain.items()}
        restore, mg1 = top_by_score(sorted(D), gain, m, scale=float(base))
        drop, mg2 = top_by_score(sorted(S), gain, m, scale=float(base))
        margin = min(margin, mg1, mg2)
        for k in sorted(restore):   # Eq. 13
            g = (g - dtype(P_row[k]) * (vbar_row - Vp[k])).astype(dtype)
            K = dtype(K + P_row[k])
        for k in sorted(drop):      # mirror of Eq. 13 for a drop
            g = (g + dtype(P_row[k]) * (vbar_row - Vp[k])).astype(dtype)
            K = dtype(K - P_row[k])
        D = (D - set(restore)) | set(drop)
        S = (S - set(drop)) | set(restore)
        out["swaps"] += len(restore)
        out["moves"].append(dict(restored=sorted(restore), dropped=sorted(drop)))
        J, G, h = objective(g, K, M, eps, dtype)
        out["J_trace"].append(float(J))
        margin = min(margin, _rel_gap(float(J), float(best_J)))
        # track-best, [ReSS] §4.3 last paragraph and Supp. B.3 (track-worst when maximising)
        if (J > best_J) if maximise else (J < best_J):
            best_D, best_J = set(D), J
    out["J_best"] = float(best_J)
    return finish(set(cand) - best_D, margin, J=best_J)


def select_blocks(method: int, P, budgets: Sequence[int], keep_k=None, dense_q=None, *,
                  s=None, v_pool=None, vbar=None, gram=None, rounds: int = 0, rho: float = 0.5,
                  eps: float = 1e-4, seed: int = 0, rows=None, sign: int = MINIMISE,
                  top_p: float = 1.0, dtype=np.float32) -> dict:
    """Selection for every (b, h, i) row, or for the listed `rows` only.

    Returns dict(kept = {(b,h,i): ascending list of kept key blocks}, margin = {...},
    info = {...: per-row dict of select_row})."""
    B, H, nq, nk = np.shape(P)
    keep_k = np.zeros(nk, np.uint8) if keep_k is None else np.asarray(keep_k)
    dense_q = np.zeros(nq, np.uint8) if dense_q is None else np.asarray(dense_q)
    always = [j for j in range(nk) if keep_k[j]]
    cand = [j for j in range(nk) if not keep_k[j]]
    if rows is None:
        rows = [(b, h, i) for b in range(B) for h in range(H) for i in range(nq)]
    kept, margins, info = {}, {}, {}
    for (b, h, i) in rows:
        if dense_q[i]:
            kept[(b, h, i)] = list(range(nk))
            margins[(b, h, i)] = math.inf
            info[(b, h, i)] = dict(selected=cand, margin=math.inf, J=0.0)
            continue
        rk = None
        if method == RANDOM:
            base = ((b * H + h) * nq + i) * nk
            rk = {j: random_key(seed, base + j) for j in cand}
        res = select_row(method, P[b, h, i], cand, budgets[h],
                         s_row=None if s is None else s[b, h, i],
                         v_pool_head=None if v_pool is None else v_pool[b, h],
                         vbar_row=None if vbar is None else vbar[b, h, i],
                         M=None if gram is None else gram[h], rounds=rounds, rho=rho, eps=eps,
                         rand_keys=rk, sign=sign, top_p=top_p,
                         fixed_mass=sum(float(P[b, h, i, j]) for j in always), dtype=dtype)
        kept[(b, h, i)] = sorted(always + res["selected"])
        margins[(b, h, i)] = res["margin"]
        info[(b, h, i)] = res
    return dict(kept=kept, margin=margins, info=info)


# ----------------------------------------------------------------------------------------
# Step (3): exact attention over the kept blocks, softmax renormalised among them.
# [ReSS] §3 step (3); [SparseVGGT] abstract ("block-sparse replacement for dense global
# attention").
# ----------------------------------------------------------------------------------------
def attention_qblock(q, k, v, b: int, h: int, i: int, kept: Sequence[int], scale: float,
                     block: int = 128, dtype=np.float32, key_block: Optional[int] = None):
    """Output rows and natural-log LSE of query block i (`block` tokens) of head (b, h)
    attending to the tokens of the kept key blocks (`key_block` tokens each, default
    `block`; ascending blocks, tokens in order); tokens >= N do not exist.  With no kept
    block the rows are zero and the LSE is -inf."""
    N = q.shape[2]
    kb = block if key_block is None else key_block
    r0, r1 = i * block, min(N, (i + 1) * block)
    rows = np.asarray(q[b, h, r0:r1], dtype=dtype)
    idx = [t for j in kept for t in range(j * kb, min(N, (j + 1) * kb))]
    if not idx:
        return np.zeros((r1 - r0, q.shape[3]), dtype), np.full(r1 - r0, -np.inf, dtype)
    kk = np.asarray(k[b, h, idx], dtype=dtype)
    vv = np.asarray(v[b, h, idx], dtype=dtype)
    logits = (rows @ kk.T) * dtype(scale)
    m = logits.max(axis=1, keepdims=True)
    p = np.exp(logits - m)
    l = p.sum(axis=1, keepdims=True)
    out = (p @ vv) / l
    lse = (m + np.log(l))[:, 0]
    return out.astype(dtype), lse.astype(dtype)


def block_sparse_attn(q, k, v, kept: dict, scale: float, rows=None, block: int = 128,
                      dtype=np.float32, key_block: Optional[int] = None):
    """Attention for the query blocks in `rows` (default: every key of `kept`).
    Returns {(b,h,i): (out rows, lse)}."""
    rows = sorted(kept) if rows is None else rows
    return {r: attention_qblock(q, k, v, *r, kept=kept[r], scale=scale, block=block, dtype=dtype,
                                key_block=key_block)
            for r in rows}


def to_numpy_f32(t) -> np.ndarray:
    """bf16 / fp32 torch tensor (any device) or array -> float32 numpy (exact widening)."""
    if hasattr(t, "detach"):
        return t.detach().float().cpu().numpy()
    return np.asarray(t, dtype=np.float32)


def layer(q, k, v, w_o, method: int, budgets, keep_k=None, dense_q=None, rounds: int = 0,
          rho: float = 0.5, eps: float = 1e-4, seed: int = 0, rows=None,
          attn_rows=None, block: int = 128, top_p: float = 1.0,
          key_block: Optional[int] = None) -> dict:
    """The whole path for one layer: pool -> P, vbar -> drift -> select -> attention.
    Query blocks hold `block` tokens, key blocks `key_block` (default `block`; the pages'
    grid is 128 x 64, [ReSS] Supp. F).  `rows` limits drift and selection to those
    (b,h,i); `attn_rows` limits the attention (default: the selected rows)."""
    qf, kf, vf = to_numpy_f32(q), to_numpy_f32(k), to_numpy_f32(v)
    B, H, N, Dh = qf.shape
    kb = block if key_block is None else key_block
    scale = 1.0 / math.sqrt(Dh)
    qp, kp, vp = pool_blocks(qf, block), pool_blocks(kf, kb), pool_blocks(vf, kb)
    P, vbar = block_scores(qp, kp, vp, scale)
    gram = head_gram(to_numpy_f32(w_o), H, Dh)
    nq = P.shape[-2]
    if rows is None:
        rows = [(b, h, i) for b in range(B) for h in range(H) for i in range(nq)]
    s = None
    if method == DRIFT:
        s = np.zeros_like(P)
        for (b, h, i) in rows:
            s[b, h, i] = drift_row(P[b, h, i], vbar[b, h, i], vp[b, h], gram[h])
    sel = select_blocks(method, P, budgets, keep_k, dense_q, s=s, v_pool=vp, vbar=vbar,
                        gram=gram, rounds=rounds, rho=rho, eps=eps, seed=seed, rows=rows,
                        top_p=top_p)
    attn = block_sparse_attn(qf, kf, vf, sel["kept"], scale,
                             rows=rows if attn_rows is None else attn_rows, block=block,
                             key_block=kb)
    return dict(q_pool=qp, k_pool=kp, v_pool=vp, P=P, vbar=vbar, gram=gram, s=s,
                kept=sel["kept"], margin=sel["margin"], info=sel["info"], attn=attn)
