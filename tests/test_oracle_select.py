"""Pins for the oracle's block selection (no GPU): swap gains against recomputed
objectives, restoration against brute-force enumeration of drop sets, attention-mass
top-k against brute-force retained mass, and the SplitMix64 random keys against the
generator's published outputs."""
import itertools
import math
import os

import numpy as np
import pytest
import torch

from oracle import ress_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _row(seed, nk=10, d=64, d_model=256, spread=1.5):
    rng = np.random.default_rng(seed)
    logits = rng.normal(size=nk) * spread
    P = np.exp(logits - logits.max())
    P /= P.sum()
    Vp = rng.normal(size=(nk, d)) / 8
    vbar = P @ Vp
    W = rng.normal(size=(d_model, d)) / math.sqrt(d_model)
    M = W.T @ W
    s = O.drift_row(P, vbar, Vp, M, dtype=np.float64)
    return logits, P, Vp, vbar, W, M, s


def _J_masked(logits, Vp, vbar, W, D):
    """||W_O (vtilde_D - vbar)||^2 from a directly recomputed masked softmax."""
    lm = torch.tensor(logits)
    lm[list(D)] = -math.inf
    vt = (torch.softmax(lm, 0) @ torch.tensor(Vp)).numpy()
    return float(np.sum((W @ (vt - vbar)) ** 2))


# ----------------------------------------------------------------- Eqs. 14-16 ([ReSS] §4.3)
def test_swap_gains_equal_recomputed_objective_change():
    for seed in range(5):
        logits, P, Vp, vbar, W, M, s = _row(20 + seed)
        rng = np.random.default_rng(seed)
        D = set(rng.choice(10, size=5, replace=False).tolist())
        S = set(range(10)) - D
        g, K = O.net_drift(D, P, Vp, vbar, np.float64)
        J, G, h = O.objective(g, K, M, 1e-12, np.float64)
        gain, base = O.swap_gains(D, S, P, {j: s[j] ** 2 for j in range(10)}, Vp, vbar, h, G, K,
                                  1e-12, np.float64)
        J0 = _J_masked(logits, Vp, vbar, W, D)
        assert base == pytest.approx(J0, rel=1e-9)
        for k in D:      # restore k: the objective falls to J(D \ {k})
            assert gain[k] == pytest.approx(J0 - _J_masked(logits, Vp, vbar, W, D - {k}), rel=1e-8, abs=1e-13)
        for k in S:      # drop k: the objective becomes J(D + {k})
            assert gain[k] == pytest.approx(J0 - _J_masked(logits, Vp, vbar, W, D | {k}), rel=1e-8, abs=1e-13)


def test_swap_count_schedule_eq17():
    # c = 107, rho = 0.5: 26.75, 13.375, 6.69, 3.34, 1.67 -> 27, 13, 7, 3, 2 (0.484 c in total)
    assert [O.swap_count(r, 107, 0.5, 1000) for r in range(5)] == [27, 13, 7, 3, 2]
    assert sum(O.swap_count(r, 107, 0.5, 1000) for r in range(5)) == round(0.5 * (1 - 2 ** -5) * 107)
    # c = 4: 1.0, 0.5 -> 1, 1 (round half up, at least one swap); never more than |D|
    assert [O.swap_count(r, 4, 0.5, 4) for r in range(2)] == [1, 1]
    assert O.swap_count(0, 40, 0.5, 3) == 3


# ------------------------------------------------- restoration vs brute force ([ReSS] §4.3)
@pytest.mark.parametrize("nk,c,rounds", [(8, 4, 2), (10, 3, 3), (12, 5, 5), (9, 2, 4), (11, 6, 5)])
def test_restoration_bounded_by_brute_force(nk, c, rounds):
    reached = 0
    for seed in range(12):
        logits, P, Vp, vbar, W, M, s = _row(100 + 7 * nk + seed, nk=nk)
        cand = list(range(nk))
        res = O.select_row(O.DRIFT, P, cand, c, s_row=s, v_pool_head=Vp, vbar_row=vbar, M=M,
                           rounds=rounds, rho=0.5, eps=1e-4, dtype=np.float64)
        assert len(res["selected"]) == c
        D_best = set(cand) - set(res["selected"])
        J_best = _J_masked(logits, Vp, vbar, W, D_best)
        assert res["J_best"] == pytest.approx(J_best, rel=1e-8)
        J_opt = min(_J_masked(logits, Vp, vbar, W, set(Dset))
                    for Dset in itertools.combinations(cand, nk - c))
        assert J_opt <= J_best * (1 + 1e-9)
        assert res["J_best"] <= res["J_init"] * (1 + 1e-12)       # track-best never worse
        sched = [O.swap_count(r, c, 0.5, nk - c) for r in range(rounds)]
        assert res["swaps"] == sum(sched)
        reached += J_best <= J_opt * (1 + 1e-9)
    assert reached >= 1


def test_drop_one_initial_selection_is_optimal():
    """With c = |P| - 1 the drop set has one block; J({j}) = kappa_j^2, so keeping the top
    c by the Eq. 7 key is exactly the brute-force optimum."""
    for seed in range(10):
        logits, P, Vp, vbar, W, M, s = _row(300 + seed, nk=9)
        res = O.select_row(O.DRIFT, P, list(range(9)), 8, s_row=s, v_pool_head=Vp, vbar_row=vbar,
                           M=M, rounds=0, dtype=np.float64)
        dropped = (set(range(9)) - set(res["selected"])).pop()
        best = min(range(9), key=lambda j: _J_masked(logits, Vp, vbar, W, {j}))
        assert dropped == best


def test_always_kept_and_dense_rows():
    rng = np.random.default_rng(3)
    B, H, nb = 1, 2, 8
    logits = rng.normal(size=(B, H, nb, nb))
    P = np.exp(logits) / np.exp(logits).sum(-1, keepdims=True)
    vp = rng.normal(size=(B, H, nb, 64)) / 8
    vbar = P @ vp
    gram = np.stack([np.eye(64)] * H)
    s = O.drift_scores(P, vp, vbar, gram, dtype=np.float64)
    keep_k = np.array([0, 0, 0, 0, 0, 0, 1, 1], np.uint8)
    dense_q = np.array([0, 0, 0, 0, 0, 0, 0, 1], np.uint8)
    for method in (O.MASS, O.DRIFT, O.RANDOM):
        res = O.select_blocks(method, P, [3, 2], keep_k, dense_q, s=s, v_pool=vp, vbar=vbar,
                              gram=gram, rounds=2, seed=99, dtype=np.float64)
        for (b, h, i), kept in res["kept"].items():
            if i == 7:
                assert kept == list(range(nb))
            else:
                assert {6, 7} <= set(kept)
                assert len(kept) == [3, 2][h] + 2
                assert kept == sorted(kept)


# ---------------------------------------------- attention-mass top-k ([ReSS] §3, SparseVGGT)
def test_mass_selection_maximises_retained_mass():
    for seed in range(20):
        rng = np.random.default_rng(seed)
        P = rng.dirichlet(np.ones(9))
        c = int(rng.integers(1, 9))
        res = O.select_row(O.MASS, P, list(range(9)), c, dtype=np.float64)
        best = max(sum(P[list(S)]) for S in itertools.combinations(range(9), c))
        assert sum(P[res["selected"]]) == pytest.approx(best, rel=1e-14)


def test_ties_go_to_the_lower_block_index():
    P = np.array([0.1, 0.3, 0.3, 0.3], np.float32)
    res = O.select_row(O.MASS, P, [0, 1, 2, 3], 2)
    assert res["selected"] == [1, 2] and res["margin"] == 0.0


# ------------------------------------------------------------ random control (SplitMix64)
def _golden_splitmix():
    rows = []
    with open(os.path.join(GOLDEN, "splitmix64.txt")) as f:
        for line in f:
            if line.strip() and not line.startswith("#"):
                vals = [int(x) for x in line.split()]
                rows.append((vals[0], vals[1:]))
    return rows


def test_splitmix64_published_outputs():
    for seed, outs in _golden_splitmix():
        assert O.splitmix64_stream(seed, len(outs)) == outs


def test_random_keys_are_the_stream_outputs():
    seed = 987654321
    stream = O.splitmix64_stream(seed, 50)
    assert [O.random_key(seed, i) for i in range(50)] == stream


def test_random_selection_keeps_largest_keys():
    B, H, nq, nk = 1, 2, 3, 7
    P = np.full((B, H, nq, nk), 1.0 / nk)
    seed = 42
    res = O.select_blocks(O.RANDOM, P, [3, 3], seed=seed)
    stream = O.splitmix64_stream(seed, B * H * nq * nk)
    for (b, h, i), kept in res["kept"].items():
        base = ((b * H + h) * nq + i) * nk
        keys = stream[base:base + nk]
        assert kept == sorted(sorted(range(nk), key=lambda j: -keys[j])[:3])


# ----------------------------------- drift-maximising control and realized J ([ReSS] §6.1)
def test_realized_drift_is_the_masked_output_change():
    """Eq. 12 on a selection's drop set equals ||W_O (vtilde - vbar)||^2 recomputed from
    the attention output with the dropped blocks masked out (Eq. 11)."""
    for seed in range(5):
        logits, P, Vp, vbar, W, M, s = _row(seed, nk=12)
        cand = list(range(12))
        for sel in ([0, 3, 5], [1, 2, 4, 7, 9, 11], [6], list(range(12))):
            J = O.realized_drift(sel, cand, P, Vp, vbar, M, 1e-12, dtype=np.float64)
            D = set(cand) - set(sel)
            assert J == pytest.approx(_J_masked(logits, Vp, vbar, W, D), rel=1e-9, abs=1e-18)


def test_full_sign_flip_keeps_the_smallest_rank_keys():
    """Fig. 8 'full': the initial selection keeps the c candidates of smallest kappa
    (ties to the lower block index), the mirror of Eq. 7's top-c."""
    for seed in range(6):
        logits, P, Vp, vbar, W, M, s = _row(seed, nk=10)
        cand = list(range(10))
        res = O.select_row(O.DRIFT, P, cand, 4, s_row=s, v_pool_head=Vp, vbar_row=vbar, M=M,
                           rounds=0, sign=O.MAXIMISE_FULL, dtype=np.float64)
        kap = O.rank_key(P, s, 1e-4, np.float64)
        assert res["selected"] == sorted(np.argsort(kap, kind="stable")[:4].tolist())


def test_swap_only_flip_starts_from_the_minimising_selection():
    for seed in range(4):
        logits, P, Vp, vbar, W, M, s = _row(seed, nk=10)
        cand = list(range(10))
        kw = dict(s_row=s, v_pool_head=Vp, vbar_row=vbar, M=M, rounds=0, dtype=np.float64)
        a = O.select_row(O.DRIFT, P, cand, 4, sign=O.MINIMISE, **kw)
        b = O.select_row(O.DRIFT, P, cand, 4, sign=O.MAXIMISE_SWAPS, **kw)
        assert a["selected"] == b["selected"] and a["J"] == b["J"]


@pytest.mark.parametrize("sign", [O.MINIMISE, O.MAXIMISE_SWAPS, O.MAXIMISE_FULL])
def test_returned_selection_is_the_extreme_of_its_trace(sign):
    """Track-best (track-worst when maximising): the returned selection's J is the
    extreme of the initial and per-round objectives, and equals the masked-output drift
    of that selection."""
    for seed in range(4):
        logits, P, Vp, vbar, W, M, s = _row(seed, nk=14)
        cand = list(range(14))
        res = O.select_row(O.DRIFT, P, cand, 6, s_row=s, v_pool_head=Vp, vbar_row=vbar, M=M,
                           rounds=4, sign=sign, dtype=np.float64)
        trace = [res["J_init"]] + res["J_trace"]
        ext = max(trace) if sign != O.MINIMISE else min(trace)
        assert res["J_best"] == ext and res["J"] == pytest.approx(ext, rel=1e-12)
        D = set(cand) - set(res["selected"])
        assert res["J"] == pytest.approx(_J_masked(logits, Vp, vbar, W, D), rel=1e-9)


def test_maximising_control_bounded_by_brute_force():
    """Every c-subset enumerated: the maximising control's J lies between its initial J
    and the largest J of any subset, and above the minimising selection's J."""
    for seed in range(5):
        logits, P, Vp, vbar, W, M, s = _row(seed, nk=9)
        cand, c = list(range(9)), 4
        allJ = [_J_masked(logits, Vp, vbar, W, set(cand) - set(S))
                for S in itertools.combinations(cand, c)]
        kw = dict(s_row=s, v_pool_head=Vp, vbar_row=vbar, M=M, rounds=5, dtype=np.float64)
        mx = O.select_row(O.DRIFT, P, cand, c, sign=O.MAXIMISE_FULL, **kw)
        mn = O.select_row(O.DRIFT, P, cand, c, sign=O.MINIMISE, **kw)
        assert mx["J_init"] - 1e-15 <= mx["J"] <= max(allJ) * (1 + 1e-9)
        assert min(allJ) * (1 - 1e-9) <= mn["J"] <= mx["J"]


def test_realized_drift_of_mass_and_dense_rows():
    """Mass selection reports the J of its drop set; a dense query block reports 0."""
    logits, P, Vp, vbar, W, M, s = _row(3, nk=8)
    P4 = np.asarray(P)[None, None, None, :].repeat(2, axis=2)
    res = O.select_blocks(O.MASS, P4, [3], dense_q=np.array([0, 1] + [0] * 6, np.uint8)[:2],
                          v_pool=np.asarray(Vp)[None, None], vbar=np.asarray(vbar)[None, None, None].repeat(2, axis=2),
                          gram=np.asarray(M)[None], dtype=np.float64)
    kept0 = res["kept"][(0, 0, 0)]
    assert res["info"][(0, 0, 0)]["J"] == pytest.approx(
        _J_masked(logits, Vp, vbar, W, set(range(8)) - set(kept0)), rel=1e-9)
    assert res["info"][(0, 0, 1)]["J"] == 0.0


# ------------------------------------------- CDF / top-p threshold (SparseVGGT's rule)
def test_cdf_keeps_the_shortest_prefix_reaching_the_threshold():
    """Against a numpy cumulative sum over the descending order: the smallest n whose
    mass (always-kept blocks included) reaches top_p, capped by the budget."""
    rng = np.random.default_rng(11)
    for trial in range(30):
        nk = int(rng.integers(4, 40))
        logits = rng.normal(size=nk) * rng.uniform(0.5, 4)
        P = np.exp(logits - logits.max())
        P /= P.sum()
        fixed = [j for j in range(nk) if rng.random() < 0.1]
        cand = [j for j in range(nk) if j not in fixed]
        if not cand:
            continue
        c = int(rng.integers(1, len(cand) + 1))
        tau = float(rng.uniform(0.05, 1.0))
        order = np.array(cand)[np.argsort(-P[cand], kind="stable")]
        csum = float(P[fixed].sum()) + np.cumsum(P[order].astype(np.float64))
        hit = np.nonzero(csum >= tau)[0]
        n = min(c, max(1, int(hit[0]) + 1 if len(hit) else c))
        kept, _ = O.cdf_keep(P, cand, c, tau, float(P[fixed].sum()))
        assert sorted(kept) == sorted(order[:n].tolist()), trial


def test_cdf_special_cases():
    P = np.array([0.5, 0.25, 0.125, 0.0625, 0.0625])
    cand = list(range(5))
    assert O.cdf_keep(P, cand, 5, 0.8, 0.0)[0] == [0, 1, 2]        # 0.75 < 0.8 <= 0.875
    assert O.cdf_keep(P, cand, 2, 0.8, 0.0)[0] == [0, 1]           # capped by the budget
    assert O.cdf_keep(P, cand, 5, 1e-9, 0.0)[0] == [0]             # at least one candidate
    assert O.cdf_keep(P, cand[1:], 4, 0.3, 0.5)[0] == [1]          # always-kept mass counts
    assert O.cdf_keep(P, cand, 0, 0.5, 0.0)[0] == []
    # top_p = 1 keeps the budget's top-c: the attention-mass selection
    rng = np.random.default_rng(2)
    P = rng.dirichlet(np.ones(20))
    mass = O.select_row(O.MASS, P, list(range(20)), 7)["selected"]
    cdf = O.select_row(O.CDF, P, list(range(20)), 7, top_p=1.0)["selected"]
    assert mass == cdf


def test_cdf_kept_sets_grow_with_the_threshold():
    rng = np.random.default_rng(4)
    P = rng.dirichlet(np.ones(30) * 0.3)
    prev = set()
    for tau in np.linspace(0.05, 1.0, 20):
        kept = set(O.cdf_keep(P, list(range(30)), 30, float(tau), 0.0)[0])
        assert prev <= kept
        prev = kept


# ------------------------------- the restoration trajectory, move by move ([ReSS] §4.3)
def _brute_round(logits, Vp, vbar, W, D, S, m, maximise=False):
    """One restoration round recomputed from its definition, independent of Eqs. 13-16:
    every candidate move is evaluated by a masked softmax.  From the start-of-round drop
    set D (reading R7), restoring k changes the objective to J(D - {k}) and dropping k to
    J(D + {k}); the m restores and the m drops with the largest decrease (largest increase
    when maximising) are taken, ties to the lower block index.  Returns (restored,
    dropped, smallest relative gap between the chosen and the next move on either side)."""
    J0 = _J_masked(logits, Vp, vbar, W, D)
    sgn = -1.0 if maximise else 1.0
    up = {k: sgn * (J0 - _J_masked(logits, Vp, vbar, W, D - {k})) for k in D}
    dn = {k: sgn * (J0 - _J_masked(logits, Vp, vbar, W, D | {k})) for k in S}
    gap = math.inf
    picks = []
    for gains in (up, dn):
        order = sorted(gains, key=lambda k: (-gains[k], k))
        if m < len(order):
            a, b = gains[order[m - 1]], gains[order[m]]
            gap = min(gap, abs(a - b) / max(abs(a), abs(b), abs(J0), 1e-300))
        picks.append(sorted(order[:m]))
    return picks[0], picks[1], gap


@pytest.mark.parametrize("sign", [O.MINIMISE, O.MAXIMISE_SWAPS])
@pytest.mark.parametrize("nk,c,rounds,rho", [(10, 2, 1, 0.5), (10, 4, 1, 0.5), (12, 6, 1, 0.5),
                                             (11, 4, 1, 1.0), (12, 6, 5, 0.5), (12, 5, 5, 1.0),
                                             (9, 3, 4, 1.0)])
def test_restoration_moves_equal_brute_force_moves(nk, c, rounds, rho, sign):
    """Every round's restored and dropped blocks are the top-m moves of D and of S, both
    evaluated by a directly recomputed masked softmax from the start-of-round drop set,
    and every entry of J_trace is the masked-softmax J of the drop set the round leaves
    (which also checks the Eq. 13 updates of g and K to within rounding).  A top-m taken
    by the smallest gain, drops chosen after the restores are applied, or drops taken
    from D instead of S each change some round's moves."""
    checked = 0
    for seed in range(10):
        logits, P, Vp, vbar, W, M, s = _row(500 + 13 * nk + seed, nk=nk)
        cand = list(range(nk))
        res = O.select_row(O.DRIFT, P, cand, c, s_row=s, v_pool_head=Vp, vbar_row=vbar, M=M,
                           rounds=rounds, rho=rho, eps=1e-12, sign=sign, dtype=np.float64)
        kap = O.rank_key(P, s, 1e-12, np.float64)
        S = set(sorted(cand, key=lambda j: (-kap[j], j))[:c])
        D = set(cand) - S
        assert len(res["moves"]) == rounds and len(res["J_trace"]) == rounds
        for r in range(rounds):
            m = O.swap_count(r, c, rho, len(D))
            restored, dropped, gap = _brute_round(logits, Vp, vbar, W, D, S, m,
                                                  maximise=sign != O.MINIMISE)
            if gap < 1e-6:     # a near tie at a cut: either choice is correct
                break
            assert res["moves"][r] == dict(restored=restored, dropped=dropped), (seed, r)
            D = (D - set(restored)) | set(dropped)
            S = (S - set(dropped)) | set(restored)
            assert res["J_trace"][r] == pytest.approx(_J_masked(logits, Vp, vbar, W, D),
                                                      rel=1e-9, abs=1e-18)
            checked += 1
    assert checked >= 8 * rounds


def test_restoration_move_check_catches_planted_mistakes():
    """The brute-force move check above fails for the three plausible slips in a round:
    restores taken by the smallest gain, drops chosen after the restores are applied
    (sequential instead of from one state), and drops taken from D instead of S.  Each
    slip is planted in a copy of one round computed here from the oracle's own Eq. 16
    gains, on the CPU."""
    caught = {"smallest": 0, "sequential": 0, "from_D": 0}
    for seed in range(12):
        logits, P, Vp, vbar, W, M, s = _row(900 + seed, nk=12)
        cand = list(range(12))
        kap = O.rank_key(P, s, 1e-12, np.float64)
        S = set(sorted(cand, key=lambda j: (-kap[j], j))[:5])
        D = set(cand) - S
        m = 3
        want_r, want_d, gap = _brute_round(logits, Vp, vbar, W, D, S, m)
        if gap < 1e-6:
            continue
        s_sq = {j: s[j] ** 2 for j in cand}
        g, K = O.net_drift(D, P, Vp, vbar, np.float64)
        J, G, h = O.objective(g, K, M, 1e-12, np.float64)
        gain, _ = O.swap_gains(D, S, P, s_sq, Vp, vbar, h, G, K, 1e-12, np.float64)
        top = lambda ks, gn, k: sorted(sorted(ks, key=lambda j: (-gn[j], j))[:k])
        ok_r, ok_d = top(D, gain, m), top(S, gain, m)
        assert (ok_r, ok_d) == (want_r, want_d)      # the correct round passes
        # 1. restores by the smallest gain
        low = sorted(sorted(D, key=lambda j: (gain[j], j))[:m])
        caught["smallest"] += low != want_r
        # 2. sequential: restores applied, gains recomputed, then drops
        D2 = D - set(ok_r)
        S2 = S | set(ok_r)
        g2, K2 = O.net_drift(D2, P, Vp, vbar, np.float64)
        J2, G2, h2 = O.objective(g2, K2, M, 1e-12, np.float64)
        gain2, _ = O.swap_gains(D2, S2 - set(ok_r), P, s_sq, Vp, vbar, h2, G2, K2, 1e-12, np.float64)
        caught["sequential"] += top(S2 - set(ok_r), gain2, m) != want_d
        # 3. drops taken from D
        caught["from_D"] += top(D, gain, m) != want_d
    assert all(v >= 3 for v in caught.values()), caught
