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
