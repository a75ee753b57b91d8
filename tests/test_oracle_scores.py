"""Pins for the oracle's pooling, pooled block map and drift score (no GPU).

Each check compares the oracle with something other than itself: a closed form, a hand
derivation (tests/golden/hand_3block.json), an exact identity of the ReSS paper, or a
library routine (torch fp64) computing the same definition.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import ress_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ---------------------------------------------------------------- pooling ([ReSS] §3 (1))
def test_pool_closed_form_arithmetic_series():
    """x[t, d] = t + 1000 d: a block's mean is (t0 + t1 - 1) / 2 + 1000 d (exact in fp32),
    including the partial last block (N = 300: blocks of 128, 128, 44 tokens)."""
    N, D = 300, 8
    t = np.arange(N, dtype=np.float32)[:, None] + 1000.0 * np.arange(D, dtype=np.float32)[None, :]
    x = np.broadcast_to(t, (2, 3, N, D)).copy()
    got = O.pool_blocks(x, block=128)
    assert got.shape == (2, 3, 3, D)
    for j, (t0, t1) in enumerate([(0, 128), (128, 256), (256, 300)]):
        want = (t0 + t1 - 1) / 2.0 + 1000.0 * np.arange(D)
        np.testing.assert_array_equal(got[:, :, j, :], np.broadcast_to(want, (2, 3, D)))


def test_pool_constant_block():
    x = np.full((1, 2, 256, 4), 3.25, np.float32)
    np.testing.assert_array_equal(O.pool_blocks(x), np.full((1, 2, 2, 4), 3.25, np.float32))


def test_pool_matches_torch_avg_pool_ceil_mode():
    """torch's average pool with ceil_mode and no padding count divides a partial last
    window by its true size: the same definition from a library routine."""
    g = torch.Generator().manual_seed(0)
    x = torch.randn(2, 3, 1000, 16, generator=g, dtype=torch.float64)
    want = torch.nn.functional.avg_pool1d(x.permute(0, 1, 3, 2).reshape(6, 16, 1000), 128,
                                          stride=128, ceil_mode=True, count_include_pad=False)
    want = want.reshape(2, 3, 16, -1).permute(0, 1, 3, 2).numpy()
    got = O.pool_blocks(x.numpy(), dtype=np.float64)
    np.testing.assert_allclose(got, want, rtol=1e-13, atol=1e-13)


# ------------------------------------------------------- pooled map, Eq. 1 ([ReSS] §4.1)
def test_block_scores_match_torch_softmax_fp64():
    g = torch.Generator().manual_seed(1)
    qp = torch.randn(2, 3, 7, 64, generator=g, dtype=torch.float64)
    kp = torch.randn(2, 3, 9, 64, generator=g, dtype=torch.float64)
    vp = torch.randn(2, 3, 9, 64, generator=g, dtype=torch.float64)
    P, vbar = O.block_scores(qp.numpy(), kp.numpy(), vp.numpy(), 0.125, dtype=np.float64)
    Pt = torch.softmax(0.125 * qp @ kp.transpose(-1, -2), dim=-1)
    np.testing.assert_allclose(P, Pt.numpy(), rtol=1e-12, atol=1e-15)
    np.testing.assert_allclose(vbar, (Pt @ vp).numpy(), rtol=1e-12, atol=1e-14)
    P32, _ = O.block_scores(qp.numpy(), kp.numpy(), vp.numpy(), 0.125)
    np.testing.assert_allclose(P32.sum(-1), 1.0, atol=1e-6)


def test_block_scores_two_blocks_is_sigmoid():
    """With two key blocks the softmax is a logistic function of the logit gap."""
    qp = np.array([[[[0.3, -1.0, 2.0, 0.5]]]])
    kp = np.array([[[[1.0, 0.0, -1.0, 2.0], [-2.0, 1.0, 0.5, 0.0]]]])
    vp = np.array([[[[1.0, 2.0, 3.0, 4.0], [-1.0, 0.0, 1.0, 0.0]]]])
    P, vbar = O.block_scores(qp, kp, vp, 0.5, dtype=np.float64)
    gap = 0.5 * (qp[0, 0, 0] @ kp[0, 0, 0] - qp[0, 0, 0] @ kp[0, 0, 1])
    p0 = 1.0 / (1.0 + math.exp(-gap))
    assert P[0, 0, 0, 0] == pytest.approx(p0, rel=1e-14)
    np.testing.assert_allclose(vbar[0, 0, 0], p0 * vp[0, 0, 0] + (1 - p0) * vp[0, 0, 1], rtol=1e-14)


def test_block_scores_equal_keys_give_uniform_map():
    qp = np.random.default_rng(2).normal(size=(1, 1, 3, 8))
    kp = np.tile(np.random.default_rng(3).normal(size=(1, 1, 1, 8)), (1, 1, 5, 1))
    vp = np.random.default_rng(4).normal(size=(1, 1, 5, 8))
    P, vbar = O.block_scores(qp, kp, vp, 0.125, dtype=np.float64)
    np.testing.assert_allclose(P, 0.2, rtol=1e-14)
    np.testing.assert_allclose(vbar[0, 0], np.tile(vp[0, 0].mean(0), (3, 1)), rtol=1e-13)


# --------------------------------------------------------- hand-derived worked example
def _hand():
    with open(os.path.join(GOLDEN, "hand_3block.json")) as f:
        return json.load(f)


def test_hand_example_scores_and_drift():
    ex = _hand()
    inp, exp = ex["inputs"], ex["expected"]
    qp = np.array(inp["q_pool"], np.float64)[None, None, None, :]
    kp = np.array(inp["k_pool"], np.float64)[None, None]
    vp = np.array(inp["v_pool"], np.float64)[None, None]
    P, vbar = O.block_scores(qp, kp, vp, inp["scale"], dtype=np.float64)
    np.testing.assert_allclose(P[0, 0, 0], exp["P"], rtol=1e-14)
    np.testing.assert_allclose(vbar[0, 0, 0], exp["vbar"], rtol=1e-14, atol=1e-16)
    M = np.eye(4)
    s = O.drift_row(P[0, 0, 0], vbar[0, 0, 0], vp[0, 0], M, dtype=np.float64)
    np.testing.assert_allclose(s, exp["s"], rtol=1e-14)
    np.testing.assert_allclose(O.rank_key(P[0, 0, 0], s, 1e-4, np.float64), exp["kappa"], rtol=1e-14)
    g, K = O.net_drift([1, 2], P[0, 0, 0], vp[0, 0], vbar[0, 0, 0], np.float64)
    J, G, h = O.objective(g, K, M, 1e-4, np.float64)
    assert K == pytest.approx(0.5, rel=1e-15)
    assert G == pytest.approx(exp["G_drop_12"], rel=1e-14)
    assert J == pytest.approx(exp["J_drop_12"], rel=1e-14)
    s_sq = {j: s[j] ** 2 for j in range(3)}
    gain, base = O.swap_gains({1, 2}, {0}, P[0, 0, 0], s_sq, vp[0, 0], vbar[0, 0, 0], h, G, K,
                              1e-4, np.float64)
    assert gain[1] == pytest.approx(exp["restore_1_gain"], rel=1e-13)
    g1, K1 = O.net_drift([2], P[0, 0, 0], vp[0, 0], vbar[0, 0, 0], np.float64)
    assert O.objective(g1, K1, M, 1e-4, np.float64)[0] == pytest.approx(exp["J_after_restore_1"], rel=1e-13)
    for method, key in ((O.MASS, "kept_mass_c1"), (O.DRIFT, "kept_drift_c1")):
        res = O.select_row(method, P[0, 0, 0], [0, 1, 2], 1, s_row=s, v_pool_head=vp[0, 0],
                           vbar_row=vbar[0, 0, 0], M=M, rounds=0, dtype=np.float64)
        assert res["selected"] == exp[key]


# ------------------------------------------------------------ Gram and drift ([ReSS] §4.2)
def _rand_head(seed, nk=11, d=64, d_model=256):
    rng = np.random.default_rng(seed)
    logits = rng.normal(size=nk) * 1.5
    P = np.exp(logits - logits.max())
    P /= P.sum()
    Vp = rng.normal(size=(nk, d)) / 8
    vbar = P @ Vp
    W = rng.normal(size=(d_model, d)) / math.sqrt(d_model)
    return logits, P, Vp, vbar, W


def test_gram_slices_the_head_columns():
    """M_h must be W_O^h^T W_O^h with W_O^h the columns of head h (Eq. 8): compare to
    ||W_O^h x||^2 for random x."""
    rng = np.random.default_rng(5)
    W = rng.normal(size=(96, 3 * 8))
    M = O.head_gram(W, heads=3, head_dim=8).astype(np.float64)
    for h in range(3):
        x = rng.normal(size=8)
        assert x @ M[h] @ x == pytest.approx(np.sum((W[:, 8 * h:8 * h + 8] @ x) ** 2), rel=1e-6)


def test_drift_equals_projected_norm_eq6():
    """s_ij = P_ij ||W_O^h e_ij|| computed with the explicit projection (Eq. 6) equals the
    oracle's Gram-based quadratic form (Eqs. 8, 9)."""
    logits, P, Vp, vbar, W = _rand_head(6)
    M = W.T @ W
    s = O.drift_row(P, vbar, Vp, M, dtype=np.float64)
    want = P * np.linalg.norm((vbar[None, :] - Vp) @ W.T, axis=1)
    np.testing.assert_allclose(s, want, rtol=1e-12)


def test_drift_identity_gram_is_euclidean():
    logits, P, Vp, vbar, _ = _rand_head(7)
    s = O.drift_row(P, vbar, Vp, np.eye(64), dtype=np.float64)
    np.testing.assert_allclose(s, P * np.linalg.norm(vbar[None, :] - Vp, axis=1), rtol=1e-13)


def test_single_block_masking_identity_eq4():
    """Masking key block j and renormalising (torch softmax with a -inf logit) moves the
    pooled output by exactly P_j / (1 - P_j) * (vbar - V_j) (Eq. 4).  The oracle's drift
    magnitude is P_j * |e_j|, so (1 - P_j) * |masked shift| must equal s_j with M = I."""
    logits, P, Vp, vbar, _ = _rand_head(8)
    s = O.drift_row(P, vbar, Vp, np.eye(64), dtype=np.float64)
    lt = torch.tensor(logits)
    for j in range(len(P)):
        lm = lt.clone()
        lm[j] = -math.inf
        vt = (torch.softmax(lm, 0) @ torch.tensor(Vp)).numpy()
        np.testing.assert_allclose(vt - vbar, P[j] / (1 - P[j]) * (vbar - Vp[j]), rtol=1e-10, atol=1e-14)
        assert (1 - P[j]) * np.linalg.norm(vt - vbar) == pytest.approx(s[j], rel=1e-10)


def test_drop_set_objective_is_masked_output_drift():
    """The spec invariant: J(D) = g^T M g / K^2 (Eqs. 10-12) equals
    ||W_O (vtilde_D - vbar)||^2 with vtilde_D from a directly recomputed softmax that
    drops every block of D."""
    logits, P, Vp, vbar, W = _rand_head(9, nk=10)
    M = W.T @ W
    rng = np.random.default_rng(10)
    lt = torch.tensor(logits)
    for _ in range(20):
        D = sorted(rng.choice(10, size=rng.integers(1, 8), replace=False).tolist())
        g, K = O.net_drift(D, P, Vp, vbar, np.float64)
        J, G, _ = O.objective(g, K, M, 1e-12, np.float64)
        lm = lt.clone()
        lm[D] = -math.inf
        vt = (torch.softmax(lm, 0) @ torch.tensor(Vp)).numpy()
        assert J == pytest.approx(np.sum((W @ (vt - vbar)) ** 2), rel=1e-9)
        np.testing.assert_allclose(g / K, vt - vbar, rtol=1e-9, atol=1e-15)


def test_single_block_objective_is_squared_rank_key():
    """Eq. 12 at D = {j} reduces to the square of the Eq. 7 key (when 1 - P_j > eps)."""
    logits, P, Vp, vbar, W = _rand_head(11)
    M = W.T @ W
    s = O.drift_row(P, vbar, Vp, M, dtype=np.float64)
    kap = O.rank_key(P, s, 1e-4, np.float64)
    for j in range(len(P)):
        g, K = O.net_drift([j], P, Vp, vbar, np.float64)
        J, _, _ = O.objective(g, K, M, 1e-4, np.float64)
        assert J == pytest.approx(kap[j] ** 2, rel=1e-10)


def test_rank_key_guard():
    P = np.array([1.0, 0.5, 0.0], np.float32)
    s = np.array([2e-4, 1.0, 3.0], np.float32)
    np.testing.assert_allclose(O.rank_key(P, s, 1e-4), [2.0, 2.0, 3.0], rtol=1e-6)
