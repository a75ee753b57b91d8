"""CUDA path (through the C ABI) against the CPU oracle on the same seeded inputs.

Small cases compare every element; the full-size VGGT-shaped layers compare the pooled
tensors and P everywhere and drift, selection and attention on seeded row samples (plus
the dense special-token rows).  Tolerances are documented in tests/parity.py."""
import math

import numpy as np
import pytest
import torch

from block_sparse_global_b200 import ress as R
from block_sparse_global_b200 import workload as W
from block_sparse_global_b200.pipeline import SparseGlobalAttention
from oracle import ress_oracle as O
from parity import (REPORT, OracleLayer, check_attention, check_drift, check_realized_drift,
                    rows_per_head,
                    close, compare_masks, ensure_built, run_gpu, sample_rows)

pytestmark = pytest.mark.gpu
METHODS = {"mass": O.MASS, "drift": O.DRIFT, "random": O.RANDOM}


def _all_rows(B, H, nb):
    return [(b, h, i) for b in range(B) for h in range(H) for i in range(nb)]


def _check_block_tensors(layer, orc, rows_for_s=None):
    close(layer.q_pool.cpu(), orc.qp, 1e-4, 1e-6, "q_pool")
    close(layer.k_pool.cpu(), orc.kp, 1e-4, 1e-6, "k_pool")
    close(layer.v_pool.cpu(), orc.vp, 1e-4, 1e-6, "v_pool")
    close(layer.P.cpu(), orc.P, 1e-4, 1e-7, "P")
    close(layer.v_bar.cpu(), orc.vbar, 1e-4, 1e-6, "v_bar")
    close(layer.gram.cpu(), orc.gram, 1e-4, 1e-6, "gram")


def _full_check(wl, method, rows, attn_rows, rounds=None):
    layer = run_gpu(wl, method=method, rounds=rounds)
    orc = OracleLayer(wl)
    _check_block_tensors(layer, orc)
    r = wl.rounds if rounds is None else rounds
    if method != O.DRIFT:
        r = 0
    s_rows = None
    if method == O.DRIFT:
        s_gpu = layer.s.cpu().numpy()
        check_drift({row: s_gpu[row] for row in rows}, orc, rows)
        s_rows = orc.drift_rows(rows)
    sel = orc.select(rows, method, r, wl.select_seed, s_rows=s_rows)
    kept = layer.kept_lists()
    stats = compare_masks(kept, sel, orc.nb, f"{wl.case.name}/{method}")
    mask = layer.mask.cpu().numpy()
    for (b, h, i) in rows:
        assert sorted(np.nonzero(mask[b, h, i])[0].tolist()) == kept[(b, h, i)]
    worst, rel = check_attention(layer, orc, attn_rows)
    REPORT.append(dict(workload=wl.case.name, key_block=wl.key_block, method=method,
                       sparsity=wl.sparsity, **stats, attn_rows=len(attn_rows),
                       attn_max_abs=worst, attn_rel_l2=rel))
    return layer, orc, stats


@pytest.mark.parametrize("method", ["mass", "drift", "random"])
def test_tiny_case_every_element(method):
    wl = W.make_workload(1)
    rows = _all_rows(1, 4, 8)
    layer, orc, stats = _full_check(wl, METHODS[method], rows, rows)
    assert all(len(v) == 4 for v in layer.kept_lists().values())


@pytest.mark.parametrize("method", ["mass", "drift", "random"])
def test_small_vggt_layer_with_specials_and_ragged_tail(method):
    # 3 views: N = 4122, 33 blocks, last block 26 tokens, 15 special tokens -> block 32
    wl = W.make_workload(2, heads=2, views=3, method=method, sparsity=0.6, rounds=4)
    rows = _all_rows(1, 2, wl.nb)
    layer, orc, stats = _full_check(wl, METHODS[method], rows, rows, rounds=4)
    kept = layer.kept_lists()
    for (b, h, i), k in kept.items():
        assert (wl.nb - 1) in k
        if i == wl.nb - 1:
            assert k == list(range(wl.nb))


def test_selection_alone_on_oracle_scores():
    """Feed the oracle's own P, s, pooled values and Gram to the GPU selection: this
    isolates the selection arithmetic (top-k, Eqs. 13-17, track-best)."""
    wl = W.make_workload(2, heads=4, views=6, method="drift", sparsity=0.75, rounds=5)
    ensure_built()
    orc = OracleLayer(wl)
    rows = _all_rows(1, 4, orc.nb)
    s_rows = orc.drift_rows(rows)
    s = np.zeros_like(orc.P)
    for r, val in s_rows.items():
        s[r] = val
    dev = torch.device("cuda")
    layer = SparseGlobalAttention(1, 4, wl.q.shape[2], device=dev, with_mask=True)
    layer.P.copy_(torch.from_numpy(orc.P))
    layer.s.copy_(torch.from_numpy(s))
    layer.v_pool.copy_(torch.from_numpy(orc.vp))
    layer.v_bar.copy_(torch.from_numpy(orc.vbar))
    layer.gram.copy_(torch.from_numpy(orc.gram))
    for method, rounds in ((O.MASS, 0), (O.DRIFT, 0), (O.DRIFT, 5), (O.RANDOM, 0)):
        layer.select(method, wl.budgets, wl.keep_k.to(dev), wl.dense_q.to(dev), rounds, wl.rho,
                     wl.eps, wl.select_seed)
        torch.cuda.synchronize()
        sel = orc.select(rows, method, rounds, wl.select_seed, s_rows=s_rows)
        stats = compare_masks(layer.kept_lists(), sel, orc.nb, f"selection-only/{method}/{rounds}")
        if method == O.RANDOM:
            assert stats["agreement"] == 1.0


@pytest.mark.parametrize("top_p", [0.3, 0.6, 0.85, 0.97])
def test_cdf_selection_on_oracle_scores(top_p):
    """SparseVGGT's top-p rule on the oracle's own P: kept lists against the oracle, in
    the selection kernel and in the fused block-map kernel (bit-identical to each other)."""
    wl = W.make_workload(2, heads=4, views=6, method="mass", sparsity=0.5)
    ensure_built()
    orc = OracleLayer(wl)
    rows = _all_rows(1, 4, orc.nb)
    dev = torch.device("cuda")
    layer = SparseGlobalAttention(1, 4, wl.q.shape[2], device=dev, with_mask=True)
    layer.P.copy_(torch.from_numpy(orc.P))
    layer.select(O.CDF, wl.budgets, wl.keep_k.to(dev), wl.dense_q.to(dev), top_p=top_p)
    torch.cuda.synchronize()
    sel = orc.select(rows, O.CDF, 0, 0, top_p=top_p)
    stats = compare_masks(layer.kept_lists(), sel, orc.nb, f"cdf/{top_p}")
    kept = sum(len(v) for v in layer.kept_lists().values())
    assert stats["rows"] == len(rows) and kept > len(rows)
    # the fused kernel on the same workload's own pooled inputs against the separate calls
    ref = SparseGlobalAttention(1, 4, wl.q.shape[2], device=dev, with_mask=True)
    ref.scores(wl.q.to(dev), wl.k.to(dev), wl.v.to(dev))
    ref.select(O.CDF, wl.budgets, wl.keep_k.to(dev), wl.dense_q.to(dev), top_p=top_p)
    fz = SparseGlobalAttention(1, 4, wl.q.shape[2], device=dev, with_mask=True)
    fz.pool(wl.q.to(dev), wl.k.to(dev), wl.v.to(dev))
    fz.scores_select(O.CDF, wl.budgets, wl.keep_k.to(dev), wl.dense_q.to(dev), top_p=top_p)
    torch.cuda.synchronize()
    assert torch.equal(fz.kv_cnt, ref.kv_cnt) and torch.equal(fz.mask, ref.mask)


@pytest.mark.parametrize("method", [O.MASS, O.RANDOM])
@pytest.mark.parametrize("case", [1, 2])
def test_fused_scores_select_equals_separate_calls(case, method):
    """ress_scores_select (block map and selection in one kernel) against
    ress_block_scores + ress_select_blocks on the same pooled inputs: identical kept
    lists, counts and masks, and identical P and v_bar when it writes them."""
    ensure_built()
    wl = W.make_workload(case, device="cuda", heads=4, views=6) if case == 2 else W.make_workload(1, device="cuda")
    B, H, N, _ = wl.q.shape
    dev = torch.device("cuda")
    ref = SparseGlobalAttention(B, H, N, device=dev, with_mask=True)
    ref.scores(wl.q, wl.k, wl.v)
    ref.select(method, wl.budgets, wl.keep_k, wl.dense_q, 0, wl.rho, wl.eps, wl.select_seed)
    for write in (False, True):
        fz = SparseGlobalAttention(B, H, N, device=dev, with_mask=True)
        fz.pool(wl.q, wl.k, wl.v)
        fz.P.fill_(-1.0)
        fz.v_bar.fill_(-1.0)
        fz.scores_select(method, wl.budgets, wl.keep_k, wl.dense_q, wl.select_seed, write_scores=write)
        torch.cuda.synchronize()
        assert torch.equal(fz.kv_cnt, ref.kv_cnt)
        assert torch.equal(fz.mask, ref.mask)
        for (b, h, i), lst in ref.kept_lists().items():
            assert fz.kept_lists()[(b, h, i)] == lst
        if write:
            assert torch.equal(fz.P, ref.P) and torch.equal(fz.v_bar, ref.v_bar)
        else:
            assert bool((fz.P == -1.0).all()) and bool((fz.v_bar == -1.0).all())


def _kv_equal(a, b):
    """Kept lists equal (counts, and every row's valid prefix of kv_idx)."""
    assert torch.equal(a.kv_cnt, b.kv_cnt)
    cnt = a.kv_cnt.unsqueeze(-1)
    pos = torch.arange(a.nk, device=a.kv_cnt.device).view(1, 1, 1, -1)
    live = pos < cnt
    assert torch.equal(torch.where(live, a.kv_idx, 0), torch.where(live, b.kv_idx, 0))


@pytest.mark.parametrize("case,kb,heads,sign,rounds", [
    (2, 128, 4, O.MINIMISE, 4), (2, 128, 4, O.MAXIMISE_FULL, 3), (2, 64, 4, O.MINIMISE, 2),
    (3, 128, 16, O.MINIMISE, 3), (3, 64, 16, O.MINIMISE, 3), (4, 128, 16, O.MINIMISE, 5),
    (2, 128, 4, O.MINIMISE, 0)])
def test_fused_drift_select_equals_separate_calls(case, kb, heads, sign, rounds):
    """ress_drift_select (block map, drift score and drift selection in one kernel, P and
    s kept on chip) against ress_block_scores + ress_drift_scores + ress_select_blocks on
    the same pooled inputs ([ReSS] §4.3 "Fused kernel implementation": the fused round
    gives the same selection): identical kept lists, masks and realized drift J, and
    identical P, v_bar and s when it writes them.  Includes the full 100-view layer
    (1074 key blocks, Dirichlet budgets, R = 5) and the 64-token key-block grid."""
    ensure_built()
    kw = dict(device="cuda", key_block=kb, method="drift", rounds=rounds)
    if case == 2:
        kw.update(heads=heads, views=6)
    wl = W.make_workload(case, **kw)
    B, H, N, _ = wl.q.shape
    dev = torch.device("cuda")
    ref = SparseGlobalAttention(B, H, N, device=dev, with_mask=True, key_block=kb)
    ref.load_output_projection(wl.w_o)
    ref.scores(wl.q, wl.k, wl.v)
    ref.drift()
    J_ref = torch.zeros(B, H, ref.nq, device=dev)
    ref.select(O.DRIFT, wl.budgets, wl.keep_k, wl.dense_q, rounds, wl.rho, wl.eps, 0,
               objective=sign, drift_out=J_ref)
    for write in (False, True):
        fz = SparseGlobalAttention(B, H, N, device=dev, with_mask=True, key_block=kb)
        fz.load_output_projection(wl.w_o)
        fz.pool(wl.q, wl.k, wl.v)
        for t in (fz.P, fz.v_bar, fz.s):
            t.fill_(-1.0)
        J = torch.full((B, H, fz.nq), -1.0, device=dev)
        fz.drift_select(wl.budgets, wl.keep_k, wl.dense_q, rounds, wl.rho, wl.eps,
                        objective=sign, drift_out=J, write_scores=write)
        torch.cuda.synchronize()
        assert fz.device_error() == 0 and ref.device_error() == 0
        _kv_equal(fz, ref)
        assert torch.equal(fz.mask, ref.mask)
        assert torch.equal(J, J_ref)
        if write:
            for name in ("P", "v_bar", "s"):
                assert torch.equal(getattr(fz, name), getattr(ref, name)), name
        else:
            for t in (fz.P, fz.v_bar, fz.s):
                assert bool((t == -1.0).all())


@pytest.mark.parametrize("sign", [O.MINIMISE, O.MAXIMISE_SWAPS, O.MAXIMISE_FULL])
def test_drift_objective_and_realized_drift_on_oracle_scores(sign):
    """The drift-maximising controls of [ReSS] Fig. 8 (swap only, full) and the realized
    drift J of every row's selection ([ReSS] §6.1), from the oracle's own P, s, pooled
    values and Gram, against the oracle.  With MINIMISE, J is also checked for the mass
    and random selections."""
    wl = W.make_workload(2, heads=4, views=6, method="drift", sparsity=0.75, rounds=5)
    ensure_built()
    orc = OracleLayer(wl)
    rows = _all_rows(1, 4, orc.nb)
    s_rows = orc.drift_rows(rows)
    s = np.zeros_like(orc.P)
    for r, val in s_rows.items():
        s[r] = val
    dev = torch.device("cuda")
    layer = SparseGlobalAttention(1, 4, wl.q.shape[2], device=dev, with_mask=True)
    layer.P.copy_(torch.from_numpy(orc.P))
    layer.s.copy_(torch.from_numpy(s))
    layer.v_pool.copy_(torch.from_numpy(orc.vp))
    layer.v_bar.copy_(torch.from_numpy(orc.vbar))
    layer.gram.copy_(torch.from_numpy(orc.gram))
    J = torch.full((1, 4, orc.nb), -1.0, device=dev)
    runs = ((O.DRIFT, 0), (O.DRIFT, 5))
    if sign == O.MINIMISE:
        runs = runs + ((O.MASS, 0), (O.RANDOM, 0))
    for method, rounds in runs:
        layer.select(method, wl.budgets, wl.keep_k.to(dev), wl.dense_q.to(dev), rounds, wl.rho,
                     wl.eps, wl.select_seed, objective=sign, drift_out=J)
        torch.cuda.synchronize()
        sel = orc.select(rows, method, rounds, wl.select_seed, s_rows=s_rows, sign=sign)
        what = f"sign {sign}/{method}/{rounds}"
        kept = layer.kept_lists()
        compare_masks(kept, sel, orc.nb, what)
        J_host = J.cpu().numpy()
        n = check_realized_drift(J_host, kept, sel, orc, what)
        assert n >= 0.9 * len(rows), (what, n)


def test_vggt_8view_mass50_full_layer():
    wl = W.make_workload(2)
    nb = wl.nb
    rows = _all_rows(1, 16, nb)
    attn_rows = sample_rows(1, 16, nb, 40, seed=1, always=[(0, h, nb - 1) for h in (0, 15)])
    layer, orc, stats = _full_check(wl, O.MASS, rows, attn_rows)
    cnt = layer.kv_cnt.cpu()
    assert int(cnt[0, 0, 0]) == 43 + 1 and int(cnt[0, 3, nb - 1]) == nb


def test_vggt_32view_drift75_r3():
    wl = W.make_workload(3)
    nb = wl.nb
    rows = sample_rows(1, 16, nb, 64, seed=2, always=[(0, 0, nb - 1), (0, 7, 0)])
    attn_rows = sample_rows(1, 16, nb, 16, seed=3, always=[(0, 5, nb - 2)])
    _full_check(wl, O.DRIFT, rows, attn_rows)


def test_vggt_100view_drift90_r5_dirichlet():
    """The headline layer (100 views, 137,400 tokens, 1074 blocks, drift 90 %, R = 5,
    Dirichlet budgets) through the fused drift selection: every head, 16 query blocks
    each (always the first, the last sparse and the last dense query block), attention on
    3 rows of every head."""
    wl = W.make_workload(4)
    nb = wl.nb
    assert sum(wl.budgets) == 16 * 107
    dense = [i for i in range(nb) if int(wl.dense_q[i])]
    assert dense == list(range(nb - 5, nb))
    rows = rows_per_head(16, nb, 16, seed=4, always_i=(0, nb - 6, nb - 1))
    attn_rows = rows_per_head(16, nb, 3, seed=5, always_i=(nb - 6,))
    layer, orc, stats = _full_check(wl, O.DRIFT, rows, attn_rows)
    cnt = layer.kv_cnt.cpu()
    for h in range(16):
        assert int(cnt[0, h, 0]) == min(wl.budgets[h], nb - 5) + 5
        assert int(cnt[0, h, nb - 1]) == nb


def test_vggt_100view_drift90_key_block_64_sampled():
    """The 100-view layer on the 128 x 64 grid (1074 query blocks, 2147 key blocks):
    drift with 5 restoration rounds on sampled rows of every head, attention on some."""
    wl = W.make_workload(4, key_block=64)
    assert (wl.nq, wl.nk) == (1074, 2147)
    rows = rows_per_head(16, wl.nq, 4, seed=14, always_i=(wl.nq - 6,))
    attn_rows = sample_rows(1, 16, wl.nq, 8, seed=15, always=[(0, 4, wl.nq - 1)])
    _full_check(wl, O.DRIFT, rows, attn_rows)


@pytest.mark.parametrize("layer_id,sparsity,method", [(0, 0.0, "mass"), (0, 0.9, "random"),
                                                       (23, 0.25, "drift"), (11, 0.5, "mass"),
                                                       (5, 0.75, "drift"), (17, 0.9, "drift"),
                                                       (8, 0.9, "mass")])
def test_vggt_64view_sweep_points(layer_id, sparsity, method):
    wl = W.make_workload(5, layer=layer_id, method=method, sparsity=sparsity)
    nb = wl.nb
    rows = sample_rows(1, 16, nb, 24, seed=layer_id + 10)
    attn_rows = sample_rows(1, 16, nb, 8, seed=layer_id + 20)
    _full_check(wl, METHODS[method], rows, attn_rows)


def test_keep_all_is_dense_attention():
    """Sparsity 0 keeps every block: the kernel computes dense attention; compare with
    torch SDPA in fp32 on a sample of query blocks (library routine, same definition)."""
    wl = W.make_workload(2, heads=4, views=4, method="mass", sparsity=0.0)
    layer = run_gpu(wl)
    assert int(layer.kv_cnt.min()) == wl.nb
    q, k, v = (t.cuda().float() for t in (wl.q, wl.k, wl.v))
    ref = torch.nn.functional.scaled_dot_product_attention(q, k, v, scale=0.125)
    err = (layer.out.float() - ref).abs().max().item()
    rel = ((layer.out.float() - ref).norm() / ref.norm()).item()
    assert err <= 2e-2 and rel <= 1e-2, (err, rel)


def _manual_attn(N, lists, B=1, H=2, seed=0, key_block=128):
    ensure_built()
    g = torch.Generator(device="cuda").manual_seed(seed)
    q, k, v = (torch.randn(B, H, N, 64, device="cuda", generator=g).to(torch.bfloat16)
               for _ in range(3))
    nq, nk = R.grid(N, key_block)
    kv_idx = torch.zeros(B, H, nq, nk, dtype=torch.int32)
    kv_cnt = torch.zeros(B, H, nq, dtype=torch.int32)
    for (b, h, i), lst in lists.items():
        kv_cnt[b, h, i] = len(lst)
        kv_idx[b, h, i, :len(lst)] = torch.tensor(lst, dtype=torch.int32)
    out = torch.full((B, H, N, 64), 7.0, device="cuda", dtype=torch.bfloat16)
    lse = torch.empty(B, H, N, device="cuda")
    err = torch.zeros(1, device="cuda", dtype=torch.int32)
    R.ress_block_sparse_attn(R.make_shape(B, H, N, key_block=key_block), q, k, v, kv_idx.cuda(),
                             kv_cnt.cuda(), None, 0.125, out, lse, err)
    torch.cuda.synchronize()
    return q, k, v, out, lse, int(err.item())


def test_edge_rows_empty_unsorted_single_partial_block():
    N = 300   # 3 blocks, last one 44 tokens
    lists = {(0, 0, 0): [2, 0], (0, 0, 1): [], (0, 0, 2): [2], (0, 1, 0): [0, 1, 2],
             (0, 1, 1): [1], (0, 1, 2): [1, 2, 0]}
    q, k, v, out, lse, err = _manual_attn(N, lists)
    assert err == 0
    qn, kn, vn = (O.to_numpy_f32(t) for t in (q, k, v))
    for (b, h, i), lst in lists.items():
        o_ref, l_ref = O.attention_qblock(qn, kn, vn, b, h, i, sorted(lst), 0.125)
        o = out[b, h, i * 128:i * 128 + o_ref.shape[0]].float().cpu().numpy()
        assert np.abs(o - o_ref).max() <= 2e-2
        if not lst:
            assert np.all(o == 0) and torch.isinf(lse[b, h, 128:256]).all()


def test_tiny_sequence_below_one_block():
    lists = {(b, h, 0): [0] for b in range(2) for h in range(2)}
    q, k, v, out, lse, err = _manual_attn(100, lists, B=2)
    ref = torch.nn.functional.scaled_dot_product_attention(q.float(), k.float(), v.float(), scale=0.125)
    assert err == 0 and (out.float() - ref).abs().max().item() <= 2e-2


def test_out_of_range_kv_index_sets_device_error_and_skips_row():
    lists = {(0, 0, 0): [0, 5], (0, 0, 1): [1], (0, 1, 0): [0], (0, 1, 1): [0, 1]}
    q, k, v, out, lse, err = _manual_attn(256, lists)
    assert err == 4   # RESS_ERR_DEVICE_BOUNDS
    assert torch.all(out[0, 0, :128].float() == 7.0)       # the bad row is left unwritten
    assert not torch.all(out[0, 1, :128].float() == 7.0)   # the others are computed


def test_repeat_runs_are_bit_identical():
    """Two runs on the same inputs give the same bytes (ReSS Supp. B.4 reports the same)."""
    wl = W.make_workload(3, heads=4, views=5, method="drift", rounds=5)
    a = run_gpu(wl)
    b = run_gpu(wl)
    for name in ("q_pool", "P", "v_bar", "s", "kv_cnt", "mask", "out", "lse"):
        assert torch.equal(getattr(a, name), getattr(b, name)), name
    for bb, h, i in _all_rows(1, 4, wl.nb):
        c = int(a.kv_cnt[bb, h, i])
        assert torch.equal(a.kv_idx[bb, h, i, :c], b.kv_idx[bb, h, i, :c])


def test_schedule_is_a_stable_descending_permutation():
    ensure_built()
    g = torch.Generator().manual_seed(0)
    shape = R.make_shape(2, 3, 1000)   # nb = 8, 48 items
    cnt = torch.randint(0, 9, (2, 3, 8), generator=g, dtype=torch.int32)
    order = torch.empty(48, dtype=torch.int32, device="cuda")
    R.ress_attn_schedule(shape, cnt.cuda(), order)
    torch.cuda.synchronize()
    flat = cnt.flatten().tolist()
    want = sorted(range(48), key=lambda it: (-flat[it], it))
    assert order.cpu().tolist() == want


def test_schedule_many_rows_and_repeated_counts():
    """384 rows spread over the 32 warps of the parallel scatter, few distinct counts
    (every bucket spans several warps' chunks), plus counts outside [0, nb]."""
    ensure_built()
    g = torch.Generator().manual_seed(5)
    shape = R.make_shape(1, 4, 96 * 128)   # nb = 96, 384 rows
    cnt = torch.randint(40, 44, (1, 4, 96), generator=g, dtype=torch.int32)
    cnt[0, 1, 7] = 96
    cnt[0, 2, 3] = -5
    cnt[0, 3, 90] = 200
    order = torch.empty(384, dtype=torch.int32, device="cuda")
    R.ress_attn_schedule(shape, cnt.cuda(), order)
    torch.cuda.synchronize()
    flat = [min(max(c, 0), 96) for c in cnt.flatten().tolist()]
    assert order.cpu().tolist() == sorted(range(384), key=lambda it: (-flat[it], it))


@pytest.mark.parametrize("method,planned", [("mass", False), ("drift", False), ("drift", True)])
def test_host_buffer_path_in_head_groups_equals_forward(method, planned):
    """forward_host (pinned host tensors, heads in groups on overlapping streams) gives the
    same bytes as forward() on device tensors: every step is per head.  `planned`: the
    heads are regrouped by budget (plan_head_order), so the staging slots are permuted."""
    ensure_built()
    wl = W.make_workload(2, heads=4, views=6, method=method, sparsity=0.75, rounds=3)
    if planned:
        wl.budgets = [wl.budgets[0] // 3, wl.budgets[1], wl.budgets[2] // 2, wl.budgets[3] * 2]
    dev = torch.device("cuda")
    B, H, N, _ = wl.q.shape
    ref = SparseGlobalAttention(B, H, N, device=dev)
    ref.load_output_projection(wl.w_o.to(dev))
    ref.forward(wl.q.to(dev), wl.k.to(dev), wl.v.to(dev), METHODS[method], wl.budgets,
                wl.keep_k.to(dev), wl.dense_q.to(dev), wl.rounds, wl.rho, wl.eps, wl.select_seed)
    layer = SparseGlobalAttention(B, H, N, device=dev)
    layer.make_groups(wl.w_o.to(dev), 3, budgets=wl.budgets if planned else None)
    if planned:
        assert layer._order != list(range(H))
    qh, kh, vh = (t.cpu().pin_memory() for t in (wl.q, wl.k, wl.v))
    outh = torch.empty(B, H, N, 64, dtype=torch.bfloat16).pin_memory()
    for _ in range(2):
        layer.forward_host(qh, kh, vh, outh, METHODS[method], wl.budgets, wl.keep_k.to(dev),
                           wl.dense_q.to(dev), wl.rounds, wl.rho, wl.eps, wl.select_seed)
    torch.cuda.synchronize()
    assert torch.equal(outh, ref.out.cpu())


def _tail_order(V, T, S):
    """Position of every view-order token after the sink-rule permutation (the layout of
    ress_token_gather written out with numpy)."""
    t = np.arange(V * T)
    v, w = t // T, t % T
    return np.where(w < S, V * (T - S) + v * S + w, v * (T - S) + (w - S))


@pytest.mark.parametrize("V,T,S", [(8, 1374, 5), (3, 300, 0), (4, 129, 129), (7, 200, 1)])
def test_token_gather_matches_the_layout_and_inverts(V, T, S):
    ensure_built()
    g = torch.Generator(device="cuda").manual_seed(V * T + S)
    x = torch.randn(2, 3, V * T, 64, device="cuda", generator=g).to(torch.bfloat16)
    shape = R.make_shape(2, 3, V * T)
    y = torch.empty_like(x)
    R.ress_token_gather(shape, V, S, False, x, y)
    back = torch.empty_like(x)
    R.ress_token_gather(shape, V, S, True, y, back)
    torch.cuda.synchronize()
    pos = torch.from_numpy(_tail_order(V, T, S)).cuda()
    want = torch.empty_like(x)
    want[:, :, pos] = x
    assert torch.equal(y, want)
    assert torch.equal(back, x)


def test_layer_in_view_order_through_the_sink_rule():
    """A layer whose tokens come in VGGT's view order (every view's 5 special tokens
    first): gather to the tail layout, run the layer (the trailing blocks holding the
    special tokens are always kept), gather the output back.  Equal, bit for bit, to the
    layer on the tail layout with its output permuted back."""
    ensure_built()
    wl = W.make_workload(2, heads=4, views=6, device="cuda")
    dev = torch.device("cuda")
    B, H, N, _ = wl.q.shape
    V, S = 6, 5
    pos = torch.from_numpy(_tail_order(V, N // V, S)).cuda()
    ref = SparseGlobalAttention(B, H, N, device=dev)
    ref.load_output_projection(wl.w_o)
    ref.forward(wl.q, wl.k, wl.v, wl.method, wl.budgets, wl.keep_k, wl.dense_q, wl.rounds,
                wl.rho, wl.eps, wl.select_seed)
    shape = R.make_shape(B, H, N)
    view_order = [x[:, :, pos] for x in (wl.q, wl.k, wl.v)]   # token t of view order
    tail = [torch.empty_like(x) for x in view_order]
    for src, dst in zip(view_order, tail):
        R.ress_token_gather(shape, V, S, False, src.contiguous(), dst)
    layer = SparseGlobalAttention(B, H, N, device=dev)
    layer.load_output_projection(wl.w_o)
    layer.forward(*tail, wl.method, wl.budgets, wl.keep_k, wl.dense_q, wl.rounds, wl.rho,
                  wl.eps, wl.select_seed)
    out_view = torch.empty_like(layer.out)
    R.ress_token_gather(shape, V, S, True, layer.out, out_view)
    torch.cuda.synchronize()
    assert torch.equal(tail[0], wl.q) and torch.equal(tail[2], wl.v)
    assert torch.equal(out_view, ref.out[:, :, pos])


def test_wide_logit_range_and_rescaling():
    """Logits spread over hundreds of units (Q scaled by 12): exp2 arguments reach the
    clamp at -126, the running max jumps between tiles and forces O rescales; a ragged
    last block masks columns.  Compared with torch SDPA in fp32."""
    ensure_built()
    g = torch.Generator(device="cuda").manual_seed(7)
    N = 1000
    q = (12.0 * torch.randn(1, 2, N, 64, device="cuda", generator=g)).to(torch.bfloat16)
    k = torch.randn(1, 2, N, 64, device="cuda", generator=g).to(torch.bfloat16)
    v = torch.randn(1, 2, N, 64, device="cuda", generator=g).to(torch.bfloat16)
    nb = 8
    # every row keeps every block, in an order that makes the max grow tile by tile
    idx = torch.arange(nb, dtype=torch.int32).expand(1, 2, nb, nb).contiguous()
    cnt = torch.full((1, 2, nb), nb, dtype=torch.int32)
    out = torch.empty(1, 2, N, 64, device="cuda", dtype=torch.bfloat16)
    lse = torch.empty(1, 2, N, device="cuda")
    R.ress_block_sparse_attn(R.make_shape(1, 2, N), q, k, v, idx.cuda(), cnt.cuda(), None, 0.125, out, lse)
    torch.cuda.synchronize()
    ref = torch.nn.functional.scaled_dot_product_attention(q.float(), k.float(), v.float(), scale=0.125)
    lref = torch.logsumexp(0.125 * q.float() @ k.float().transpose(-1, -2), dim=-1)
    assert torch.isfinite(out.float()).all()
    assert (out.float() - ref).abs().max().item() <= 2e-2
    assert ((out.float() - ref).norm() / ref.norm()).item() <= 1e-2
    assert ((lse - lref).abs() <= 1e-3 + 1e-4 * lref.abs()).all()


# ------------------------------------------- key blocks of 64 tokens (ReSS Supp. F grid)
def test_key_block_64_edge_rows_odd_even_ragged_unsorted():
    """Query blocks of 128 against key blocks of 64: N = 300 gives 3 query blocks and 5
    key blocks, the last 44 tokens.  Rows with odd counts (the last tile's second half
    empty), even counts, the ragged block in either half, unsorted lists, one block, the
    ragged block alone and an empty row; oracle per query block."""
    N = 300
    lists = {(0, 0, 0): [4, 0, 2], (0, 0, 1): [], (0, 0, 2): [4], (0, 1, 0): [0, 1, 2, 3, 4],
             (0, 1, 1): [1, 4], (0, 1, 2): [3, 1, 0, 2], (1, 0, 0): [2], (1, 0, 1): [4, 3],
             (1, 0, 2): [0, 1, 2, 3], (1, 1, 0): [1, 0], (1, 1, 1): [0, 2, 4, 1, 3],
             (1, 1, 2): [3]}
    q, k, v, out, lse, err = _manual_attn(N, lists, B=2, key_block=64)
    assert err == 0
    qn, kn, vn = (O.to_numpy_f32(t) for t in (q, k, v))
    for (b, h, i), lst in lists.items():
        o_ref, l_ref = O.attention_qblock(qn, kn, vn, b, h, i, sorted(lst), 0.125, key_block=64)
        r0 = i * 128
        o = out[b, h, r0:r0 + o_ref.shape[0]].float().cpu().numpy()
        assert np.abs(o - o_ref).max() <= 2e-2, (b, h, i, lst)
        if lst:
            close(lse[b, h, r0:r0 + o_ref.shape[0]].cpu(), l_ref, 1e-4, 1e-3, f"lse{(b, h, i)}")
        else:
            assert np.all(o == 0) and torch.isinf(lse[b, h, r0:r0 + o_ref.shape[0]]).all()


def test_key_block_64_out_of_range_index_sets_device_error():
    # 256 tokens: 4 key blocks of 64; index 4 is out of range and its row is skipped
    lists = {(0, 0, 0): [0, 4], (0, 0, 1): [3], (0, 1, 0): [0], (0, 1, 1): [2, 1]}
    q, k, v, out, lse, err = _manual_attn(256, lists, key_block=64)
    assert err == 4   # RESS_ERR_DEVICE_BOUNDS
    assert torch.all(out[0, 0, :128].float() == 7.0)       # the bad row is left unwritten
    qn, kn, vn = (O.to_numpy_f32(t) for t in (q, k, v))
    for r in ((0, 0, 1), (0, 1, 0), (0, 1, 1)):
        o_ref, _ = O.attention_qblock(qn, kn, vn, *r, sorted(lists[r]), 0.125, key_block=64)
        o = out[r[0], r[1], r[2] * 128:r[2] * 128 + 128].float().cpu().numpy()
        assert np.abs(o - o_ref).max() <= 2e-2


@pytest.mark.parametrize("method", ["mass", "drift", "random"])
@pytest.mark.parametrize("sparsity", [0.6, 0.61])
def test_key_block_64_small_layer_every_row(method, sparsity):
    """The whole path on the 128 x 64 grid: 3 views, N = 4122 -> 33 query blocks and 65
    key blocks, both ragged (58 and 26 tokens); the 15 special tokens sit in key block 64
    (always kept) and query block 32 (dense).  Sparsity 0.6 keeps 26 candidates + 1 (an
    odd count: the last score tile is half empty), 0.61 keeps 25 + 1 (even)."""
    wl = W.make_workload(2, heads=2, views=3, method=method, sparsity=sparsity, rounds=4,
                         key_block=64)
    assert (wl.nq, wl.nk) == (33, 65)
    assert wl.keep_k.nonzero().flatten().tolist() == [64]
    assert wl.dense_q.nonzero().flatten().tolist() == [32]
    rows = _all_rows(1, 2, wl.nq)
    layer, orc, stats = _full_check(wl, METHODS[method], rows, rows, rounds=4)
    kept = layer.kept_lists()
    want = wl.budgets[0] + 1
    assert want % 2 == (1 if sparsity == 0.6 else 0)
    for (b, h, i), lst in kept.items():
        assert 64 in lst
        assert lst == list(range(65)) if i == 32 else len(lst) == want


def test_key_block_64_vggt_8view_mass50_sampled():
    """The 8-view layer (N = 10992: 86 query blocks, 172 key blocks) on the 128 x 64 grid:
    block tensors everywhere, selection on every row, attention on sampled rows."""
    wl = W.make_workload(2, key_block=64)
    assert (wl.nq, wl.nk) == (86, 172)
    rows = _all_rows(1, 16, wl.nq)
    attn_rows = sample_rows(1, 16, wl.nq, 32, seed=7,
                            always=[(0, 0, wl.nq - 1), (0, 15, wl.nq - 2), (0, 3, 0)])
    layer, orc, stats = _full_check(wl, O.MASS, rows, attn_rows)
    cnt = layer.kv_cnt.cpu()
    assert int(cnt[0, 0, 0]) == wl.budgets[0] + int(wl.keep_k.sum())
    assert int(cnt[0, 3, wl.nq - 1]) == wl.nk


def test_key_block_64_vggt_32view_drift75_sampled():
    wl = W.make_workload(3, key_block=64)
    rows = sample_rows(1, 16, wl.nq, 48, seed=8, always=[(0, 0, wl.nq - 1), (0, 7, 0)])
    attn_rows = sample_rows(1, 16, wl.nq, 12, seed=9, always=[(0, 5, wl.nq - 2)])
    _full_check(wl, O.DRIFT, rows, attn_rows)


@pytest.mark.parametrize("top_p", [0.5, 0.9])
def test_key_block_64_cdf_on_oracle_scores(top_p):
    wl = W.make_workload(2, heads=4, views=6, method="mass", sparsity=0.5, key_block=64)
    ensure_built()
    orc = OracleLayer(wl)
    rows = _all_rows(1, 4, orc.nq)
    dev = torch.device("cuda")
    layer = SparseGlobalAttention(1, 4, wl.q.shape[2], device=dev, with_mask=True, key_block=64)
    layer.P.copy_(torch.from_numpy(orc.P))
    layer.select(O.CDF, wl.budgets, wl.keep_k.to(dev), wl.dense_q.to(dev), top_p=top_p)
    torch.cuda.synchronize()
    sel = orc.select(rows, O.CDF, 0, 0, top_p=top_p)
    compare_masks(layer.kept_lists(), sel, orc.nk, f"cdf64/{top_p}")
    fz = SparseGlobalAttention(1, 4, wl.q.shape[2], device=dev, with_mask=True, key_block=64)
    fz.pool(wl.q.to(dev), wl.k.to(dev), wl.v.to(dev))
    fz.scores_select(O.CDF, wl.budgets, wl.keep_k.to(dev), wl.dense_q.to(dev), top_p=top_p)
    ref = SparseGlobalAttention(1, 4, wl.q.shape[2], device=dev, with_mask=True, key_block=64)
    ref.scores(wl.q.to(dev), wl.k.to(dev), wl.v.to(dev))
    ref.select(O.CDF, wl.budgets, wl.keep_k.to(dev), wl.dense_q.to(dev), top_p=top_p)
    torch.cuda.synchronize()
    # entries past kv_cnt are unspecified: compare the kept lists
    assert torch.equal(fz.kv_cnt, ref.kv_cnt) and fz.kept_lists() == ref.kept_lists()


def test_key_block_64_keep_all_is_dense_attention():
    wl = W.make_workload(2, heads=4, views=4, method="mass", sparsity=0.0, key_block=64)
    layer = run_gpu(wl)
    assert int(layer.kv_cnt.min()) == wl.nk
    q, k, v = (t.cuda().float() for t in (wl.q, wl.k, wl.v))
    ref = torch.nn.functional.scaled_dot_product_attention(q, k, v, scale=0.125)
    err = (layer.out.float() - ref).abs().max().item()
    rel = ((layer.out.float() - ref).norm() / ref.norm()).item()
    assert err <= 2e-2 and rel <= 1e-2, (err, rel)


def test_maximum_grid_4096_key_blocks():
    """The largest grid the library accepts: 4096 key blocks per row (one head of 524,288
    tokens, N(0,1) inputs, no special tokens), drift selection of 40 blocks with two
    restoration rounds.  At this size the selection runs 4 rows per CTA, the block map 8,
    and the launch order uses the single-warp scatter; checked against the oracle on
    sampled rows like the VGGT-shaped layers."""
    N = 4096 * 128
    gen = torch.Generator().manual_seed(4096)
    q, k, v = (torch.randn(1, 1, N, 64, generator=gen).to(torch.bfloat16) for _ in range(3))
    w_o = torch.randn(64, 64, generator=gen) / 8.0
    case = W.Case(0, "max-grid-1head-524288tok", heads=1, views=0, seq_len=N, method="drift",
                  sparsity=1.0 - 40 / 4096, rounds=2, tiny=True)
    wl = W.Workload(case=case, layer=0, seed=4096, q=q, k=k, v=v, w_o=w_o,
                    keep_k=torch.zeros(4096, dtype=torch.uint8),
                    dense_q=torch.zeros(4096, dtype=torch.uint8), budgets=[40],
                    method=O.DRIFT, rounds=2, select_seed=99, sparsity=case.sparsity)
    rows = sample_rows(1, 1, 4096, 12, seed=7, always=[(0, 0, 0), (0, 0, 4095)])
    attn_rows = rows[:6]
    layer, orc, stats = _full_check(wl, O.DRIFT, rows, attn_rows)
    cnt = layer.kv_cnt.cpu()
    assert int(cnt.min()) == 40 and int(cnt.max()) == 40


@pytest.mark.parametrize("method", ["mass", "drift"])
def test_batch_of_two_full_layer(method):
    """Two batch elements with different seeded inputs through the whole path (pool, block
    map, drift, selection with restoration, attention): every row against the oracle, so
    that batch and head indexing (per-head Gram matrix and budget) are both exercised."""
    a = W.make_workload(2, layer=0, heads=2, views=3, method=method, sparsity=0.6, rounds=3)
    b = W.make_workload(2, layer=1, heads=2, views=3, method=method, sparsity=0.6, rounds=3)
    wl = W.Workload(case=a.case, layer=0, seed=a.seed, q=torch.cat([a.q, b.q]),
                    k=torch.cat([a.k, b.k]), v=torch.cat([a.v, b.v]), w_o=a.w_o,
                    keep_k=a.keep_k, dense_q=a.dense_q, budgets=[a.budgets[0], a.budgets[1] - 3],
                    method=a.method, rounds=a.rounds, select_seed=a.select_seed,
                    sparsity=a.sparsity)
    rows = _all_rows(2, 2, wl.nb)
    layer, orc, stats = _full_check(wl, METHODS[method], rows, rows)
    assert stats["rows"] == len(rows)
    cnt = layer.kv_cnt.cpu()
    for bb in range(2):
        assert int(cnt[bb, 1, 0]) == wl.budgets[1] + int(wl.keep_k.sum())


@pytest.mark.parametrize("method,key_block", [("mass", 128), ("drift", 128), ("drift", 64)])
def test_cuda_graph_replay_equals_eager(method, key_block):
    """forward() captured into a CUDA graph and replayed gives the eager result bit for
    bit; after new inputs are copied into the captured tensors, a replay computes the new
    layer (again equal to eager)."""
    dev = torch.device("cuda")
    wls = [W.make_workload(2, layer=i, heads=4, views=6, method=method, sparsity=0.75,
                           rounds=3, key_block=key_block) for i in (0, 1)]
    wl = wls[0]
    B, H, N, _ = wl.q.shape
    q, k, v = wl.q.to(dev), wl.k.to(dev), wl.v.to(dev)
    keep_k, dense_q = wl.keep_k.to(dev), wl.dense_q.to(dev)
    args = (METHODS[method], wl.budgets, keep_k, dense_q, wl.rounds, wl.rho, wl.eps, wl.select_seed)

    def eager(src):
        ref = SparseGlobalAttention(B, H, N, device=dev, key_block=key_block)
        ref.load_output_projection(src.w_o.to(dev))
        ref.forward(src.q.to(dev), src.k.to(dev), src.v.to(dev), *args)
        torch.cuda.synchronize()
        return ref.out.clone(), ref.kv_idx.clone(), ref.kv_cnt.clone()

    layer = SparseGlobalAttention(B, H, N, device=dev, key_block=key_block)
    layer.load_output_projection(wl.w_o.to(dev))
    graph = layer.capture_forward(q, k, v, *args)
    for src in wls:
        if src is not wl:
            q.copy_(src.q)
            k.copy_(src.k)
            v.copy_(src.v)
            layer.load_output_projection(src.w_o.to(dev))
        layer.out.zero_()
        graph.replay()
        torch.cuda.synchronize()
        assert layer.device_error() == 0
        out, idx, cnt = eager(src)
        assert torch.equal(layer.kv_cnt, cnt)
        for r in range(layer.nq):
            c = int(cnt[0, 0, r])
            assert torch.equal(layer.kv_idx[0, 0, r, :c], idx[0, 0, r, :c])
        assert torch.equal(layer.out, out)
