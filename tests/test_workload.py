"""Host-side checks of the seeded synthetic workloads (no GPU)."""
import numpy as np
import pytest
import torch

from block_sparse_global_b200 import workload as W
from oracle import ress_oracle as O


def test_special_token_tail_blocks():
    # 8 views: 10992 tokens, 40 specials -> only the last block (112 tokens) holds them
    assert W.special_tail_blocks(8 * 1374, 40) == [85]
    assert W.special_tail_blocks(32 * 1374, 160) == [342, 343]
    assert W.special_tail_blocks(100 * 1374, 500) == [1069, 1070, 1071, 1072, 1073]
    assert W.special_tail_blocks(64 * 1374, 320) == [684, 685, 686]
    assert W.num_blocks(100 * 1374) == 1074


def test_uniform_budgets():
    assert W.uniform_budget(0.5, 85) == 43
    assert W.uniform_budget(0.75, 342) == 86
    assert W.uniform_budget(0.9, 1069) == 107
    assert [W.uniform_budget(s, 684) for s in W.SWEEP_SPARSITIES] == [684, 513, 342, 171, 68]
    assert W.uniform_budget(0.99, 8) == 2          # two-block floor
    assert W.uniform_budget(0.5, 1) == 1


def test_allocation_respects_total_cap_floor():
    rng = np.random.default_rng(0)
    for _ in range(50):
        w = rng.dirichlet(np.ones(16)).tolist()
        out = W.allocate_budgets(w, 16 * 107, cap=1069, floor=2)
        assert sum(out) == 16 * 107
        assert min(out) >= 2 and max(out) <= 1069
    out = W.allocate_budgets([0.97] + [0.002] * 15, 16 * 107, cap=1069, floor=2)
    assert out[0] == 1069 and sum(out) == 16 * 107
    out = W.allocate_budgets([0.25] * 4, 40, cap=12, floor=2)
    assert out == [10, 10, 10, 10]


def test_tiny_workload_shapes_and_layout():
    wl = W.make_workload(1)
    assert wl.q.shape == (1, 4, 1024, 64) and wl.q.dtype == torch.bfloat16
    assert wl.budgets == [4, 4, 4, 4] and wl.rounds == 2
    assert int(wl.keep_k.sum()) == 0 and int(wl.dense_q.sum()) == 0
    wl2 = W.make_workload(1)
    assert torch.equal(wl.q, wl2.q) and torch.equal(wl.w_o, wl2.w_o)


def test_vggt_workload_small_variant():
    wl = W.make_workload(2, heads=2, views=2)
    n = 2 * 1374
    assert wl.q.shape == (1, 2, n, 64)
    assert wl.keep_k.tolist()[-1] == 1 and wl.dense_q.tolist()[-1] == 1
    q = wl.q.float()
    # special tokens (tail) carry the high norm
    assert q[0, :, -10:].norm(dim=-1).mean() > 2 * q[0, :, :100].norm(dim=-1).mean()


def test_near_duplicate_views_cosine():
    wl = W.make_workload(4, heads=2, views=6)
    assert len(wl.extras["near_duplicate_views"]) == 5
    assert wl.extras["near_duplicate_min_cos"] >= 0.9
    assert sum(wl.budgets) == 2 * W.uniform_budget(0.9, wl.nb - 1) or sum(wl.budgets) >= 2 * 2


def test_oracle_layer_runs_on_tiny_case():
    wl = W.make_workload(1)
    for method in (O.MASS, O.DRIFT, O.RANDOM):
        res = O.layer(wl.q, wl.k, wl.v, wl.w_o, method, wl.budgets, rounds=2, seed=wl.select_seed,
                      rows=[(0, h, i) for h in range(4) for i in range(8)])
        assert all(len(v) == 4 for v in res["kept"].values())
        o, lse = res["attn"][(0, 1, 3)]
        assert o.shape == (128, 64) and np.isfinite(o).all()


def test_host_path_head_group_sizes():
    """Head groups of the host-buffer call: they cover every head once, in contiguous
    ranges of at least one head; sizes never grow, so the last group is the smallest;
    the default (near-equal) split differs by at most one."""
    from block_sparse_global_b200.pipeline import SparseGlobalAttention as S
    for heads in (1, 2, 3, 7, 16, 24):
        for groups in (1, 2, 3, 4, 5, 8, 16, 40):
            for taper in (True, False):
                sizes = S.group_sizes(heads, groups, taper)
                assert sum(sizes) == heads and min(sizes) >= 1
                assert len(sizes) == min(groups, heads)
                assert all(a >= b for a, b in zip(sizes, sizes[1:])), (heads, groups, sizes)
                if not taper:
                    assert max(sizes) - min(sizes) <= 1
    assert S.group_sizes(16, 4, taper=True) == [6, 5, 3, 2]
    assert S.group_sizes(16, 6) == [3, 3, 3, 3, 2, 2]


def test_host_path_head_order_by_budget():
    """plan_head_order: a permutation of the heads; the last group holds the cheapest
    heads; the other groups' work per head is balanced (largest first to the least loaded
    group per head); identity with one group; ascending within each group."""
    from block_sparse_global_b200.pipeline import SparseGlobalAttention as S
    budgets = [142, 80, 226, 14, 104, 207, 58, 58, 85, 123, 25, 74, 52, 254, 135, 75]
    sizes = S.group_sizes(16, 6)
    order = S.plan_head_order(budgets, sizes)
    assert sorted(order) == list(range(16))
    assert sorted(order[-sizes[-1]:]) == sorted(sorted(range(16), key=lambda h: (budgets[h], h))[:sizes[-1]])
    groups, s0 = [], 0
    for n in sizes:
        groups.append(order[s0:s0 + n])
        s0 += n
    assert all(g == sorted(g) for g in groups)
    per_head = [sum(budgets[h] + 16 for h in g) / len(g) for g in groups[:-1]]
    assert max(per_head) - min(per_head) <= max(budgets) / 3, per_head
    assert S.plan_head_order(budgets, [16]) == list(range(16))
    assert S.plan_head_order([5, 5, 5, 5], [2, 2]) == [0, 1, 2, 3]
    assert S.plan_head_order([5, 5, 5, 6], [2, 2]) == [2, 3, 0, 1]


def test_host_path_group_plan_rejects_bad_input_and_maps_every_head():
    """make_groups: sizes must cover the heads, budgets must name every head; the planned
    groups' slots and heads form a bijection and each group's W_O columns are its heads'."""
    import pytest
    import torch
    from block_sparse_global_b200.pipeline import SparseGlobalAttention as S
    layer = S.__new__(S)  # host-side planning only: no device buffers
    layer.B, layer.H, layer.N, layer.key_block = 1, 6, 256, 128
    layer.device = torch.device("cpu")
    calls = []

    class _Sub:
        def __init__(self, B, H, N, device=None, key_block=128):
            self.H = H

        def load_output_projection(self, w):
            calls.append(w)

    import block_sparse_global_b200.pipeline as P
    real, P.SparseGlobalAttention = P.SparseGlobalAttention, _Sub
    real_stream = torch.cuda.Stream
    torch.cuda.Stream = lambda *a, **k: None
    try:
        w_o = torch.arange(64 * 6, dtype=torch.float32).repeat(3, 1)  # column c holds c
        with pytest.raises(ValueError):
            S.make_groups(layer, w_o, 2, sizes=[3, 2])
        with pytest.raises(ValueError):
            S.make_groups(layer, w_o, 2, sizes=[6, 0])
        with pytest.raises(ValueError):
            S.make_groups(layer, w_o, 2, budgets=[1, 2, 3])  # not one budget per head
        groups = S.make_groups(layer, w_o, 3, budgets=[9, 1, 5, 7, 2, 8])
    finally:
        P.SparseGlobalAttention = real
        torch.cuda.Stream = real_stream
    slots, heads = [], []
    for (s0, s1, sub, hs), w in zip(groups, calls[-len(groups):]):
        assert s1 - s0 == len(hs) == sub.H
        slots += list(range(s0, s1))
        heads += hs
        want = torch.cat([torch.arange(64 * h, 64 * h + 64, dtype=torch.float32) for h in hs])
        assert torch.equal(w[0], want)
    assert slots == list(range(6)) and sorted(heads) == list(range(6))
    assert groups[-1][3] == sorted([1, 4])  # the two cheapest heads last
