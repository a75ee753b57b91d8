"""Host-side pieces of bench.py that its reported numbers rest on (CPU only)."""
import itertools
import os
import sys

import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _brute_flops(kv_idx, kv_cnt, N, kb):
    """4 * rows * cols * 64 summed over every kept (query block, key block) pair, rows and
    cols counting only real tokens, by plain enumeration."""
    B, H, nq, _ = kv_idx.shape
    total = 0
    for b, h, i in itertools.product(range(B), range(H), range(nq)):
        rows = min(128, N - 128 * i)
        for t in range(int(kv_cnt[b, h, i])):
            j = int(kv_idx[b, h, i, t])
            total += 4 * rows * min(kb, N - kb * j) * 64
    return float(total)


def test_kept_tile_flops_matches_enumeration():
    g = torch.Generator().manual_seed(3)
    for N, kb in ((300, 128), (300, 64), (1024, 128), (1000, 64), (130, 64)):
        nq, nk = -(-N // 128), -(-N // kb)
        B, H = 2, 3
        kv_idx = torch.zeros(B, H, nq, nk, dtype=torch.int32)
        kv_cnt = torch.randint(0, nk + 1, (B, H, nq), generator=g, dtype=torch.int32)
        for b, h, i in itertools.product(range(B), range(H), range(nq)):
            perm = torch.randperm(nk, generator=g)[: int(kv_cnt[b, h, i])].sort().values
            kv_idx[b, h, i, : len(perm)] = perm.to(torch.int32)
            kv_idx[b, h, i, len(perm):] = 7777   # unspecified tail entries must not count
        assert bench.kept_tile_flops(kv_idx, kv_cnt, N, kb) == _brute_flops(kv_idx, kv_cnt, N, kb)


def test_dense_layer_flops_closed_form():
    """Every block kept: 4 * N * N * 64 per (batch, head)."""
    N, kb = 10992, 128
    nq = nk = -(-N // kb)
    kv_idx = torch.arange(nk, dtype=torch.int32).expand(1, 2, nq, nk).contiguous()
    kv_cnt = torch.full((1, 2, nq), nk, dtype=torch.int32)
    assert bench.kept_tile_flops(kv_idx, kv_cnt, N, kb) == 2 * 4.0 * N * N * 64


def test_traffic_record_follows_the_kernel_source():
    """roofline.traffic comes from a committed ncu record only for its own workload and
    only while the attention kernel's source is the one the counters were taken on."""
    rec = os.path.join(ROOT, "profiles", "attn_kernel_vggt-8view-16head-mass50_traffic.txt")
    kv = dict(l.strip().split("=", 1) for l in open(rec) if "=" in l and not l.startswith("#"))
    import hashlib
    src = os.path.join(ROOT, "block_sparse_global_b200", "csrc", "k_attn.cu")
    same = hashlib.sha256(open(src, "rb").read()).hexdigest() == kv["kernel_source_sha256"]
    got = bench.measured_traffic("vggt-8view-16head-mass50")
    want = int(kv["dram_bytes_read"]) + int(kv["dram_bytes_write"]) if same else None
    assert got == want
    assert bench.measured_traffic("no-such-workload") is None
