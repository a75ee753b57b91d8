"""Pins for the oracle's block-sparse attention (no GPU): a keep-all mask reproduces dense
softmax attention, any mask equals dense attention with the dropped logits at -inf (torch
fp64 scaled-dot-product attention), a block of identical keys gives its closed form, and
the LSE equals torch.logsumexp."""
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F

from oracle import ress_oracle as O


def _qkv(seed, B=1, H=2, N=300, D=64):
    g = torch.Generator().manual_seed(seed)
    return [torch.randn(B, H, N, D, generator=g, dtype=torch.float64) for _ in range(3)]


def test_keep_all_equals_dense_sdpa():
    q, k, v = _qkv(0)
    nb = 3
    kept = {(0, h, i): list(range(nb)) for h in range(2) for i in range(nb)}
    got = O.block_sparse_attn(q.numpy(), k.numpy(), v.numpy(), kept, 0.125, dtype=np.float64)
    want = F.scaled_dot_product_attention(q, k, v, scale=0.125).numpy()
    lse = torch.logsumexp(0.125 * q @ k.transpose(-1, -2), dim=-1).numpy()
    for (b, h, i), (o, l) in got.items():
        r0, r1 = 128 * i, min(300, 128 * (i + 1))
        np.testing.assert_allclose(o, want[b, h, r0:r1], rtol=1e-11, atol=1e-12)
        np.testing.assert_allclose(l, lse[b, h, r0:r1], rtol=1e-12)


def test_mask_equals_dense_with_dropped_logits_at_minus_inf():
    q, k, v = _qkv(1, N=640)
    nb = 5
    rng = np.random.default_rng(1)
    kept = {}
    for h in range(2):
        for i in range(nb):
            kept[(0, h, i)] = sorted(rng.choice(nb, size=int(rng.integers(1, nb + 1)), replace=False).tolist())
    got = O.block_sparse_attn(q.numpy(), k.numpy(), v.numpy(), kept, 0.125, dtype=np.float64)
    for (b, h, i), (o, l) in got.items():
        allow = torch.zeros(128, 640, dtype=torch.bool)
        for j in kept[(b, h, i)]:
            allow[:, 128 * j:128 * (j + 1)] = True
        qi = q[b, h, 128 * i:128 * (i + 1)]
        want = F.scaled_dot_product_attention(qi[None], k[b, h][None], v[b, h][None],
                                              attn_mask=allow[None], scale=0.125)[0]
        np.testing.assert_allclose(o, want.numpy(), rtol=1e-11, atol=1e-12)


def test_one_block_of_identical_keys_closed_form():
    """All 128 keys of the only kept block equal k0: attention is uniform, the output is the
    block's mean value row and the LSE is tau q.k0 + ln 128."""
    q, k, v = _qkv(2, N=384)
    k[0, 0, 128:256] = k[0, 0, 128]
    got, lse = O.attention_qblock(q.numpy(), k.numpy(), v.numpy(), 0, 0, 2, [1], 0.125, dtype=np.float64)
    np.testing.assert_allclose(got, np.tile(v[0, 0, 128:256].mean(0).numpy(), (128, 1)), rtol=1e-12)
    want_lse = 0.125 * (q[0, 0, 256:384] @ k[0, 0, 128]).numpy() + math.log(128)
    np.testing.assert_allclose(lse, want_lse, rtol=1e-13)


def test_partial_last_block_ignores_missing_tokens():
    """N = 300: the last key block holds 44 tokens; keeping it alone must equal SDPA over
    those 44 keys."""
    q, k, v = _qkv(3, N=300)
    got, lse = O.attention_qblock(q.numpy(), k.numpy(), v.numpy(), 0, 1, 0, [2], 0.125, dtype=np.float64)
    want = F.scaled_dot_product_attention(q[0, 1, :128][None], k[0, 1, 256:][None], v[0, 1, 256:][None],
                                          scale=0.125)[0]
    np.testing.assert_allclose(got, want.numpy(), rtol=1e-11, atol=1e-12)
    assert got.shape == (128, 64)
    got2, _ = O.attention_qblock(q.numpy(), k.numpy(), v.numpy(), 0, 1, 2, [0, 2], 0.125, dtype=np.float64)
    assert got2.shape == (44, 64)


def test_no_kept_block_gives_zero_rows():
    q, k, v = _qkv(4, N=256)
    o, l = O.attention_qblock(q.numpy(), k.numpy(), v.numpy(), 0, 0, 0, [], 0.125)
    assert np.all(o == 0) and np.all(np.isneginf(l))


# ------------------------------------------- the pages' grid: key blocks of 64 tokens
def test_key_blocks_of_64_pool_and_attend_like_their_pairs():
    """[ReSS] Supp. F grid (query blocks of 128, key blocks of 64): two consecutive 64-token
    pools average to the 128-token pool, and keeping both 64-blocks of a pair attends
    exactly like keeping the 128-block that holds them."""
    rng = np.random.default_rng(8)
    N = 700                                        # 6 query blocks, 11 key blocks of 64
    q, k, v = (rng.normal(size=(1, 2, N, 64)).astype(np.float32) for _ in range(3))
    p128 = O.pool_blocks(k, 128, dtype=np.float64)
    p64 = O.pool_blocks(k, 64, dtype=np.float64)
    for j in range(5):                             # full 128-blocks
        assert np.allclose(p128[:, :, j], 0.5 * (p64[:, :, 2 * j] + p64[:, :, 2 * j + 1]), atol=1e-12)
    # last 128-block: 60 tokens = one partial 64-block
    assert np.allclose(p128[:, :, 5], p64[:, :, 10], atol=1e-12)
    for i in range(6):
        kept128 = [0, 2, 5]
        kept64 = [0, 1, 4, 5, 10]
        o1, l1 = O.attention_qblock(q, k, v, 0, 1, i, kept128, 0.125, dtype=np.float64)
        o2, l2 = O.attention_qblock(q, k, v, 0, 1, i, kept64, 0.125, dtype=np.float64,
                                    key_block=64)
        assert np.allclose(o1, o2, atol=1e-12) and np.allclose(l1, l2, atol=1e-12)
    # a single 64-block is half of its 128-block: brute force against a direct softmax
    o3, _ = O.attention_qblock(q, k, v, 0, 0, 2, [3], 0.125, dtype=np.float64, key_block=64)
    lg = q[0, 0, 256:384].astype(np.float64) @ k[0, 0, 192:256].astype(np.float64).T * 0.125
    pr = np.exp(lg - lg.max(1, keepdims=True))
    assert np.allclose(o3, (pr / pr.sum(1, keepdims=True)) @ v[0, 0, 192:256], atol=1e-12)
