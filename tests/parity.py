"""Helpers shared by the GPU parity tests: run the CUDA path through the C ABI, run the
oracle on the same inputs, and compare with the tolerances below.

Tolerances (fp32 intermediates, bf16 attention output):
    pooled means, P, vbar : |gpu - oracle| <= 1e-4 |oracle| + floor  (summation order only)
    drift s               : |gpu - oracle| <= 1e-4 |s| + P sqrt(1e-6 (a + 2|b| + c)), the
                            cancellation bound of the Eq. 9 expansion a - 2b + c evaluated
                            in fp32 (a = vbar^T M vbar, b = vbar^T M V_j, c = V_j^T M V_j)
    kept-block lists      : identical on every row whose oracle decision margin exceeds
                            1e-3 (relative); at least 99.9 % of all mask bits equal
    attention             : max |gpu - oracle| <= 2e-2 and relative L2 <= 1e-2, the oracle
                            run in fp32 on the GPU's own kept lists; LSE within 1e-3 + 1e-4|lse|
"""
from __future__ import annotations

import math

import numpy as np
import torch

from block_sparse_global_b200 import build as B
from block_sparse_global_b200 import ress as R
from block_sparse_global_b200.pipeline import SparseGlobalAttention
from oracle import ress_oracle as O

MARGIN = 1e-3


def ensure_built():
    B.build()
    R.load()


def run_gpu(wl, method=None, rounds=None, with_mask=True, seed=None):
    ensure_built()
    dev = torch.device("cuda")
    method = wl.method if method is None else method
    rounds = wl.rounds if rounds is None else rounds
    if method != O.DRIFT:
        rounds = 0
    q, k, v = wl.q.to(dev), wl.k.to(dev), wl.v.to(dev)
    b, h, n, _ = q.shape
    layer = SparseGlobalAttention(b, h, n, device=dev, with_mask=with_mask,
                                  key_block=wl.key_block)
    layer.load_output_projection(wl.w_o.to(dev))
    # the fused kernels write the block map, vbar and (drift) s as well, for the checks
    layer.forward(q, k, v, method, wl.budgets, wl.keep_k.to(dev), wl.dense_q.to(dev), rounds,
                  wl.rho, wl.eps, wl.select_seed if seed is None else seed, write_scores=True)
    torch.cuda.synchronize()
    assert layer.device_error() == 0, f"device error {layer.device_error()}"
    return layer


class OracleLayer:
    """Oracle intermediates for one workload (pooled tensors and P for every row)."""

    def __init__(self, wl):
        self.q = O.to_numpy_f32(wl.q)
        self.k = O.to_numpy_f32(wl.k)
        self.v = O.to_numpy_f32(wl.v)
        self.B, self.H, self.N, _ = self.q.shape
        self.scale = 1.0 / math.sqrt(64)
        self.key_block = wl.key_block
        self.qp = O.pool_blocks(self.q)
        self.kp = O.pool_blocks(self.k, wl.key_block)
        self.vp = O.pool_blocks(self.v, wl.key_block)
        self.P, self.vbar = O.block_scores(self.qp, self.kp, self.vp, self.scale)
        self.gram = O.head_gram(O.to_numpy_f32(wl.w_o), self.H)
        self.nq, self.nk = self.P.shape[-2:]
        self.nb = self.nk  # key blocks: the width of a kept-block mask
        self.keep_k = wl.keep_k.cpu().numpy()
        self.dense_q = wl.dense_q.cpu().numpy()
        self.wl = wl

    def drift_rows(self, rows):
        s = {}
        for (b, h, i) in rows:
            s[(b, h, i)] = O.drift_row(self.P[b, h, i], self.vbar[b, h, i], self.vp[b, h], self.gram[h])
        return s

    def select(self, rows, method, rounds, seed, P=None, s_rows=None, vp=None, vbar=None,
               sign=O.MINIMISE, top_p=1.0):
        P = self.P if P is None else P
        vp = self.vp if vp is None else vp
        vbar = self.vbar if vbar is None else vbar
        s_full = None
        if method == O.DRIFT:
            s_full = np.zeros_like(P)
            s_rows = s_rows if s_rows is not None else self.drift_rows(rows)
            for r, val in s_rows.items():
                s_full[r] = val
        return O.select_blocks(method, P, self.wl.budgets, self.keep_k, self.dense_q, s=s_full,
                               v_pool=vp, vbar=vbar, gram=self.gram, rounds=rounds,
                               rho=self.wl.rho, eps=self.wl.eps, seed=seed, rows=rows, sign=sign,
                               top_p=top_p)

    def attention(self, kept, rows):
        return O.block_sparse_attn(self.q, self.k, self.v, kept, self.scale, rows=rows,
                                   key_block=self.key_block)


# per full-layer parity check: mask agreement and attention error (written out at the end
# of the session when RESS_PARITY_REPORT names a file; see conftest.py)
REPORT: list = []


def close(got, want, rtol, atol, what):
    got = np.asarray(got, np.float64)
    want = np.asarray(want, np.float64)
    err = np.abs(got - want)
    lim = rtol * np.abs(want) + atol
    bad = err > lim
    assert not bad.any(), (f"{what}: {int(bad.sum())} of {bad.size} outside tolerance; "
                           f"worst excess {float((err - lim).max()):.3g}")


def check_drift(s_gpu_rows, orc: OracleLayer, rows):
    s_orc = orc.drift_rows(rows)
    for (b, h, i) in rows:
        vb = orc.vbar[b, h, i].astype(np.float64)
        M = orc.gram[h].astype(np.float64)
        V = orc.vp[b, h].astype(np.float64)
        a = vb @ M @ vb
        bb = np.abs(V @ (M @ vb))
        c = np.einsum("jd,de,je->j", V, M, V)
        tol = orc.P[b, h, i] * np.sqrt(1e-6 * (a + 2 * bb + c))
        close(s_gpu_rows[(b, h, i)], s_orc[(b, h, i)], 1e-4, tol + 1e-12, f"s{(b, h, i)}")


def compare_masks(gpu_kept, orc_sel, nb, what):
    """Kept lists identical on non-ambiguous rows; >= 99.9 % of mask bits agree."""
    rows = sorted(orc_sel["kept"])
    diff_bits, amb, same, mism = 0, 0, 0, []
    for r in rows:
        g = set(gpu_kept[r])
        o = set(orc_sel["kept"][r])
        d = len(g ^ o)
        diff_bits += d
        same += d == 0
        if orc_sel["margin"][r] <= MARGIN:
            amb += 1
        elif d:
            mism.append((r, sorted(g - o), sorted(o - g), orc_sel["margin"][r]))
    agree = 1.0 - diff_bits / (len(rows) * nb)
    assert not mism, f"{what}: {len(mism)} non-ambiguous rows differ, e.g. {mism[:3]}"
    assert agree >= 0.999, f"{what}: mask agreement {agree:.5f}"
    # rows whose kept list is identical to the oracle's, ambiguous or not
    return dict(rows=len(rows), ambiguous=amb, identical_rows=same, agreement=agree)


def check_realized_drift(J_gpu, gpu_kept, sel, orc: OracleLayer, what):
    """Realized J per row against the oracle's, on rows whose kept lists agree.  Both sides
    sum g in fp32 over a hundred-odd terms (the GPU over the drop set or, through Eq. 1,
    the kept set): the tolerance is 1e-4 of J plus 3e-5 of the scale
    T = (sum over the larger side of P_j |vbar - V_j|)^2 |M| / K^2, which bounds the
    cancellation in g."""
    checked = 0
    for r, res in sel["info"].items():
        if res.get("J") is None or sorted(gpu_kept[r]) != sorted(sel["kept"][r]):
            continue
        b, h, i = r
        if orc.dense_q[i]:
            assert float(J_gpu[r]) == 0.0, (what, r)
            continue
        P = orc.P[b, h, i].astype(np.float64)
        e = np.linalg.norm(orc.vbar[b, h, i].astype(np.float64) - orc.vp[b, h].astype(np.float64), axis=1)
        kept = set(sel["kept"][r])
        drop = [j for j in range(orc.nb) if j not in kept]
        sd = float((P[drop] * e[drop]).sum()) if drop else 0.0
        sk = float((P[list(kept)] * e[list(kept)]).sum()) if kept else 0.0
        K = max(1.0 - float(P[drop].sum()), orc.wl.eps)
        T = max(sd, sk) ** 2 * float(np.linalg.norm(orc.gram[h].astype(np.float64), 2)) / K ** 2
        close([float(J_gpu[r])], [res["J"]], 1e-4, 3e-5 * T + 1e-30, f"{what} J{r}")
        checked += 1
    return checked


def check_attention(layer, orc: OracleLayer, rows):
    kept = layer.kept_lists()
    ref = orc.attention(kept, rows)
    out = layer.out.float().cpu().numpy()
    lse = layer.lse.cpu().numpy()
    num, den, worst = 0.0, 0.0, 0.0
    for (b, h, i) in rows:
        o_ref, l_ref = ref[(b, h, i)]
        r0 = i * 128
        o_gpu = out[b, h, r0:r0 + o_ref.shape[0]]
        worst = max(worst, float(np.abs(o_gpu - o_ref).max()))
        num += float(((o_gpu - o_ref) ** 2).sum())
        den += float((o_ref ** 2).sum())
        l_gpu = lse[b, h, r0:r0 + o_ref.shape[0]]
        if len(kept[(b, h, i)]):
            close(l_gpu, l_ref, 1e-4, 1e-3, f"lse{(b, h, i)}")
    rel = math.sqrt(num / max(den, 1e-30))
    assert worst <= 2e-2, f"attention max-abs {worst:.4g}"
    assert rel <= 1e-2, f"attention rel-L2 {rel:.4g}"
    return worst, rel


def sample_rows(B, H, nb, count, seed, always=()):
    rng = np.random.default_rng(seed)
    rows = set(always)
    while len(rows) < min(count, B * H * nb):
        rows.add((int(rng.integers(B)), int(rng.integers(H)), int(rng.integers(nb))))
    return sorted(rows)


def rows_per_head(H, nb, per_head, seed, always_i=()):
    """per_head seeded query blocks of every head (batch 0), always including the query
    blocks listed in always_i."""
    rng = np.random.default_rng(seed)
    rows = set()
    for h in range(H):
        pick = set(int(i) for i in always_i)
        while len(pick) < min(per_head, nb):
            pick.add(int(rng.integers(nb)))
        rows |= {(0, h, i) for i in pick}
    return sorted(rows)
