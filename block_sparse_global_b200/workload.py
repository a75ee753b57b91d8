"""Seeded synthetic inputs shaped like the global-attention layers of a VGGT-style 3D ViT.

This module only draws random numbers and lays tokens out; it holds none of the
attention or selection arithmetic.  Both the CUDA path and the CPU oracle are fed
from here, so that they always see the same bytes.

Token layout (one batch element):
    [ patch tokens of view 0 | view 1 | ... | view V-1 | special tokens, view-major ]
Each view has 1 camera + 4 register tokens ("special tokens") and 37 x 37 = 1369 patch
tokens, 1374 in all, as in VGGT.  The specials are moved to the tail so that they fill
the trailing key blocks: the block grid then has a set of always-kept key blocks at
the end, which is the "sink rule that always keeps the trailing block holding the
special tokens" of the ReSS paper (Supp. F, "Common conditions").  Query blocks that
hold special tokens are computed densely (special tokens are excluded from
sparsification, ReSS paper §3).

Value distributions:
    tiny case   : Q, K, V ~ N(0, 1) drawn in fp32, then rounded to bf16.
    VGGT-shaped : per (view, head) base vector b ~ N(0, I_64); patch Q = b + 0.5 e,
                  patch K = b + 0.5 e' (independent e, e'); special-token Q, K = 4 e''
                  (high norm); V ~ N(0, 1) for every token.
    near-duplicate views (100-view case): 10 seeded views v in 1..99 are rebuilt as
                  x_v = 0.97 x_{v-1} + 0.243 e for the patch tokens of Q, K and V, which
                  keeps the flattened per-view cosine to the neighbour >= 0.9.
    W_O         : the layer's output projection, entries N(0, 1/d), d = heads * 64.

Seeds: seed = 1234 + 100 * case_index + layer, one torch.Generator per workload on the
requested device (a CUDA generator gives different numbers than a CPU one; each run
feeds the same tensors to both sides, so only the recipe has to match).
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import Optional

import torch

HEAD_DIM = 64
BLOCK = 128
VIEW_PATCH = 37 * 37          # patch tokens per view
VIEW_SPECIAL = 5              # 1 camera + 4 register tokens
VIEW_TOKENS = VIEW_PATCH + VIEW_SPECIAL

METHOD_MASS = 0
METHOD_DRIFT = 1
METHOD_RANDOM = 2
METHOD_CDF = 3
METHOD_NAMES = {"mass": METHOD_MASS, "drift": METHOD_DRIFT, "random": METHOD_RANDOM,
                "cdf": METHOD_CDF}


@dataclass(frozen=True)
class Case:
    """One synthetic workload recipe."""
    index: int
    name: str
    heads: int
    views: int                    # 0 = unstructured tiny case
    seq_len: int
    method: str
    sparsity: float
    rounds: int
    dirichlet: bool = False
    near_duplicates: int = 0
    tiny: bool = False


CASES = {
    1: Case(1, "tiny-1024tok-4head", heads=4, views=0, seq_len=1024, method="drift",
            sparsity=0.5, rounds=2, tiny=True),
    2: Case(2, "vggt-8view-16head-mass50", heads=16, views=8, seq_len=8 * VIEW_TOKENS,
            method="mass", sparsity=0.5, rounds=0),
    3: Case(3, "vggt-32view-16head-drift75-r3", heads=16, views=32, seq_len=32 * VIEW_TOKENS,
            method="drift", sparsity=0.75, rounds=3),
    4: Case(4, "vggt-100view-16head-drift90-r5-dirichlet", heads=16, views=100,
            seq_len=100 * VIEW_TOKENS, method="drift", sparsity=0.9, rounds=5,
            dirichlet=True, near_duplicates=10),
    5: Case(5, "vggt-64view-16head-sweep", heads=16, views=64, seq_len=64 * VIEW_TOKENS,
            method="drift", sparsity=0.75, rounds=5),
}

SWEEP_SPARSITIES = (0.0, 0.25, 0.5, 0.75, 0.9)
SWEEP_LAYERS = 24


def num_blocks(n: int, block: int = BLOCK) -> int:
    return (n + block - 1) // block


def special_tail_blocks(seq_len: int, n_special: int, block: int = BLOCK) -> list[int]:
    """Indices of the blocks that overlap the trailing n_special tokens."""
    if n_special <= 0:
        return []
    first_special = seq_len - n_special
    return list(range(first_special // block, num_blocks(seq_len, block)))


def uniform_budget(sparsity: float, n_cand: int) -> int:
    """Candidate blocks kept per row for a target sparsity: round((1 - s) * |P|), at least
    min(2, |P|) (the two-block floor of ReSS Supp. F) and at most |P|."""
    c = int(math.floor((1.0 - sparsity) * n_cand + 0.5))
    return max(min(2, n_cand), min(c, n_cand))


def allocate_budgets(weights: list[float], total: int, cap: int, floor: int) -> list[int]:
    """Head-wise budgets from head weights: proportional allocation with iterative
    clipping at the cap (and at the two-block floor), then a largest-remainder split to
    integers.  This is the allocation step that HeSS uses to turn head scores into
    budgets (ReSS paper, Supp. D "Procedure"); ReSS itself takes the budgets as given."""
    h = len(weights)
    total = max(min(total, cap * h), floor * h)
    fixed: dict[int, float] = {}
    while True:
        free = [i for i in range(h) if i not in fixed]
        left = total - sum(fixed.values())
        wsum = sum(weights[i] for i in free)
        share = {i: left * weights[i] / wsum if wsum > 0 else left / len(free) for i in free}
        over = [i for i in free if share[i] > cap]
        under = [i for i in free if share[i] < floor]
        if not over and not under:
            break
        for i in over:
            fixed[i] = float(cap)
        for i in under:
            fixed[i] = float(floor)
        if len(fixed) == h:
            share = {}
            break
    real = [fixed.get(i, share.get(i, 0.0)) for i in range(h)]
    out = [int(math.floor(x)) for x in real]
    rem = total - sum(out)
    order = sorted(range(h), key=lambda i: (-(real[i] - out[i]), i))
    for i in order:
        if rem <= 0:
            break
        if out[i] < cap:
            out[i] += 1
            rem -= 1
    return out


@dataclass
class Workload:
    case: Case
    layer: int
    seed: int
    q: torch.Tensor               # bf16 [B, H, N, 64]
    k: torch.Tensor
    v: torch.Tensor
    w_o: torch.Tensor             # fp32 [d, H*64]: output projection, head h = columns 64h..64h+63
    keep_k: torch.Tensor          # uint8 [nk]: always-kept key blocks (hold special tokens)
    dense_q: torch.Tensor         # uint8 [nq]: query blocks computed densely
    budgets: list[int]            # per head, candidate blocks kept per row
    method: int
    rounds: int
    rho: float = 0.5
    eps: float = 1e-4
    select_seed: int = 0
    sparsity: float = 0.0
    extras: dict = field(default_factory=dict)
    key_block: int = BLOCK        # tokens per key block (query blocks are always BLOCK)

    @property
    def shape(self):
        b, h, n, d = self.q.shape
        return b, h, n, d

    @property
    def nb(self) -> int:
        return num_blocks(self.q.shape[2])

    @property
    def nq(self) -> int:
        return num_blocks(self.q.shape[2])

    @property
    def nk(self) -> int:
        return num_blocks(self.q.shape[2], self.key_block)


def _vggt_qkv(case: Case, gen: torch.Generator, device) -> tuple:
    H, V = case.heads, case.views
    n_patch = V * VIEW_PATCH
    N = case.seq_len
    f32 = dict(device=device, dtype=torch.float32)
    base = torch.randn(V, H, HEAD_DIM, generator=gen, **f32)
    q = torch.empty(1, H, N, HEAD_DIM, **f32)
    k = torch.empty(1, H, N, HEAD_DIM, **f32)
    # patch tokens: view-major, each view's base vector plus independent noise on Q and K
    bq = base.permute(1, 0, 2).unsqueeze(2).expand(H, V, VIEW_PATCH, HEAD_DIM).reshape(H, n_patch, HEAD_DIM)
    q[0, :, :n_patch] = bq + 0.5 * torch.randn(H, n_patch, HEAD_DIM, generator=gen, **f32)
    k[0, :, :n_patch] = bq + 0.5 * torch.randn(H, n_patch, HEAD_DIM, generator=gen, **f32)
    # special tokens (camera + 4 registers per view) at the tail: high-norm noise
    n_sp = N - n_patch
    q[0, :, n_patch:] = 4.0 * torch.randn(H, n_sp, HEAD_DIM, generator=gen, **f32)
    k[0, :, n_patch:] = 4.0 * torch.randn(H, n_sp, HEAD_DIM, generator=gen, **f32)
    v = torch.randn(1, H, N, HEAD_DIM, generator=gen, **f32)
    if case.near_duplicates:
        pick = torch.randperm(V - 1, generator=gen, device=device)[: case.near_duplicates] + 1
        views = sorted(int(x) for x in pick.cpu())
        cos = []
        for vi in views:
            a, b = vi * VIEW_PATCH, (vi + 1) * VIEW_PATCH
            pa, pb = (vi - 1) * VIEW_PATCH, vi * VIEW_PATCH
            for t in (q, k, v):
                noise = torch.randn(H, VIEW_PATCH, HEAD_DIM, generator=gen, **f32)
                t[0, :, a:b] = 0.97 * t[0, :, pa:pb] + 0.243 * noise
                x, y = t[0, :, a:b].flatten(), t[0, :, pa:pb].flatten()
                cos.append(float(torch.dot(x, y) / (x.norm() * y.norm())))
        assert min(cos) >= 0.9, f"near-duplicate views fell below cosine 0.9: {min(cos)}"
        return q, k, v, {"near_duplicate_views": views, "near_duplicate_min_cos": min(cos)}
    return q, k, v, {}


def head_range(heads: int, world: int, rank: int) -> tuple[int, int]:
    """Contiguous heads [h0, h1) of rank `rank` when `heads` heads are split over `world`
    ranks: sizes differ by at most one, the larger ranges first."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("rank must lie in [0, world)")
    base, extra = divmod(heads, world)
    h0 = rank * base + min(rank, extra)
    return h0, h0 + base + (1 if rank < extra else 0)


def shard_heads(wl: "Workload", h0: int, h1: int) -> "Workload":
    """The heads [h0, h1) of a workload: Q, K, V and the budgets of those heads and the
    W_O columns 64 h0 .. 64 h1 - 1 that multiply them (every step of the path is per
    head, so a shard is computed exactly as inside the whole layer; random-selection keys
    are drawn per call and so differ from the unsplit layer's)."""
    import dataclasses
    return dataclasses.replace(
        wl, q=wl.q[:, h0:h1].contiguous(), k=wl.k[:, h0:h1].contiguous(),
        v=wl.v[:, h0:h1].contiguous(), w_o=wl.w_o[:, 64 * h0:64 * h1].contiguous(),
        budgets=list(wl.budgets[h0:h1]))


def make_workload(index: int, layer: int = 0, device="cpu", method: Optional[str] = None,
                  sparsity: Optional[float] = None, rounds: Optional[int] = None,
                  heads: Optional[int] = None, views: Optional[int] = None,
                  key_block: int = BLOCK) -> Workload:
    """Build the seeded inputs of one synthetic case.  `method`, `sparsity`, `rounds`,
    `heads` and `views` override the case's own values (used by the sweep and by tests
    that need a smaller VGGT-shaped layer).  `key_block` (128 or 64) sets the key-block
    grid: keep_k and the budgets count key blocks of that size, dense_q query blocks of
    128; Q, K, V and W_O do not depend on it."""
    case = CASES[index]
    if heads is not None or views is not None:
        hv = heads if heads is not None else case.heads
        vv = views if views is not None else case.views
        case = Case(case.index, f"{case.name}-h{hv}-v{vv}", heads=hv, views=vv,
                    seq_len=(vv * VIEW_TOKENS if not case.tiny else case.seq_len),
                    method=case.method, sparsity=case.sparsity, rounds=case.rounds,
                    dirichlet=case.dirichlet,
                    near_duplicates=min(case.near_duplicates, max(vv - 1, 0)), tiny=case.tiny)
    seed = 1234 + 100 * index + layer
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    H, N = case.heads, case.seq_len
    extras: dict = {}
    if case.tiny:
        q = torch.randn(1, H, N, HEAD_DIM, generator=gen, device=device)
        k = torch.randn(1, H, N, HEAD_DIM, generator=gen, device=device)
        v = torch.randn(1, H, N, HEAD_DIM, generator=gen, device=device)
        n_special = 0
    else:
        q, k, v, extras = _vggt_qkv(case, gen, device)
        n_special = case.views * VIEW_SPECIAL
    d_model = H * HEAD_DIM
    w_o = torch.randn(d_model, d_model, generator=gen, device=device) / math.sqrt(d_model)
    nq, nk = num_blocks(N), num_blocks(N, key_block)
    tail_q = special_tail_blocks(N, n_special)
    tail_k = special_tail_blocks(N, n_special, key_block)
    keep_k = torch.zeros(nk, dtype=torch.uint8, device=device)
    dense_q = torch.zeros(nq, dtype=torch.uint8, device=device)
    if tail_k:
        keep_k[tail_k] = 1
    if tail_q:
        dense_q[tail_q] = 1
    n_cand = nk - len(tail_k)
    s = case.sparsity if sparsity is None else sparsity
    c = uniform_budget(s, n_cand)
    budgets = [c] * H
    if case.dirichlet:
        e = -torch.log(torch.rand(H, generator=gen, device=device, dtype=torch.float64).clamp_min(1e-300))
        w = (e / e.sum()).cpu().tolist()
        budgets = allocate_budgets(w, c * H, cap=n_cand, floor=min(2, n_cand))
        extras["dirichlet_weights"] = w
    m = case.method if method is None else method
    r = case.rounds if rounds is None else rounds
    if m != "drift":
        r = 0
    bf = torch.bfloat16
    return Workload(case=case, layer=layer, seed=seed,
                    q=q.to(bf).contiguous(), k=k.to(bf).contiguous(), v=v.to(bf).contiguous(),
                    w_o=w_o.float().contiguous(), keep_k=keep_k, dense_q=dense_q,
                    budgets=budgets, method=METHOD_NAMES[m], rounds=r,
                    select_seed=seed * 7919 + 17, sparsity=s, extras=extras,
                    key_block=key_block)
