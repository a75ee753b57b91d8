"""One global-attention layer through libress: device buffers (torch) + the C-ABI calls.

    layer = SparseGlobalAttention(batch, heads, seq_len)
    layer.load_output_projection(w_o)          # M_h, once per layer
    out = layer.forward(q, k, v, method=..., budgets=[...], keep_k=..., dense_q=...)

Every step runs in the library's kernels; this class only owns the buffers and orders
the calls on one stream: pool -> block map + selection (one kernel; for the drift method
the block map, drift score and restoration rounds in one kernel) -> schedule -> attention.
"""
from __future__ import annotations

import math
from typing import Optional, Sequence

import torch

from . import ress as R


class SparseGlobalAttention:
    def __init__(self, batch: int, heads: int, seq_len: int, device="cuda", with_mask: bool = False,
                 key_block: int = 128):
        """key_block: tokens per key block, 128 (the query block's size) or 64 (ReSS
        Supp. F).  Query blocks are always 128 tokens."""
        self.B, self.H, self.N = batch, heads, seq_len
        self.key_block = key_block
        self.nq, self.nk = R.grid(seq_len, key_block)
        self.nb = self.nq  # rows of the block map
        self.shape = R.make_shape(batch, heads, seq_len, key_block=key_block)
        self.device = torch.device(device)
        B, H, nq, nk, N = batch, heads, self.nq, self.nk, seq_len
        f32 = dict(device=self.device, dtype=torch.float32)
        i32 = dict(device=self.device, dtype=torch.int32)
        self.q_pool = torch.empty(B, H, nq, 64, **f32)
        self.k_pool = torch.empty(B, H, nk, 64, **f32)
        self.v_pool = torch.empty(B, H, nk, 64, **f32)
        self.P = torch.empty(B, H, nq, nk, **f32)
        self.v_bar = torch.empty(B, H, nq, 64, **f32)
        self.s = torch.empty(B, H, nq, nk, **f32)
        self.workspace = torch.empty(max(R.ress_drift_workspace_bytes(self.shape),
                                         R.ress_drift_select_workspace_bytes(self.shape), 16),
                                     device=self.device, dtype=torch.uint8)
        self.kv_idx = torch.empty(B, H, nq, nk, **i32)
        self.kv_cnt = torch.empty(B, H, nq, **i32)
        self.order = torch.empty(B * H * nq, **i32)
        self.mask = torch.empty(B, H, nq, nk, device=self.device, dtype=torch.uint8) if with_mask else None
        self.out = torch.empty(B, H, N, 64, device=self.device, dtype=torch.bfloat16)
        self.lse = torch.empty(B, H, N, **f32)
        self.dev_err = torch.zeros(4, **i32)
        self.gram = torch.empty(H, 64, 64, **f32)
        self.scale = 1.0 / math.sqrt(64)

    def load_output_projection(self, w_o: torch.Tensor, stream=None):
        """M_h = W_O^h^T W_O^h for every head (ReSS Eq. 8), computed once per layer."""
        R.ress_head_gram(self.shape, w_o.contiguous().float(), self.gram, stream)

    # ------------------------------------------------------------------ the path
    def pool(self, q, k, v, stream=None):
        R.ress_pool_blocks(self.shape, q, k, v, self.q_pool, self.k_pool, self.v_pool, stream)

    def scores(self, q, k, v, stream=None):
        self.pool(q, k, v, stream)
        R.ress_block_scores(self.shape, self.q_pool, self.k_pool, self.v_pool, self.scale, self.P,
                            self.v_bar, stream)

    def scores_select(self, method: int, budgets: Sequence[int], keep_k=None, dense_q=None,
                      seed: int = 0, write_scores: bool = False, stream=None, top_p: float = 1.0):
        """Block map and MASS / CDF / RANDOM selection in one kernel (after pool()).  P and
        v_bar are written only with write_scores."""
        params = R.select_params(method, budgets, keep_k, dense_q, 0, 0.5, 1e-4, seed, top_p=top_p)
        R.ress_scores_select(self.shape, params, self.q_pool, self.k_pool,
                             self.v_pool if write_scores else None, self.scale,
                             self.P if write_scores else None,
                             self.v_bar if write_scores else None, self.kv_idx, self.kv_cnt,
                             self.mask, self.dev_err, stream)

    def drift(self, stream=None):
        R.ress_drift_scores(self.shape, self.P, self.v_pool, self.v_bar, self.gram, self.s,
                            self.workspace, stream)

    def select(self, method: int, budgets: Sequence[int], keep_k=None, dense_q=None, rounds: int = 0,
               rho: float = 0.5, eps: float = 1e-4, seed: int = 0, stream=None,
               objective: int = R.DRIFT_MINIMISE, drift_out: Optional[torch.Tensor] = None,
               top_p: float = 1.0):
        """Block selection.  `objective` flips the sign of the drift objective (the
        maximising controls, drift only); `drift_out` (fp32 [B,H,nq]) receives each row's
        realized drift J."""
        params = R.select_params(method, budgets, keep_k, dense_q, rounds, rho, eps, seed,
                                 objective, drift_out, top_p)
        drift = method == R.SELECT_DRIFT
        state = drift or drift_out is not None
        R.ress_select_blocks(self.shape, params, self.P, self.s if drift else None,
                             self.v_pool if state else None, self.v_bar if state else None,
                             self.gram if state else None, self.kv_idx, self.kv_cnt, self.mask,
                             self.dev_err, stream)

    def drift_select(self, budgets: Sequence[int], keep_k=None, dense_q=None, rounds: int = 0,
                     rho: float = 0.5, eps: float = 1e-4, stream=None,
                     objective: int = R.DRIFT_MINIMISE, drift_out: Optional[torch.Tensor] = None,
                     write_scores: bool = False):
        """Block map, drift score and DRIFT selection in one kernel (after pool()); P, v_bar
        and s are written only with write_scores."""
        params = R.select_params(R.SELECT_DRIFT, budgets, keep_k, dense_q, rounds, rho, eps, 0,
                                 objective, drift_out)
        R.ress_drift_select(self.shape, params, self.q_pool, self.k_pool, self.v_pool, self.gram,
                            self.scale, self.P if write_scores else None,
                            self.v_bar if write_scores else None,
                            self.s if write_scores else None, self.kv_idx, self.kv_cnt,
                            self.workspace, self.mask, self.dev_err, stream)

    def attend(self, q, k, v, stream=None, schedule: bool = True):
        if schedule:
            R.ress_attn_schedule(self.shape, self.kv_cnt, self.order, stream)
        R.ress_block_sparse_attn(self.shape, q, k, v, self.kv_idx, self.kv_cnt,
                                 self.order if schedule else None, self.scale, self.out, self.lse,
                                 self.dev_err, stream)

    def forward(self, q, k, v, method: int, budgets: Sequence[int], keep_k=None, dense_q=None,
                rounds: int = 0, rho: float = 0.5, eps: float = 1e-4, seed: int = 0, stream=None,
                top_p: float = 1.0, write_scores: bool = False, fused: bool = True):
        """pool -> block map + selection (one kernel: drift_select for DRIFT, scores_select
        otherwise; with fused=False, DRIFT runs the separate block-map, drift and selection
        calls) -> schedule -> attention.  write_scores: the fused kernels also write P,
        v_bar (and s for DRIFT)."""
        self.pool(q, k, v, stream)
        if method == R.SELECT_DRIFT and fused:
            self.drift_select(budgets, keep_k, dense_q, rounds, rho, eps, stream,
                              write_scores=write_scores)
        elif method == R.SELECT_DRIFT:
            R.ress_block_scores(self.shape, self.q_pool, self.k_pool, self.v_pool, self.scale,
                                self.P, self.v_bar, stream)
            self.drift(stream)
            self.select(method, budgets, keep_k, dense_q, rounds, rho, eps, seed, stream)
        else:
            self.scores_select(method, budgets, keep_k, dense_q, seed, write_scores, stream=stream,
                               top_p=top_p)
        self.attend(q, k, v, stream)
        return self.out

    # ------------------------------------------------------------- CUDA graphs
    @staticmethod
    def capture(fn, warmup: int = 2) -> "torch.cuda.CUDAGraph":
        """Captures the library calls that `fn()` enqueues on the current stream into a CUDA
        graph, after `warmup` eager runs on a side stream; `graph.replay()` then launches
        the same kernels with the same arguments on the current stream.  The library
        allocates nothing and its launches take only host-side attribute calls, so a layer
        captures as is; the tensors `fn` uses must keep their addresses (copy new inputs
        into them before a replay)."""
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            for _ in range(warmup):
                fn()
        torch.cuda.current_stream().wait_stream(side)
        graph = torch.cuda.CUDAGraph()
        # thread-local capture: CUDA calls of other threads (a process group's watchdog,
        # for one) do not invalidate it; the captured calls themselves allocate nothing
        with torch.cuda.graph(graph, capture_error_mode="thread_local"):
            fn()
        return graph

    def capture_forward(self, q, k, v, method: int, budgets: Sequence[int], keep_k=None,
                        dense_q=None, rounds: int = 0, rho: float = 0.5, eps: float = 1e-4,
                        seed: int = 0, top_p: float = 1.0) -> "torch.cuda.CUDAGraph":
        """forward() on these tensors as one CUDA graph (pool, block map, drift, selection,
        schedule and attention in one launch of the graph)."""
        return self.capture(lambda: self.forward(q, k, v, method, budgets, keep_k, dense_q,
                                                 rounds, rho, eps, seed, top_p=top_p))

    # ------------------------------------------------ end to end from host buffers
    @staticmethod
    def group_sizes(heads: int, groups: int, taper: bool = False) -> list[int]:
        """Heads per group for forward_host().  The copies in run back to back and set the
        pace as long as each group's kernels end before the next group's copy in does;
        after the last copy in, the last group's kernels and copy out are what is left.
        By default the groups are near-equal, the larger ones first (sizes differ by at
        most one and never grow), which keeps the kernels behind the copies when they take
        nearly as long per head (the 100-view layer); with `taper` the sizes fall off
        linearly (weights groups, groups-1, ..., 1; largest-remainder rounding, at least
        one head each), which suits layers whose kernels are much shorter than their
        copies."""
        groups = max(1, min(groups, heads))
        if not taper:
            return [heads // groups + (1 if g < heads % groups else 0) for g in range(groups)]
        w = [groups - g for g in range(groups)]
        extra = heads - groups                     # one head each, then the rest by weight
        real = [extra * x / sum(w) for x in w]
        sizes = [1 + int(r) for r in real]
        order = sorted(range(groups), key=lambda g: (-(real[g] - int(real[g])), g))
        for g in order[: heads - sum(sizes)]:
            sizes[g] += 1
        return sizes

    @staticmethod
    def plan_head_order(budgets: Sequence[int], sizes: Sequence[int]) -> list[int]:
        """Heads in processing order for groups of the given sizes.  The kernels of a
        head take time roughly in proportion to its budget (its kept blocks), the copies
        the same time for every head, so the cheapest heads go to the last group (what is
        left after the last copy in), and the other heads are spread over the other groups
        largest first, each to the group with the least work per head so far, so that no
        group's kernels outlast the next group's copy in.  Heads keep ascending order
        within a group.  With equal budgets the heads stay in order (contiguous heads are
        copied in one piece)."""
        H, G = len(budgets), len(sizes)
        if G <= 1 or len(set(int(b) for b in budgets)) == 1:
            return list(range(H))  # equal budgets: nothing to balance, keep the copies whole
        cost = [int(b) + 16 for b in budgets]  # kept candidates + always-kept / fixed work
        asc = sorted(range(H), key=lambda h: (cost[h], h))
        last = asc[:sizes[-1]]
        rest = sorted(asc[sizes[-1]:], key=lambda h: (-cost[h], h))
        members: list[list[int]] = [[] for _ in range(G - 1)]
        load = [0] * (G - 1)
        for h in rest:
            g = min((g for g in range(G - 1) if len(members[g]) < sizes[g]),
                    key=lambda g: (load[g] / sizes[g], g))
            members[g].append(h)
            load[g] += cost[h]
        return [h for m in members for h in sorted(m)] + sorted(last)

    def make_groups(self, w_o: torch.Tensor, groups: int, taper: bool = False,
                    sizes: Optional[Sequence[int]] = None,
                    budgets: Optional[Sequence[int]] = None):
        """Splits the heads into groups for forward_host(): `sizes` heads per group if
        given (positive, summing to the head count), else `groups` groups sized by
        group_sizes().  With `budgets`, the heads are assigned by plan_head_order();
        without, group g takes the next contiguous range.  One layer object per group,
        with the W_O columns of its heads (head h owns columns 64h .. 64h+63)."""
        if self.B != 1:
            raise ValueError("forward_host splits heads of one batch element (B = 1)")
        if sizes is not None:
            sizes = [int(n) for n in sizes]
            if min(sizes) < 1 or sum(sizes) != self.H:
                raise ValueError(f"group sizes {sizes} must be positive and sum to {self.H}")
        else:
            sizes = self.group_sizes(self.H, groups, taper)
        order = self.plan_head_order(budgets, sizes) if budgets is not None else list(range(self.H))
        if sorted(order) != list(range(self.H)):
            raise ValueError("the head order must be a permutation of the heads")
        self._order = order
        self._groups = []
        s0 = 0
        for n in sizes:
            heads = order[s0:s0 + n]
            sub = SparseGlobalAttention(1, n, self.N, device=self.device, key_block=self.key_block)
            cols = torch.cat([torch.arange(64 * h, 64 * h + 64, device=w_o.device) for h in heads])
            sub.load_output_projection(w_o[:, cols])
            self._groups.append((s0, s0 + n, sub, heads))
            s0 += n
        # copies in, kernels of even groups, copies out, kernels of odd groups
        self._streams = [torch.cuda.Stream(self.device) for _ in range(4)]
        return self._groups

    def forward_host(self, q_host, k_host, v_host, out_host, method: int, budgets: Sequence[int],
                     keep_k=None, dense_q=None, rounds: int = 0, rho: float = 0.5,
                     eps: float = 1e-4, seed: int = 0, q_dev=None, k_dev=None, v_dev=None,
                     top_p: float = 1.0):
        """The layer end to end from pinned host tensors [1,H,N,64] bf16 to the pinned host
        output.  Heads are processed in the groups of make_groups(): the copy in of group
        g+1, the kernels of group g and the copy out of group g-1 overlap, and the kernels
        of consecutive groups run on two streams (every group has its own buffers), so that
        a group's selection can fill the SMs that the previous group's attention leaves
        idle in its last wave.  The device staging tensors hold the heads in processing order (slot s
        holds head make_groups' order[s]); contiguous runs of heads are copied in one piece.
        RANDOM selection runs as one group in head order (its keys depend on the head index
        within the call).  The caller's current stream waits for the whole layer.
        q_dev, k_dev, v_dev: optional device staging tensors of the same shape."""
        groups = getattr(self, "_groups", None)
        if not groups:
            raise RuntimeError("call make_groups() first")
        if method == R.SELECT_RANDOM and (len(groups) > 1 or self._order != list(range(self.H))):
            raise ValueError("random selection runs as one group in head order")
        q_dev = torch.empty_like(q_host, device=self.device) if q_dev is None else q_dev
        k_dev = torch.empty_like(k_host, device=self.device) if k_dev is None else k_dev
        v_dev = torch.empty_like(v_host, device=self.device) if v_dev is None else v_dev
        budgets = list(budgets)
        s_in, s_even, s_out, s_odd = self._streams
        main = torch.cuda.current_stream(self.device)
        for s in self._streams:
            s.wait_stream(main)

        def runs(s0, heads):
            # (first slot, first head, count) of every run of consecutive heads
            out, i = [], 0
            while i < len(heads):
                j = i
                while j + 1 < len(heads) and heads[j + 1] == heads[j] + 1:
                    j += 1
                out.append((s0 + i, heads[i], j - i + 1))
                i = j + 1
            return out

        for gi, (s0, s1, sub, heads) in enumerate(groups):
            s_cmp = s_odd if gi % 2 else s_even
            with torch.cuda.stream(s_in):
                for (sl, h, n) in runs(s0, heads):
                    for dev, host in ((q_dev, q_host), (k_dev, k_host), (v_dev, v_host)):
                        dev[:, sl:sl + n].copy_(host[:, h:h + n], non_blocking=True)
                arrived = torch.cuda.Event()
                arrived.record(s_in)
            s_cmp.wait_event(arrived)
            with torch.cuda.stream(s_cmp):
                sub.forward(q_dev[:, s0:s1], k_dev[:, s0:s1], v_dev[:, s0:s1], method,
                            [budgets[h] for h in heads], keep_k, dense_q, rounds, rho, eps, seed,
                            stream=s_cmp, top_p=top_p)
                done = torch.cuda.Event()
                done.record(s_cmp)
            s_out.wait_event(done)
            with torch.cuda.stream(s_out):
                for (sl, h, n) in runs(0, heads):
                    out_host[:, h:h + n].copy_(sub.out[:, sl:sl + n], non_blocking=True)
        for s in self._streams:
            main.wait_stream(s)
        return out_host

    def kernel_launches(self, method: int, fused: bool = True) -> int:
        """Kernels one forward() launches: drift fused: pool, drift prep (c_j), fused
        block map + drift + select, schedule, attention; drift unfused: pool, scores, drift
        prep, drift, select, schedule, attention; mass / cdf / random: pool, fused scores +
        select, schedule, attention."""
        if method == R.SELECT_DRIFT:
            return 5 if fused else 7
        return 4

    def device_error(self) -> int:
        return int(self.dev_err[0].item())

    def kept_lists(self):
        """{(b,h,i): ascending kept key blocks} from the device kv list (host copy); i runs
        over the nq query blocks."""
        idx = self.kv_idx.cpu()
        cnt = self.kv_cnt.cpu()
        out = {}
        for b in range(self.B):
            for h in range(self.H):
                for i in range(self.nq):
                    c = int(cnt[b, h, i])
                    out[(b, h, i)] = idx[b, h, i, :c].tolist()
        return out
