#!/usr/bin/env python
"""Benchmark of one block-sparse global-attention layer on B200 (one JSON line).

A step is one pass of the whole path over one layer of synthetic VGGT-shaped input:
pool -> pooled block map -> (drift) -> selection -> schedule -> block-sparse attention.
Default workload: 100 views x 1374 tokens (137400), 16 heads, head_dim 64, block 128, 90 %
sparsity, drift selection with 5 restoration rounds and Dirichlet head budgets (the largest
single-GPU layer).  `--case 2/3` runs the 8-view mass and 32-view drift layers instead.

    python bench.py [--gpus N --steps K --warmup W] [--case 4] [--impl reference]

value      whole-job effective TFLOP/s over kept tiles (kept-tile FLOPs of all ranks /
           max over ranks of the summed per-step device time); inputs resident in HBM,
           L2 flushed (256 MiB write) before every timed step; the step's kernels are
           replayed from two CUDA graphs (selection part, attention; `--eager` launches
           them one by one).
e2e        the same metric with Q, K, V copied from pinned host memory and the output
           copied back inside every timed step.
roofline   the attention kernel (dominant): kept-tile FLOPs per launch / its mean CUDA-
           event duration, against the measured dense bf16 tensor-core peak.
With N > 1 (torchrun) the heads of the layer are split over the ranks (--shard heads,
strong scaling) or every rank runs its own layer (--shard layers, weak scaling); either
way no collective on the data path.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "global-attn layer latency (ms) & effective TFLOP/s on kept tiles vs bf16 peak"
PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
FALLBACK_BF16_TFLOPS = 1590.0
L2_FLUSH_BYTES = 256 << 20


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--case", type=int, default=4,
                    help="synthetic case index (4 = 100 views, drift 90%%, R = 5, Dirichlet budgets; "
                         "2 = 8 views, mass 50%%; 3 = 32 views, drift 75%%, R = 3)")
    ap.add_argument("--method", choices=["mass", "drift", "random", "cdf"], default=None)
    ap.add_argument("--top-p", type=float, default=0.9,
                    help="mass threshold of the cdf method (the budget from --sparsity caps it)")
    ap.add_argument("--sparsity", type=float, default=None)
    ap.add_argument("--key-block", type=int, choices=[128, 64], default=128,
                    help="tokens per key block (query blocks are 128); 64 = ReSS Supp. F grid")
    ap.add_argument("--objective", choices=["min", "max-swaps", "max-full"], default="min",
                    help="drift objective: the method, or a drift-maximising control (drift only)")
    ap.add_argument("--l2-flush", choices=["write", "write+read"], default="write+read",
                    help="L2 flush before every timed step: a 256 MiB write, then (default) a "
                         "256 MiB read of another buffer, so that the write's dirty lines go back "
                         "to HBM before the step instead of during its first kernel's reads")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--e2e-groups", type=int, default=None,
                    help="head groups of the host-buffer call (copy in / kernels / copy out overlap); "
                         "default: 9 when a head's Q, K and V take at least 32 MB, else 6")
    ap.add_argument("--e2e-split", default=None,
                    help="explicit heads per group of the host-buffer call, e.g. 8,4,2,1,1")
    ap.add_argument("--e2e-taper", action="store_true",
                    help="linearly tapered head groups instead of near-equal ones (last group smallest)")
    ap.add_argument("--quick", action="store_true", help="timed loop only (profiling runs)")
    ap.add_argument("--shard", choices=["heads", "layers"], default="heads",
                    help="with N > 1 GPUs: split the heads of one layer over the ranks (strong "
                         "scaling), or give every rank its own layer (weak scaling)")
    ap.add_argument("--unfused", action="store_true",
                    help="drift: separate block-map, drift-score and selection calls instead of "
                         "the fused drift-selection kernel")
    ap.add_argument("--eager", action="store_true",
                    help="launch the kernels one by one instead of replaying the step from CUDA "
                         "graphs (selection part and attention, each captured once)")
    ap.add_argument("--sweep", action="store_true",
                    help="64-view sweep: sparsity {0,25,50,75,90}%% x {mass, drift, random} over "
                         "--layers independent layers, one JSON line per point (not the bench line)")
    ap.add_argument("--layers", type=int, default=24, help="layers of the --sweep")
    ap.add_argument("--sweep-out", default=None,
                    help="JSONL file the --sweep appends each finished point to; points already "
                         "in it are skipped (resume)")
    return ap.parse_args()


def measured_traffic(workload: str):
    """DRAM bytes (read + write) of one attention launch from the committed ncu record,
    or None when the record is for another workload or the kernel source has changed
    since the counters were taken."""
    import hashlib
    rec = os.path.join(ROOT, "profiles", f"attn_kernel_{workload}_traffic.txt")
    src = os.path.join(ROOT, "block_sparse_global_b200", "csrc", "k_attn.cu")
    try:
        kv = dict(l.strip().split("=", 1) for l in open(rec) if "=" in l and not l.startswith("#"))
        with open(src, "rb") as f:
            sha = hashlib.sha256(f.read()).hexdigest()
    except OSError:
        return None
    if kv.get("kernel_source_sha256") != sha or kv.get("workload") != workload:
        return None
    return int(kv["dram_bytes_read"]) + int(kv["dram_bytes_write"])


class L2Flush:
    """Evicts the layer's inputs from L2 before a timed step: writes a 256 MiB buffer
    (twice the 126 MB L2).  With `clean`, it then also reads a second 256 MiB buffer, so
    that the dirty lines the write left in L2 are written back to HBM here, outside the
    timed region, instead of during the step's first reads."""

    def __init__(self, dev, clean: bool):
        import torch
        self.buf = torch.empty(L2_FLUSH_BYTES // 4, device=dev, dtype=torch.float32)
        self.clean = clean
        self.other = torch.ones(L2_FLUSH_BYTES // 4, device=dev, dtype=torch.float32) if clean else None

    def __call__(self):
        self.buf.fill_(1.0)
        if self.clean:
            self.other.sum()

    def describe(self) -> str:
        return ("flushed before every timed step (256 MiB write, then a 256 MiB read of "
                "another buffer, so the write's dirty lines leave L2 before the step)"
                if self.clean else "flushed before every timed step (256 MiB write)")


FP32_PEAK_SOURCE = ("derived: 148 SMs x 128 fp32 FMA lanes x 2 FLOP x clocks.max.sm "
                    "(1965 MHz), no measured fp32 figure")


def fp32_fma_peak_tflops(sm_mhz: float = 1965.0) -> float:
    """fp32 FMA-pipe peak of a B200 from its unit counts: 148 SMs x 128 lanes x 2 FLOP per
    clock at the maximum SM clock."""
    return 148 * 128 * 2 * sm_mhz * 1e6 / 1e12


def peaks():
    try:
        with open(PEAKS_FILE) as f:
            p = json.load(f)
        return float(p["bf16_tflops"]), float(p.get("hbm_gbs", 0.0)), "measured"
    except Exception:
        return FALLBACK_BF16_TFLOPS, 6650.0, "fallback"


# ------------------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return None
        mhz = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        maxmhz = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[k] for r in rows for k in range(4) if r[5 + k].lower() == "active"})
        loaded = [m for m in mhz if m > 0.5 * max(mhz)] if mhz else []
        return {"sm_mhz": statistics.median(loaded) if loaded else None,
                "sm_max_mhz": max(maxmhz) if maxmhz else None, "reasons": reasons,
                "samples": len(rows)}


# ---------------------------------------------------------------------- workload
def build_case(args, rank: int):
    from block_sparse_global_b200 import workload as W
    return W.make_workload(args.case, layer=rank, device="cuda", method=args.method,
                           sparsity=args.sparsity, key_block=getattr(args, "key_block", 128))


def workload_name(wl) -> str:
    return wl.case.name + ("" if wl.key_block == 128 else f"-kb{wl.key_block}")


def kept_tile_flops(kv_idx, kv_cnt, N: int, key_block: int = 128) -> float:
    """Algorithmic FLOPs over the kept (query block, key block) pairs: sum of
    4 * rows * cols * 64 (QK^T and PV), rows and cols counting only tokens < N (query
    blocks of 128 tokens, key blocks of key_block)."""
    import torch
    B, H, nq, nk = kv_idx.shape
    dev = kv_idx.device
    rows = torch.clamp(N - torch.arange(nq, device=dev) * 128, max=128).to(torch.float64)
    valid = torch.clamp(N - torch.arange(nk, device=dev) * key_block, max=key_block).to(torch.float64)
    pos = torch.arange(nk, device=dev).view(1, 1, 1, nk)
    live = pos < kv_cnt.unsqueeze(-1)
    cols = torch.where(live, valid[kv_idx.clamp(0, nk - 1).long()],
                       torch.zeros((), dtype=torch.float64, device=dev))
    per_row = cols.sum(-1) * rows.view(1, 1, nq)
    return float(per_row.sum().item()) * 4.0 * 64.0


def reduce_over_ranks(ms: float, work: float) -> tuple[float, float]:
    """Whole-job figures of a weak-scaling run: (max over ranks of the device time, sum over
    ranks of the work).  Identity without an initialised process group; the reduction runs
    on the backend's own device (CUDA tensors for NCCL, host tensors for gloo)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(ms), float(work)
    dev = torch.device("cuda", torch.cuda.current_device()) if dist.get_backend() == "nccl" \
        else torch.device("cpu")
    t = torch.tensor([float(ms)], dtype=torch.float64, device=dev)
    w = torch.tensor([float(work)], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    dist.all_reduce(w, op=dist.ReduceOp.SUM)
    return float(t.item()), float(w.item())


def run_ours(args):
    import torch
    import torch.distributed as dist

    from block_sparse_global_b200 import build as B
    from block_sparse_global_b200 import ress as R
    from block_sparse_global_b200.pipeline import SparseGlobalAttention

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if rank == 0:
        B.build()
    if world > 1:
        dist.barrier()
    R.load()

    if world > 1 and args.shard == "heads":
        # one layer, its heads split over the ranks: each rank runs the whole path on its
        # heads (every step is per head, so nothing crosses ranks on the data path)
        from block_sparse_global_b200 import workload as W
        full = build_case(args, 0)
        h0, h1 = W.head_range(full.q.shape[1], world, rank)
        wl = W.shard_heads(full, h0, h1)
        del full
    else:
        wl = build_case(args, rank)
    objective = {"min": R.DRIFT_MINIMISE, "max-swaps": R.DRIFT_MAXIMISE_SWAPS,
                 "max-full": R.DRIFT_MAXIMISE_FULL}[args.objective]
    if objective != R.DRIFT_MINIMISE and wl.method != R.SELECT_DRIFT:
        raise SystemExit("--objective max-* is a control of drift selection (use --case 3/4 or --method drift)")
    Bsz, H, N, _ = wl.q.shape
    q, k, v = wl.q, wl.k, wl.v
    keep_k, dense_q = wl.keep_k, wl.dense_q
    layer = SparseGlobalAttention(Bsz, H, N, device=dev, key_block=wl.key_block)
    layer.load_output_projection(wl.w_o)
    flush = L2Flush(dev, args.l2_flush == "write+read")
    stream = torch.cuda.current_stream()

    drift_method = wl.method == R.SELECT_DRIFT
    unfused = drift_method and args.unfused   # separate block-map, drift and select calls

    def step():
        layer.pool(q, k, v)
        if unfused:
            R.ress_block_scores(layer.shape, layer.q_pool, layer.k_pool, layer.v_pool, layer.scale,
                                layer.P, layer.v_bar)
            layer.drift()
            layer.select(wl.method, wl.budgets, keep_k, dense_q, wl.rounds, wl.rho, wl.eps,
                         wl.select_seed, objective=objective)
        elif drift_method:   # block map, drift score and selection in one kernel
            layer.drift_select(wl.budgets, keep_k, dense_q, wl.rounds, wl.rho, wl.eps,
                               objective=objective)
        else:                # block map and selection in one kernel
            layer.scores_select(wl.method, wl.budgets, keep_k, dense_q, wl.select_seed,
                                top_p=args.top_p)
        R.ress_attn_schedule(layer.shape, layer.kv_cnt, layer.order)

    def attn():
        R.ress_block_sparse_attn(layer.shape, q, k, v, layer.kv_idx, layer.kv_cnt, layer.order,
                                 layer.scale, layer.out, layer.lse, layer.dev_err)

    for _ in range(args.warmup):
        flush()
        step()
        attn()
    torch.cuda.synchronize()
    if layer.device_error():
        raise SystemExit(f"device error {layer.device_error()} during warm-up")
    flops = kept_tile_flops(layer.kv_idx, layer.kv_cnt, N, wl.key_block)
    kept_frac = float(layer.kv_cnt.sum().item()) / (Bsz * H * layer.nq * layer.nk)
    # realized drift J of every row's selection (extra, untimed passes: the block map
    # written out, then the selection with its J output)
    J = torch.zeros(Bsz, H, layer.nq, device=dev)
    layer.pool(q, k, v)
    if drift_method and not unfused:
        layer.drift_select(wl.budgets, keep_k, dense_q, wl.rounds, wl.rho, wl.eps,
                           objective=objective, drift_out=J)
    else:
        R.ress_block_scores(layer.shape, layer.q_pool, layer.k_pool, layer.v_pool, layer.scale,
                            layer.P, layer.v_bar)
        if drift_method:
            layer.drift()
        layer.select(wl.method, wl.budgets, keep_k, dense_q, wl.rounds, wl.rho, wl.eps,
                     wl.select_seed, objective=objective, drift_out=J, top_p=args.top_p)
    torch.cuda.synchronize()
    sparse_rows = J[:, :, ~wl.dense_q.bool().to(dev)] if wl.dense_q is not None else J
    drift_mean = float(sparse_rows.mean().item())

    # the timed steps replay CUDA graphs of the same calls (one launch per part instead of
    # one per kernel); eager launches if asked, or if the capture fails
    run_step, run_attn = step, attn
    launch_mode = "eager launches"
    if not args.eager:
        try:
            g_step = SparseGlobalAttention.capture(step)
            g_attn = SparseGlobalAttention.capture(attn)
            torch.cuda.synchronize()
            run_step, run_attn = g_step.replay, g_attn.replay
            launch_mode = "CUDA graph replay (selection part, attention)"
        except Exception as exc:   # the step still runs, eagerly
            torch.cuda.synchronize()
            launch_mode = f"eager launches (graph capture failed: {type(exc).__name__})"
    clocks = ClockSampler(local)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clocks.start()
    for s in range(args.steps):
        flush()
        ev[s][0].record(stream)
        run_step()
        ev[s][1].record(stream)
        run_attn()
        ev[s][2].record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clk = clocks.stop()
    step_ms = [e[0].elapsed_time(e[2]) for e in ev]
    attn_ms = [e[1].elapsed_time(e[2]) for e in ev]
    total_ms = sum(step_ms)
    total_ms_max, flops_all = reduce_over_ranks(total_ms, flops * args.steps)
    value = flops_all / (total_ms_max * 1e-3) / 1e12

    extra = {}
    if not args.quick:
        # per-kernel breakdown (separate pass, same inputs)
        # the step's own kernels, then (drift) the separate calls the fused kernel replaces
        if not drift_method:
            names = ["pool", "scores_select", "schedule", "attention"]
        elif unfused:
            names = ["pool", "block_scores", "drift", "select", "schedule", "attention"]
        else:
            names = ["pool", "drift_select", "schedule", "attention", "block_scores", "drift", "select"]
        calls = {
            "drift_select": lambda: layer.drift_select(wl.budgets, keep_k, dense_q, wl.rounds, wl.rho,
                                                       wl.eps, objective=objective),
            "scores_select": lambda: layer.scores_select(wl.method, wl.budgets, keep_k, dense_q,
                                                         wl.select_seed, top_p=args.top_p),
            "pool": lambda: R.ress_pool_blocks(layer.shape, q, k, v, layer.q_pool, layer.k_pool, layer.v_pool),
            "block_scores": lambda: R.ress_block_scores(layer.shape, layer.q_pool, layer.k_pool, layer.v_pool,
                                                        layer.scale, layer.P, layer.v_bar),
            "drift": layer.drift,
            "select": lambda: layer.select(wl.method, wl.budgets, keep_k, dense_q, wl.rounds, wl.rho,
                                           wl.eps, wl.select_seed, objective=objective),
            "schedule": lambda: R.ress_attn_schedule(layer.shape, layer.kv_cnt, layer.order),
            "attention": attn,
        }
        per = {}
        for name in names:
            times = []
            for _ in range(5):
                flush()
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record(stream)
                calls[name]()
                b.record(stream)
                torch.cuda.synchronize()
                times.append(a.elapsed_time(b))
            per[name] = round(statistics.median(times), 4)
        extra["kernels_ms"] = per
        if drift_method and not unfused:
            extra["kernels_ms_note"] = ("drift_select = block map + drift score + selection in one "
                                        "kernel (with its c_j prep launch), the step's path; "
                                        "block_scores, drift and select are the separate calls it "
                                        "replaces, timed for comparison")
        # the HBM-bound step: pooling reads Q, K, V once and writes the fp32 block means
        _, hbm_peak_gbs, _ = peaks()
        pool_bytes = 3 * q.numel() * q.element_size() + 4 * Bsz * H * (layer.nq + 2 * layer.nk) * 64
        # algorithmic HBM bytes of each block-level step: pooling reads Q, K, V and writes
        # the fp32 means (HBM-bound); the block map writes P, the drift pass reads P and
        # writes s, the selection reads P (and s) and writes the kept lists -- those three
        # are fp32 / latency bound, their GB/s is reported for completeness
        maps = 4 * Bsz * H * layer.nq * layer.nk
        lists = 4 * Bsz * H * layer.nq * (layer.nk + 1)
        bytes_of = {"pool": (pool_bytes, "hbm"),
                    "block_scores": (maps, "fp32 / latency"),
                    "drift": (2 * maps, "fp32 / latency"),
                    "select": ((2 if wl.method == R.SELECT_DRIFT else 1) * maps + lists, "fp32 / latency"),
                    "scores_select": (lists, "fp32 / latency"),
                    "drift_select": (lists, "fp32 / latency")}
        hk = {}
        for name, (nbytes, bound) in bytes_of.items():
            if per.get(name):
                gbs = nbytes / (per[name] * 1e-3) / 1e9
                hk[name] = {"algorithmic_bytes": nbytes, "gbs": round(gbs, 1), "bound": bound,
                            "frac": round(gbs / hbm_peak_gbs, 4) if hbm_peak_gbs else None}
        extra["hbm_kernels"] = dict(hk, peak_gbs=hbm_peak_gbs)
        # the fp32 block-level kernels against the FMA pipes: algorithmic FMAs per launch
        # (each 2 FLOP) / event time, as a fraction of the fp32 FMA peak derived from the
        # unit counts (no measured fp32 figure exists for this machine)
        fma_peak = fp32_fma_peak_tflops()
        rows_cols = Bsz * H * layer.nq * layer.nk
        restore_rounds = wl.rounds if wl.method == R.SELECT_DRIFT else 0
        fma_of = {"block_scores": 2 * rows_cols * 64,          # logits and vbar
                  "drift": rows_cols * 64,                      # w_i . V_j
                  "select": (restore_rounds + 1) * rows_cols * 64 if restore_rounds else 0,
                  # all three in one kernel
                  "drift_select": (restore_rounds + 4) * rows_cols * 64 if drift_method else 0}
        fk = {}
        for name, fma in fma_of.items():
            if fma and per.get(name):
                tf = 2.0 * fma / (per[name] * 1e-3) / 1e12
                fk[name] = {"fma": fma, "tflops": round(tf, 2), "frac": round(tf / fma_peak, 4)}
        extra["fp32_kernels"] = dict(fk, peak_tflops=round(fma_peak, 1),
                                     peak_source=FP32_PEAK_SOURCE)
        # same-shape dense attention: every query block keeps every key block
        nq, nk = layer.nq, layer.nk
        dense_idx = torch.arange(nk, device=dev, dtype=torch.int32).expand(Bsz, H, nq, nk).contiguous()
        dense_cnt = torch.full((Bsz, H, nq), nk, device=dev, dtype=torch.int32)
        dense_out = torch.empty_like(layer.out)
        dts = []
        for _ in range(5):
            flush()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            R.ress_block_sparse_attn(layer.shape, q, k, v, dense_idx, dense_cnt, None, layer.scale, dense_out)
            b.record(stream)
            torch.cuda.synchronize()
            dts.append(a.elapsed_time(b))
        dense_flops = kept_tile_flops(dense_idx, dense_cnt, N, wl.key_block)
        dms = statistics.median(dts)
        extra["dense_attention"] = {"ms": round(dms, 4), "tflops": round(dense_flops / dms / 1e9, 1)}
        del dense_idx, dense_cnt, dense_out
        # end to end through the API with host buffers
        if not args.no_e2e:
            qh, kh, vh = (x.cpu().pin_memory() for x in (q, k, v))
            outh = torch.empty(layer.out.shape, dtype=layer.out.dtype).pin_memory()
            qd, kd, vd = (torch.empty_like(x) for x in (q, k, v))
            # head groups: copies in, kernels and copies out overlap on three streams
            # more, smaller groups once a head's copy is long enough that the per-copy
            # overhead no longer shows (the 100-view layer); the kernels of consecutive
            # groups overlap on two streams
            per_head = 3 * q[0, 0].numel() * q.element_size()
            want = args.e2e_groups if args.e2e_groups else (9 if per_head >= 32 << 20 else 6)
            groups = 1 if wl.method == R.SELECT_RANDOM else max(1, min(want, H))
            split = [int(x) for x in args.e2e_split.split(",")] if args.e2e_split else None
            layer.make_groups(wl.w_o, groups, taper=args.e2e_taper,
                              sizes=split if wl.method != R.SELECT_RANDOM else None,
                              budgets=wl.budgets if wl.method != R.SELECT_RANDOM else None)
            e2e_ms = []
            for s in range(max(3, args.steps // 2) + 2):
                flush()
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record(stream)
                layer.forward_host(qh, kh, vh, outh, wl.method, wl.budgets, keep_k, dense_q,
                                   wl.rounds, wl.rho, wl.eps, wl.select_seed, q_dev=qd, k_dev=kd,
                                   v_dev=vd, top_p=args.top_p)
                b.record(stream)
                torch.cuda.synchronize()
                if s >= 2:
                    e2e_ms.append(a.elapsed_time(b))
            em, e2e_flops = reduce_over_ranks(statistics.mean(e2e_ms), flops)
            extra["e2e"] = {"value": round(e2e_flops / (em * 1e-3) / 1e12, 3), "unit": "TFLOP/s",
                            "ms_per_step": round(em, 4), "head_groups": [heads for _, _, _, heads in layer._groups],
                            "h2d_bytes_per_step": 3 * q.numel() * q.element_size(),
                            "d2h_bytes_per_step": layer.out.numel() * layer.out.element_size()}
    bf16_peak, hbm_peak, peak_kind = peaks()
    attn_mean = statistics.mean(attn_ms)
    achieved = flops / (attn_mean * 1e-3) / 1e12
    line = {
        "metric": METRIC,
        "value": round(value, 3),
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(total_ms_max / args.steps, 4),
        "higher_is_better": True,
        "scaling": "strong" if world > 1 and args.shard == "heads" else "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic (seeded, VGGT-shaped)",
        "config": {
            "workload": workload_name(wl), "batch": Bsz, "heads": H, "seq_len": N, "head_dim": 64,
            "block": 128, "key_block": wl.key_block, "method": ["mass", "drift", "random", "cdf"][wl.method], "sparsity": wl.sparsity,
            "rounds": wl.rounds, "budgets": sorted(set(wl.budgets)) if len(set(wl.budgets)) < 4 else "dirichlet",
            "drift_objective": args.objective, "realized_drift_J_mean": float(f"{drift_mean:.6g}"),
            **({"top_p": args.top_p} if wl.method == R.SELECT_CDF else {}),
            "kept_tile_fraction": round(kept_frac, 4), "kept_tile_gflop": round(flops / 1e9, 3),
            "selection_dtype": "f32", "l2": flush.describe(),
            "parallelism": ("single GPU" if world == 1 else
                            f"heads of one layer split over {world} GPUs ({H} on this rank)"
                            if args.shard == "heads" else f"{world} independent layers, one per GPU"),
            "launch": launch_mode,
            "selection_kernel": ("separate block map, drift score and selection calls" if unfused else
                                 "fused drift selection (block map, drift score, selection)"
                                 if drift_method else "fused block map + selection"),
        },
        "roofline": {"kernel": "block_sparse_attn", "bound": "tensor", "achieved": round(achieved, 2),
                     "peak": bf16_peak, "unit": "TFLOP/s", "frac": round(achieved / bf16_peak, 4),
                     "peak_source": f"{peak_kind} dense bf16 (burst)",
                     "traffic": measured_traffic(workload_name(wl)), "traffic_unit": "bytes per launch (ncu)",
                     "mean_launch_ms": round(attn_mean, 4)},
        "gpu_launches": args.steps * layer.kernel_launches(wl.method, fused=not unfused),
    }
    if clk:
        line["clocks"] = clk
    line.update({k_: v_ for k_, v_ in extra.items() if k_ != "e2e"})
    if not args.quick:
        # the exact inputs of this run (seeded generator on the device), for reproducibility
        import hashlib
        line["inputs_sha256"] = {n: hashlib.sha256(t.contiguous().view(torch.uint8).cpu().numpy().tobytes()).hexdigest()[:16]
                                 for n, t in (("q", q), ("k", k), ("v", v))}
    if "e2e" in extra:
        line["e2e"] = extra["e2e"]
    if rank == 0 and not args.no_cpu_baseline and world == 1 and not args.quick:
        line["cpu_baseline"] = cpu_baseline(wl, top_p=args.top_p)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


# ------------------------------------------------------------- CPU oracle timing
def _oracle_sample(wl, heads, rows_per_head: int, seed: int, top_p: float = 1.0):
    """Runs the oracle's whole path on a seeded sample of the layer: for each listed head,
    the per-head steps in full (pooling of that head's Q, K, V, its block map and Gram
    matrix), then the per-row steps (drift, selection with its restoration rounds,
    attention) for `rows_per_head` query blocks of that head, drawn uniformly without
    replacement by a generator seeded with `seed`.  Returns (seconds of per-head steps,
    seconds of per-row steps, rows in the sample, kept-tile FLOPs of the sampled rows)."""
    import numpy as np

    from oracle import ress_oracle as O
    N, kb = wl.q.shape[2], wl.key_block
    nq = (N + 127) // 128
    scale = 1.0 / math.sqrt(64)
    keep_k = wl.keep_k.cpu().numpy()
    dense_q = wl.dense_q.cpu().numpy()
    rng = np.random.default_rng(seed)
    t_head = t_rows = 0.0
    n_rows, flops = 0, 0.0
    rows_tok = [min(128, N - 128 * i) for i in range(nq)]
    valid = [min(kb, N - kb * j) for j in range((N + kb - 1) // kb)]
    for h in heads:
        q = O.to_numpy_f32(wl.q[:, h:h + 1])
        k = O.to_numpy_f32(wl.k[:, h:h + 1])
        v = O.to_numpy_f32(wl.v[:, h:h + 1])
        w_o = O.to_numpy_f32(wl.w_o)[:, 64 * h:64 * h + 64]
        t0 = time.perf_counter()
        qp, kp, vp = O.pool_blocks(q, 128), O.pool_blocks(k, kb), O.pool_blocks(v, kb)
        P, vbar = O.block_scores(qp, kp, vp, scale)
        gram = O.head_gram(w_o, 1)
        t1 = time.perf_counter()
        pick = rng.choice(nq, size=min(rows_per_head, nq), replace=False)
        rows = [(0, 0, int(i)) for i in sorted(pick)]
        s = np.zeros_like(P) if wl.method == 1 else None
        if s is not None:
            for (_, _, i) in rows:
                s[0, 0, i] = O.drift_row(P[0, 0, i], vbar[0, 0, i], vp[0, 0], gram[0])
        sel = O.select_blocks(wl.method, P, [wl.budgets[h]], keep_k, dense_q, s=s, v_pool=vp,
                              vbar=vbar, gram=gram, rounds=wl.rounds, rho=wl.rho, eps=wl.eps,
                              seed=wl.select_seed, rows=rows, top_p=top_p)
        O.block_sparse_attn(q, k, v, sel["kept"], scale, rows=rows, key_block=kb)
        t2 = time.perf_counter()
        t_head += t1 - t0
        t_rows += t2 - t1
        n_rows += len(rows)
        flops += sum(4.0 * 64 * rows_tok[i] * sum(valid[j] for j in kept)
                     for (_, _, i), kept in sel["kept"].items())
    return t_head, t_rows, n_rows, flops


def _extrapolated(t_head: float, t_rows: float, n_rows: int, flops: float, n_heads_sampled: int,
                  nq: int) -> float:
    """Oracle throughput on the whole layer, extrapolated from a sample: the per-row time
    is charged as measured on the sampled rows, the per-head time pro rata over the
    head's nq rows (a full layer pays it once per head).  Returns FLOP/s."""
    per_row_head = t_head / (n_heads_sampled * nq)
    return flops / (t_rows + per_row_head * n_rows)


def _cores():
    try:
        from threadpoolctl import threadpool_info
        n = max((int(x.get("num_threads", 1)) for x in threadpool_info()), default=1)
        return max(1, n)
    except Exception:
        return os.cpu_count() or 1


def cpu_baseline(wl, seconds: float = 45.0, top_p: float = 1.0):
    """The oracle as it stands on the host cores, on a bounded seeded sample of the same
    layer: every head, 2 query blocks per head at a time (rounds continue until about
    `seconds` of host time), the per-head steps charged pro rata (see _extrapolated)."""
    H = wl.q.shape[1]
    nq = (wl.q.shape[2] + 127) // 128
    th = tr = fl = 0.0
    nr = rounds = 0
    while th + tr < seconds and rounds * 2 < nq:
        a, b, c, d = _oracle_sample(wl, list(range(H)), 2, seed=7000 + rounds, top_p=top_p)
        th, tr, nr, fl = th + a, tr + b, nr + c, fl + d
        rounds += 1
    value = _extrapolated(th, tr, nr, fl, rounds * H, nq)
    return {"value": round(value / 1e12, 6), "unit": "TFLOP/s", "cores": _cores(),
            "kind": "oracle",
            "sample": f"extrapolated: whole path for {nr} seeded query blocks ({nr // H} per head, "
                      f"all {H} heads, {nr} of {H * nq} rows); per-head steps (pooling, block map, "
                      f"Gram) timed in full and charged pro rata over each head's {nq} rows; "
                      f"{th + tr:.1f} s of host time"}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if rank != 0:
        return
    from block_sparse_global_b200 import workload as W
    wl = W.make_workload(args.case, layer=0, device="cpu", method=args.method, sparsity=args.sparsity,
                         key_block=getattr(args, "key_block", 128))
    H, N = wl.q.shape[1], wl.q.shape[2]
    nq = (N + 127) // 128
    rows = 4 if nq > 8 else nq
    per_step, times = [], []
    for s in range(args.warmup + args.steps):
        t0 = time.perf_counter()
        th, tr, nr, fl = _oracle_sample(wl, [s % H], rows, seed=9000 + s, top_p=args.top_p)
        dt = time.perf_counter() - t0
        if s >= args.warmup:
            per_step.append((th, tr, nr, fl))
            times.append(dt)
    th, tr, nr, fl = (sum(x[i] for x in per_step) for i in range(4))
    value = _extrapolated(th, tr, nr, fl, len(per_step), nq)
    sample = (f"extrapolated: per step, one head (heads rotate) in full for the per-head steps "
              f"(pooling, block map, Gram) and {rows} seeded query blocks of it through drift, "
              f"selection and attention; per-head time charged pro rata over the head's {nq} rows")
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value / 1e12, 6), "unit": "TFLOP/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(1e3 * statistics.mean(times), 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic (seeded, VGGT-shaped)",
        "config": {"workload": workload_name(wl), "batch": 1, "heads": H, "seq_len": N,
                   "head_dim": 64, "block": 128, "key_block": wl.key_block, "method": ["mass", "drift", "random", "cdf"][wl.method],
                   "sparsity": wl.sparsity, "rounds": wl.rounds,
                   "step": f"oracle: one head's per-head steps and {rows} of its query blocks (heads rotate)"},
        "cpu_baseline": {"value": round(value / 1e12, 6), "unit": "TFLOP/s", "cores": _cores(), "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": round(value / 1e12, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def sweep_todo(path, methods, sparsities, key_block: int, layers: int):
    """The (method name, method, sparsity) points of the sweep still to run: every point
    minus those already recorded in the JSONL file `path` (same key block and layer count).
    Lines that do not parse (a run cut off mid-write) are ignored."""
    done = set()
    if path and os.path.exists(path):
        with open(path) as f:
            for line in f:
                try:
                    d = json.loads(line)
                    c = d["config"]
                    done.add((c["method"], float(c["sparsity"]), int(c["key_block"]), int(d["layers"])))
                except (ValueError, KeyError, TypeError):
                    continue
    return [(mn, m, sp) for mn, m in methods for sp in sparsities
            if (mn, float(sp), int(key_block), int(layers)) not in done]


def run_sweep(args):
    """The 64-view sweep: `layers` layers (independent seeded Q, K, V, W_O, all resident in
    HBM, about 0.55 GB each) and, for each (method, sparsity) point in turn, the whole path
    (pool, block map, drift for the drift method, selection, schedule, attention) on every
    layer: one warm-up step, then two timed steps, each after an L2 flush.  One JSON line
    per point, printed as soon as the point is done: mean layer latency over the layers and
    kept-tile TFLOP/s (kept-tile FLOPs of all timed steps / their summed device time).
    Sparsity 0 keeps every key block: the same-shape dense layer through the same kernels.
    With --sweep-out FILE each line is also appended to FILE, and points already in FILE
    are skipped, so an interrupted sweep resumes at the next point.  Single GPU (rank 0)."""
    import torch

    from block_sparse_global_b200 import build as B
    from block_sparse_global_b200 import ress as R
    from block_sparse_global_b200 import workload as W
    from block_sparse_global_b200.pipeline import SparseGlobalAttention

    if int(os.environ.get("RANK", "0")) != 0:
        return
    B.build()
    R.load()
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    flush = L2Flush(dev, args.l2_flush == "write+read")
    methods = [("mass", R.SELECT_MASS), ("drift", R.SELECT_DRIFT), ("random", R.SELECT_RANDOM)]
    todo = sweep_todo(args.sweep_out, methods, W.SWEEP_SPARSITIES, args.key_block, args.layers)
    if not todo:
        return
    wls = [W.make_workload(5, layer=li, device="cuda", key_block=args.key_block)
           for li in range(args.layers)]
    Bsz, H, N, _ = wls[0].q.shape
    layer = SparseGlobalAttention(Bsz, H, N, device=dev, key_block=args.key_block)
    n_cand = layer.nk - int(wls[0].keep_k.sum().item())
    sdpa_ms = None
    try:   # printed context only: torch's own dense attention on layer 0
        import torch.nn.functional as F
        for _ in range(2):
            F.scaled_dot_product_attention(wls[0].q, wls[0].k, wls[0].v)
        flush()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        F.scaled_dot_product_attention(wls[0].q, wls[0].k, wls[0].v)
        b.record()
        torch.cuda.synchronize()
        sdpa_ms = a.elapsed_time(b)
    except Exception:
        sdpa_ms = None
    bf16_peak, _, peak_kind = peaks()
    for mname, m, sp in todo:
        c = W.uniform_budget(sp, n_cand)
        budgets = [c] * H
        tot_ms = tot_fl = kept = 0.0
        n = 0
        clocks = ClockSampler(0)
        clocks.start()
        for wl in wls:
            layer.load_output_projection(wl.w_o)
            rounds = wl.rounds if m == R.SELECT_DRIFT else 0

            def step():
                layer.forward(wl.q, wl.k, wl.v, m, budgets, wl.keep_k, wl.dense_q, rounds,
                              wl.rho, wl.eps, wl.select_seed)
            flush()
            step()
            for _ in range(2):
                flush()
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record()
                step()
                b.record()
                torch.cuda.synchronize()
                tot_ms += a.elapsed_time(b)
                n += 1
            if layer.device_error():
                raise SystemExit(f"device error {layer.device_error()} in the sweep")
            fl = kept_tile_flops(layer.kv_idx, layer.kv_cnt, N, args.key_block)
            tot_fl += 2 * fl
            kept += float(layer.kv_cnt.sum().item()) / (Bsz * H * layer.nq * layer.nk)
        clk = clocks.stop()
        tf = tot_fl / (tot_ms * 1e-3) / 1e12
        line = {"metric": METRIC, "sweep": True, "value": round(tf, 3), "unit": "TFLOP/s",
                "ms_per_layer": round(tot_ms / n, 4), "layers": args.layers, "steps_per_layer": 2,
                "dtype": "bf16", "data": "synthetic (seeded, VGGT-shaped)",
                "config": {"workload": W.CASES[5].name, "method": mname, "sparsity": sp,
                           "budget": c, "key_block": args.key_block,
                           "rounds": W.CASES[5].rounds if mname == "drift" else 0,
                           "kept_tile_fraction": round(kept / args.layers, 4),
                           "l2": flush.describe()},
                "frac_of_bf16_peak": round(tf / bf16_peak, 4), "peak_source": f"{peak_kind} dense bf16 (burst)"}
        if sp == 0.0 and sdpa_ms is not None:
            line["torch_sdpa_dense_ms_layer0"] = round(sdpa_ms, 4)
        if clk:
            line["clocks"] = clk
        text = json.dumps(line)
        print(text, flush=True)
        if args.sweep_out:
            with open(args.sweep_out, "a") as f:
                f.write(text + "\n")


def main():
    args = parse()
    if args.sweep:
        run_sweep(args)
    elif args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
