"""Host logic of the multi-GPU (weak-scaling) bench path, run as two gloo ranks on CPU.

With N GPUs every rank processes its own layer (independent seeds) and nothing crosses
ranks on the data path; the only collectives are the barriers and the final reduction
(max over ranks of the device time, sum of the work).  These tests run that reduction,
the per-rank workload assignment and the reference arm's rank gating in world-size-2
process groups on the gloo backend.
"""
from __future__ import annotations

import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _init(rank: int, world: int, port: int) -> None:
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))


def _reduce_worker(rank: int, world: int, port: int, out) -> None:
    _init(rank, world, port)
    try:
        import bench
        ms, work = bench.reduce_over_ranks(10.0 + 5.0 * rank, 100.0 * (rank + 1))
        out.put((rank, ms, work))
    finally:
        dist.destroy_process_group()


def _shard_worker(rank: int, world: int, port: int, out) -> None:
    _init(rank, world, port)
    try:
        from block_sparse_global_b200 import workload as W
        wl = W.make_workload(1, layer=rank, device="cpu")
        digest = torch.tensor([float(wl.q.float().sum()), float(wl.k.float().sum())],
                              dtype=torch.float64)
        gathered = [torch.zeros(2, dtype=torch.float64) for _ in range(world)]
        dist.all_gather(gathered, digest)
        out.put((rank, [g.tolist() for g in gathered]))
    finally:
        dist.destroy_process_group()


def _reference_worker(rank: int, world: int, port: int, out) -> None:
    import contextlib
    import io
    _init(rank, world, port)
    try:
        import bench

        class A:
            case, method, sparsity, steps, warmup, top_p = 1, None, None, 1, 0, 1.0
        buf = io.StringIO()
        with contextlib.redirect_stdout(buf):
            bench.run_reference(A)
        out.put((rank, buf.getvalue()))
    finally:
        dist.destroy_process_group()


def _guarded(worker, rank, world, port, out):
    """Runs a worker; an exception is sent to the parent instead of leaving it waiting."""
    try:
        worker(rank, world, port, out)
    except BaseException as e:  # noqa: BLE001 - reported to the parent, then re-raised
        out.put((rank, "error", repr(e)))
        raise


def _run(worker, world: int = 2, timeout: float = 240.0):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_guarded, args=(worker, r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = {}
    try:
        for _ in range(world):
            item = q.get(timeout=timeout)
            assert not (len(item) == 3 and item[1] == "error"), f"rank {item[0]} failed: {item[2]}"
            res[item[0]] = item[1:]
    finally:
        for p in procs:
            p.join(timeout=30)
            if p.is_alive():
                p.kill()
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    return res


def test_reduce_over_ranks_max_time_sum_work():
    res = _run(_reduce_worker)
    for r in range(2):
        ms, work = res[r]
        assert ms == 15.0          # max of 10 and 15
        assert work == 300.0       # 100 + 200


def test_reduce_over_ranks_single_process_identity():
    import bench
    assert not dist.is_initialized()
    assert bench.reduce_over_ranks(3.5, 7.0) == (3.5, 7.0)


def test_each_rank_gets_its_own_layer():
    res = _run(_shard_worker)
    g0, g1 = res[0][0], res[1][0]
    assert g0 == g1                # every rank saw the same gathered digests
    assert g0[0] != g0[1]          # rank 0 and rank 1 hold different inputs
    # rank r's layer is the same as a fresh single-process build of layer r
    from block_sparse_global_b200 import workload as W
    for r in range(2):
        wl = W.make_workload(1, layer=r, device="cpu")
        assert float(wl.q.float().sum()) == g0[r][0]


@pytest.mark.timeout(600)
def test_reference_arm_runs_on_rank0_only():
    import json
    res = _run(_reference_worker, timeout=500.0)
    assert res[1][0] == ""
    line = json.loads(res[0][0].strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["n_gpus"] == 2
    assert line["value"] > 0 and line["e2e"]["h2d_bytes_per_step"] == 0


def test_sweep_resume_skips_recorded_points(tmp_path):
    """An interrupted sweep resumes at the next point: points already in the JSONL file
    (same key block and layer count) are skipped; a torn last line is ignored."""
    import json

    import bench
    methods = [("mass", 0), ("drift", 1)]
    sp = (0.0, 0.5, 0.9)
    out = tmp_path / "sweep.jsonl"
    assert len(bench.sweep_todo(str(out), methods, sp, 128, 24)) == 6
    rec = lambda m, s, kb=128, layers=24: json.dumps(
        {"layers": layers, "config": {"method": m, "sparsity": s, "key_block": kb}})
    out.write_text("\n".join([rec("mass", 0.0), rec("mass", 0.5), rec("drift", 0.9, kb=64),
                              rec("drift", 0.0, layers=2)]) + "\n" + '{"layers": 24, "conf')
    todo = bench.sweep_todo(str(out), methods, sp, 128, 24)
    assert [(m, s) for m, _, s in todo] == [("mass", 0.9), ("drift", 0.0), ("drift", 0.5),
                                           ("drift", 0.9)]


# ------------------------------------------------ heads of one layer split over the ranks
def test_head_ranges_cover_every_head_once():
    from block_sparse_global_b200 import workload as W
    for heads in (1, 2, 5, 16, 17, 128):
        for world in (1, 2, 3, 4, 8):
            if world > heads:
                continue
            ranges = [W.head_range(heads, world, r) for r in range(world)]
            covered = [h for a, b in ranges for h in range(a, b)]
            assert covered == list(range(heads)), (heads, world)
            sizes = [b - a for a, b in ranges]
            assert max(sizes) - min(sizes) <= 1 and min(sizes) >= 1
    with pytest.raises(ValueError):
        W.head_range(16, 2, 2)


def _head_shard_worker(rank: int, world: int, port: int, out) -> None:
    _init(rank, world, port)
    try:
        import numpy as np

        from block_sparse_global_b200 import workload as W
        from oracle import ress_oracle as O
        full = W.make_workload(2, heads=5, views=3, method="drift", device="cpu")
        h0, h1 = W.head_range(5, world, rank)
        wl = W.shard_heads(full, h0, h1)
        ok = (torch.equal(wl.q, full.q[:, h0:h1]) and torch.equal(wl.v, full.v[:, h0:h1])
              and wl.budgets == full.budgets[h0:h1] and torch.equal(wl.keep_k, full.keep_k))
        # the Gram matrices of the shard's W_O columns are the full layer's, heads h0..h1-1
        g_shard = O.head_gram(wl.w_o.numpy(), h1 - h0)
        g_full = O.head_gram(full.w_o.numpy(), 5)[h0:h1]
        ok = ok and bool(np.array_equal(g_shard, g_full))
        # every head of the layer is processed by exactly one rank
        mine = torch.zeros(5, dtype=torch.int64)
        mine[h0:h1] = 1
        dist.all_reduce(mine)
        out.put((rank, ok, mine.tolist()))
    finally:
        dist.destroy_process_group()


def test_head_sharded_layer_two_ranks():
    port = _free_port()
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    procs = [ctx.Process(target=_head_shard_worker, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    res = [out.get(timeout=120) for _ in range(2)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, ok, count in res:
        assert ok, rank
        assert count == [1, 1, 1, 1, 1]
