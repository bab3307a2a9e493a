"""The multi-rank plumbing of bench.py, run as two gloo ranks on the CPU.

`bench.py --gpus N` under torchrun gives every rank one full workload (weak scaling: every
(batch, kv head) group is independent, so the path needs no data-path collective), times it on
the device, takes the slowest rank's time with one all-reduce of a scalar, and rank 0 alone
prints.  These tests run that host logic with world size 2 on the gloo backend:
 * max_over_ranks returns the same maximum on every rank, and weak_scaling_tops turns it into
   the whole-job rate;
 * the reference arm under two ranks: rank 1 exits without work, rank 0 prints one JSON line.
"""
import json
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _init(rank, world, port):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import datetime
    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    return dist


def _reduce_worker(rank, world, port, out):
    sys.path.insert(0, ROOT)
    dist = _init(rank, world, port)
    import bench
    local_ms = [12.5, 20.0][rank]
    m = bench.max_over_ranks(local_ms, world)
    value = bench.weak_scaling_tops(8.8e12, 10, world, m)
    out.put((rank, m, value))
    dist.barrier()
    dist.destroy_process_group()


def _reference_worker(rank, world, port, out):
    sys.path.insert(0, ROOT)
    dist = _init(rank, world, port)
    import contextlib
    import io
    import bench
    buf = io.StringIO()
    with contextlib.redirect_stdout(buf):
        bench.main(["--impl", "reference", "--gpus", str(world), "--workload", "tiny",
                    "--steps", "1", "--warmup", "1", "--cpu-seconds", "1"])
    out.put((rank, buf.getvalue()))
    dist.barrier()
    dist.destroy_process_group()


def _run(fn, world=2):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=fn, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=240) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    return sorted(res)


def test_max_over_ranks_and_weak_scaling_value():
    res = _run(_reduce_worker)
    assert [r[1] for r in res] == [20.0, 20.0]          # the slowest rank's time, on every rank
    expected = 2 * 8.8e12 * 10 / (20.0 / 1e3) / 1e12      # both ranks' work in that time
    assert all(abs(r[2] - expected) < 1e-9 * expected for r in res)


def test_reference_arm_prints_on_rank_zero_only():
    res = _run(_reference_worker)
    assert res[1][1] == ""                               # rank 1: no line, no work
    line = json.loads(res[0][1].strip())
    assert line["impl"] == "reference" and line["n_gpus"] == 2
    assert line["config"]["workload"] == "tiny" and line["value"] > 0
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["cpu_baseline"]["kind"] == "oracle"


def test_bench_modes_parse():
    """The FP4-path mode is selected by --fp4-topk (-1: all FP4); omitted, the INT8 path."""
    import bench
    assert bench.parse_args([]).fp4_topk is None
    assert bench.parse_args(["--fp4-topk", "16"]).fp4_topk == 16
    assert bench.parse_args(["--fp4-topk", "-1"]).fp4_topk == -1
    assert bench.parse_args(["--sparse-topk", "8"]).sparse_topk == 8
