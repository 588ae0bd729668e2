"""The N>1 host logic of bench.py on CPU: two gloo ranks (127.0.0.1).

Checks the max-over-ranks timing reduction, the per-rank workload seeds
(same shapes, different data: weak scaling with no data-path exchange),
the whole-job throughput arithmetic, and that the reference arm prints only
on rank 0.
"""

import io
import os
import socket
import sys
import types
from contextlib import redirect_stdout

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
import synth  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    import torch.distributed as dist
    os.environ["RANK"] = str(rank)
    os.environ["WORLD_SIZE"] = str(world)
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world)
    try:
        mine = [10.0 + rank, 5.0 - rank, 0.5 * (rank + 1)]
        got = bench.max_over_ranks(mine, "cpu")
        # the reference arm: only rank 0 prints its line
        args = types.SimpleNamespace(config="c0", steps=1, warmup=0, gpus=world)
        buf = io.StringIO()
        if rank != 0:
            with redirect_stdout(buf):
                bench.run_reference(args)
        dist.barrier()
        q.put((rank, got, buf.getvalue()))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_max_and_only_rank0_reports():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    expect = [11.0, 5.0, 1.0]
    for rank, got, out in res:
        assert got == pytest.approx(expect)
        if rank != 0:
            assert out == ""


def test_rank_workloads_share_shapes_not_data():
    a = synth.config("c0", seed=bench.rank_seed("c0", 0))
    b = synth.config("c0", seed=bench.rank_seed("c0", 1))
    assert bench.rank_seed("c0", 0) != bench.rank_seed("c0", 1)
    for k in ("q", "a", "k_idx", "q_idx"):  # (c0 compresses every entry in the step: kv starts empty)
        assert np.asarray(a[k]).shape == np.asarray(b[k]).shape
        assert not np.array_equal(np.asarray(a[k]), np.asarray(b[k]))


def test_job_value_is_all_ranks_over_the_slowest_step():
    # 2 ranks x 32 queries in 0.1 ms (the max over ranks) -> 640k queries/s
    assert bench.job_value(2, 32, 0.1) == pytest.approx(640000.0)
    assert bench.job_value(1, 32, 0.1) == pytest.approx(320000.0)


def test_attention_flops_closed_form():
    # HCA: every visible entry plus the window, 4d flops per (head, row)
    w = synth.config("c3", B=2, L=4096)
    p = w["params"]
    n_t = 4096 // p.m
    assert bench.algorithmic_flops(w) == 2 * p.n_h * (n_t + p.W) * 4 * p.d
    # CSA: min(k, n_t) selected entries plus the window
    w = synth.config("c1", B=1, L=8192)
    p = w["params"]
    assert bench.algorithmic_flops(w) == p.n_h * (min(p.k, 8192 // p.m) + p.W) * 4 * p.d
