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


def test_index_flops_closed_form():
    w = synth.config("c1", B=2, L=8192)
    p = w["params"]
    n_t = 8192 // p.m
    assert bench.index_flops(w) == 2 * 2 * p.H_I * p.c_I * n_t
    assert bench.index_flops(synth.config("c3", B=1, L=4096)) == 0


def test_dominant_roofline_binds_the_right_roof():
    hbm, bf16 = (6451.8, "measured"), (1655.5, "measured")
    # CSA decode: the index call against HBM
    w = synth.config("c1", B=2, L=8192)
    _, idx_bytes = bench.algorithmic_bytes(w)
    r = bench.dominant_roofline(w, 0.01, 0.005, idx_bytes, 2 * idx_bytes, hbm, bf16, 123)
    assert r["bound"] == "hbm" and r["unit"] == "GB/s" and r["traffic"] == 123
    assert r["achieved"] == pytest.approx(idx_bytes / 1e-5 / 1e9)
    assert r["frac"] == pytest.approx(r["achieved"] / 6451.8)
    assert r["frac_vs_8tbs_datasheet"] == pytest.approx(r["achieved"] / 8000.0)
    # CSA prefill, index call longer: the indexer's MXFP4 contraction
    # against the FP4 peak (here, without a GPU to probe: 4x the BF16 peak)
    w = synth.config("c4", B=1, L=1024)
    r = bench.dominant_roofline(w, 2.0, 1.0, 1e6, 2e6, hbm, bf16, None)
    assert r["bound"] == "tensor" and r["peak"] == pytest.approx(4 * 1655.5) and r["kernel"] == "csa_index_topk"
    assert r["achieved"] == pytest.approx(bench.index_flops(w) / 2e-3 / 1e12)
    # CSA prefill, attention longer: the sparse attention against the BF16
    # peak, the index call's entry beside it
    r = bench.dominant_roofline(w, 1.0, 3.0, 1e6, 2e6, hbm, bf16, None)
    assert r["bound"] == "tensor" and r["kernel"] == "csa_sparse_attn" and r["peak"] == 1655.5
    assert r["achieved"] == pytest.approx(bench.algorithmic_flops(w) / 3e-3 / 1e12)
    assert r["index_call"]["kernel"] == "csa_index_topk"
    # HCA: the dense attention against the BF16 peak
    w = synth.config("c3", B=1, L=4096)
    r = bench.dominant_roofline(w, 0.1, 0.1, 0, 1e6, hbm, bf16, None)
    assert r["bound"] == "tensor" and r["peak"] == 1655.5 and r["kernel"] == "hca_dense_attn"
    assert r["achieved"] == pytest.approx(bench.algorithmic_flops(w) / 1e-4 / 1e12)
    s = bench.step_roofline_entry(w, 0.2, 1e6, 6451.8, 1655.5)
    assert s["frac"] == pytest.approx(1e6 / 2e-4 / 1e9 / 6451.8) and s["index_fp4_tflops"] == 0


def test_cpu_baseline_entry_reports_threads_and_model():
    e = bench.cpu_baseline_entry(synth.config("c0"), "c0")
    assert e["kind"] == "oracle" and e["value"] > 0 and e["cores"] >= 1
    assert e["nproc"] >= 1 and isinstance(e["cpu_model"], str)
    assert e.get("value_1_thread", 1.0) > 0
