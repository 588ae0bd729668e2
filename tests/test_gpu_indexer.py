"""The tensor-core (tcgen05 kind::mxf4) Lightning Indexer against the oracle.

On MXFP4 workloads whose scores are exactly representable in fp32 (the
workload generator checks the bound), the fp32 scores the indexer writes to
its workspace must equal the oracle's exact fp64 scores bit for bit; so must
the CUDA-core indexer, which serves the shapes the tensor-core one does not
(here: 32 index heads).
"""

import numpy as np
import pytest
import torch

import synth
from oracle import csa, pipeline

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from long_context_sparse_gated_b200 import build
    build.build()


def _scores(dw):
    """The fp32 scores the indexer leaves at the start of its workspace
    (rows padded to a multiple of 32 entries)."""
    ld = (dw.n_max + 31) // 32 * 32
    n = dw.p.B * dw.T * ld
    return dw.ws_idx.view(torch.float32)[:n].view(dw.p.B * dw.T, ld)[:, :dw.n_max].cpu().numpy()


def _run_index(w):
    from long_context_sparse_gated_b200.runner import DeviceWorkload
    dw = DeviceWorkload(w)
    dw.index_topk()
    torch.cuda.synchronize()
    assert dw.err_bits() == 0
    return dw


@pytest.mark.parametrize("name,kw", [
    ("c1", dict(B=2, L=4096)),                        # 1024 entries: 8 tiles per query
    ("c1", dict(B=3, L=[16384, 9001, 4099])),          # ragged tails inside tiles
    ("c2", dict(B=1, L=131072, cluster=(1, 1024, 3.0))),
])
def test_tc_scores_exact(name, kw):
    w = synth.config(name, **kw)
    dw = _run_index(w)
    g = _scores(dw)
    _, scores = pipeline.index_topk(w, return_scores=True)
    p = w["params"]
    for (b, tq), sc in scores.items():
        t = int(w["q_pos0"][b]) + tq
        n_t = csa.n_visible(t, p.m)
        row = g[b * w["T"] + tq, :n_t].astype(np.float64)
        bad = np.flatnonzero(row != sc)
        assert bad.size == 0, f"b={b}: {bad.size} inexact scores, first {bad[:5]} gpu {row[bad[:5]]} ref {sc[bad[:5]]}"


def test_cuda_core_indexer_scores_and_topk_exact():
    """32 index heads run on the CUDA-core scorer (no histogram: the staged
    selector); scores and top-k sets equal the oracle's exactly."""
    w = synth.with_index_heads(synth.config("c1", B=2, L=8192), 32)
    dw = _run_index(w)
    g = _scores(dw)
    idx, scores = pipeline.index_topk(w, return_scores=True)
    for (b, tq), sc in scores.items():
        np.testing.assert_array_equal(g[b, :len(sc)].astype(np.float64), sc)
        np.testing.assert_array_equal(dw.idx[b, tq].cpu().numpy(), idx[(b, tq)])


def test_tc_prefill_many_queries():
    """Many queries per sequence (each its own tile row of queries)."""
    w = synth.config("c4", B=1, L=2048, T=300, q_pos0=1500)
    dw = _run_index(w)
    g = _scores(dw)
    _, scores = pipeline.index_topk(w, return_scores=True)
    for (b, tq), sc in scores.items():
        n_t = len(sc)
        np.testing.assert_array_equal(g[tq, :n_t].astype(np.float64), sc)


@pytest.mark.parametrize("score_fmt", ["f32", "bf16"])
def test_tc_prefill_query_pairs(score_fmt):
    """Prefill shape (T > 4): the scorer pairs consecutive queries of one
    sequence into one N=128 MMA.  Two sequences (pairs never cross them),
    an odd T (the last pair has one query), queries at the start of a
    sequence that see no entry yet, ragged rows; scores and top-k sets
    equal the oracle's exactly."""
    w = synth.with_score_fmt(synth.config("c4", B=2, L=[6000, 4100], T=301, q_pos0=[0, 3700]), score_fmt)
    dw = _run_index(w)
    idx, scores = pipeline.index_topk(w, return_scores=True, score_fmt=score_fmt)
    if score_fmt == "f32":
        g = _scores(dw)
        for (b, tq), sc in scores.items():
            np.testing.assert_array_equal(g[b * w["T"] + tq, :len(sc)].astype(np.float64), sc)
    got = dw.idx.cpu().numpy()
    for (b, tq), ref in idx.items():
        np.testing.assert_array_equal(got[b, tq], ref, err_msg=f"b={b} tq={tq}")


@pytest.mark.parametrize("T,B", [(5, 3), (6, 1), (2, 4)])
def test_tc_short_query_runs(T, B):
    """The smallest prefill shapes (T = 5: two pairs and a single query per
    sequence; T = 6: three pairs) and a multi-query decode (T = 2, one query
    per stage): scores bit for bit and top-k sets equal the oracle's."""
    w = synth.config("c1", B=B, L=[20000 + 97 * b for b in range(B)], T=T)
    dw = _run_index(w)
    g = _scores(dw)
    idx, scores = pipeline.index_topk(w, return_scores=True)
    got = dw.idx.cpu().numpy()
    for (b, tq), sc in scores.items():
        np.testing.assert_array_equal(g[b * T + tq, :len(sc)].astype(np.float64), sc, err_msg=f"b={b} tq={tq}")
        np.testing.assert_array_equal(got[b, tq], idx[(b, tq)], err_msg=f"b={b} tq={tq}")
