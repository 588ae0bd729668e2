"""The tensor-core (tcgen05 kind::mxf4) Lightning Indexer against the oracle.

On MXFP4 workloads whose scores are exactly representable in fp32 (the
workload generator checks the bound), the fp32 scores the indexer writes to
its workspace must equal the oracle's exact fp64 scores bit for bit, and the
CUDA-core indexer (CSA_INDEXER=simt) must produce the same bits.
"""

import os

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


def _run_index(w, simt=False):
    from long_context_sparse_gated_b200.runner import DeviceWorkload
    dw = DeviceWorkload(w)
    old = os.environ.get("CSA_INDEXER")
    try:
        if simt:
            os.environ["CSA_INDEXER"] = "simt"
        else:
            os.environ.pop("CSA_INDEXER", None)
        dw.index_topk()
        torch.cuda.synchronize()
    finally:
        if old is None:
            os.environ.pop("CSA_INDEXER", None)
        else:
            os.environ["CSA_INDEXER"] = old
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


def test_tc_matches_simt_bits():
    w = synth.config("c1", B=2, L=8192)
    a = _scores(_run_index(w))
    b = _scores(_run_index(w, simt=True))
    np.testing.assert_array_equal(a.view(np.uint32), b.view(np.uint32))


def test_tc_prefill_many_queries():
    """Many queries per sequence (each its own tile row of queries)."""
    w = synth.config("c4", B=1, L=2048, T=300, q_pos0=1500)
    dw = _run_index(w)
    g = _scores(dw)
    _, scores = pipeline.index_topk(w, return_scores=True)
    for (b, tq), sc in scores.items():
        n_t = len(sc)
        np.testing.assert_array_equal(g[tq, :n_t].astype(np.float64), sc)
