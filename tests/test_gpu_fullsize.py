"""Full-size workloads, in the launch configuration the benchmark times,
checked on sampled queries the oracle computes one by one.

config 1: V4-Flash CSA decode, B=32, L=131072 (8 sampled sequences)
config 2: V4-Pro CSA decode at 1M context with the planted cluster (all 4)
config 3: HCA decode at 1M context, with the incremental compress (all 16)
config 4: CSA chunked prefill, 2 x 32768 tokens (sampled query positions)
Top-k sets must match exactly; attention within the BF16/FP8 tolerances.
"""

import numpy as np
import pytest
import torch

import synth
from oracle import csa, pipeline
from parity_util import check_attn, check_fp8_rows, check_topk, valid_topk_layout

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from long_context_sparse_gated_b200 import build
    build.build()


def _run(w, hca=False):
    from long_context_sparse_gated_b200.runner import DeviceWorkload
    dw = DeviceWorkload(w)
    if hca:
        dw.hca_step()
    else:
        dw.csa_step()
    torch.cuda.synchronize()
    assert dw.err_bits() == 0
    return dw


def _check_sampled_csa(w, dw, queries):
    p = w["params"]
    seqs = sorted(set(b for b, _ in queries))
    comp = pipeline.compress(w, seqs=seqs) if w["S"] else None
    if comp:
        for b in seqs:
            ent, pos, packed = comp[b]
            e = pos // p.m
            np.testing.assert_array_equal(dw.kv_pos[b].cpu().numpy()[e], pos)
            check_fp8_rows(dw.kv[b].cpu().numpy()[e], dw.kv_scale[b].cpu().numpy()[e], *packed, p.d, p.r,
                           what=f"compress b={b}")
    idx_o, scores = pipeline.index_topk(w, queries, return_scores=True)
    g_idx = dw.idx.cpu().numpy()
    for (b, tq), oi in idx_o.items():
        t = int(w["q_pos0"][b]) + tq
        valid_topk_layout(g_idx[b, tq], csa.n_visible(t, p.m), p.k)
        check_topk(g_idx[b, tq], oi, what=f"b={b} t={t}")
    out_o = pipeline.sparse_attn(w, idx_o, comp, queries)
    g = dw.out_f64()
    ref = np.stack([out_o[q] for q in queries])
    got = np.stack([g[b, tq] for b, tq in queries])
    check_attn(got, ref, what="attention")


def test_c1_fullsize_sampled():
    w = synth.config("c1")
    dw = _run(w)
    _check_sampled_csa(w, dw, [(b, 0) for b in (0, 5, 11, 17, 23, 26, 30, 31)])


def test_c2_fullsize_with_cluster():
    w = synth.config("c2")
    dw = _run(w)
    _check_sampled_csa(w, dw, [(b, 0) for b in range(4)])
    b, off, ln = w["cluster"][0]
    sel = dw.idx[b, 0].cpu().numpy()
    assert np.sum((sel >= off) & (sel < off + ln)) == ln  # the cluster fills the top-1024


def test_c3_fullsize_hca():
    w = synth.config("c3")
    dw = _run(w, hca=True)
    p = w["params"]
    comp = pipeline.compress(w)
    for b in range(p.B):
        ent, pos, packed = comp[b]
        e = pos // p.m
        check_fp8_rows(dw.kv[b].cpu().numpy()[e], dw.kv_scale[b].cpu().numpy()[e], *packed, p.d, p.r,
                       what=f"hca compress b={b}")
    out_o = pipeline.dense_attn(w, comp)
    ref = np.stack([[out_o[(b, 0)]] for b in range(p.B)])
    check_attn(dw.out_f64(), ref, what="hca attention")


def test_c4_fullsize_prefill_sampled():
    w = synth.config("c4")
    dw = _run(w)
    qs = [(0, 0), (0, 3), (0, 127), (0, 2047), (0, 2048), (0, 4099), (1, 8191), (1, 16000), (1, 24575),
          (1, 32700), (1, 32766), (1, 32767)]
    _check_sampled_csa(w, dw, qs)
