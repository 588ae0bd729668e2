"""CUDA path vs the fp64 oracle, element by element, on seeded workloads.

Sizes the oracle finishes in seconds that still span several tiles and a
ragged tail, the five configurations' shapes (reduced B/L), and the edge
cases: ragged batches, queries before the window fills, fewer visible
entries than k, zero visible entries, heavy ties.  Full-size workloads, in
the launch configuration the benchmark times, live in test_gpu_fullsize.py.
"""

import numpy as np
import pytest
import torch

import synth
from oracle import csa, pipeline
from parity_util import (bf16_to_f64, check_attn, check_fp8_rows, check_topk,
                         valid_topk_layout)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from long_context_sparse_gated_b200 import build
    build.build()


def _run(w, which="csa"):
    from long_context_sparse_gated_b200.runner import DeviceWorkload
    dw = DeviceWorkload(w)
    if which == "csa":
        dw.csa_step()
    else:
        dw.hca_step()
    torch.cuda.synchronize()
    assert dw.err_bits() == 0, f"device error bits {dw.err_bits()}"
    return dw


def _check_compress(w, dw, comp):
    p = w["params"]
    for b, (ent, pos, packed) in comp.items():
        if not len(pos):
            continue
        e = pos // p.m
        np.testing.assert_array_equal(dw.kv_pos[b].cpu().numpy()[e], pos)
        if p.kv_fmt == "f32":
            g = dw.kv[b].cpu().numpy()[e].astype(np.float64)
            rel = np.abs(g - ent).max() / np.abs(ent).max()
            assert rel <= 1e-5, f"compress rel {rel}"
        else:
            check_fp8_rows(dw.kv[b].cpu().numpy()[e], dw.kv_scale[b].cpu().numpy()[e],
                           packed[0], packed[1], packed[2], p.d, p.r, what=f"compress b={b}")


def _check_csa(w, dw, exact_topk=True):
    p = w["params"]
    comp = pipeline.compress(w) if w["S"] else None
    if comp:
        _check_compress(w, dw, comp)
    idx_o, scores = pipeline.index_topk(w, return_scores=True)
    g_idx = dw.idx.cpu().numpy()
    use = {}
    for (b, tq), oi in idx_o.items():
        t = int(w["q_pos0"][b]) + tq
        n_t = csa.n_visible(t, p.m)
        valid_topk_layout(g_idx[b, tq], n_t, p.k)
        check_topk(g_idx[b, tq], oi, scores[(b, tq)], n_t, exact=exact_topk, what=f"b={b} t={t}")
        use[(b, tq)] = g_idx[b, tq]  # equal to oi, or a legitimate near-tie
    out_o = pipeline.sparse_attn(w, use, comp)
    g_out = dw.out_f64()
    ref = np.stack([[out_o[(b, tq)] for tq in range(w["T"])] for b in range(p.B)])
    return check_attn(g_out, ref, f32=p.act_fmt == "f32", what="csa attention")


def _check_hca(w, dw):
    p = w["params"]
    comp = pipeline.compress(w) if w["S"] else None
    if comp:
        _check_compress(w, dw, comp)
    out_o = pipeline.dense_attn(w, comp)
    ref = np.stack([[out_o[(b, tq)] for tq in range(w["T"])] for b in range(p.B)])
    return check_attn(dw.out_f64(), ref, f32=p.act_fmt == "f32", what="hca attention")


# ----------------------------------------------------------------------------
# config 0: tiny fp32 CSA decode
# ----------------------------------------------------------------------------


def test_c0_decode_fp32():
    w = synth.config("c0")
    _check_csa(w, _run(w), exact_topk=False)


def test_c0_decode_mxfp4_indexer_exact():
    w = synth.config("c0", idx_fmt="mxfp4")
    _check_csa(w, _run(w), exact_topk=True)


def test_c0_multi_query_ragged_batch():
    """Three sequences of different lengths, 6 queries each: early queries
    see fewer than k entries and a partial window."""
    w = synth.config("c0", B=3, L=[2048, 333, 130], T=6, q_pos0=[0, 200, 124], idx_fmt="mxfp4")
    _check_csa(w, _run(w), exact_topk=True)


def test_c0_hca_shape_fp32():
    p = synth.Params(B=2, d=128, r=32, m=128, H_I=4, c_I=64, k=0, n_h=8, W=128, tau=1.0,
                     kv_fmt="f32", idx_fmt="f32", act_fmt="f32")
    w = synth.make_workload(7, p, L=[1200, 700], T=3, compress="all", sink="normal")
    _check_hca(w, _run(w, "hca"))


# ----------------------------------------------------------------------------
# reduced shapes of configs 1-4 (FP8/BF16 storage, MXFP4 indexer)
# ----------------------------------------------------------------------------


def test_c1_shape_reduced():
    w = synth.config("c1", B=3, L=[16384, 9001, 4099])
    _check_csa(w, _run(w))


def test_c2_shape_reduced_with_cluster():
    w = synth.config("c2", B=2, L=65536, cluster=(1, 1024, 3.0))
    dw = _run(w)
    _check_csa(w, dw)
    # the planted cluster dominates sequence 0's selection
    b, off, ln = w["cluster"][0]
    sel = dw.idx[0, 0].cpu().numpy()
    assert np.sum((sel >= off) & (sel < off + ln)) >= 0.9 * min(ln, w["params"].k)


def test_c3_shape_reduced_hca():
    w = synth.config("c3", B=2, L=[131072, 65536 + 128 * 3 + 5])
    _check_hca(w, _run(w, "hca"))


def test_c4_shape_reduced_prefill():
    w = synth.config("c4", B=1, L=3000)
    _check_csa(w, _run(w))


def test_prefill_two_sequences_ragged():
    w = synth.config("c4", B=2, L=[1500, 1500], T=700, q_pos0=[800, 0])
    _check_csa(w, _run(w))


# ----------------------------------------------------------------------------
# edge cases
# ----------------------------------------------------------------------------


def test_no_visible_entries_window_only():
    """Queries before the first block completes: no entries, top-k all -1,
    attention over the window tokens and the sink only."""
    w = synth.config("c4", B=1, L=64, T=3, q_pos0=0)
    dw = _run(w)
    assert np.all(dw.idx[0, :3].cpu().numpy() == -1)
    _check_csa(w, dw)


def test_topk_heavy_ties_exact():
    """All index keys equal within a sequence: every score ties and the
    lowest indices must win."""
    w = synth.config("c1", B=2, L=8192)
    w["k_idx"][...] = w["k_idx"][:, :1]
    w["k_idx_sf"][...] = w["k_idx_sf"][:, :1]
    dw = _run(w)
    for b in range(2):
        np.testing.assert_array_equal(dw.idx[b, 0].cpu().numpy(), np.arange(512))
    _check_csa(w, dw)


def test_topk_many_zero_scores():
    """Negative-only head weights are not allowed to break ReLU: queries whose
    dot products are all negative give all-zero scores -> lowest indices."""
    w = synth.config("c1", B=1, L=8192)
    # flip the sign bit of every query element: every q.k of the original
    # positive-only keys becomes <= 0
    w["k_idx"][...] = w["k_idx"] & 0x77  # clear sign bits: keys >= 0
    w["q_idx"][...] = w["q_idx"] | 0x88  # set sign bits: queries <= 0
    dw = _run(w)
    np.testing.assert_array_equal(dw.idx[0, 0].cpu().numpy(), np.arange(512))
    _check_csa(w, dw)


def test_device_error_on_bad_index():
    """An out-of-range top-k index is skipped and reported in *err."""
    from long_context_sparse_gated_b200.runner import DeviceWorkload
    w = synth.config("c1", B=1, L=4096)
    dw = DeviceWorkload(w)
    dw.compress()
    dw.index_topk()
    dw.idx[0, 0, 3] = 10 ** 6
    dw.sparse_attn()
    torch.cuda.synchronize()
    assert dw.err_bits() & 1
