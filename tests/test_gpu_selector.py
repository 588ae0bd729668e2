"""The top-k selector, with fp32 index scores and with the BF16 scores of
kwkr.cn notes 4.4 (index scores quantised from FP32 to BF16 before the
selector), against the oracle's selection (oracle.pipeline.index_topk with
score_fmt "f32" / "bf16": exact scores, or the same rounded to BF16 by round
to nearest even, ranked by score then lower index).

The sets are unique, so they must be identical.  Paths: one CTA per query
(rows up to 32768 entries), chunked rows (longer), the heavy-tie fallback,
and the staged selector behind the CUDA-core scorer."""

import numpy as np
import pytest
import torch

import synth
from oracle import csa, pipeline

pytestmark = pytest.mark.gpu

FMTS = ["f32", "bf16"]


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from long_context_sparse_gated_b200 import build
    build.build()


def _run(w):
    from long_context_sparse_gated_b200.runner import DeviceWorkload
    dw = DeviceWorkload(w)
    dw.index_topk()
    torch.cuda.synchronize()
    assert dw.err_bits() == 0
    return dw


def _check(w, dw, queries=None):
    fmt = w["params"].score_fmt
    ref = pipeline.index_topk(w, queries, score_fmt=fmt)
    got = dw.idx.cpu().numpy()
    for (b, tq), r in ref.items():
        np.testing.assert_array_equal(got[b, tq], r, err_msg=f"{fmt} b={b} tq={tq}")


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("name,kw", [
    ("c1", dict(B=3, L=[16384, 9001, 4099])),                   # one CTA per query, ragged rows
    ("c1", dict(B=2, L=[200000, 131072 + 12])),                 # 50000 / 32771 entries: chunked rows
    ("c2", dict(B=2, L=262144, cluster=(1, 1024, 3.0))),        # 65536 entries, planted cluster, k = 1024
    ("c1", dict(B=1, L=1200000)),                               # 300000 entries: bitmap beyond the finish's shared copy
])
def test_topk_exact(fmt, name, kw):
    w = synth.with_score_fmt(synth.config(name, **kw), fmt)
    _check(w, _run(w))


def test_bf16_scores_are_the_rounded_exact_scores():
    w = synth.with_score_fmt(synth.config("c1", B=2, L=16384), "bf16")
    dw = _run(w)
    ld = (dw.n_max + 31) // 32 * 32
    g = dw.ws_idx.view(torch.int16)[:2 * ld].view(2, ld).cpu().numpy().view(np.uint16)
    _, scores = pipeline.index_topk(w, return_scores=True, score_fmt="bf16")
    from oracle import codecs
    for (b, tq), sc in scores.items():
        np.testing.assert_array_equal(g[b, :len(sc)], codecs.bf16_encode(sc))


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("L", [32768, 200000])
def test_topk_duplicate_keys_in_threshold_bin(fmt, L):
    """Every index key repeated 16 times: the threshold bin's ties come in
    groups of equal scores that only the index order separates (one CTA per
    row, and chunked rows)."""
    w = synth.with_score_fmt(synth.config("c1", B=2, L=L), fmt)
    for key in ("k_idx", "k_idx_sf"):
        a = w[key]
        w[key] = np.ascontiguousarray(np.repeat(a[:, ::16], 16, axis=1)[:, :a.shape[1]])
    _check(w, _run(w))


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("L", [8192, 262144])
def test_topk_all_ties_fallback(fmt, L):
    """All keys equal: the threshold bin holds every entry (more than the
    tie list keeps), the global-memory fallback takes the lowest indices."""
    w = synth.with_score_fmt(synth.config("c1", B=1, L=L), fmt)
    w["k_idx"][...] = w["k_idx"][:, :1]
    w["k_idx_sf"][...] = w["k_idx_sf"][:, :1]
    dw = _run(w)
    np.testing.assert_array_equal(dw.idx[0, 0].cpu().numpy(), np.arange(512))


@pytest.mark.parametrize("fmt", FMTS)
def test_topk_staged_selector(fmt):
    """32 index heads: the CUDA-core scorer, no histogram, the staged
    selector (fp32 or BF16 keys)."""
    w = synth.with_score_fmt(synth.with_index_heads(synth.config("c1", B=2, L=8192), 32), fmt)
    _check(w, _run(w))


@pytest.mark.parametrize("fmt", FMTS)
def test_topk_prefill_rows(fmt):
    w = synth.with_score_fmt(synth.config("c4", B=1, L=4096, T=200, q_pos0=3000), fmt)
    _check(w, _run(w))


@pytest.mark.parametrize("fmt", FMTS)
def test_topk_rows_heavy_ties(fmt):
    """No-histogram mode with every score of a row equal (all index keys
    the same): the row selector keeps the k lowest indices."""
    w = synth.with_score_fmt(synth.with_index_heads(synth.config("c1", B=2, L=8192), 32), fmt)
    w["k_idx"][...] = w["k_idx"][:, :1]
    w["k_idx_sf"][...] = w["k_idx_sf"][:, :1]
    dw = _run(w)
    for b in range(2):
        np.testing.assert_array_equal(dw.idx[b, 0].cpu().numpy(), np.arange(512))
