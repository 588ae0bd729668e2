"""The tensor-core (tcgen05 kind::f16) attention against the oracle.

Covers: sparse and dense, single split (prefill) and split + merge (decode),
multi-tile online softmax, the lazy running-max rescale, 64 and 128 heads,
and the CUDA-core kernel on the same FP8/BF16 layout (a head count that is
not a multiple of 64 runs there).
"""

import numpy as np
import pytest
import torch

import synth
from oracle import pipeline
from parity_util import check_attn, check_attn_scaled

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from long_context_sparse_gated_b200 import build
    build.build()


def _attn(w, dense=False, idx=None, expect_err=0):
    from long_context_sparse_gated_b200.runner import DeviceWorkload
    dw = DeviceWorkload(w)
    if dense:
        dw.dense_attn()
    else:
        if idx is not None:
            dw.idx.copy_(torch.from_numpy(idx))
        else:
            dw.index_topk()
        dw.sparse_attn()
    torch.cuda.synchronize()
    assert dw.err_bits() == expect_err, dw.err_bits()
    return dw


def _ref_sparse(w, dw):
    idx = dw.idx.cpu().numpy()
    o = pipeline.sparse_attn(w, {(b, t): idx[b, t] for b in range(w["params"].B) for t in range(w["T"])})
    return np.stack([[o[(b, t)] for t in range(w["T"])] for b in range(w["params"].B)])


def _ref_dense(w):
    o = pipeline.dense_attn(w)
    return np.stack([[o[(b, t)] for t in range(w["T"])] for b in range(w["params"].B)])


@pytest.mark.parametrize("name,kw", [
    ("c1", dict(B=2, L=8192, compress="none")),
    ("c2", dict(B=1, L=65536, compress="none")),   # 128 heads: two head groups
])
def test_tc_sparse_decode(name, kw):
    w = synth.config(name, **kw)
    dw = _attn(w)
    check_attn(dw.out_f64(), _ref_sparse(w, dw), what=name)


def test_tc_dense_decode_multi_tile_and_merge():
    # 2048 + 128 rows: 17 tiles -> splits of 8 tiles -> 3 splits + merge
    w = synth.config("c3", B=2, L=[262144, 200000], compress="none")
    dw = _attn(w, dense=True)
    check_attn(dw.out_f64(), _ref_dense(w), what="dense")


def test_tc_prefill_single_split_multi_tile():
    w = synth.config("c4", B=1, L=1024, T=40, q_pos0=900, compress="none")
    dw = _attn(w)
    check_attn(dw.out_f64(), _ref_sparse(w, dw), what="prefill")


def test_tc_lazy_rescale_path():
    """The query's own window row is replaced by head 0's query vector, so
    head 0's logit there (~ |q|^2 / sqrt(d) ~ 22) exceeds the running max of
    the earlier tiles (~3) by far more than the lazy threshold, and the
    accumulated O of head 0 must be rescaled in TMEM."""
    import ml_dtypes
    w = synth.config("c3", B=1, L=131072 + 64, compress="none")  # 1024 entries + window
    t = int(w["q_pos0"][0])
    slot = t % w["Wcap"]
    q0 = (w["q"][0, 0, 0].astype(np.uint32) << 16).view(np.float32)
    sc = np.float32(np.abs(q0[:448]).max() / 448.0)
    codes = (q0[:448] / sc).astype(ml_dtypes.float8_e4m3fn).view(np.uint8)
    w["win"][0, slot, :448] = codes
    w["win"][0, slot, 448:] = w["q"][0, 0, 0, 448:].view(np.uint8)
    w["win_scale"][0, slot] = sc
    dw = _attn(w, dense=True)
    ref = _ref_dense(w)
    check_attn(dw.out_f64(), ref, what="rescale")


@pytest.mark.parametrize("dense", [False, True])
def test_cuda_core_path_fp8(dense):
    """96 heads (not a whole number of 64-head groups) run on the CUDA-core
    kernel: same layout, same oracle, same tolerance."""
    w = synth.config("c3" if dense else "c2", B=2, L=65536 if dense else 8192, compress="none")
    w = synth.with_heads(w, 96)
    dw = _attn(w, dense=dense)
    ref = _ref_dense(w) if dense else _ref_sparse(w, dw)
    check_attn(dw.out_f64(), ref, what="cuda-core fp8")


# ---- input range: row scales, RoPE magnitudes and queries over many binades

@pytest.mark.parametrize("q_log2", [None, (-24.0, 20.0)])
def test_tc_wide_range_sparse_decode(q_log2):
    """Per-row FP8 scales 2^-16 .. 2^4 and RoPE/non-RoPE magnitude ratios
    1 .. 10^4 (cache and window rows); optionally queries whose heads span
    2^-24 .. 2^20 (beyond FP16's range).  Outputs must stay finite and match
    the oracle per head."""
    w = synth.config("c1", B=2, L=8192, compress="none")
    w = synth.with_wide_rows(w, 11, q_log2=q_log2)
    dw = _attn(w)
    check_attn_scaled(dw.out_f64(), _ref_sparse(w, dw), what="wide sparse")


def test_tc_wide_range_dense_split_merge():
    """The same ranges through the dense kernel with several splits (fp32
    partials and the merge) and 128 heads."""
    w = synth.config("c3", B=2, L=[262144, 200000], compress="none")
    w = synth.with_wide_rows(w, 12, q_log2=(-8.0, 8.0))
    dw = _attn(w, dense=True)
    check_attn_scaled(dw.out_f64(), _ref_dense(w), what="wide dense")


def test_tc_wide_range_prefill():
    w = synth.config("c4", B=1, L=1024, T=40, q_pos0=900, compress="none")
    w = synth.with_wide_rows(w, 13, scale_log2=(-12.0, 2.0), rope_ratio_log10=(-2.0, 3.0))
    dw = _attn(w)
    check_attn_scaled(dw.out_f64(), _ref_sparse(w, dw), what="wide prefill")


def test_tc_rope_heavy_rows_unit_scale():
    """RoPE dims 10^4 times the non-RoPE amax with scales near the
    workloads' own (the case a single FP16 accumulator of rope/s overflowed),
    queries scaled so the logits stay moderate."""
    w = synth.config("c1", B=2, L=8192, compress="none")
    w = synth.with_wide_rows(w, 14, scale_log2=(-7.0, -6.0), rope_ratio_log10=(3.5, 4.0),
                             q_log2=(-14.0, -12.0))
    dw = _attn(w)
    check_attn_scaled(dw.out_f64(), _ref_sparse(w, dw), what="rope heavy")


def test_tc_out_of_range_scale_rows_are_dropped():
    """A row whose scale is outside [2^-90, 2^90] (or not finite) takes no
    part and raises CSA_DEV_ERR_RANGE; the output stays finite and equals
    the oracle's over the remaining rows."""
    w = synth.config("c1", B=1, L=8192, compress="none")
    t = int(w["q_pos0"][0])
    slot = t % w["Wcap"]
    w["win_scale"][0, slot] = np.float32(2.0 ** -100)
    dw = _attn(w, expect_err=2)
    # the oracle over the same rows without that window row
    from oracle import csa
    p = w["params"]
    idx = dw.idx.cpu().numpy()[0, 0]
    rows = pipeline.cache_rows(w, 0)
    win = pipeline.window_rows(w, 0, t)
    pos = csa.window_positions(t, p.W)
    keep = (pos % w["Wcap"]) != slot
    J = csa.csa_rows(rows, idx, win[keep])
    ref = csa.attend(pipeline._query(w, 0, 0), J, w["sink"], p.tau, t, p.theta, p.r)
    check_attn(dw.out_f64()[0, 0], ref, what="dropped row")
