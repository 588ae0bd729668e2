"""The tensor-core (tcgen05 kind::f16) attention against the oracle and
against the CUDA-core attention (CSA_ATTN=simt).

Covers: sparse and dense, single split (prefill) and split + merge (decode),
multi-tile online softmax, the lazy running-max rescale, 64 and 128 heads.
"""

import os

import numpy as np
import pytest
import torch

import synth
from oracle import pipeline
from parity_util import check_attn

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from long_context_sparse_gated_b200 import build
    build.build()


def _attn(w, dense=False, simt=False, idx=None):
    from long_context_sparse_gated_b200.runner import DeviceWorkload
    dw = DeviceWorkload(w)
    old = os.environ.get("CSA_ATTN")
    try:
        if simt:
            os.environ["CSA_ATTN"] = "simt"
        else:
            os.environ.pop("CSA_ATTN", None)
        # workspace sized for whichever path is selected
        from long_context_sparse_gated_b200 import (csa_sparse_attn_workspace_bytes,
                                                    hca_dense_attn_workspace_bytes)
        nb = hca_dense_attn_workspace_bytes(dw.params, dw.T, dw.n_max) if dense else \
            csa_sparse_attn_workspace_bytes(dw.params, dw.T)
        dw.ws_attn = torch.empty(max(nb, 16), dtype=torch.uint8, device="cuda")
        if dense:
            dw.dense_attn()
        else:
            if idx is not None:
                dw.idx.copy_(torch.from_numpy(idx))
            else:
                dw.index_topk()
            dw.sparse_attn()
        torch.cuda.synchronize()
    finally:
        if old is None:
            os.environ.pop("CSA_ATTN", None)
        else:
            os.environ["CSA_ATTN"] = old
    assert dw.err_bits() == 0, dw.err_bits()
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


def test_tc_matches_simt():
    w = synth.config("c1", B=2, L=8192, compress="none")
    a = _attn(w)
    b = _attn(w, simt=True, idx=a.idx.cpu().numpy())
    check_attn(a.out_f64(), b.out_f64(), what="tc vs simt")
