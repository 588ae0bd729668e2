"""Batch invariance (kwkr.cn notes 4.3 and Qiaomu blog 批次不变和确定性内核:
DeepSeek-V4's kernels give a query the same bits whatever batch it runs
in).  Each sequence is run alone (B = 1) and inside the full batch; its
compressed entry, top-k indices and attention output must be bitwise equal.
The batches mix sequence lengths, so the host bounds (n_max, the split
grid) differ between the two runs."""

import numpy as np
import pytest
import torch

import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from long_context_sparse_gated_b200 import build
    build.build()


def _run(w):
    from long_context_sparse_gated_b200.runner import DeviceWorkload
    dw = DeviceWorkload(w)
    dw.step()
    torch.cuda.synchronize()
    assert dw.err_bits() == 0
    res = {"out": dw.out.cpu().numpy()}
    if w["params"].k > 0:
        res["idx"] = dw.idx.cpu().numpy()
    res["kv"] = dw.kv.cpu().numpy()
    if dw.kv_scale is not None:
        res["kv_scale"] = dw.kv_scale.cpu().numpy()
    return res


@pytest.mark.parametrize("name,kw", [
    ("c1", dict(B=6, L=[8192, 8192 + 4, 16384, 6000, 8192, 12000])),   # 64 heads, split decode
    ("c2", dict(B=3, L=[65536, 40000, 65536 - 8])),                     # 128 heads
    ("c3", dict(B=4, L=[262144, 200000, 131072 + 64, 65536])),         # dense, n_t differs per sequence
])
def test_query_alone_equals_query_in_batch(name, kw):
    w = synth.config(name, **kw)
    full = _run(w)
    for b in range(w["params"].B):
        one = _run(synth.select_seqs(w, [b]))
        np.testing.assert_array_equal(one["out"][0], full["out"][b], err_msg=f"{name} seq {b}: output")
        if "idx" in full:
            np.testing.assert_array_equal(one["idx"][0], full["idx"][b], err_msg=f"{name} seq {b}: top-k")
        np.testing.assert_array_equal(one["kv"][0], full["kv"][b], err_msg=f"{name} seq {b}: cache rows")
