"""The allocation-free indexer call, csa_index_topk_noalloc.

It exists for callers that cannot allocate device memory (a plugin given
only its inputs and outputs, a loop that must stay off the allocator) and
so cannot hand csa_index_topk a workspace; it uses a static device array
inside the library instead.  Checked through the C ABI against the regular
entry point, on two calls in a row with different workloads (the shared
scratch keeps the previous call's contents), plus the host-side rejection of
a problem larger than the scratch.  This file is collected last.
"""

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


def _regular_and_noalloc(w):
    from long_context_sparse_gated_b200 import csa_index_topk_noalloc
    from long_context_sparse_gated_b200.runner import DeviceWorkload
    dw = DeviceWorkload(w)
    dw.index_topk()
    ref = dw.idx.clone()
    out = torch.full_like(dw.idx, -7)
    csa_index_topk_noalloc(dw.params, dw.q_idx, dw.q_idx_sf, dw.w_idx, dw.k_idx, dw.k_idx_sf, dw.q_pos0,
                           dw.T, dw.n_max, out, err=dw.err)
    torch.cuda.synchronize()
    assert dw.err_bits() == 0
    return ref, out


def test_noalloc_matches_regular_entry_point_twice():
    ref1, out1 = _regular_and_noalloc(synth.config("c1", B=3, L=[16384, 9001, 4099]))
    assert torch.equal(out1, ref1)
    ref2, out2 = _regular_and_noalloc(synth.config("c2", B=2, L=65536, cluster=(1, 1024, 3.0)))
    assert torch.equal(out2, ref2)


def test_noalloc_rejects_problems_beyond_the_scratch():
    from long_context_sparse_gated_b200 import CsaError, csa_index_topk_noalloc
    from long_context_sparse_gated_b200.runner import DeviceWorkload
    w = synth.config("c1", B=1, L=8192)
    dw = DeviceWorkload(w)
    # n_max / T that would need > 16 MiB of workspace; rejected on the host
    with pytest.raises(CsaError) as e:
        csa_index_topk_noalloc(dw.params, dw.q_idx, dw.q_idx_sf, dw.w_idx, dw.k_idx, dw.k_idx_sf, dw.q_pos0,
                               5000, dw.n_max, dw.idx, err=dw.err)
    assert e.value.status == -4
