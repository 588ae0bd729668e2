"""The allocation-free indexer call, csa_index_topk_noalloc.

It exists for callers that cannot allocate device memory (a plugin given
only its inputs and outputs, a loop that must stay off the allocator) and
so cannot hand csa_index_topk a workspace; it uses a static device array
inside the library instead.  Checked through the C ABI against the regular
entry point on several calls in a row (the shared scratch keeps the previous
call's contents), including a row longer than 32768 entries whose candidate
lists live in the scratch, run after a larger call has left stale data
there; then that the calls allocate nothing, and the host-side rejection of
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


def _prepare(w):
    """Device workload and the regular entry point's indices."""
    from long_context_sparse_gated_b200.runner import DeviceWorkload
    dw = DeviceWorkload(w)
    dw.index_topk()
    torch.cuda.synchronize()
    assert dw.err_bits() == 0
    return dw, dw.idx.clone(), torch.full_like(dw.idx, -7)


def _noalloc(dw, out):
    from long_context_sparse_gated_b200 import csa_index_topk_noalloc
    csa_index_topk_noalloc(dw.params, dw.q_idx, dw.q_idx_sf, dw.w_idx, dw.k_idx, dw.k_idx_sf, dw.q_pos0,
                           dw.T, dw.n_max, out, err=dw.err)


def test_noalloc_matches_regular_entry_point_in_a_row():
    cases = [
        synth.config("c1", B=3, L=[16384, 9001, 4099]),
        synth.config("c2", B=2, L=65536, cluster=(1, 1024, 3.0)),
        synth.config("c1", B=32, L=131072),            # 4.5 MiB of workspace: leaves stale data
        synth.config("c2", B=2, L=262144, cluster=(1, 1024, 3.0)),  # n_max 65536: chunked candidates
    ]
    for i, w in enumerate(cases):
        dw, ref, out = _prepare(w)
        _noalloc(dw, out)
        torch.cuda.synchronize()
        assert dw.err_bits() == 0
        assert torch.equal(out, ref), f"call {i}"


def test_noalloc_allocates_nothing():
    """After the first call on the device (which loads the library module
    holding the scratch), further calls change neither torch's allocator
    nor the device's free memory."""
    dw, ref, out = _prepare(synth.config("c2", B=2, L=262144, cluster=(1, 1024, 3.0)))
    _noalloc(dw, out)  # first call on this device in a fresh process: module load
    torch.cuda.synchronize()
    torch_before = torch.cuda.memory_allocated()
    free_before = torch.cuda.mem_get_info()[0]
    for _ in range(3):
        out.fill_(-7)
        _noalloc(dw, out)
        torch.cuda.synchronize()
        assert torch.equal(out, ref)
    assert torch.cuda.memory_allocated() == torch_before
    assert torch.cuda.mem_get_info()[0] == free_before


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
