"""Decode-time state (kwkr.cn notes 4.4: a state cache beside the classical
KV cache, periodic checkpointing every 1024 tokens): csa_state_append and
csa_state_restore against the token-by-token oracle (oracle.state).

A sequence is fed in uneven chunks (prefill-like and single-token decode
appends) past 1024 and 2048 tokens.  Checked: the window ring, the stream
rings, every entry the appends completed, both checkpoints; then a fresh
state restored from the 1024 checkpoint and fed the rest in other chunks
ends bit-identical to the uninterrupted run."""

import numpy as np
import pytest
import torch

import synth
from oracle import codecs, csa, state as ostate
from parity_util import check_fp8_rows

pytestmark = pytest.mark.gpu

B, D, R, M, W = 2, 512, 64, 4, 128
EVERY, SLOTS = 1024, 3
CHUNKS = [300, 1, 1, 700, 1, 21, 1, 1000, 3, 100]   # 2128 tokens: crosses 1024 and 2048
L = sum(CHUNKS)
T_MAX = max(CHUNKS)


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from long_context_sparse_gated_b200 import build
    build.build()


def _inputs(seed=31):
    rng = np.random.default_rng(seed)
    kv = synth.normal_bf16(rng, (B, L, D))      # window KV vectors (already normalised/rotated)
    a = synth.normal_bf16(rng, (B, L, D))
    b = synth.normal_bf16(rng, (B, L, D))
    gate = synth.normal_f32(rng, (B, L, 2))
    return kv, a, b, gate


class _Dev:
    def __init__(self):
        from long_context_sparse_gated_b200 import make_ckpt, make_state, make_params
        self.p = make_params(B=B, d=D, r=R, m=M, n_idx_heads=64, idx_dim=128, topk=512, n_heads=64, window=W,
                             softmax_scale=1.0 / np.sqrt(D))
        cu = dict(device="cuda")
        self.win = torch.zeros((B, W + T_MAX, D + R), dtype=torch.uint8, **cu)
        self.win_sc = torch.zeros((B, W + T_MAX), dtype=torch.float32, **cu)
        s_cap = ((T_MAX + 2 * M + M - 1) // M) * M
        self.a = torch.zeros((B, s_cap, D), dtype=torch.int16, **cu)
        self.b = torch.zeros((B, s_cap, D), dtype=torch.int16, **cu)
        self.g = torch.zeros((B, s_cap, 2), dtype=torch.float32, **cu)
        self.cache = torch.zeros((B, L // M + 4, D + R), dtype=torch.uint8, **cu)
        self.cache_sc = torch.zeros((B, L // M + 4), dtype=torch.float32, **cu)
        self.cache_pos = torch.full((B, L // M + 4), -1, dtype=torch.int32, **cu)
        self.ck = [torch.zeros((B, SLOTS, W, D + R), dtype=torch.uint8, **cu),
                   torch.zeros((B, SLOTS, W), dtype=torch.float32, **cu),
                   torch.zeros((B, SLOTS, M, D), dtype=torch.int16, **cu),
                   torch.zeros((B, SLOTS, M, D), dtype=torch.int16, **cu),
                   torch.zeros((B, SLOTS, M, 2), dtype=torch.float32, **cu)]
        self.err = torch.zeros(4, dtype=torch.int32, **cu)
        self.state = make_state(self.win, self.win_sc, self.a, self.b, self.g)
        self.ckpt = make_ckpt(*self.ck, every=EVERY)

    def append(self, kv, a, b, gate, p0, T):
        from long_context_sparse_gated_b200 import csa_state_append
        sl = slice(p0, p0 + T)
        t = lambda x: torch.from_numpy(np.ascontiguousarray(x[:, sl])).cuda()
        pos0 = torch.full((B,), p0, dtype=torch.int32, device="cuda")
        csa_state_append(self.p, t(kv.view(np.int16)), t(a.view(np.int16)), t(b.view(np.int16)), t(gate), pos0,
                         self.state, self.cache, self.cache_sc, self.cache_pos, self.ckpt, err=self.err)

    def restore(self, P):
        from long_context_sparse_gated_b200 import csa_state_restore
        csa_state_restore(self.p, torch.full((B,), P, dtype=torch.int32, device="cuda"), self.ckpt, self.state,
                          err=self.err)


def _feed(dev, inputs, start, chunks):
    p0 = start
    for T in chunks:
        dev.append(*inputs, p0, T)
        p0 += T
    torch.cuda.synchronize()
    assert int(dev.err[0]) == 0
    return p0


def _packed(rows, scale):
    rows = np.asarray(rows)
    return rows[..., : D - R], np.asarray(scale), np.ascontiguousarray(rows[..., D - R:]).view(np.uint16)


def test_state_append_matches_oracle():
    inputs = _inputs()
    kv, a, b, gate = inputs
    dev = _Dev()
    end = _feed(dev, inputs, 0, CHUNKS)
    assert end == L
    win, win_sc = dev.win.cpu().numpy(), dev.win_sc.cpu().numpy()
    cache, cache_sc = dev.cache.cpu().numpy(), dev.cache_sc.cpu().numpy()
    cpos = dev.cache_pos.cpu().numpy()
    for s in range(B):
        kv64, a64, b64 = (codecs.bf16_decode(x[s]) for x in (kv, a, b))
        # window ring: tokens L-W .. L-1 at row p mod cap
        ws = ostate.window_state(kv64, L, W, R, "fp8")
        pos = sorted(ws)
        rows = [(p % dev.win.shape[1]) for p in pos]
        oc = np.stack([ws[p][0] for p in pos]); osc = np.array([ws[p][1] for p in pos])
        ob = np.stack([ws[p][2] for p in pos])
        check_fp8_rows(win[s, rows], win_sc[s, rows], oc, osc, ob, D, R, what=f"window seq {s}")
        # stream rings: the last s_cap tokens, bit copies
        s_cap = dev.a.shape[1]
        a_r, b_r, g_r = dev.a.cpu().numpy()[s], dev.b.cpu().numpy()[s], dev.g.cpu().numpy()[s]
        for p in range(L - s_cap, L):
            assert np.array_equal(a_r[p % s_cap].view(np.uint16), a[s, p])
            assert np.array_equal(b_r[p % s_cap].view(np.uint16), b[s, p])
            assert np.array_equal(g_r[p % s_cap], gate[s, p])
        # entries: every complete block, as the compressor over the whole prefix
        ent, epos = ostate.entries_after(a64, b64, gate[s], L, M, R, 1e4, 1e-6)
        n = len(epos)
        assert n == L // M
        np.testing.assert_array_equal(cpos[s, :n], epos)
        oc, osc, ob = csa.pack_entries(ent, R)
        check_fp8_rows(cache[s, :n], cache_sc[s, :n], oc, osc, ob, D, R, what=f"entries seq {s}")
        # checkpoints at 1024 (slot 0) and 2048 (slot 1)
        ck = [x.cpu().numpy() for x in dev.ck]
        for P in (1024, 2048):
            slot = (P // EVERY - 1) % SLOTS
            ws = ostate.window_state(kv64, P, W, R, "fp8")
            pos = sorted(ws)
            oc = np.stack([ws[p][0] for p in pos]); osc = np.array([ws[p][1] for p in pos])
            ob = np.stack([ws[p][2] for p in pos])
            check_fp8_rows(ck[0][s, slot], ck[1][s, slot], oc, osc, ob, D, R, what=f"ckpt {P} window seq {s}")
            ss = ostate.stream_state(a64, b64, gate[s], P, M)
            for i, p in enumerate(sorted(ss)):
                assert np.array_equal(ck[2][s, slot, i].view(np.uint16), a[s, p])
                assert np.array_equal(ck[3][s, slot, i].view(np.uint16), b[s, p])
                assert np.array_equal(ck[4][s, slot, i], gate[s, p])


def test_restore_from_checkpoint_resumes_bit_identically():
    inputs = _inputs()
    full = _Dev()
    _feed(full, inputs, 0, CHUNKS)
    part = _Dev()
    _feed(part, inputs, 0, [700, 324])              # reaches 1024: checkpoint slot 0
    resumed = _Dev()
    resumed.cache.copy_(part.cache)                 # the classical cache survives
    resumed.cache_sc.copy_(part.cache_sc)
    resumed.cache_pos.copy_(part.cache_pos)
    for src, dst in zip(part.ck, resumed.ck):
        dst.copy_(src)
    resumed.restore(1024)
    end = _feed(resumed, inputs, 1024, [1, 2, 500, 601])
    assert end == L
    for name in ("cache", "cache_sc", "cache_pos"):
        assert torch.equal(getattr(resumed, name), getattr(full, name)), name
    cap = full.win.shape[1]
    rows = [p % cap for p in range(L - W, L)]
    assert torch.equal(resumed.win[:, rows], full.win[:, rows])
    assert torch.equal(resumed.win_sc[:, rows], full.win_sc[:, rows])
