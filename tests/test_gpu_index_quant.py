"""On-device index keys and queries in FP4 (kwkr.cn notes 3.1, 3.4, 4.4;
Qiaomu blog FP4量化感知训练): csa_index_quantize and csa_index_compress
against the oracle's OCP MX conversion (oracle.codecs.mxfp4_encode) and its
compressor (oracle.csa.index_key_compress).

Quantising given values is deterministic arithmetic on both sides, so the
packed bytes and scales must be bit-identical.  Compressed keys come from
fp32 (GPU) and fp64 (oracle) merges, so a value may straddle an E2M1
rounding boundary or a block's amax a power of two: codes may then differ by
one step, scales by one binade where the oracle's amax is within 1e-5 of a
power of two, and nowhere else."""

import numpy as np
import pytest
import torch

import synth
from oracle import codecs, csa

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from long_context_sparse_gated_b200 import build
    build.build()


def _params(idx_dim, act, m=4, B=1):
    from long_context_sparse_gated_b200 import ACT_BF16, ACT_F32, make_params
    return make_params(B=B, d=512, r=64, m=m, n_idx_heads=64, idx_dim=idx_dim,
                       act_fmt=ACT_BF16 if act == "bf16" else ACT_F32)


def _rows(rng, n, c):
    """Values spanning many binades, plus blocks of exact E2M1 ties and
    all-zero blocks."""
    x = rng.normal(size=(n, c)) * np.exp2(rng.uniform(-30, 30, size=(n, 1)))
    ties = np.array([6, 3, 1.5, 0.75, -0.25, 5, 2.5, -7, 0.25, -1.25, 3.5, -5] + [0] * 20, np.float64)
    x[0, :32] = ties
    x[1, :32] = ties * 2.0 ** -9
    x[2, :] = 0.0
    if c > 32:
        x[3, 32:64] = -ties * 2.0 ** 17
    return x


@pytest.mark.parametrize("act,c", [("bf16", 128), ("f32", 128), ("bf16", 64)])
def test_index_quantize_bit_exact(act, c):
    from long_context_sparse_gated_b200 import csa_index_quantize
    rng = np.random.default_rng(21)
    x = _rows(rng, 4096, c)
    if act == "bf16":
        host = synth._bf16_of(x)
        vals = codecs.bf16_decode(host)
        dev = torch.from_numpy(host.view(np.int16)).cuda()
    else:
        host = x.astype(np.float32)
        vals = host.astype(np.float64)
        dev = torch.from_numpy(host).cuda()
    out = torch.zeros((4096, c // 2), dtype=torch.uint8, device="cuda")
    sf = torch.zeros((4096, c // 32), dtype=torch.uint8, device="cuda")
    csa_index_quantize(_params(c, act), dev, out, sf)
    torch.cuda.synchronize()
    o_packed, o_sf = codecs.mxfp4_encode(vals)
    np.testing.assert_array_equal(sf.cpu().numpy(), o_sf)
    np.testing.assert_array_equal(out.cpu().numpy(), o_packed)


def _e2m1_line(nib):
    n = np.asarray(nib).astype(np.int64)
    return np.where(n & 8, -(n & 7), n & 7)


@pytest.mark.parametrize("act,c,m,rope", [("bf16", 128, 4, 64), ("f32", 64, 4, 32), ("bf16", 128, 128, 0)])
def test_index_compress_matches_oracle(act, c, m, rope):
    from long_context_sparse_gated_b200 import csa_index_compress
    rng = np.random.default_rng(22)
    B, n_ent = 3, 40
    S = m * n_ent
    if act == "bf16":
        a = synth.normal_bf16(rng, (B, S, c))
        b = synth.normal_bf16(rng, (B, S, c))
        a64, b64 = codecs.bf16_decode(a), codecs.bf16_decode(b)
        ta, tb = (torch.from_numpy(v.view(np.int16)).cuda() for v in (a, b))
    else:
        a = synth.normal_f32(rng, (B, S, c))
        b = synth.normal_f32(rng, (B, S, c))
        a64, b64 = a.astype(np.float64), b.astype(np.float64)
        ta, tb = torch.from_numpy(a).cuda(), torch.from_numpy(b).cuda()
    gate = synth.normal_f32(rng, (B, S, 2)) * np.float32(2.0)
    zeros = torch.zeros(B, dtype=torch.int32, device="cuda")
    e_end = torch.full((B,), n_ent, dtype=torch.int32, device="cuda")
    k_cap = n_ent + 4
    k = torch.zeros((B, k_cap, c // 2), dtype=torch.uint8, device="cuda")
    ksf = torch.zeros((B, k_cap, c // 32), dtype=torch.uint8, device="cuda")
    err = torch.zeros(4, dtype=torch.int32, device="cuda")
    p = _params(c, act, m, B=B)
    csa_index_compress(p, ta, tb, torch.from_numpy(gate).cuda(), zeros, zeros, e_end, n_ent, rope, k, ksf, err=err)
    torch.cuda.synchronize()
    assert int(err[0]) == 0
    g_packed, g_sf = k.cpu().numpy()[:, :n_ent], ksf.cpu().numpy()[:, :n_ent]
    n_diff = 0
    for bb in range(B):
        o_packed, o_sf, pos = csa.index_key_compress(a64[bb], b64[bb], gate[bb], m, rope, 1e4, 1e-6)
        assert pos.tolist() == [m * e for e in range(n_ent)]
        keys, _ = csa.compress(a64[bb], b64[bb], gate[bb], m, rope, 1e4, 1e-6)
        amax = np.abs(keys.reshape(n_ent, c // 32, 32)).max(axis=-1)
        near_pow2 = np.abs(np.log2(amax) - np.round(np.log2(amax))) < 1e-5 / np.log(2)
        sdiff = g_sf[bb].astype(int) - o_sf.astype(int)
        assert np.all((sdiff == 0) | ((np.abs(sdiff) == 1) & near_pow2)), "scale differs away from a power of two"
        gn = np.stack([g_packed[bb] & 0xF, g_packed[bb] >> 4], -1).reshape(n_ent, c)
        on = np.stack([o_packed & 0xF, o_packed >> 4], -1).reshape(n_ent, c)
        same_scale = np.repeat(sdiff == 0, 32, axis=-1)
        step = np.abs(_e2m1_line(gn) - _e2m1_line(on))
        assert step[same_scale].max() <= 1
        n_diff += int((step[same_scale] > 0).sum())
    assert n_diff <= 0.01 * B * n_ent * c
