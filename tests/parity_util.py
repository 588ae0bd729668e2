"""Comparison helpers for the GPU-vs-oracle parity tests.

Tolerances (stated once, used everywhere):
  * BF16/FP8 attention outputs: max |gpu - oracle| <= 2e-2 and
    mean |gpu - oracle| / mean |oracle| <= 5e-3.
  * fp32 (config 0) outputs and compressed entries: max |diff| / max |oracle|
    <= 1e-5.
  * FP8 pack: E4M3 codes within one code step, per-row scale within 1e-6
    relative (fp32 vs fp64 values may straddle a rounding boundary); BF16
    RoPE dims within one BF16 ulp of the oracle's value plus 1e-6 absolute
    (the kernel rotates in fp32: a rotated value near zero carries the
    fp32 cancellation error of its unit-size inputs, ~1e-7).
  * Wide-range attention workloads (row scales, RoPE magnitudes or queries
    spanning many binades, so outputs are far from unit size): the two
    BF16/FP8 bounds applied to each head's output divided by the largest
    magnitude of the oracle's output of that head.
  * Top-k sets: identical (they are unique: ties go to the lower index).
    On fp32 index data (config 0) a mismatch is accepted only where the
    oracle's k-th and (k+1)-th scores are within 1e-5 relative.
  * Entry positions: identical.
"""

import numpy as np

from oracle import codecs, csa

ATTN_MAX_ABS = 2e-2
ATTN_MEAN_REL = 5e-3
F32_REL = 1e-5


def bf16_to_f64(x):
    return (np.asarray(x).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def check_attn(gpu, ref, f32=False, what=""):
    gpu = np.asarray(gpu, np.float64)
    ref = np.asarray(ref, np.float64)
    assert gpu.shape == ref.shape, (gpu.shape, ref.shape)
    assert np.all(np.isfinite(gpu)), f"{what}: non-finite GPU output"
    diff = np.abs(gpu - ref)
    if f32:
        rel = diff.max() / max(np.abs(ref).max(), 1e-30)
        assert rel <= F32_REL, f"{what}: max rel {rel:.3e} > {F32_REL}"
        return rel
    mx = diff.max()
    mrel = diff.mean() / max(np.abs(ref).mean(), 1e-30)
    assert mx <= ATTN_MAX_ABS, f"{what}: max abs {mx:.3e} > {ATTN_MAX_ABS}"
    assert mrel <= ATTN_MEAN_REL, f"{what}: mean rel {mrel:.3e} > {ATTN_MEAN_REL}"
    return mx, mrel


def check_attn_scaled(gpu, ref, what=""):
    """check_attn on every (query, head) output normalised by the oracle's
    largest magnitude of that head (heads with an all-zero oracle output must
    be all zero)."""
    gpu = np.asarray(gpu, np.float64)
    ref = np.asarray(ref, np.float64)
    assert gpu.shape == ref.shape, (gpu.shape, ref.shape)
    assert np.all(np.isfinite(gpu)), f"{what}: non-finite GPU output"
    mag = np.abs(ref).max(axis=-1, keepdims=True)
    zero = mag[..., 0] == 0
    assert np.all(gpu[zero] == 0), f"{what}: nonzero output where the oracle's is 0"
    mag = np.where(mag == 0, 1.0, mag)
    return check_attn(gpu / mag, ref / mag, what=what)


def _mag_index(codes):
    """Position of an E4M3 code on the signed magnitude line (+-0 -> 0)."""
    c = np.asarray(codes).astype(np.int64)
    mag = c & 0x7F
    return np.where(c & 0x80, -mag, mag)


def check_fp8_rows(g_rows, g_scale, o_codes, o_scale, o_rbits, d, r, what=""):
    """GPU packed rows [n, d+r] + scale [n] vs oracle codes/scale/bits."""
    g_rows = np.asarray(g_rows)
    g_codes = g_rows[:, : d - r]
    g_rbits = np.ascontiguousarray(g_rows[:, d - r:]).view(np.uint16)
    np.testing.assert_allclose(np.asarray(g_scale, np.float64), np.asarray(o_scale, np.float64),
                               rtol=1e-6, err_msg=f"{what}: scale")
    step = np.abs(_mag_index(g_codes) - _mag_index(o_codes))
    assert step.max() <= 1, f"{what}: E4M3 codes differ by {step.max()} steps"
    gv = bf16_to_f64(g_rbits)
    ov = bf16_to_f64(o_rbits)
    ulp = np.exp2(np.floor(np.log2(np.maximum(np.abs(ov), 2.0 ** -126))) - 7)
    bad = np.abs(gv - ov) > ulp + 1e-6
    assert not bad.any(), f"{what}: bf16 RoPE dims differ: {gv[bad][:4]} vs {ov[bad][:4]}"


def check_topk(g_idx, o_idx, o_scores=None, n_t=None, exact=True, what=""):
    g = np.asarray(g_idx)
    o = np.asarray(o_idx)
    if exact or o_scores is None:
        np.testing.assert_array_equal(g, o, err_msg=f"{what}: top-k sets differ")
        return
    if np.array_equal(g, o):
        return
    # fp32 data: accept only a near-tie at the k-th place
    k = len(o)
    sc = np.sort(np.asarray(o_scores)[:n_t])[::-1]
    assert n_t > k, f"{what}: differ although every entry is selected"
    gap = abs(sc[k - 1] - sc[k]) / max(abs(sc[k - 1]), 1e-30)
    assert gap < 1e-5, f"{what}: top-k differs with k-th gap {gap:.2e}"
    # and the GPU's set must be a valid top-k up to that tie
    gs = set(int(x) for x in g if x >= 0)
    assert len(gs) == k and all(0 <= x < n_t for x in gs)
    assert min(o_scores[list(gs)]) >= sc[k - 1] * (1 - 2e-5)


def valid_topk_layout(g_idx, n_t, k):
    g = np.asarray(g_idx)
    n = min(k, n_t)
    assert np.all(g[n:] == -1)
    assert np.all(np.diff(g[:n]) > 0) and (n == 0 or (g[0] >= 0 and g[n - 1] < n_t))
