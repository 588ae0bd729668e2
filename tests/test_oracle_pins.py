"""Pins of the oracle's method arithmetic: closed forms, invariants,
hand-worked fixtures (tests/golden), brute force on tiny inputs and a
textbook reduction.  None of these re-types the oracle's own formula."""

import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest

import synth
from oracle import codecs, csa, pipeline

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _gold(name):
    with open(os.path.join(GOLD, name)) as f:
        return json.load(f)


def _num(v):
    if v == "ln3":
        return math.log(3.0)
    if v == "ln2":
        return math.log(2.0)
    return float(v)


# --------------------------------------------------------------------------
# compressor
# --------------------------------------------------------------------------


def test_compress_hand_worked_fixture():
    g = _gold("compress_8tok_d4.json")
    a = np.array(g["a"], float)
    b = np.array(g["b"], float)
    gate = np.stack([[_num(x) for x in g["gate_a"]], [_num(x) for x in g["gate_b"]]], axis=1)
    ent, pos = csa.compress(a, b, gate, m=4, r=2, theta=1e4, eps=0.0)
    np.testing.assert_array_equal(pos, g["expected"]["pos"])
    np.testing.assert_allclose(ent[0], g["expected"]["entry0"], rtol=0, atol=1e-14)
    np.testing.assert_allclose(ent[1], g["expected"]["entry1"], rtol=0, atol=1e-14)


def test_gate_weights_convex():
    rng = np.random.default_rng(1)
    for m in (4, 128):
        for _ in range(20):
            ga, gb = rng.standard_normal(m) * 5, rng.standard_normal(m) * 5
            wa, wb = csa.gate_weights(ga, gb)
            assert np.all(wa >= 0) and np.all(wb >= 0)
            assert abs(wa.sum() + wb.sum() - 1.0) < 1e-15 * 4 * m
        wa, wb = csa.gate_weights(rng.standard_normal(m), np.zeros(0))
        assert abs(wa.sum() - 1) < 1e-14 and len(wb) == 0


def test_merge_equal_logits_is_mean():
    rng = np.random.default_rng(2)
    m, d = 4, 16
    A, Bp = rng.standard_normal((m, d)), rng.standard_normal((m, d))
    x = csa.merge_entry(A, Bp, np.full(m, 0.7), np.full(m, 0.7))
    np.testing.assert_allclose(x, np.concatenate([A, Bp]).mean(axis=0), atol=1e-15)


def test_merge_b_stream_off_is_block_mean():
    rng = np.random.default_rng(3)
    m, d = 128, 8
    A, Bp = rng.standard_normal((m, d)), rng.standard_normal((m, d))
    x = csa.merge_entry(A, Bp, np.zeros(m), np.full(m, -np.inf))
    np.testing.assert_allclose(x, A.mean(axis=0), atol=1e-14)


def test_compress_rms_one_and_positions():
    rng = np.random.default_rng(4)
    L, d, r, m = 64, 32, 8, 4
    a, b = rng.standard_normal((L, d)), rng.standard_normal((L, d))
    gate = rng.standard_normal((L, 2))
    ent, pos = csa.compress(a, b, gate, m, r, 1e4, 0.0)
    assert ent.shape == (L // m, d)
    np.testing.assert_array_equal(pos, np.arange(L // m) * m)
    # RoPE preserves the norm, so RMS is 1 after it as well
    np.testing.assert_allclose(np.sqrt((ent ** 2).mean(axis=1)), 1.0, atol=1e-12)
    # the first d-r dims are untouched by RoPE: equal to the normalised merge
    e3 = csa.rmsnorm(csa.merge_entry(a[12:16], b[8:12], gate[12:16, 0], gate[8:12, 1]), None, 0.0)
    np.testing.assert_allclose(ent[3, : d - r], e3[: d - r], atol=1e-14)


def test_compress_incremental_equals_full():
    """Entries computed from a trailing token buffer (decode) equal the same
    entries computed from the whole sequence."""
    rng = np.random.default_rng(5)
    L, d, r, m = 40, 16, 4, 4
    a, b, gate = rng.standard_normal((L, d)), rng.standard_normal((L, d)), rng.standard_normal((L, 2))
    full, _ = csa.compress(a, b, gate, m, r, 1e4, 1e-6)
    base = L - 2 * m
    last, pos = csa.compress(a[base:], b[base:], gate[base:], m, r, 1e4, 1e-6,
                             e_begin=L // m - 1, e_end=L // m, tok_base=base)
    assert pos[0] == L - m
    np.testing.assert_array_equal(last[0], full[-1])


# --------------------------------------------------------------------------
# RoPE
# --------------------------------------------------------------------------


def test_rope_known_rotations():
    v = np.array([5.0, 1.0, 0.0, 1.0, 0.0])  # d=5, r=4: pairs (1,2), (3,4)
    out = csa.rope(v, 1, 1e4, 4)
    assert out[0] == 5.0
    # pair 0: angle 1 * 1e4^0 = 1; pair 1: angle 1 * 1e4^(-2/4) = 0.01
    np.testing.assert_allclose(out[1:3], [math.cos(1), math.sin(1)], atol=1e-15)
    np.testing.assert_allclose(out[3:5], [math.cos(0.01), math.sin(0.01)], atol=1e-15)


def test_rope_norm_and_inverse():
    rng = np.random.default_rng(6)
    v = rng.standard_normal((10, 64))
    for t in (0, 3, 4095, 1048575):
        w = csa.rope(v, t, 1e4, 32)
        np.testing.assert_allclose(np.linalg.norm(w, axis=1), np.linalg.norm(v, axis=1), rtol=1e-13)
        np.testing.assert_allclose(csa.rope(w, -t, 1e4, 32), v, atol=1e-9)


# --------------------------------------------------------------------------
# packing
# --------------------------------------------------------------------------


def test_pack_scale_and_roundtrip():
    rng = np.random.default_rng(7)
    y = rng.standard_normal(512)
    codes, scale, rbits = csa.pack_entry(y, 64)
    amax = np.abs(y[:448]).max()
    assert scale == np.float32(amax / 448)
    # the largest element lands on (or within rounding of) the top code
    assert codecs.e4m3_decode(codes).__abs__().max() in (448.0, 416.0)
    back = csa.unpack_rows(codes[None], np.array([scale]), rbits[None])[0]
    # E4M3 has 3 mantissa bits: relative half-step 2^-4 for normals
    err = np.abs(back[:448] - y[:448])
    assert np.all(err <= np.maximum(np.abs(y[:448]) * 2 ** -4, 2 ** -10 * scale) + 1e-12)
    np.testing.assert_allclose(back[448:], y[448:], rtol=2 ** -8)
    c0, s0, _ = csa.pack_entry(np.zeros(512), 64)
    assert s0 == 1.0 and not c0.any()


def test_storage_fraction_two_percent():
    """The mixed layout's bytes reproduce the '~2% of a BF16 GQA8 (head dim
    128) cache at 1M context' figure (WeChat 1.1; kwkr 3.4) for alternating
    CSA (580 B entry + 68 B MXFP4 index key per 4 tokens) and HCA (580 B per
    128 tokens) layers."""
    L = 2 ** 20
    base = L * 8 * 128 * 2 * 2  # K and V, 8 groups, dim 128, bf16
    entry = 448 + 64 * 2 + 4
    key = 128 // 2 + 128 // 32
    csa_l = (L // 4) * (entry + key)
    hca_l = (L // 128) * entry
    frac = (csa_l + hca_l) / 2 / base
    assert entry == 580 and key == 68
    assert 0.015 < frac < 0.025


# --------------------------------------------------------------------------
# indexer and top-k
# --------------------------------------------------------------------------


def test_index_scores_brute_force():
    rng = np.random.default_rng(8)
    H, c, n = 3, 5, 7
    q, k = rng.standard_normal((H, c)), rng.standard_normal((n, c))
    w = rng.uniform(0.1, 1, H)
    got = csa.index_scores(q, w, k)
    for s in range(n):
        ref = 0.0
        for h in range(H):
            dot = sum(q[h, j] * k[s, j] for j in range(c))
            ref += w[h] * (dot if dot > 0 else 0.0)
        assert abs(got[s] - ref) < 1e-12


def test_index_scores_exact_on_mxfp4_grid():
    """On MXFP4 inputs with dyadic head weights, the fp64 score equals the
    exact rational score (Fractions)."""
    w = synth.config("c0", idx_fmt="mxfp4", L=256)
    q, wt = pipeline.index_query(w, 0, 0)
    k = pipeline.index_keys(w, 0, 64)
    got = csa.index_scores(q, wt, k)
    for s in range(0, 64, 7):
        tot = Fraction(0)
        for h in range(q.shape[0]):
            dot = sum(Fraction(q[h, j]) * Fraction(k[s, j]) for j in range(q.shape[1]))
            tot += Fraction(wt[h]) * max(dot, Fraction(0))
        assert Fraction(got[s]) == tot


def _brute_topk(scores, n_t, k):
    order = sorted(range(n_t), key=lambda s: (-scores[s], s))[:k]
    return sorted(order) + [-1] * (k - min(k, n_t))


@pytest.mark.parametrize("n,k", [(10, 3), (10, 10), (5, 8), (0, 4), (64, 16)])
def test_topk_brute_force_with_ties(n, k):
    rng = np.random.default_rng(n * 31 + k)
    for trial in range(20):
        sc = rng.integers(0, 4, n).astype(float)  # many ties, many zeros
        if trial % 2:
            sc = rng.standard_normal(n)
        got = csa.topk_select(sc, n, k)
        assert list(got) == _brute_topk(sc, n, k)


def test_topk_ties_lower_index_and_padding():
    sc = np.array([1.0, 2.0, 2.0, 0.0, 2.0])
    assert list(csa.topk_select(sc, 5, 2)) == [1, 2]
    assert list(csa.topk_select(sc, 3, 5)) == [0, 1, 2, -1, -1]
    assert list(csa.topk_select(sc, 0, 2)) == [-1, -1]


def test_n_visible_causality():
    # entry i (tokens m*i..m*i+m-1) is visible to t iff its last token <= t
    for m in (4, 128):
        for t in range(0, 3 * m):
            n = csa.n_visible(t, m)
            assert all(m * (i + 1) - 1 <= t for i in range(n))
            assert m * (n + 1) - 1 > t


# --------------------------------------------------------------------------
# attention
# --------------------------------------------------------------------------


def test_attend_hand_worked_fixture():
    g = _gold("attend_1head_d4.json")
    rows = np.array(g["rows"], float)
    q = np.array([[_num(x) for x in g["q"]]])
    o = csa.attend(q, rows, np.array([g["sink"]]), 1.0, g["t"], 1e4, 2)
    np.testing.assert_allclose(o[0], g["expected"]["o"], atol=1e-15)
    p, ps = csa.attention_weights(q, rows, np.array([g["sink"]]), 1.0)
    np.testing.assert_allclose(p[0], g["expected"]["p"], atol=1e-15)
    assert abs(ps[0] - g["expected"]["sink_weight"]) < 1e-15


def test_attend_weights_sum_with_sink():
    rng = np.random.default_rng(9)
    q, rows = rng.standard_normal((6, 32)), rng.standard_normal((50, 32))
    sig = rng.standard_normal(6) * 3
    p, ps = csa.attention_weights(q, rows, sig, 0.3)
    assert np.all(p >= 0)
    s = p.sum(axis=1)
    assert np.all(s <= 1 + 1e-15)
    np.testing.assert_allclose(1 - s, ps, atol=1e-14)


def test_attend_single_candidate_no_sink_is_value():
    rng = np.random.default_rng(10)
    v = rng.standard_normal((1, 16))
    q = rng.standard_normal((3, 16))
    o = csa.attend(q, v, np.full(3, -np.inf), 0.5, 77, 1e4, 8)
    for h in range(3):
        np.testing.assert_allclose(o[h], csa.rope(v[0], -77, 1e4, 8), atol=1e-14)


def test_attend_no_rows_is_zero():
    o = csa.attend(np.ones((2, 8)), np.zeros((0, 8)), np.zeros(2), 1.0, 5, 1e4, 4)
    assert np.all(o == 0)


def test_attend_equals_textbook_softmax():
    rng = np.random.default_rng(11)
    q, rows = rng.standard_normal((4, 24)), rng.standard_normal((30, 24))
    sig = rng.standard_normal(4)
    o = csa.attend(q, rows, sig, 0.2, 123, 1e4, 8)
    ref = csa.rope(csa.dense_softmax_with_null_value(q, rows, sig, 0.2), -123, 1e4, 8)
    np.testing.assert_allclose(o, ref, atol=1e-13)


def test_csa_reduces_to_dense_when_k_and_window_cover_all():
    """With k >= n_t and W >= t+1, CSA = plain softmax attention over every
    visible entry and every raw token, plus the sink (textbook routine)."""
    p = synth.Params(B=1, d=32, r=8, m=4, H_I=2, c_I=32, k=64, n_h=3, W=64, tau=0.25,
                     kv_fmt="f32", idx_fmt="f32", act_fmt="f32")
    L = 40
    w = synth.make_workload(21, p, L=L, T=3, compress="all", sink="normal")
    comp, idx, out = pipeline.csa_step(w)
    cache = pipeline.cache_rows(w, 0, comp)
    for tq in range(3):
        t = L - 3 + tq
        n_t = (t + 1) // 4
        assert list(idx[(0, tq)][:n_t]) == list(range(n_t))
        slots = np.arange(0, t + 1) % w["Wcap"]
        toks = w["win"][0][slots].astype(np.float64)
        vals = np.concatenate([cache[:n_t], toks])
        q = w["q"][0, tq].astype(np.float64)
        ref = csa.rope(csa.dense_softmax_with_null_value(q, vals, w["sink"], p.tau), -t, 1e4, 8)
        np.testing.assert_allclose(out[(0, tq)], ref, atol=1e-12)


def test_hca_pipeline_window_and_causality():
    """HCA attends exactly the n_t visible entries plus the window."""
    p = synth.Params(B=2, d=32, r=8, m=8, H_I=2, c_I=32, k=0, n_h=2, W=4, tau=0.3,
                     kv_fmt="f32", idx_fmt="f32", act_fmt="f32")
    w = synth.make_workload(22, p, L=[37, 20], T=2, compress="all")
    comp, out = pipeline.hca_step(w)
    for b in range(2):
        cache = pipeline.cache_rows(w, b, comp)
        for tq in range(2):
            t = int(w["q_pos0"][b]) + tq
            n_t = (t + 1) // 8
            pos = np.arange(max(0, t - 3), t + 1)
            vals = np.concatenate([cache[:n_t], w["win"][b][pos % w["Wcap"]].astype(np.float64)])
            q = w["q"][b, tq].astype(np.float64)
            ref = csa.rope(csa.dense_softmax_with_null_value(q, vals, w["sink"], p.tau), -t, 1e4, 8)
            np.testing.assert_allclose(out[(b, tq)], ref, atol=1e-12)


# ---- BF16 index scores (the selector's low-precision variant) -------------

def test_bf16_scores_round_to_nearest_even_like_torch():
    import torch
    rng = np.random.default_rng(7)
    x = np.concatenate([rng.normal(size=2000) * 37.0, [0.0, 1.0, 1.00390625, 1.01171875, 3.0e-3]])
    ref = torch.tensor(x, dtype=torch.float32).to(torch.bfloat16).to(torch.float64).numpy()
    np.testing.assert_array_equal(csa.bf16_scores(x.astype(np.float32).astype(np.float64)), ref)


def test_bf16_topk_ranks_collisions_by_index():
    # 1 + 2^-9 and 1 + 2^-10 both round to 1.0 in BF16: after rounding the
    # three entries tie and the lowest indices win
    sc = np.array([1.0, 1.0 + 2.0 ** -10, 1.0 + 2.0 ** -9, 0.5])
    assert csa.topk_select(sc, 4, 2).tolist() == [1, 2]
    assert csa.topk_select(csa.bf16_scores(sc), 4, 2).tolist() == [0, 1]


def test_bf16_recall_is_one_when_everything_is_selected():
    w = synth.config("c1", B=1, L=1024)  # n_t = 256 <= k = 512
    assert pipeline.bf16_score_recall(w, [(0, 0)]) == {(0, 0): 1.0}


def _f32_index_workload(score_rows, k):
    """A one-head f32 indexer workload whose scores are given directly:
    query q = e_0 with weight 1 and key s = (score_s, 0, ...), so that
    I(t, s) = max(0, score_s).  One query per row of ``score_rows``, each at
    a position that sees exactly len(row) entries (m = 4)."""
    n = max(len(r) for r in score_rows)
    T = len(score_rows)
    p = synth.Params(B=1, d=128, r=32, m=4, H_I=1, c_I=64, k=k, n_h=1, W=1, tau=1.0,
                     kv_fmt="f32", idx_fmt="f32", act_fmt="f32")
    # one key array serves every query: column t of key s holds query t's
    # score of entry s
    assert all(len(r) == n for r in score_rows)
    keys = np.zeros((1, n, 64), np.float32)
    keys[0, :, :T] = np.asarray(score_rows, np.float32).T   # key s, column t = score of query t
    q = np.zeros((1, T, 1, 64), np.float32)
    for t in range(T):
        q[0, t, 0, t] = 1.0
    return dict(params=p, T=T, q_pos0=np.array([4 * n - 1], np.int32), Ncap=n, k_idx=keys, q_idx=q,
                w_idx=np.ones((1, T, 1), np.float32))


def test_bf16_recall_hand_worked_half():
    # FP32 scores 1, 1 + 2^-10, 1 + 2^-9, 0.5: the FP32 top-2 is {1, 2}.  In
    # BF16 (8 significant bits) the first three all round to 1.0, the tie
    # goes to the lower indices and the BF16 top-2 is {0, 1}: recall 1/2.
    w = _f32_index_workload([[1.0, 1.0 + 2.0 ** -10, 1.0 + 2.0 ** -9, 0.5]], k=2)
    w["q_pos0"] = np.array([15], np.int32)   # n_t = 16 // 4 = 4
    assert pipeline.index_topk(w)[(0, 0)].tolist() == [1, 2]
    assert pipeline.index_topk(w, score_fmt="bf16")[(0, 0)].tolist() == [0, 1]
    assert pipeline.bf16_score_recall(w, [(0, 0)]) == {(0, 0): 0.5}


def test_bf16_recall_hand_worked_two_thirds():
    # scores 3, 2 + 2^-8, 2, 2 + 2^-7, 1 with k = 3: FP32 top-3 = {0, 1, 3};
    # BF16 keeps 8 significant bits, so near 2 the step is 2^-6: 2 + 2^-8
    # and 2 + 2^-7 round to 2 and tie with entry 2, which now wins on its
    # index over entry 3: BF16 top-3 = {0, 1, 2}, recall 2/3.
    w = _f32_index_workload([[3.0, 2.0 + 2.0 ** -8, 2.0, 2.0 + 2.0 ** -7, 1.0]], k=3)
    w["q_pos0"] = np.array([19], np.int32)   # n_t = 5
    assert pipeline.index_topk(w)[(0, 0)].tolist() == [0, 1, 3]
    assert pipeline.index_topk(w, score_fmt="bf16")[(0, 0)].tolist() == [0, 1, 2]
    assert pipeline.bf16_score_recall(w, [(0, 0)])[(0, 0)] == pytest.approx(2.0 / 3.0, abs=0)


def test_fp8_row_bytes_decode_hand_built():
    """A stored row built byte by byte from the format definitions: E4M3
    codes 0x38 (1.0), 0x40 (2.0), 0xB8 (-1.0), 0x01 (2^-9, the smallest
    subnormal), 0x7E (448, the largest finite), 0x00 (0), times the row
    scale 0.5; then two BF16 RoPE dims stored little-endian, 0x3F80 (1.0)
    as bytes 80 3F and 0xC040 (-3.0) as bytes 40 C0."""
    p = synth.Params(B=1, d=8, r=2, m=4, H_I=1, c_I=64, k=1, n_h=1, W=1, tau=1.0)
    row = np.array([[0x38, 0x40, 0xB8, 0x01, 0x7E, 0x00, 0x80, 0x3F, 0x40, 0xC0]], np.uint8)
    got = pipeline.decode_rows(row, np.array([0.5], np.float32), p)
    np.testing.assert_array_equal(got[0], [0.5, 1.0, -0.5, 2.0 ** -10, 224.0, 0.0, 1.0, -3.0])


# ---- decode-time state (oracle.state) --------------------------------------

def test_state_checkpoint_positions_brute_force():
    from oracle import state
    for a0 in range(0, 3000, 37):
        for T in (1, 5, 1024, 1500):
            ref = [P for P in range(a0 + 1, a0 + T + 1) if P % 1024 == 0]
            assert state.checkpoints(a0, a0 + T, 1024) == ref


def test_state_window_and_stream_extent():
    from oracle import state
    rng = np.random.default_rng(5)
    kv = rng.normal(size=(300, 8))
    ws = state.window_state(kv, 200, 128, 2, "fp8")
    assert sorted(ws) == list(range(72, 200))
    c, s, rb = ws[100]
    # a window row is the token's own vector in the entry layout
    np.testing.assert_allclose(csa.unpack_rows(c[None], np.array([s]), rb[None])[0], kv[100], rtol=0.07, atol=1e-2)
    assert sorted(state.window_state(kv, 50, 128, 2, "fp8")) == list(range(50))
    ss = state.stream_state(kv, kv, kv[:, :2], 256, 4)
    assert sorted(ss) == [252, 253, 254, 255]


def test_state_entries_after_are_the_complete_blocks():
    from oracle import state
    rng = np.random.default_rng(6)
    a, b, g = rng.normal(size=(23, 8)), rng.normal(size=(23, 8)), rng.normal(size=(23, 2))
    ent, pos = state.entries_after(a, b, g, 23, 4, 2, 1e4, 1e-6)
    assert pos.tolist() == [0, 4, 8, 12, 16]          # entry 5 would need token 23
    ref, _ = csa.compress(a[:20], b[:20], g[:20], 4, 2, 1e4, 1e-6)
    np.testing.assert_array_equal(ent, ref)
