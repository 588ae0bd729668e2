"""fp64 CPU oracle of DeepSeek-V4's hybrid compressed attention (CSA / HCA).

TEST INFRASTRUCTURE. Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU
baseline leg of ``bench.py`` may import anything under ``oracle/``.  It shares
no code with the CUDA library and never imports it.

Everything here is plain numpy in float64, one sequence and one query at a
time, in the order the pages state the method.  A matmul is used as a library
primitive where the method is a plain contraction; there is no blocking,
fusion or reordering beyond the formulas.

Sources (cited by page title and section):

* [PACMAN] "DeepSeek-V4 技术报告分享" (10100.com talk notes), §3.1 CSA,
  §3.2 HCA, §5 Muon 与训练稳定性, §6 MoE.
* [Qiaomu] "DeepSeek-V4论文解析：百万上下文、水平接近闭源模型是如何做到的？"
  (乔木博客), sections 混合注意力机制, FP4量化感知训练, 训练配置.
* [WeChat] 未来科技 article on DeepSeek-V4 (cdjax.com), §1.1 混合注意力.
* [fengweifeng] "DeepSeek-V4: Towards Highly Efficient Million-Token Context
  Intelligence" (fengweifeng.com notes), second part, 2. 技术实现与架构细节.
* [kwkr] kwkr.cn DeepSeek-V4 notes, §3.1 CSA 的工作方式, §3.3 层间排布与滑窗补充,
  §3.4 两个降开销的设计, §4.4 FP4 QAT 与 KV Cache 层级.

Readings where the pages are silent or garbled (each is listed with its
reason in the design notes):

1. Overlap: entry i merges stream a over block i and stream b over block i-1
   (entry 0 has only stream a).  [kwkr §3.1: two KV sequences, adjacent
   blocks share part of their indices.]
2. One gate logit per token per stream.
3. One softmax over the union of both streams' logits of an entry (so the
   merge weights are convex).
4. HCA's compressor is the same operator with m = 128.
5. RMSNorm eps and weight are parameters (eps 1e-6, weight 1 in the
   workloads).
6. RoPE rotates interleaved pairs (d-r+2j, d-r+2j+1) of the last r dims by
   pos * theta^(-2j/r); an entry sits at position m*i (its block start).
7. The output's inverse RoPE uses angle -t, t the query position.
8. The softmax scale tau is a parameter.
9. The window is the W raw tokens max(0, t-W+1) .. t (t included), with no
   de-duplication against compressed entries.
10. Entry i is visible to query t iff m*(i+1) - 1 <= t, i.e. i < n_t =
    floor((t+1)/m).
11. One index key per entry, shared by all index heads; one weight per
    (query, head); ReLU before the weighted head sum; no score scale.
12. Top-k ties go to the lower entry index; k >= n_t selects all n_t;
    output ascending, padded with -1.
15. The sink adds exp(sigma_h) to the softmax denominator and has no value.
"""

from __future__ import annotations

import numpy as np

from . import codecs

# ----------------------------------------------------------------------------
# Compressor  [kwkr §3.1; Qiaomu 混合注意力机制; PACMAN §3.1, §3.2]
# ----------------------------------------------------------------------------


def gate_weights(ga: np.ndarray, gb: np.ndarray) -> tuple[np.ndarray, np.ndarray]:
    """Softmax over the union of stream-a logits ``ga`` (block i) and stream-b
    logits ``gb`` (block i-1, possibly empty).  Max-subtracted for range.

    Returns (wa, wb) with wa, wb >= 0 and sum(wa) + sum(wb) = 1.
    """
    ga = np.asarray(ga, dtype=np.float64)
    gb = np.asarray(gb, dtype=np.float64)
    allg = np.concatenate([ga, gb])
    mx = np.max(allg)
    ea = np.exp(ga - mx)
    eb = np.exp(gb - mx)
    z = ea.sum() + eb.sum()
    return ea / z, eb / z


def merge_entry(a_blk: np.ndarray, b_prev: np.ndarray, ga: np.ndarray, gb: np.ndarray) -> np.ndarray:
    """Pre-norm compressed vector x = sum_u wa_u a_u + sum_u wb_u b_u.

    a_blk: [m, d] stream a over block i; b_prev: [m', d] stream b over block
    i-1 (m' = 0 for i = 0).
    """
    wa, wb = gate_weights(ga, gb)
    x = wa @ np.asarray(a_blk, dtype=np.float64)
    if len(wb):
        x = x + wb @ np.asarray(b_prev, dtype=np.float64)
    return x


def rmsnorm(x: np.ndarray, gamma: np.ndarray | None, eps: float) -> np.ndarray:
    """y = gamma * x / sqrt(mean(x^2) + eps) along the last axis.
    [PACMAN §5 / Qiaomu 混合注意力机制: KV entries and queries are RMS-normalised.]"""
    x = np.asarray(x, dtype=np.float64)
    y = x / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps)
    if gamma is not None:
        y = y * np.asarray(gamma, dtype=np.float64)
    return y


def rope(v: np.ndarray, pos, theta: float, r: int) -> np.ndarray:
    """Rotate the last r dims of v (interleaved pairs) by angle pos*theta^(-2j/r).

    [Qiaomu 混合注意力机制: RoPE on part of the dims; WeChat §1.1: the last
    64 dims.]  ``pos`` may be negative (inverse RoPE) and may be an array
    broadcasting against v's leading axes.
    """
    v = np.array(v, dtype=np.float64, copy=True)
    d = v.shape[-1]
    j = np.arange(r // 2, dtype=np.float64)
    freq = np.power(float(theta), -2.0 * j / r)  # [r/2]
    ang = np.asarray(pos, dtype=np.float64)[..., None] * freq  # [..., r/2]
    c, s = np.cos(ang), np.sin(ang)
    x = v[..., d - r + 0::2].copy()
    y = v[..., d - r + 1::2].copy()
    v[..., d - r + 0::2] = x * c - y * s
    v[..., d - r + 1::2] = x * s + y * c
    return v


def compress(a, b, gate, m: int, r: int, theta: float, eps: float, gamma=None,
             e_begin: int = 0, e_end: int | None = None, tok_base: int = 0):
    """Compressed entries e in [e_begin, e_end) of one sequence.

    a, b: [S, d] float64 streams for absolute token positions tok_base ..
    tok_base+S-1; gate: [S, 2] logits (column 0 stream a, column 1 stream b).
    Entry e uses a over tokens m*e .. m*e+m-1 and b over m*(e-1) .. m*e-1.
    Returns (entries [n, d] float64, pos [n] int64 = m*e).
    """
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    gate = np.asarray(gate, dtype=np.float64)
    S = a.shape[0]
    if e_end is None:
        e_end = (tok_base + S) // m
    out, pos = [], []
    for e in range(e_begin, e_end):
        ia0 = m * e - tok_base
        ia1 = ia0 + m
        ib0 = max(m * (e - 1), 0) - tok_base
        ib1 = m * e - tok_base
        assert 0 <= ia0 and ia1 <= S and 0 <= ib0 <= ib1, "token range not in the buffer"
        x = merge_entry(a[ia0:ia1], b[ib0:ib1], gate[ia0:ia1, 0], gate[ib0:ib1, 1])
        y = rmsnorm(x, gamma, eps)
        y = rope(y, m * e, theta, r)
        out.append(y)
        pos.append(m * e)
    d = a.shape[1]
    return np.array(out, dtype=np.float64).reshape(-1, d), np.array(pos, dtype=np.int64)


# ----------------------------------------------------------------------------
# Mixed KV-entry layout  [WeChat §1.1: RoPE dims BF16, the others FP8]
# ----------------------------------------------------------------------------


def pack_entry(y: np.ndarray, r: int):
    """One entry [d] -> (e4m3 codes [d-r], fp32 scale, bf16 bits [r]).

    scale = fp32(amax / 448) over the d-r non-RoPE dims (1 when amax = 0);
    code = E4M3 round-to-nearest-even, saturating, of x / scale.
    """
    y = np.asarray(y, dtype=np.float64)
    d = y.shape[-1]
    nope = y[: d - r]
    amax = float(np.max(np.abs(nope))) if d > r else 0.0
    scale = np.float32(amax / codecs.E4M3_MAX) if amax > 0 else np.float32(1.0)
    codes = codecs.e4m3_encode(nope / np.float64(scale))
    rbits = codecs.bf16_encode(y[d - r:])
    return codes, scale, rbits


def pack_entries(ys: np.ndarray, r: int):
    codes, scales, rbits = [], [], []
    for y in ys:
        c, s, rb = pack_entry(y, r)
        codes.append(c)
        scales.append(s)
        rbits.append(rb)
    n = len(ys)
    d = ys.shape[-1] if n else r
    return (np.array(codes, dtype=np.uint8).reshape(n, d - r),
            np.array(scales, dtype=np.float32).reshape(n),
            np.array(rbits, dtype=np.uint16).reshape(n, r))


def unpack_rows(codes: np.ndarray, scale: np.ndarray, rbits: np.ndarray) -> np.ndarray:
    """Stored rows -> float64 [n, d] = (code * scale) || bf16 value."""
    nope = codecs.e4m3_decode(codes) * np.asarray(scale, dtype=np.float64)[..., None]
    return np.concatenate([nope, codecs.bf16_decode(rbits)], axis=-1)


# ----------------------------------------------------------------------------
# Index keys and queries in FP4  [kwkr §3.1, §3.4, §4.4; Qiaomu FP4量化感知训练]
# ----------------------------------------------------------------------------


def index_key_compress(a, b, gate, m: int, rope_dims: int, theta: float, eps: float, gamma=None,
                       e_begin: int = 0, e_end: int | None = None, tok_base: int = 0):
    """Index keys of entries e in [e_begin, e_end): the same gated
    compressor as the KV entries (kwkr §3.1: the indexer scores the
    compressed entries; §3.4: its QK runs in FP4), run over the c_I-dim
    indexer streams with RoPE on their last ``rope_dims`` dims, then
    quantised to MXFP4 by the OCP MX conversion.

    Returns (packed [n, c_I/2], scales [n, c_I/32], pos [n])."""
    keys, pos = compress(a, b, gate, m, rope_dims, theta, eps, gamma, e_begin=e_begin, e_end=e_end,
                         tok_base=tok_base)
    packed, scales = codecs.mxfp4_encode(keys)
    return packed, scales, pos


def index_query_quantize(q):
    """Index queries [..., c_I] -> MXFP4 (packed, scales) by the OCP MX
    conversion (kwkr §3.4: the indexer QK runs directly in FP4)."""
    return codecs.mxfp4_encode(q)


# ----------------------------------------------------------------------------
# Lightning Indexer  [Qiaomu 混合注意力机制; kwkr §3.4; WeChat §1.1]
# ----------------------------------------------------------------------------


def n_visible(t: int, m: int) -> int:
    """Number of entries a query at position t may see: floor((t+1)/m)."""
    return (t + 1) // m


def index_scores(q: np.ndarray, w: np.ndarray, k: np.ndarray) -> np.ndarray:
    """I_s = sum_h w_h * max(0, q_h . k_s) for every key row s.

    q: [H, c] index queries; w: [H] head weights; k: [n, c] index keys.
    """
    q = np.asarray(q, dtype=np.float64)
    w = np.asarray(w, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    dots = k @ q.T  # [n, H]
    return np.maximum(dots, 0.0) @ w


def bf16_scores(scores: np.ndarray) -> np.ndarray:
    """Index scores rounded to BF16 (round to nearest even) and widened
    back: the selector's input in the BF16-score variant (Qiaomu blog
    FP4量化感知训练 and kwkr.cn notes 4.4: the index scores are quantised
    from FP32 to BF16 before the top-k selector).  The selection rule is
    unchanged, so entries whose scores collide after rounding are ranked by
    index."""
    return codecs.bf16_decode(codecs.bf16_encode(np.asarray(scores, dtype=np.float64)))


def topk_select(scores: np.ndarray, n_t: int, k: int) -> np.ndarray:
    """The min(k, n_t) entries s < n_t ranked by (score descending, s
    ascending), returned in ascending order and padded with -1 to length k."""
    sc = np.asarray(scores, dtype=np.float64)[:n_t]
    s = np.arange(n_t)
    order = np.lexsort((s, -sc))  # last key is the primary key
    chosen = np.sort(order[: min(k, n_t)])
    out = np.full(k, -1, dtype=np.int32)
    out[: len(chosen)] = chosen
    return out


# ----------------------------------------------------------------------------
# Core attention with window, sink and inverse RoPE
# [WeChat §1.1; kwkr §3.3; fengweifeng 2.; Qiaomu 混合注意力机制]
# ----------------------------------------------------------------------------


def window_positions(t: int, W: int) -> np.ndarray:
    """Raw-token positions of the sliding window of query t (t included)."""
    return np.arange(max(0, t - W + 1), t + 1, dtype=np.int64)


def attend(q: np.ndarray, rows: np.ndarray, sigma: np.ndarray, tau: float,
           t: int, theta: float, r: int) -> np.ndarray:
    """MQA over shared key=value rows with a sink logit, then inverse RoPE.

    q: [n_h, d]; rows: [J, d] (each row is both key and value); sigma: [n_h].
    z_hj = tau * q_h . v_j;  M_h = max(sigma_h, max_j z_hj);
    p_hj = exp(z_hj - M_h) / (exp(sigma_h - M_h) + sum_j exp(z_hj - M_h));
    o_h = sum_j p_hj v_j, then the last r dims rotated by angle -t.
    """
    q = np.asarray(q, dtype=np.float64)
    rows = np.asarray(rows, dtype=np.float64).reshape(-1, q.shape[-1])
    sigma = np.asarray(sigma, dtype=np.float64)
    z = tau * (q @ rows.T)  # [n_h, J]
    zmax = z.max(axis=1) if rows.shape[0] else np.full(q.shape[0], -np.inf)
    M = np.maximum(sigma, zmax)
    e = np.exp(z - M[:, None])
    den = np.exp(sigma - M) + e.sum(axis=1)
    p = e / den[:, None]
    o = p @ rows
    return rope(o, -t, theta, r)


def attention_weights(q, rows, sigma, tau):
    """The p_hj of ``attend`` and the sink weight exp(sigma_h-M)/den (for
    the invariant checks)."""
    q = np.asarray(q, dtype=np.float64)
    rows = np.asarray(rows, dtype=np.float64)
    sigma = np.asarray(sigma, dtype=np.float64)
    z = tau * (q @ rows.T)
    M = np.maximum(sigma, z.max(axis=1))
    e = np.exp(z - M[:, None])
    es = np.exp(sigma - M)
    den = es + e.sum(axis=1)
    return e / den[:, None], es / den


def csa_rows(cache_rows: np.ndarray, sel: np.ndarray, win_rows: np.ndarray) -> np.ndarray:
    """Candidate rows of a CSA query: the selected entries (ignoring -1
    padding), then the window tokens."""
    sel = np.asarray(sel)
    sel = sel[sel >= 0]
    return np.concatenate([cache_rows[sel], win_rows], axis=0)


def hca_rows(cache_rows: np.ndarray, n_t: int, win_rows: np.ndarray) -> np.ndarray:
    """Candidate rows of an HCA query: every visible entry, then the window."""
    return np.concatenate([cache_rows[:n_t], win_rows], axis=0)


# ----------------------------------------------------------------------------
# A separate textbook routine for the oracle's self-check
# ----------------------------------------------------------------------------


def dense_softmax_with_null_value(q, values, sigma, tau):
    """Plain softmax attention over [sink] + values, where the sink is an
    extra logit sigma_h whose value vector is zero.  Uses scipy's softmax so
    it shares no arithmetic with ``attend``.  No RoPE."""
    from scipy.special import softmax

    q = np.asarray(q, dtype=np.float64)
    values = np.asarray(values, dtype=np.float64)
    n_h, d = q.shape
    logits = np.concatenate([np.asarray(sigma, dtype=np.float64)[:, None], tau * (q @ values.T)], axis=1)
    vals = np.concatenate([np.zeros((1, d)), values], axis=0)
    return softmax(logits, axis=1) @ vals
