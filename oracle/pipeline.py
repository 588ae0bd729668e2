"""The oracle run over a whole workload's stored bytes, one call at a time.

TEST INFRASTRUCTURE. Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU
baseline leg of ``bench.py`` may import anything under ``oracle/``.

Each function mirrors one of the library's five calls and reads the same
stored bytes (decoded with ``oracle.codecs``), but computes in float64 with
the plain formulas of ``oracle.csa``.  ``queries`` arguments restrict the work
to a sample of (sequence, query-offset) pairs for full-size workloads.
"""

from __future__ import annotations

import numpy as np

from . import codecs
from . import csa


def _f64_stream(x, fmt):
    if fmt == "f32":
        return np.asarray(x, dtype=np.float64)
    return codecs.bf16_decode(x)


def decode_rows(rows, scale, p):
    """Stored KV rows -> float64 [..., d]."""
    if p.kv_fmt == "f32":
        return np.asarray(rows, dtype=np.float64)
    n_nope = p.d - p.r
    codes = rows[..., :n_nope]
    rbits = np.ascontiguousarray(rows[..., n_nope:]).view(np.uint16)
    return csa.unpack_rows(codes, scale, rbits)


def compress(w, seqs=None):
    """csa_compress / hca_compress over the workload's entry ranges.

    Returns {b: (entries_f64 [n, d], pos [n], packed)} where packed is
    (codes, scale, rope_bits) in the fp8 format, or None in the f32 format.
    """
    p = w["params"]
    out = {}
    for b in (range(p.B) if seqs is None else seqs):
        eb, ee = int(w["e_begin"][b]), int(w["e_end"][b])
        if ee <= eb:
            out[b] = (np.zeros((0, p.d)), np.zeros(0, np.int64), None)
            continue
        a = _f64_stream(w["a"][b], p.act_fmt)
        bb = _f64_stream(w["b"][b], p.act_fmt)
        ent, pos = csa.compress(a, bb, w["gate"][b], p.m, p.r, p.theta, p.eps, None,
                                e_begin=eb, e_end=ee, tok_base=int(w["tok_base"][b]))
        packed = csa.pack_entries(ent, p.r) if p.kv_fmt == "fp8" else None
        out[b] = (ent, pos, packed)
    return out


def cache_rows(w, b, comp=None):
    """float64 cache rows [Ncap, d] of sequence b as the attention reads
    them: stored rows, with the entries the compressor produced (taken from
    ``comp``, the oracle's own compress output, after packing) in place."""
    p = w["params"]
    rows = decode_rows(w["kv"][b], w.get("kv_scale", [None] * p.B)[b] if p.kv_fmt == "fp8" else None, p)
    if comp is not None and b in comp:
        ent, pos, packed = comp[b]
        if len(pos):
            idx = pos // p.m
            if packed is None:
                rows[idx] = ent
            else:
                rows[idx] = csa.unpack_rows(*packed)
    return rows


def window_rows(w, b, t):
    """float64 window rows of query position t of sequence b (ring lookup)."""
    p = w["params"]
    pos = csa.window_positions(t, p.W)
    slots = pos % w["Wcap"]
    sc = w["win_scale"][b][slots] if p.kv_fmt == "fp8" else None
    return decode_rows(w["win"][b][slots], sc, p)


def index_query(w, b, tq):
    p = w["params"]
    if p.idx_fmt == "mxfp4":
        q = codecs.mxfp4_decode(w["q_idx"][b, tq], w["q_idx_sf"][b, tq], p.c_I)
    else:
        q = np.asarray(w["q_idx"][b, tq], dtype=np.float64)
    return q, np.asarray(w["w_idx"][b, tq], dtype=np.float64)


def index_keys(w, b, n):
    p = w["params"]
    if p.idx_fmt == "mxfp4":
        return codecs.mxfp4_decode(w["k_idx"][b, :n], w["k_idx_sf"][b, :n], p.c_I)
    return np.asarray(w["k_idx"][b, :n], dtype=np.float64)


def all_queries(w):
    p = w["params"]
    return [(b, tq) for b in range(p.B) for tq in range(w["T"])]


def index_topk(w, queries=None, return_scores=False, score_fmt="f32"):
    """csa_index_topk: {(b, tq): int32 [k]} (and the fp64 scores).
    score_fmt "bf16" selects on the scores rounded to BF16."""
    p = w["params"]
    queries = all_queries(w) if queries is None else queries
    res, scores = {}, {}
    keys_cache = {}
    for b, tq in queries:
        t = int(w["q_pos0"][b]) + tq
        n_t = csa.n_visible(t, p.m)
        if b not in keys_cache:
            keys_cache = {b: index_keys(w, b, int(w["Ncap"]))}
        k = keys_cache[b][:n_t]
        q, wt = index_query(w, b, tq)
        sc = csa.index_scores(q, wt, k)
        if score_fmt == "bf16":
            sc = csa.bf16_scores(sc)
        res[(b, tq)] = csa.topk_select(sc, n_t, p.k)
        if return_scores:
            scores[(b, tq)] = sc
    return (res, scores) if return_scores else res


def bf16_score_recall(w, queries):
    """Recall of the FP32-score top-k by the BF16-score top-k, per query:
    |selected with BF16 scores  and  selected with FP32 scores| / min(k, n_t)."""
    p = w["params"]
    f32 = index_topk(w, queries)
    b16 = index_topk(w, queries, score_fmt="bf16")
    out = {}
    for q in queries:
        a, b = f32[q], b16[q]
        n = int((a >= 0).sum())
        out[q] = len(set(a[a >= 0].tolist()) & set(b[b >= 0].tolist())) / max(n, 1)
    return out


def _query(w, b, tq):
    p = w["params"]
    if p.act_fmt == "f32":
        return np.asarray(w["q"][b, tq], dtype=np.float64)
    return codecs.bf16_decode(w["q"][b, tq])


def sparse_attn(w, idx, comp=None, queries=None):
    """csa_sparse_attn: {(b, tq): float64 [n_h, d]} given top-k lists ``idx``
    ({(b, tq): int32 [k]} or an array [B, T, k])."""
    p = w["params"]
    queries = all_queries(w) if queries is None else queries
    out = {}
    rows_cache = {}
    for b, tq in queries:
        t = int(w["q_pos0"][b]) + tq
        if b not in rows_cache:
            rows_cache = {b: cache_rows(w, b, comp)}
        sel = idx[(b, tq)] if isinstance(idx, dict) else idx[b, tq]
        J = csa.csa_rows(rows_cache[b], sel, window_rows(w, b, t))
        out[(b, tq)] = csa.attend(_query(w, b, tq), J, w["sink"], p.tau, t, p.theta, p.r)
    return out


def dense_attn(w, comp=None, queries=None):
    """hca_dense_attn: {(b, tq): float64 [n_h, d]}."""
    p = w["params"]
    queries = all_queries(w) if queries is None else queries
    out = {}
    rows_cache = {}
    for b, tq in queries:
        t = int(w["q_pos0"][b]) + tq
        if b not in rows_cache:
            rows_cache = {b: cache_rows(w, b, comp)}
        J = csa.hca_rows(rows_cache[b], csa.n_visible(t, p.m), window_rows(w, b, t))
        out[(b, tq)] = csa.attend(_query(w, b, tq), J, w["sink"], p.tau, t, p.theta, p.r)
    return out


def csa_step(w, queries=None):
    """compress -> index_topk -> sparse_attn for a CSA workload."""
    comp = compress(w) if w["S"] else None
    idx = index_topk(w, queries)
    out = sparse_attn(w, idx, comp, queries)
    return comp, idx, out


def hca_step(w, queries=None):
    """compress -> dense_attn for an HCA workload."""
    comp = compress(w) if w["S"] else None
    return comp, dense_attn(w, comp, queries)
