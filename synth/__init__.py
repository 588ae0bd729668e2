"""Seeded synthetic workloads for the CSA/HCA hot path.

This module serves both the oracle side (tests, CPU baseline) and the CUDA
side (tests, bench).  It holds none of the method's arithmetic: it never
compresses, normalises, rotates, scores, selects or attends.  Every array is
drawn directly in its storage format, and every float-to-code conversion is
a library cast (``ml_dtypes``), never one of this repository's codecs.

Shapes follow DeepSeek-V4's published configuration (Qiaomu blog,
训练配置: V4-Flash 64 query heads, V4-Pro 128, head dim 512, indexer 64 heads
x 128, top-k 512 / 1024, window 128; compression 4 for CSA and 128 for HCA).
No public dataset is involved; values are N(0,1)-like throughout.

Storage layouts (all little-endian, C-contiguous):

* stream a / b      ``[B, S, d]``  f32, or bf16 bits (uint16)
* gate logits       ``[B, S, 2]``  f32 (column 0 stream a, column 1 stream b)
* KV rows (fp8 fmt) ``[B, cap, d + r]`` uint8: d-r E4M3 codes, then r bf16
  values (2r bytes); per-row f32 scale ``[B, cap]``
* KV rows (f32 fmt) ``[B, cap, d]`` f32, no scale
* index keys        ``[B, cap, c/2]`` uint8 MXFP4 (low nibble = lower
  element) + ``[B, cap, c/32]`` uint8 UE8M0 scales, or f32 ``[B, cap, c]``
* index queries     ``[B, T, H, c/2]`` + ``[B, T, H, c/32]``, or f32
* head weights      ``[B, T, H]`` f32
* queries           ``[B, T, n_h, d]`` bf16 bits or f32
* sink logits       ``[n_h]`` f32
* window ring       same row format as the cache, ``[B, Wcap, ...]``;
  the token at position p lives in slot p mod Wcap.

Draw order for a workload (one ``numpy.random.default_rng(seed)``): streams
a, b, gate; cache rows (codes, scales, RoPE dims); window rows; index keys;
index queries; head weights; queries; sinks; planted cluster.
"""

from __future__ import annotations

import dataclasses
import math

import ml_dtypes
import numpy as np
from scipy.special import ndtri

FMT_F32 = "f32"
FMT_FP8 = "fp8"     # E4M3 non-RoPE dims + BF16 RoPE dims + per-row f32 scale
FMT_MXFP4 = "mxfp4"
FMT_BF16 = "bf16"


@dataclasses.dataclass
class Params:
    B: int
    d: int
    r: int
    m: int
    H_I: int
    c_I: int
    k: int
    n_h: int
    W: int
    tau: float
    theta: float = 1e4
    eps: float = 1e-6
    kv_fmt: str = FMT_FP8
    idx_fmt: str = FMT_MXFP4
    act_fmt: str = FMT_BF16
    score_fmt: str = "f32"   # index-score precision the selector ranks ("f32" or "bf16")

    @property
    def row_bytes(self) -> int:
        return self.d + self.r if self.kv_fmt == FMT_FP8 else 4 * self.d


# ---------------------------------------------------------------------------
# samplers (inverse-CDF lookup tables, built once from library casts)
# ---------------------------------------------------------------------------

_Q = ndtri((np.arange(65536, dtype=np.float64) + 0.5) / 65536.0)  # N(0,1) quantiles
_LUT_BF16 = _Q.astype(np.float32).astype(ml_dtypes.bfloat16).view(np.uint16)
_FP8_SPREAD = 112.0  # codes ~ N(0, 112^2): amax of a 448-vector lands near 448
_LUT_E4M3 = np.clip(_Q * _FP8_SPREAD, -448.0, 448.0).astype(np.float32).astype(
    ml_dtypes.float8_e4m3fn).view(np.uint8)


def _u16(rng, shape):
    """Uniform 16-bit words from the generator's raw 64-bit output."""
    n = int(np.prod(shape))
    raw = rng.bit_generator.random_raw((n + 3) // 4)
    return raw.view(np.uint16)[:n].reshape(shape)


def normal_bf16(rng, shape) -> np.ndarray:
    """N(0,1) samples already in bf16 bit patterns."""
    return _LUT_BF16[_u16(rng, shape)]


def normal_e4m3(rng, shape) -> np.ndarray:
    """E4M3 codes of N(0, 112^2) samples."""
    return _LUT_E4M3[_u16(rng, shape)]


_LUT_F32 = _Q.astype(np.float32)


def normal_f32(rng, shape) -> np.ndarray:
    """N(0,1) samples, 16-bit quantile resolution (ample for synthetic data)."""
    return _LUT_F32[_u16(rng, shape)]


# E2M1 code of every fp16 bit pattern (library cast, built once); NaN/inf
# patterns never occur in the sampler's inputs.
with np.errstate(invalid="ignore", over="ignore"):
    _F16_ALL = np.arange(65536, dtype=np.uint32).astype(np.uint16).view(np.float16).astype(np.float32)
    _LUT_E2M1_F16 = (np.nan_to_num(np.clip(_F16_ALL, -6.0, 6.0))
                     .astype(ml_dtypes.float4_e2m1fn).view(np.uint8) & 0xF).astype(np.uint8)
_E2M1_VAL = np.array([0, .5, 1, 1.5, 2, 3, 4, 6, -0.0, -.5, -1, -1.5, -2, -3, -4, -6], np.float32)


def mxfp4_from_float(x: np.ndarray):
    """Library-cast float32 [..., c] to MXFP4 (packed nibbles, UE8M0 scales).

    Block exponent E = max(-2, ceil(log2(amax/6))) so no element saturates and
    every scale is at least 2^-2 (keeps the score lattice at 2^-10); elements
    are ml_dtypes' E2M1 cast of fp16(x / 2^E) (a sampler, not a quantiser
    contract: the hot path consumes the codes as given).
    """
    c = x.shape[-1]
    blk = x.reshape(x.shape[:-1] + (c // 32, 32)).astype(np.float32)
    amax = np.max(np.abs(blk), axis=-1)
    with np.errstate(divide="ignore"):
        E = np.ceil(np.log2(np.maximum(amax, 1e-30) / 6.0))
    E = np.maximum(E, -2.0).astype(np.int32)
    y = (blk / np.exp2(E.astype(np.float32))[..., None]).astype(np.float16)
    nib = _LUT_E2M1_F16[y.view(np.uint16)]
    scales = (E + 127).astype(np.uint8)
    nib = nib.reshape(x.shape[:-1] + (c,))
    packed = (nib[..., 0::2] | (nib[..., 1::2] << 4)).astype(np.uint8)
    return packed, scales, (nib, E)


def fp8_rows(rng, shape_rows, d, r) -> tuple[np.ndarray, np.ndarray]:
    """KV rows in the mixed layout drawn directly in storage format.

    Non-RoPE codes ~ E4M3(N(0, 112^2)); per-row scale ~ U(0.9, 1.1)/112, so
    the decoded values are ~N(0,1), like an RMS-normalised vector; RoPE dims
    bf16 N(0,1).
    """
    n_nope = d - r
    rows = np.empty(shape_rows + (d + r,), dtype=np.uint8)
    rows[..., :n_nope] = normal_e4m3(rng, shape_rows + (n_nope,))
    scale = (rng.uniform(0.9, 1.1, size=shape_rows) / _FP8_SPREAD).astype(np.float32)
    rb = normal_bf16(rng, shape_rows + (r,))
    rows[..., n_nope:] = rb.view(np.uint8).reshape(shape_rows + (2 * r,))
    return rows, scale


# ---------------------------------------------------------------------------
# workload builder
# ---------------------------------------------------------------------------


def make_workload(seed: int, p: Params, *, L, T=1, q_pos0=None, compress="last",
                  sink="normal", w_denom=16, cluster=None, w_levels=None,
                  exact_bound=True):
    """Build one seeded workload.

    L: context length per sequence (int or list of B ints).  Queries sit at
       positions q_pos0[b] .. q_pos0[b]+T-1 (default: the last T tokens).
    compress: "all"  -> streams for every token, the cache is produced by
                        the compressor (entries 0 .. L//m - 1);
              "last" -> streams for the last 2m tokens only, entries
                        0 .. L//m - 2 are drawn in storage format, the last
                        entry is produced by the compressor;
              "none" -> every entry drawn, no streams.
    cluster: (n_seqs, length, amp) planted cluster of index keys aligned
             with the query of each planted sequence (last query).
    """
    B = p.B
    Ls = np.array([L] * B if np.isscalar(L) else list(L), dtype=np.int64)
    if q_pos0 is None:
        q_pos0 = Ls - T
    q_pos0 = np.array([q_pos0] * B if np.isscalar(q_pos0) else list(q_pos0), dtype=np.int64)
    assert np.all(q_pos0 + T <= Ls) and np.all(q_pos0 >= 0)
    rng = np.random.default_rng(seed)
    m, d, r = p.m, p.d, p.r
    Ncap = int(max(Ls.max() // m, 1))
    w = dict(params=p, L=Ls, T=T, q_pos0=q_pos0.astype(np.int32), Ncap=Ncap, seed=seed,
             compress=compress)

    # --- streams ------------------------------------------------------------
    if compress == "all":
        S = int(Ls.max())
        tok_base = np.zeros(B, dtype=np.int64)
        e_begin = np.zeros(B, dtype=np.int64)
        e_end = Ls // m
    elif compress == "last":
        S = 2 * m
        tok_base = np.maximum((Ls // m) * m - 2 * m, 0)
        e_end = Ls // m
        e_begin = np.maximum(e_end - 1, 0)
    else:
        S = 0
        tok_base = e_begin = e_end = np.zeros(B, dtype=np.int64)
    if S:
        if p.act_fmt == FMT_F32:
            w["a"] = normal_f32(rng, (B, S, d))
            w["b"] = normal_f32(rng, (B, S, d))
        else:
            w["a"] = normal_bf16(rng, (B, S, d))
            w["b"] = normal_bf16(rng, (B, S, d))
        w["gate"] = normal_f32(rng, (B, S, 2))
    w["S"] = S
    w["tok_base"] = tok_base.astype(np.int32)
    w["e_begin"] = e_begin.astype(np.int32)
    w["e_end"] = e_end.astype(np.int32)

    # --- cache rows -----------------------------------------------------------
    if p.kv_fmt == FMT_FP8:
        kv, kv_scale = fp8_rows(rng, (B, Ncap), d, r)
        w["kv_scale"] = kv_scale
    else:
        kv = normal_f32(rng, (B, Ncap, d))
    if compress == "all":
        kv[...] = 0  # filled by the compressor
        if p.kv_fmt == FMT_FP8:
            w["kv_scale"][...] = 0
    w["kv"] = kv

    # --- window ring ------------------------------------------------------------
    lo = np.maximum(q_pos0 - p.W + 1, 0)
    hi = q_pos0 + T - 1
    Wcap = int(max(p.W, (hi - lo + 1).max()))
    w["Wcap"] = Wcap
    if p.kv_fmt == FMT_FP8:
        win, win_scale = fp8_rows(rng, (B, Wcap), d, r)
        w["win_scale"] = win_scale
    else:
        win = normal_f32(rng, (B, Wcap, d))
    w["win"] = win

    # --- indexer ---------------------------------------------------------------
    H, c = p.H_I, p.c_I
    kf = normal_f32(rng, (B, Ncap, c))
    qf = normal_f32(rng, (B, T, H, c))
    if w_levels is None:
        w_levels = w_denom
    wj = rng.integers(1, w_levels + 1, size=(B, T, H))
    w["w_idx"] = (wj / float(w_denom)).astype(np.float32)
    if cluster is not None:
        n_seq, clen, amp = cluster
        w["cluster"] = []
        for bb in range(n_seq):
            off = int(rng.integers(0, max(int(Ls[bb] // m) - clen, 1)))
            # aligned with the weighted sum of the sequence's last index query
            u = np.sign((w["w_idx"][bb, T - 1][:, None] * qf[bb, T - 1]).sum(axis=0))
            kf[bb, off:off + clen] += amp * u[None, :]
            w["cluster"].append((bb, off, clen))
    if p.idx_fmt == FMT_MXFP4:
        w["k_idx"], w["k_idx_sf"], kcodes = mxfp4_from_float(kf)
        w["q_idx"], w["q_idx_sf"], qcodes = mxfp4_from_float(qf)
        if exact_bound:
            check_score_exactness(kcodes, qcodes, w["w_idx"])
    else:
        w["k_idx"], w["q_idx"] = kf, qf

    # --- attention queries and sinks ----------------------------------------------
    if p.act_fmt == FMT_F32:
        w["q"] = (normal_f32(rng, (B, T, p.n_h, d)) / np.float32(math.sqrt(d))).astype(np.float32)
    else:
        w["q"] = normal_bf16(rng, (B, T, p.n_h, d))
    if sink == "normal":
        w["sink"] = normal_f32(rng, (p.n_h,))
    else:
        w["sink"] = np.zeros(p.n_h, dtype=np.float32)
    return w


SCORE_LIMIT = 2.0 ** 14  # lattice 2^-10 x 2^24 significand


def _abs_vals(nib_E):
    nib, E = nib_E
    c = nib.shape[-1]
    a = np.abs(_E2M1_VAL[nib]).reshape(nib.shape[:-1] + (c // 32, 32))
    return (a * np.exp2(E.astype(np.float32))[..., None]).reshape(nib.shape)


def check_score_exactness(k_codes, q_codes, wts, chunk=1024):
    """Assert every index score of the workload is exactly representable in
    fp32 whatever the summation order: with element lattice 2^-3 (scales >=
    2^-2) and dyadic weights j/16, every partial sum is a multiple of 2^-10,
    so a bound of 2^14 on sum_h w_h sum_c |q_hc k_sc| keeps it within fp32's
    24-bit significand.  Raises if a workload breaks the bound."""
    knib, kE = k_codes
    qnib, qE = q_codes
    B, T = qnib.shape[:2]
    for b in range(B):
        kabs = _abs_vals((knib[b], kE[b]))  # [N, c] float32 (exact)
        if kabs.shape[0] == 0:
            continue
        for t0 in range(0, T, chunk):
            qabs = _abs_vals((qnib[b, t0:t0 + chunk], qE[b, t0:t0 + chunk]))  # [t, H, c]
            u = (wts[b, t0:t0 + chunk][:, :, None] * qabs).sum(axis=1)  # [t, c]
            mx = float((kabs @ u.T).max())
            # float32 products/sums here bound the exact value to a relative
            # 1e-6; keep a margin
            if mx >= SCORE_LIMIT * (1 - 1e-4):
                raise ValueError(f"index-score exactness bound broken at b={b}, t0={t0}: {mx}")


# ---------------------------------------------------------------------------
# the five workloads (configurations of the method; seeds are choices)
# ---------------------------------------------------------------------------


def config(name: str, **over):
    """Named workloads.  ``over`` shrinks B/L for parity tests."""
    if name == "c0":
        p = Params(B=over.pop("B", 1), d=128, r=32, m=4, H_I=4, c_I=64, k=64, n_h=8, W=128,
                   tau=1.0, kv_fmt=FMT_F32, idx_fmt=over.pop("idx_fmt", FMT_F32), act_fmt=FMT_F32)
        kw = dict(L=2048, compress="all", sink="zero", w_denom=8)
        kw.update(over)
        return make_workload(kw.pop("seed", 0), p, **kw)
    if name == "c1":
        p = Params(B=over.pop("B", 32), d=512, r=64, m=4, H_I=64, c_I=128, k=512, n_h=64, W=128,
                   tau=1.0 / math.sqrt(512))
        kw = dict(L=131072, compress="last")
        kw.update(over)
        return make_workload(kw.pop("seed", 1), p, **kw)
    if name == "c2":
        p = Params(B=over.pop("B", 4), d=512, r=64, m=4, H_I=64, c_I=128, k=1024, n_h=128, W=128,
                   tau=1.0 / math.sqrt(512))
        kw = dict(L=1048576, compress="last", cluster=(1, 1024, 3.0))
        kw.update(over)
        return make_workload(kw.pop("seed", 2), p, **kw)
    if name == "c3":
        p = Params(B=over.pop("B", 16), d=512, r=64, m=128, H_I=64, c_I=128, k=0, n_h=128, W=128,
                   tau=1.0 / math.sqrt(512), idx_fmt=FMT_MXFP4)
        kw = dict(L=1048576, compress="last")
        kw.update(over)
        return make_workload(kw.pop("seed", 3), p, **kw)
    if name == "c4":
        p = Params(B=over.pop("B", 2), d=512, r=64, m=4, H_I=64, c_I=128, k=512, n_h=64, W=128,
                   tau=1.0 / math.sqrt(512))
        L = over.pop("L", 32768)
        kw = dict(L=L, T=over.pop("T", L), q_pos0=0, compress="all")
        kw.update(over)
        return make_workload(kw.pop("seed", 4), p, **kw)
    raise KeyError(name)


# ---------------------------------------------------------------------------
# workload variants (still draws and slices only)
# ---------------------------------------------------------------------------


def with_heads(w, n_h: int):
    """The workload with only its first ``n_h`` query heads (queries and
    sinks sliced; nothing else changes)."""
    p = w["params"]
    assert n_h <= p.n_h
    w = dict(w)
    w["params"] = dataclasses.replace(p, n_h=n_h)
    w["q"] = np.ascontiguousarray(w["q"][:, :, :n_h])
    w["sink"] = np.ascontiguousarray(w["sink"][:n_h])
    return w


def with_score_fmt(w, fmt: str):
    """The workload with index scores ranked in ``fmt`` ("f32" or "bf16")."""
    w = dict(w)
    w["params"] = dataclasses.replace(w["params"], score_fmt=fmt)
    return w


def with_index_heads(w, n: int):
    """The workload with only its first ``n`` index heads (index queries,
    their scales and head weights sliced)."""
    p = w["params"]
    assert n <= p.H_I
    w = dict(w)
    w["params"] = dataclasses.replace(p, H_I=n)
    for k in ("q_idx", "q_idx_sf", "w_idx"):
        if k in w and w[k] is not None:
            w[k] = np.ascontiguousarray(w[k][:, :, :n])
    return w


def _bf16_of(x):
    return np.asarray(x, np.float32).astype(ml_dtypes.bfloat16).view(np.uint16)


def with_wide_rows(w, seed: int, *, scale_log2=(-16.0, 4.0), rope_ratio_log10=(0.0, 4.0),
                   q_log2=None):
    """Redraw the FP8 rows' scales and RoPE dims over wide ranges, in storage
    format: per-row scale 2^u with u ~ U(scale_log2) (codes kept); RoPE dims
    bf16 of N(0,1) * amax * 10^v, v ~ U(rope_ratio_log10), where amax is the
    row's decoded non-RoPE amax (so the RoPE/non-RoPE magnitude ratio spans
    10^v).  With ``q_log2`` the queries are redrawn as
    bf16 of N(0,1) * 2^u per (query, head), u ~ U(q_log2).  Cache rows and
    window rows are both redrawn."""
    p = w["params"]
    assert p.kv_fmt == FMT_FP8
    rng = np.random.default_rng(seed)
    w = dict(w)
    n_nope = p.d - p.r
    for key, skey in (("kv", "kv_scale"), ("win", "win_scale")):
        rows = w[key].copy()
        shp = rows.shape[:-1]
        sc = np.exp2(rng.uniform(*scale_log2, size=shp)).astype(np.float32)
        codes = rows[..., :n_nope].view(ml_dtypes.float8_e4m3fn).astype(np.float32)
        amax = np.abs(codes).max(axis=-1) * sc
        ratio = 10.0 ** rng.uniform(*rope_ratio_log10, size=shp)
        rope = normal_f32(rng, shp + (p.r,)) * (amax * ratio)[..., None].astype(np.float32)
        rows[..., n_nope:] = _bf16_of(rope).view(np.uint8).reshape(shp + (2 * p.r,))
        w[key] = rows
        w[skey] = sc
    if q_log2 is not None:
        B, T = w["q"].shape[:2]
        mag = np.exp2(rng.uniform(*q_log2, size=(B, T, p.n_h, 1))).astype(np.float32)
        w["q"] = _bf16_of(normal_f32(rng, (B, T, p.n_h, p.d)) * mag)
    return w


_PER_SEQ = ("L", "q_pos0", "a", "b", "gate", "tok_base", "e_begin", "e_end", "kv", "kv_scale", "win",
            "win_scale", "q_idx", "q_idx_sf", "w_idx", "k_idx", "k_idx_sf", "q")


def select_seqs(w, seqs):
    """The workload restricted to the listed sequences (every per-sequence
    array sliced along its first axis; capacities unchanged)."""
    p = w["params"]
    seqs = list(seqs)
    out = dict(w)
    out["params"] = dataclasses.replace(p, B=len(seqs))
    for k in _PER_SEQ:
        if k in w and w[k] is not None and not np.isscalar(w[k]):
            out[k] = np.ascontiguousarray(np.asarray(w[k])[seqs])
    return out
