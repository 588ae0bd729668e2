"""Storage-format codecs for the oracle, written from the public format specs.

TEST INFRASTRUCTURE. Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU
baseline leg of ``bench.py`` may import anything under ``oracle/``. The product
path (the CUDA library and its Python binding) never does.

Formats (all decoders return float64):

* FP8 E4M3 ("e4m3fn", OCP 8-bit floating point specification v1.0): 1 sign
  bit, 4 exponent bits with bias 7, 3 mantissa bits, no infinities, only
  S.1111.111 is NaN, largest finite magnitude 448.  The KV-cache entries keep
  their non-RoPE dims in this format (WeChat 未来科技 article, §1.1
  混合注意力: RoPE dims in BF16, the other dims in FP8).
* BF16: the upper 16 bits of an IEEE-754 binary32.
* FP4 E2M1 (OCP Microscaling Formats (MX) v1.0, element type): 1 sign bit,
  2 exponent bits with bias 1, 1 mantissa bit, no infinities, no NaN.
* UE8M0 (OCP MX v1.0, shared scale): an unsigned biased exponent,
  value 2^(E-127); 0xFF is NaN.  One scale per 32 consecutive elements.
  The Lightning Indexer's QK runs in FP4 (PACMAN talk notes, §6 MoE:
  FP4 QAT covers the CSA indexer QK path; kwkr.cn notes, §3.4).

Packing of MXFP4 (a choice of this library, stated once here): two E2M1
codes per byte, the element with the lower index in the low nibble.

Encoders round to nearest, ties to even, as the specs' default rounding.
The E4M3 encoder saturates to +-448 ("satfinite"), which is the conversion
the KV packer uses.  Every encoder is a plain nearest-value search over the
enumerated code table, so it can be checked against the table by eye.
"""

from __future__ import annotations

import numpy as np

# ----------------------------------------------------------------------------
# FP8 E4M3
# ----------------------------------------------------------------------------


def e4m3_decode(codes) -> np.ndarray:
    """Decode E4M3 codes (uint8) to float64 from the bit fields.

    exponent field 0 -> subnormal: (-1)^s * (mant/8) * 2^(1-7)
    otherwise        -> normal:    (-1)^s * (1 + mant/8) * 2^(e-7)
    S.1111.111       -> NaN
    """
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    s = (c >> 7) & 1
    e = (c >> 3) & 0xF
    mant = c & 0x7
    sign = np.where(s == 1, -1.0, 1.0)
    sub = sign * (mant / 8.0) * 2.0 ** (1 - 7)
    nrm = sign * (1.0 + mant / 8.0) * np.power(2.0, (e - 7).astype(np.float64))
    out = np.where(e == 0, sub, nrm)
    out = np.where((e == 0xF) & (mant == 0x7), np.nan, out)
    return out.astype(np.float64)


# The 127 non-negative finite E4M3 values, in code order 0x00..0x7E; the
# values rise strictly with the code, so nearest-value search is a sorted
# search.
_E4M3_POS = e4m3_decode(np.arange(0, 127, dtype=np.uint8))


def _nearest_even(table_vals: np.ndarray, mag: np.ndarray) -> np.ndarray:
    """Index of the nearest entry of a strictly increasing table to each
    magnitude; on an exact tie the even index wins (ties-to-even on the code,
    whose last bit is the mantissa LSB)."""
    hi = np.searchsorted(table_vals, mag, side="left")
    hi = np.clip(hi, 1, len(table_vals) - 1)
    lo = hi - 1
    dlo = mag - table_vals[lo]
    dhi = table_vals[hi] - mag
    pick_hi = (dhi < dlo) | ((dhi == dlo) & (hi % 2 == 0))
    idx = np.where(pick_hi, hi, lo)
    # below the first entry / above the last
    idx = np.where(mag <= table_vals[0], 0, idx)
    idx = np.where(mag >= table_vals[-1], len(table_vals) - 1, idx)
    return idx


def e4m3_encode(x) -> np.ndarray:
    """float64 -> E4M3 code, round to nearest even, saturating at +-448.

    NaN maps to 0x7F (positive NaN).  Zero keeps its sign.
    """
    x = np.asarray(x, dtype=np.float64)
    mag = np.abs(x)
    idx = _nearest_even(_E4M3_POS, np.nan_to_num(mag, nan=0.0))
    code = idx.astype(np.uint8) | np.where(np.signbit(x), 0x80, 0).astype(np.uint8)
    code = np.where(np.isnan(x), np.uint8(0x7F), code)
    return code.astype(np.uint8)


E4M3_MAX = 448.0

# ----------------------------------------------------------------------------
# BF16
# ----------------------------------------------------------------------------


def bf16_decode(bits) -> np.ndarray:
    """BF16 bit patterns (uint16) -> float64 (exact)."""
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return b.view(np.float32).astype(np.float64)


# All non-negative finite BF16 values in code order 0x0000..0x7F7F.
_BF16_POS = bf16_decode(np.arange(0, 0x7F80, dtype=np.uint32).astype(np.uint16))


def bf16_encode(x) -> np.ndarray:
    """float64 -> BF16 bits, round to nearest even (values beyond the largest
    finite BF16 saturate; none of the library's data reaches them)."""
    x = np.asarray(x, dtype=np.float64)
    mag = np.abs(x)
    idx = _nearest_even(_BF16_POS, np.nan_to_num(mag, nan=0.0))
    bits = idx.astype(np.uint16) | np.where(np.signbit(x), 0x8000, 0).astype(np.uint16)
    bits = np.where(np.isnan(x), np.uint16(0x7FC0), bits)
    return bits.astype(np.uint16)


# ----------------------------------------------------------------------------
# MXFP4: E2M1 elements + UE8M0 scale per 32 elements
# ----------------------------------------------------------------------------


def e2m1_decode(nibbles) -> np.ndarray:
    """E2M1 codes (0..15) -> float64 from the bit fields.

    exponent field 0 -> subnormal: (-1)^s * (mant/2) * 2^(1-1)
    otherwise        -> normal:    (-1)^s * (1 + mant/2) * 2^(e-1)
    """
    n = np.asarray(nibbles).astype(np.int64) & 0xF
    s = (n >> 3) & 1
    e = (n >> 1) & 0x3
    mant = n & 0x1
    sign = np.where(s == 1, -1.0, 1.0)
    sub = sign * (mant / 2.0)
    nrm = sign * (1.0 + mant / 2.0) * np.power(2.0, (e - 1).astype(np.float64))
    return np.where(e == 0, sub, nrm).astype(np.float64)


def ue8m0_decode(codes) -> np.ndarray:
    """UE8M0 scale bytes -> float64 2^(E-127); 0xFF -> NaN."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    v = np.power(2.0, (c - 127).astype(np.float64))
    return np.where(c == 0xFF, np.nan, v)


def mxfp4_decode(packed, scales, n: int) -> np.ndarray:
    """Decode MXFP4 vectors.

    packed: uint8 [..., n/2], element 2i in the low nibble of byte i,
            element 2i+1 in the high nibble.
    scales: uint8 [..., n/32] UE8M0, scale j covers elements 32j..32j+31.
    returns float64 [..., n] = e2m1(element) * 2^(E_j - 127).
    """
    packed = np.asarray(packed, dtype=np.uint8)
    lo = packed & 0xF
    hi = packed >> 4
    codes = np.stack([lo, hi], axis=-1).reshape(packed.shape[:-1] + (n,))
    vals = e2m1_decode(codes)
    sc = ue8m0_decode(scales)
    sc = np.repeat(sc, 32, axis=-1)
    return vals * sc


# The 8 non-negative E2M1 values in code order 0..7 (strictly increasing).
_E2M1_POS = e2m1_decode(np.arange(0, 8))
E2M1_MAX = 6.0


def e2m1_encode(x) -> np.ndarray:
    """float64 -> E2M1 code (0..15), round to nearest, ties to even,
    saturating at +-6 (OCP MX v1.0: FP4 has no infinity or NaN, conversions
    clamp to the largest magnitude).  The sign is kept, so a negative value
    that rounds to zero becomes -0 (code 8)."""
    x = np.asarray(x, dtype=np.float64)
    idx = _nearest_even(_E2M1_POS, np.abs(x))
    return (idx.astype(np.uint8) | np.where(np.signbit(x), 8, 0).astype(np.uint8)).astype(np.uint8)


def mxfp4_encode(x):
    """float64 [..., n] (n a multiple of 32) -> (packed [..., n/2],
    scales [..., n/32]) by the OCP MX v1.0 conversion (section 6.3):
    for each block of 32, the shared exponent is
        X = floor(log2(max |v|)) - emax_elem,   emax_elem = 2 for E2M1,
    clamped to the UE8M0 range [-127, 127] (an all-zero block takes
    X = -127), stored as X + 127; each element becomes the E2M1 code of
    v / 2^X (nearest even, saturating at +-6: the block's largest magnitude
    lands in [4, 8) before rounding)."""
    x = np.asarray(x, dtype=np.float64)
    n = x.shape[-1]
    blk = x.reshape(x.shape[:-1] + (n // 32, 32))
    amax = np.max(np.abs(blk), axis=-1)
    with np.errstate(divide="ignore"):
        X = np.where(amax > 0, np.floor(np.log2(np.where(amax > 0, amax, 1.0))) - 2.0, -127.0)
    X = np.clip(X, -127.0, 127.0)
    codes = e2m1_encode(blk / np.power(2.0, X)[..., None]).reshape(x.shape)
    packed = (codes[..., 0::2] | (codes[..., 1::2] << 4)).astype(np.uint8)
    return packed, (X + 127).astype(np.uint8)
