"""Pins of the oracle's storage codecs against the format specs and against
independent library casts (torch, ml_dtypes)."""

import ml_dtypes
import numpy as np
import torch

from oracle import codecs


def test_e4m3_decode_spec_points():
    # OCP FP8 spec: E4M3 bias 7, max 448 (S.1111.110), NaN only S.1111.111,
    # min normal 2^-6 (0.0001.000), min subnormal 2^-9 (0.0000.001).
    v = codecs.e4m3_decode(np.array([0x00, 0x01, 0x08, 0x38, 0x7E, 0x7F, 0xFE, 0x80, 0x07], np.uint8))
    assert v[0] == 0.0 and v[1] == 2.0 ** -9 and v[2] == 2.0 ** -6 and v[3] == 1.0
    assert v[4] == 448.0 and np.isnan(v[5]) and v[6] == -448.0
    assert v[7] == 0.0 and np.signbit(v[7])
    assert v[8] == 7 * 2.0 ** -9  # largest subnormal


def test_e4m3_decode_matches_libraries_all_codes():
    codes = np.arange(256, dtype=np.uint8)
    ours = codecs.e4m3_decode(codes)
    lib = codes.view(ml_dtypes.float8_e4m3fn).astype(np.float64)
    tor = torch.from_numpy(codes.copy()).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    np.testing.assert_array_equal(np.isnan(ours), np.isnan(lib))
    ok = ~np.isnan(ours)
    np.testing.assert_array_equal(ours[ok], lib[ok])
    np.testing.assert_array_equal(ours[ok], tor[ok])


def test_e4m3_encode_vs_torch_rne_in_range():
    rng = np.random.default_rng(5)
    x = np.concatenate([
        rng.standard_normal(20000) * 100,
        rng.uniform(-448, 448, 20000),
        rng.standard_normal(2000) * 1e-3,
        # exact midpoints between adjacent codes (ties -> even code)
        (codecs._E4M3_POS[:-1] + codecs._E4M3_POS[1:]) / 2,
    ]).astype(np.float32)
    ours = codecs.e4m3_encode(x.astype(np.float64))
    tor = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    np.testing.assert_array_equal(ours, tor)


def test_e4m3_encode_saturates():
    c = codecs.e4m3_encode(np.array([449.0, 1e6, -500.0, 464.0, 463.9]))
    np.testing.assert_array_equal(c, [0x7E, 0x7E, 0xFE, 0x7E, 0x7E])


def test_bf16_roundtrip_vs_torch():
    rng = np.random.default_rng(6)
    x = np.concatenate([rng.standard_normal(50000).astype(np.float32),
                        (rng.standard_normal(5000) * 1e-30).astype(np.float32),
                        np.float32([1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -2.0 - 2 ** -7])])
    ours = codecs.bf16_encode(x.astype(np.float64))
    tor = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(ours, tor)
    np.testing.assert_array_equal(codecs.bf16_decode(tor), torch.from_numpy(x).to(torch.bfloat16).double().numpy())


def test_e2m1_table_and_library():
    # OCP MX spec E2M1 magnitudes
    np.testing.assert_array_equal(codecs.e2m1_decode(np.arange(8)), [0, .5, 1, 1.5, 2, 3, 4, 6])
    np.testing.assert_array_equal(codecs.e2m1_decode(np.arange(8, 16)), -np.array([0, .5, 1, 1.5, 2, 3, 4, 6]))
    lib = np.arange(16, dtype=np.uint8).view(ml_dtypes.float4_e2m1fn).astype(np.float64)
    np.testing.assert_array_equal(codecs.e2m1_decode(np.arange(16)), lib)


def test_ue8m0_and_mxfp4_layout():
    assert codecs.ue8m0_decode(np.uint8(127)) == 1.0
    assert codecs.ue8m0_decode(np.uint8(125)) == 0.25
    assert np.isnan(codecs.ue8m0_decode(np.uint8(255)))
    # element 0 in the low nibble, element 1 in the high nibble; scale per 32
    packed = np.zeros(32, np.uint8)
    packed[0] = 0x72  # elem0 = code 2 (1.0), elem1 = code 7 (6.0)
    packed[16] = 0x0B  # elem32 = code 11 (-1.5)
    sc = np.array([127, 128], np.uint8)
    v = codecs.mxfp4_decode(packed, sc, 64)
    assert v[0] == 1.0 and v[1] == 6.0 and v[32] == -3.0 and np.count_nonzero(v) == 3


# ---- the OCP MX conversion to MXFP4 (index keys and queries) ---------------

def test_mxfp4_encode_hand_worked_blocks():
    """Blocks worked by hand from the OCP MX v1.0 conversion rule
    X = floor(log2 amax) - 2, elements RNE(v / 2^X) on the E2M1 grid
    {0, .5, 1, 1.5, 2, 3, 4, 6}, saturating."""
    blk_a = [6.0, 3.0, 1.5, 0.75, -0.25, 5.0, 2.5, -7.0] + [0.0] * 24
    # amax 7 -> X = floor(2.807) - 2 = 0, scale byte 127
    # 0.75 ties between .5 and 1 -> 1 (even); -0.25 ties between 0 and .5 ->
    # -0; 5 ties between 4 and 6 -> 4; 2.5 -> 2; -7 saturates to -6
    want_a = [0x7, 0x5, 0x3, 0x2, 0x8, 0x6, 0x4, 0xF] + [0x0] * 24
    blk_b = [0.3, -0.1, 0.05, 0.2] + [0.0] * 28
    # amax 0.3 -> X = floor(-1.737) - 2 = -4 (byte 123); v * 16 = 4.8 -> 4,
    # -1.6 -> -1.5, 0.8 -> 1, 3.2 -> 3
    want_b = [0x6, 0xB, 0x2, 0x5] + [0x0] * 28
    blk_c = [0.0] * 32  # all zero -> X = -127 (byte 0), codes 0
    x = np.array([blk_a + blk_b + blk_c + blk_a])
    packed, scales = codecs.mxfp4_encode(x)
    assert scales.tolist() == [[127, 123, 0, 127]]
    nib = np.stack([packed & 0xF, packed >> 4], axis=-1).reshape(1, 128)
    assert nib[0, :32].tolist() == want_a
    assert nib[0, 32:64].tolist() == want_b
    assert nib[0, 64:96].tolist() == [0] * 32
    # decode: the block's values back on the scaled grid
    dec = codecs.mxfp4_decode(packed, scales, 128)
    np.testing.assert_array_equal(dec[0, :8], [6, 3, 1.5, 1, -0.0, 4, 2, -6])
    np.testing.assert_array_equal(dec[0, 32:36], [0.25, -0.09375, 0.0625, 0.1875])


def test_mxfp4_encode_elements_match_library_cast():
    """Element codes equal ml_dtypes' E2M1 cast (round to nearest even) of
    v / 2^X, and X is floor(log2 amax) - 2, over values spanning binades."""
    import ml_dtypes
    rng = np.random.default_rng(3)
    y = rng.normal(size=(200, 128)) * np.exp2(rng.uniform(-20, 20, size=(200, 1)))
    packed, scales = codecs.mxfp4_encode(y)
    X = scales.astype(np.float64) - 127
    amax = np.abs(y.reshape(200, 4, 32)).max(axis=-1)
    np.testing.assert_array_equal(X, np.floor(np.log2(amax)) - 2)
    ref = (y.reshape(200, 4, 32) / np.exp2(X)[..., None]).astype(np.float32)
    ref = ref.astype(ml_dtypes.float4_e2m1fn).view(np.uint8).reshape(200, 128) & 0xF
    nib = np.stack([packed & 0xF, packed >> 4], axis=-1).reshape(200, 128)
    np.testing.assert_array_equal(nib, ref)
