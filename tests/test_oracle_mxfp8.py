"""Pins for the oracle's MXFP8 codec and blockwise quantisation (CPU only).

torch's float8_e4m3fn and float8_e8m0fnu dtypes are independent
implementations of the same OCP formats, so all 256 codes of each and the
round-to-nearest-even encode are checked against them.  The scale rule is
checked by brute force, exactly representable blocks must round-trip
bit-exactly, and the quantisation error must respect E4M3's half-ulp bound.
"""
import numpy as np
import pytest
import torch

from oracle import mxfp8_ref as M


def test_e4m3_decode_all_codes_match_torch():
    codes = np.arange(256, dtype=np.uint8)
    ours = M.e4m3_decode(codes)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    np.testing.assert_array_equal(np.isnan(ours), np.isnan(ref))
    ok = ~np.isnan(ref)
    np.testing.assert_array_equal(ours[ok], ref[ok])
    assert np.nanmax(ours) == 448.0
    assert M.e4m3_decode(np.array([1]))[0] == 2.0 ** -9     # smallest subnormal


def test_e8m0_decode_all_codes_match_torch():
    codes = np.arange(256, dtype=np.uint8)
    ours = M.e8m0_decode(codes)
    ref = torch.from_numpy(codes).view(torch.float8_e8m0fnu).to(torch.float64).numpy()
    np.testing.assert_array_equal(np.isnan(ours), np.isnan(ref))
    ok = ~np.isnan(ref)
    np.testing.assert_array_equal(ours[ok], ref[ok])


def test_e4m3_encode_matches_torch_rne():
    rng = np.random.default_rng(0)
    v = np.concatenate([rng.uniform(-463, 463, 50000),
                        rng.standard_normal(50000) * 2.0 ** rng.integers(-12, 6, 50000),
                        # exact midpoints between neighbouring codes
                        0.5 * (M.e4m3_decode(np.arange(0, 0x7E)) + M.e4m3_decode(np.arange(1, 0x7F))),
                        [0.0, -0.0, 448.0, -448.0]])
    v = v.astype(np.float32).astype(np.float64)
    ours = M.e4m3_encode(v)
    ref = torch.tensor(v, dtype=torch.float32).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    np.testing.assert_array_equal(ours, ref)


def test_e4m3_encode_saturates():
    big = np.array([464.0, 1000.0, 1e30, -500.0])
    np.testing.assert_array_equal(M.e4m3_decode(M.e4m3_encode(big)), [448, 448, 448, -448])


def test_scale_rule_brute_force():
    rng = np.random.default_rng(1)
    amax = np.concatenate([rng.standard_normal(2000) ** 2 * 2.0 ** rng.integers(-60, 60, 2000),
                           2.0 ** np.arange(-133, 140, dtype=np.float64), [448.0, 512.0, 511.9],
                           # both clamps: bf16 subnormals reach e < -127 (2^-133 is the
                           # smallest), huge float64 values e > 127
                           [1.5 * 2.0 ** -119, 1.9 * 2.0 ** -120, 1e-40, 3.0 * 2.0 ** 135]])
    amax = np.abs(amax)
    got = M.scale_exponent(amax)
    for a, e in zip(amax, got):
        # the unique e with 2^8 <= a / 2^e < 2^9
        cand = [s for s in range(-160, 161) if 256.0 <= a / 2.0 ** s < 512.0]
        assert len(cand) == 1 and e == max(-127, min(127, cand[0]))
    assert M.scale_exponent(np.array([0.0]))[0] == -127


@pytest.mark.parametrize("axis", [0, 1])
def test_exact_blocks_round_trip(axis):
    rng = np.random.default_rng(2 + axis)
    R_, C_ = 64, 96
    finite = np.array([c for c in range(0x7F)])
    codes = rng.choice(finite, size=(R_, C_)) | (rng.integers(0, 2, (R_, C_)) << 7)
    vals = M.e4m3_decode(codes)
    nb = (R_ // 32, C_) if axis == 0 else (R_, C_ // 32)
    s = rng.integers(-20, 20, size=nb)
    # force each block's max magnitude into [256, 448] so that its scale is exactly 2^s
    if axis == 1:
        vals.reshape(R_, C_ // 32, 32)[:, :, 0] = 448.0
        a = vals * np.repeat(2.0 ** s, 32, axis=1)
    else:
        vals.reshape(R_ // 32, 32, C_)[:, 0, :] = 320.0
        a = vals * np.repeat(2.0 ** s, 32, axis=0)
    q, sc = M.quantize_blocks(a, axis)
    np.testing.assert_array_equal(sc.astype(np.int64) - 127, s)
    np.testing.assert_array_equal(M.dequantize_blocks(q, sc, axis), a)


def test_quantisation_error_bound():
    rng = np.random.default_rng(4)
    a = rng.standard_normal((128, 256)) * np.exp(rng.standard_normal((128, 1)) * 3)
    q, s = M.quantize_blocks(a, 1)
    back = M.dequantize_blocks(q, s, 1)
    scale = np.repeat(M.e8m0_decode(s), 32, axis=1)
    scaled = np.abs(a) / scale
    normal = (scaled >= 2.0 ** -6) & (scaled <= 448)
    rel = np.abs(back - a)[normal] / np.abs(a)[normal]
    assert rel.max() <= 2.0 ** -4 + 1e-12
    sub = scaled < 2.0 ** -6                      # subnormal range: absolute half-ulp
    assert np.all(np.abs(back - a)[sub] <= 2.0 ** -10 * scale[sub] + 1e-300)


def test_zero_block():
    q, s = M.quantize_blocks(np.zeros((2, 64)), 1)
    assert np.all(q == 0) and np.all(s == 0)
