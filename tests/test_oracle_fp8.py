"""Pins of the oracle's 8-bit (e4m3) compressed cache against things outside the oracle.

* Code values: torch's float8_e4m3fn type (a library implementation of the same OCP
  format) for all 256 codes, plus facts of the format definition typed in by hand
  (largest finite 448, smallest normal 2^-6, smallest subnormal 2^-9, one = 0x38, NaN
  codes 0x7f / 0xff).
* Rounding: torch's float32 -> float8_e4m3fn cast (round to nearest, ties to even) on
  every exact value, every midpoint between neighbouring values, one float32 step either
  side of each midpoint, and random values; saturation at 448 (where torch gives NaN
  instead, only the oracle's saturating reading is checked).
* Block quantisation: a block whose mean is exactly a code value times the scale gives
  that code; any block's dequantised entry lies within half a quantisation step of the
  float32 mean.
* Decode on a dequantised cache equals decode on the same values built by torch.
Each planted mistake below (a wrong exponent bias, ties away from zero, no saturation, a
multiplied scale, K and V scales swapped) fails at least one pin.
"""

import numpy as np
import pytest
import torch

import oracle.hca_oracle as ORC


def _torch_values(codes):
    return torch.from_numpy(np.asarray(codes, np.uint8).copy()).view(
        torch.float8_e4m3fn).to(torch.float64).numpy()


def _torch_codes(x32):
    return torch.from_numpy(np.asarray(x32, np.float32).copy()).to(
        torch.float8_e4m3fn).view(torch.uint8).numpy()


# ------------------------------------------------------------------------------ pins
def pin_values_match_library(orc):
    codes = np.arange(256, dtype=np.uint8)
    got = orc.e4m3_value(codes)
    assert np.array_equal(got, _torch_values(codes), equal_nan=True)


def pin_values_by_hand(orc):
    v = orc.e4m3_value(np.array([0x7E, 0x08, 0x01, 0x38, 0x00, 0x80, 0xFE, 0x07, 0x3C],
                                np.uint8))
    want = [448.0, 2.0 ** -6, 2.0 ** -9, 1.0, 0.0, -0.0, -448.0, 7 * 2.0 ** -9, 1.5]
    assert np.array_equal(v, want)
    assert np.isnan(orc.e4m3_value(np.array([0x7F, 0xFF], np.uint8))).all()


def _test_points():
    table = _torch_values(np.arange(127, dtype=np.uint8))
    mids = (table[:-1] + table[1:]) / 2.0          # exact in float64 and in float32
    m32 = mids.astype(np.float32)
    up = np.nextafter(m32, np.float32(np.inf))
    down = np.nextafter(m32, np.float32(-np.inf))
    rng = np.random.default_rng(7)
    rand = np.concatenate([rng.standard_normal(4000) * s for s in (1e-3, 0.05, 1.0, 60.0)])
    pts = np.concatenate([table, m32, up, down, rand]).astype(np.float32)
    pts = pts[np.abs(pts) < 448.0]
    return np.concatenate([pts, -pts])


def pin_rounding_matches_library(orc):
    x = _test_points()
    assert np.array_equal(orc.e4m3_quantize(x), _torch_codes(x))


def pin_saturation(orc):
    x = np.array([448.0, 460.0, 464.0, 500.0, 1e6, 3e38], np.float32)
    assert (orc.e4m3_quantize(x) == 0x7E).all()
    assert (orc.e4m3_quantize(-x) == 0xFE).all()
    assert orc.e4m3_quantize(np.array([np.nan], np.float32))[0] == 0x7F


def pin_exact_block_means(orc):
    # every non-negative finite code c: a block of 4 tokens whose mean is value(c) * s
    # (float32-exact for this power-of-two-free scale only where the product is; keep
    # those) must store c
    s = np.float32(0.375)
    codes = np.arange(127, dtype=np.uint8)
    vals = _torch_values(codes) * np.float64(s)
    keep = vals.astype(np.float32).astype(np.float64) == vals
    X = np.repeat(vals[keep][None, None, :], 4, axis=0)       # [4 tokens, 1, n]
    got = orc.compress_blocks_e4m3(X, 4, float(s))
    assert np.array_equal(got[0, 0], codes[keep])
    got_neg = orc.compress_blocks_e4m3(-X, 4, float(s))
    nz = codes[keep] != 0     # a zero mean is +0 (a sum that starts at +0)
    assert np.array_equal(got_neg[0, 0][nz], codes[keep][nz] | 0x80)
    assert (got_neg[0, 0][~nz] == 0).all()


def pin_block_quantisation_error(orc):
    rng = np.random.default_rng(3)
    X = rng.standard_normal((300, 2, 64))
    s = 0.0021
    codes = orc.compress_blocks_e4m3(X, 128, s)
    mean = np.stack([X[j * 128:(j + 1) * 128].mean(0) for j in range(3)]).astype(np.float32)
    back = _torch_values(codes) * np.float64(np.float32(s))
    # half a step of the code's binade (the subnormal step below 2^-6), in stored units
    y = np.abs(mean.astype(np.float64) / np.float32(s))
    step = np.where(y < 2.0 ** -6, 2.0 ** -9, 2.0 ** (np.floor(np.log2(np.maximum(y, 1e-30))) - 3))
    # a float32 ulp of y covers the float32 division
    assert (np.abs(back - mean) <= (step / 2 + 2.0 ** -23 * y) * np.float32(s) * (1 + 1e-12)).all()


def pin_decode_on_dequantised_cache(orc):
    rng = np.random.default_rng(11)
    D, hq, W, block = 32, 4, 8, 4
    ctx = 45
    nc = orc.visible_compressed_count(ctx - 1, block, W)
    ck = rng.integers(0, 0x7F, size=(nc + 2, 1, D), dtype=np.uint8) ^ np.uint8(0x80) * rng.integers(0, 2, size=(nc + 2, 1, D), dtype=np.uint8)
    cv = rng.integers(0, 0x7F, size=(nc + 2, 1, D), dtype=np.uint8)
    sk, sv = 0.0625, 0.011
    q = rng.standard_normal((hq, D))
    rk = rng.standard_normal((W, 1, D))
    rv = rng.standard_normal((W, 1, D))
    got, lse = orc.hca_decode(q, orc.e4m3_dequantize(ck, sk), orc.e4m3_dequantize(cv, sv),
                              rk, rv, ctx, block, W, 0.3)
    Kc = _torch_values(ck) * np.float64(np.float32(sk))
    Vc = _torch_values(cv) * np.float64(np.float32(sv))
    want, lse2 = orc.hca_decode(q, Kc, Vc, rk, rv, ctx, block, W, 0.3)
    assert np.allclose(got, want, rtol=0, atol=1e-13)
    assert np.allclose(lse, lse2, rtol=0, atol=1e-13)


PINS = [pin_values_match_library, pin_values_by_hand, pin_rounding_matches_library,
        pin_saturation, pin_exact_block_means, pin_block_quantisation_error,
        pin_decode_on_dequantised_cache]


@pytest.mark.parametrize("pin", PINS, ids=[p.__name__ for p in PINS])
def test_fp8_oracle_pin(pin):
    pin(ORC)


# ------------------------------------------------------------------ planted mistakes
def _mut_bias8(codes):
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = c & 0x7
    mag = np.where(e == 0, m / 8.0 * 2.0 ** -7, (1.0 + m / 8.0) * np.exp2(e - 8.0))
    return sign * np.where((e == 15) & (m == 7), np.nan, mag)


def _mut_ties_away(x):
    real = ORC.__dict__["_orig_quantize"]
    x = np.asarray(x, np.float32)
    code = real(x)
    table = ORC.e4m3_value(np.arange(127, dtype=np.uint8))
    a = np.abs(x.astype(np.float64))
    # at an exact midpoint take the larger magnitude
    hi = np.clip(np.searchsorted(table, a, side="left"), 1, 126)
    tie = (table[hi] - a) == (a - table[hi - 1])
    bump = tie & (a < 448.0) & (a > 0)
    return np.where(bump, (hi | np.where(np.signbit(x), 0x80, 0)).astype(np.uint8), code)


def _mut_no_saturation(x):
    real = ORC.__dict__["_orig_quantize"]
    code = real(x)
    x = np.asarray(x, np.float32)
    return np.where(np.abs(x) >= 448.0, np.uint8(0x7F), code).astype(np.uint8)


def _mut_scale_multiplied(X, block, scale):
    mean32 = ORC.compress_blocks(X, block).astype(np.float32)
    return ORC.e4m3_quantize((mean32 * np.float32(scale)).astype(np.float32))


def _mut_dequant_swapped(codes, scale):
    # uses the reciprocal of the scale (a typical direction mistake)
    return ORC.e4m3_value(codes) / np.float64(np.float32(scale))


FP8_MUTANTS = {
    "bias8": ("e4m3_value", _mut_bias8),
    "ties_away": ("e4m3_quantize", _mut_ties_away),
    "no_saturation": ("e4m3_quantize", _mut_no_saturation),
    "scale_multiplied": ("compress_blocks_e4m3", _mut_scale_multiplied),
    "dequant_divides": ("e4m3_dequantize", _mut_dequant_swapped),
}


@pytest.mark.parametrize("name", sorted(FP8_MUTANTS))
def test_fp8_planted_mistakes_are_caught(name, monkeypatch):
    attr, fn = FP8_MUTANTS[name]
    monkeypatch.setitem(ORC.__dict__, "_orig_quantize", ORC.e4m3_quantize)
    monkeypatch.setattr(ORC, attr, fn)
    failed = []
    for pin in PINS:
        try:
            pin(ORC)
        except (AssertionError, ValueError, IndexError):
            failed.append(pin.__name__)
    assert failed, f"planted mistake {name!r} passed every pin"


def test_two_part_e4m3_query_split():
    """The reading the 8-bit decode's scores rest on: with r_h the power of two that puts a
    row's largest |q| in [128, 256), x = q / r_h and Q1 = e4m3(x), Q2 = e4m3(x - Q1), the
    two parts give x exactly wherever |x| >= 1/4 (the remainder's last bit is still an e4m3
    step) and within 2^-10 below, for bf16 rows over a wide range of magnitudes."""
    rng = np.random.default_rng(12)
    for trial in range(40):
        scale = 2.0 ** rng.integers(-30, 30)
        q = torch.tensor(rng.standard_normal(512) * scale, dtype=torch.float32)
        q = q.to(torch.bfloat16).to(torch.float64).numpy()
        amax = np.abs(q).max()
        e = int(np.floor(np.log2(amax))) - 7   # r_h = 2^e: amax / r_h in [128, 256)
        x = q / 2.0 ** e
        assert 128.0 <= np.abs(x).max() < 256.0
        q1 = ORC.e4m3_value(ORC.e4m3_quantize(x))
        q2 = ORC.e4m3_value(ORC.e4m3_quantize(x - q1))
        err = np.abs(x - (q1 + q2))
        big = np.abs(x) >= 0.25
        assert (err[big] == 0).all(), f"trial {trial}: inexact at |x| >= 1/4"
        assert (err <= 2.0 ** -10).all(), f"trial {trial}: error above 2^-10"
