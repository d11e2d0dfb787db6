"""Pins of the oracle's FP8 E4M3 cache format against what the format and the
mathematics fix, independent of the oracle's own code:

  * special values of E4M3 as the OCP 8-bit floating point specification
    (OFP8, E4M3 column of its table of special values) lists them;
  * the code <-> value round trip, monotonicity, ties to even and saturation;
  * PyTorch's CPU cast to float8_e4m3fn (a library routine) for in-range values;
  * decode over an fp8 cache equals the already pinned 16-bit decode of the
    same cache dequantized, when the dequantized values are exactly
    representable in half precision (power-of-two scales).
Planted mistakes show each pin has teeth."""

import numpy as np
import pytest
import torch

from oracle import attention as A
from oracle import cache_ops as C
from oracle import fp8 as F
from oracle.fpbits import bits_to_f64
from workloads import gen


# -- pins -------------------------------------------------------------------
def pin_special_values():
    # OFP8 specification, E4M3: bias 7; max normal S.1111.110 = 448; min normal
    # S.0001.000 = 2^-6; max subnormal S.0000.111 = 0.875 * 2^-6; min subnormal
    # S.0000.001 = 2^-9; NaN S.1111.111; zeros S.0000.000
    assert F.decode_e4m3(0b0_1111_110) == 448.0
    assert F.decode_e4m3(0b1_1111_110) == -448.0
    assert F.decode_e4m3(0b0_0001_000) == 2.0 ** -6
    assert F.decode_e4m3(0b0_0000_111) == 0.875 * 2.0 ** -6
    assert F.decode_e4m3(0b0_0000_001) == 2.0 ** -9
    assert F.decode_e4m3(0b0_0111_000) == 1.0
    assert F.decode_e4m3(0b0_1000_100) == 3.0
    assert np.isnan(F.decode_e4m3(0x7F)) and np.isnan(F.decode_e4m3(0xFF))
    assert F.decode_e4m3(0x00) == 0.0 and np.signbit(F.decode_e4m3(0x80))
    assert F.encode_e4m3(448.0) == 0x7E and F.encode_e4m3(1.0) == 0x38


def pin_round_trip_and_order():
    vals = [F.decode_e4m3(c) for c in range(0x7F)]
    assert all(a < b for a, b in zip(vals, vals[1:]))
    for c in range(256):
        if c in (0x7F, 0xFF):
            continue
        assert F.encode_e4m3(F.decode_e4m3(c)) == c, hex(c)
    codes = F.encode_e4m3_array(np.array([F.decode_e4m3(c) for c in range(256)
                                          if c not in (0x7F, 0xFF)]))
    assert codes.tolist() == [c for c in range(256) if c not in (0x7F, 0xFF)]


def pin_ties_and_saturation():
    for c in range(0x7E):
        lo, hi = F.decode_e4m3(c), F.decode_e4m3(c + 1)
        mid = (lo + hi) / 2          # exact in binary floating point
        even = c if c % 2 == 0 else c + 1
        assert F.encode_e4m3(mid) == even, hex(c)
        assert F.encode_e4m3(-mid) == 0x80 | even
        assert F.encode_e4m3(np.nextafter(mid, 0)) == c
        assert F.encode_e4m3(np.nextafter(mid, 1e9)) == c + 1
    for big in (448.0, 448.5, 464.0, 480.0, 1e6, float(np.finfo(np.float32).max)):
        assert F.encode_e4m3(big) == 0x7E and F.encode_e4m3(-big) == 0xFE
    assert F.encode_e4m3(-1e-30) == 0x80 and F.encode_e4m3(1e-30) == 0x00
    assert F.encode_e4m3(float("nan")) == 0x7F


def pin_library_cast():
    rng = np.random.default_rng(3)
    x = np.concatenate([
        rng.standard_normal(20000) * 30,
        rng.standard_normal(5000) * 2.0 ** -8,                    # subnormal range
        [(F.decode_e4m3(c) + F.decode_e4m3(c + 1)) / 2 for c in range(0x7E)],
    ]).astype(np.float32)
    x = np.clip(x, -448, 448)
    x = np.concatenate([x, -x])
    want = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(F.encode_e4m3_array(x), want)
    assert np.array_equal([F.encode_e4m3(v) for v in x[:3000].tolist()], want[:3000])


def pin_quantize_divides_in_float32():
    """Against torch's float32 division and cast, over random values and over
    every positive finite 16-bit value at scales (0.11, 1.3) where dividing in
    float32 and dividing exactly give different codes for some inputs."""
    every = {"f16": np.arange(1, 0x7C00, dtype=np.uint16),
             "bf16": np.arange(1, 0x7F80, dtype=np.uint16)}
    for dt, tdt in (("f16", torch.float16), ("bf16", torch.bfloat16)):
        bits = np.concatenate([gen.normal_bits([9, 1], (4096,), dt, scale=40.0), every[dt]])
        for scale in (0.37, 1.0, 0.05, 3.3, 0.11, 1.3):
            x = torch.from_numpy(bits.view(np.int16)).view(tdt).float()
            q = (x / torch.tensor(scale, dtype=torch.float32)).clamp(-448, 448)
            want = q.to(torch.float8_e4m3fn).view(torch.uint8).numpy()
            assert np.array_equal(F.quantize(bits, dt, scale), want), (dt, scale)


def _fp8_cache(seed, nb, hkv, d):
    rng = np.random.default_rng(seed)
    codes = rng.integers(0, 256, (2, nb, hkv, 16, d)).astype(np.uint8)
    codes[(codes & 0x7F) == 0x7F] = 0x3A      # no NaN codes in a cache
    return codes[0], codes[1]


def pin_decode_matches_16bit_decode():
    """With a power-of-two scale every dequantized value is an exact half, so the
    fp8 decode must equal the 16-bit decode of the dequantized cache."""
    nb, hkv, hq, d = 12, 2, 8, 64
    kc8, vc8 = _fp8_cache(1, nb, hkv, d)
    ks, vs = 0.25, 2.0 ** -3
    # dequantized by the library's float8 type, not by the oracle
    def lib_dequant(codes, sc):
        x = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float32) * sc
        return x.to(torch.float16).view(torch.int16).numpy().view(np.uint16)
    kc16, vc16 = lib_dequant(kc8, ks), lib_dequant(vc8, vs)
    assert np.array_equal(bits_to_f64(kc16, "f16"), F.dequantize(kc8, ks))
    q = gen.normal_bits([9, 2], (3, hq, d), "f16")
    tables = np.array([[3, 7, 1, -1], [0, 11, -1, -1], [5, 2, 9, 4]], np.int32)
    ctx = np.array([40, 17, 64], np.int32)
    got = F.paged_decode_fp8(q, kc8, vc8, tables, ctx, 0.125, ks, vs, "f16")
    want = A.paged_decode(q, kc16, vc16, tables, ctx, 0.125, "f16")
    assert np.array_equal(got, want)


def pin_cache_write_layout():
    nb, hkv, d = 6, 2, 64
    key = gen.normal_bits([9, 3], (5, hkv, d), "bf16", scale=20.0)
    val = gen.normal_bits([9, 4], (5, hkv, d), "bf16", scale=20.0)
    slots = np.array([17, -1, 90, 0, 33], np.int64)
    kc = np.zeros((nb, hkv, 16, d), np.uint8)
    vc = np.zeros_like(kc)
    F.reshape_and_cache_fp8(kc, vc, key, val, slots, 16, "bf16", 0.5, 0.25)
    kw = np.zeros_like(kc)
    vw = np.zeros_like(kc)
    C.reshape_and_cache(kw, vw, F.quantize(key, "bf16", 0.5), F.quantize(val, "bf16", 0.25),
                        slots, 16)
    assert np.array_equal(kc, kw) and np.array_equal(vc, vw)
    assert kc[1, 1, 1, 5] == F.encode_e4m3(np.float32(bits_to_f64(key[0, 1, 5], "bf16"))
                                           / np.float32(0.5))


PINS = [pin_special_values, pin_round_trip_and_order, pin_ties_and_saturation, pin_library_cast,
        pin_quantize_divides_in_float32, pin_decode_matches_16bit_decode, pin_cache_write_layout]


@pytest.mark.parametrize("pin", PINS, ids=lambda f: f.__name__)
def test_fp8_pin(pin):
    pin()


# -- planted mistakes -------------------------------------------------------
_ORIG_DECODE = F.decode_e4m3
_ORIG_ENCODE = F.encode_e4m3
_ORIG_ENCODE_ARRAY = F.encode_e4m3_array


def _decode_bias8(code):
    v = _ORIG_DECODE(code)
    e = (int(code) >> 3) & 0xF
    return v / 2 if e else v


def _encode_truncate(x):
    x = float(x)
    a = abs(x)
    best = max(c for c in range(0x7F) if _ORIG_DECODE(c) <= min(a, 448.0))
    return (0x80 if np.signbit(x) else 0) | best


def _encode_ties_up(x):
    x = float(x)
    sign = 0x80 if np.signbit(x) else 0
    a = abs(x)
    if a >= 448.0:
        return sign | 0x7E
    for c in range(0x7E):
        lo, hi = _ORIG_DECODE(c), _ORIG_DECODE(c + 1)
        if lo <= a <= hi:
            return sign | (c if a - lo < hi - a else c + 1)


def _encode_array_ties_up(x):
    x = np.asarray(x, dtype=np.float64)
    return np.array([_encode_ties_up(v) for v in x.reshape(-1).tolist()],
                    np.uint8).reshape(x.shape)


def _encode_no_saturation(x):
    return 0x7F if abs(float(x)) > 448.0 else _ORIG_ENCODE(x)


def _encode_array_no_saturation(x):
    x = np.asarray(x, dtype=np.float64)
    out = _ORIG_ENCODE_ARRAY(x)
    out[np.abs(x) > 448.0] = 0x7F
    return out


def _dequantize_ignores_scale(codes, scale):
    table = np.array([_ORIG_DECODE(c) for c in range(256)], dtype=np.float64)
    return table[np.asarray(codes, dtype=np.uint8)]


def _quantize_multiplies_by_f64_reciprocal(bits, dtype, scale):
    x = bits_to_f64(np.asarray(bits), dtype)
    return _ORIG_ENCODE_ARRAY(x * (1.0 / scale))


MISTAKES = {
    "decode_bias_8": [("decode_e4m3", _decode_bias8)],
    "encode_truncates": [("encode_e4m3", _encode_truncate)],
    "ties_round_up": [("encode_e4m3", _encode_ties_up),
                      ("encode_e4m3_array", _encode_array_ties_up)],
    "no_saturation": [("encode_e4m3", _encode_no_saturation),
                      ("encode_e4m3_array", _encode_array_no_saturation)],
    "dequantize_ignores_scale": [("dequantize", _dequantize_ignores_scale)],
    "quantize_in_float64": [("quantize", _quantize_multiplies_by_f64_reciprocal)],
}


def _fails_some_pin():
    for pin in PINS:
        try:
            pin()
        except (Exception, pytest.fail.Exception):
            return True
    return False


@pytest.mark.parametrize("name", sorted(MISTAKES))
def test_planted_mistake_is_caught(name, monkeypatch):
    for attr, bad in MISTAKES[name]:
        monkeypatch.setattr(F, attr, bad)
    assert _fails_some_pin(), f"planted mistake {name!r} passed every pin"
