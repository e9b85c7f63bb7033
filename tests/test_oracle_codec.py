"""Pins for the oracle's element codecs (CPU only).

E4M3 follows the OCP 8-bit floating point format (the FP8 KV cache of
"PagedAttention 与 Continuous Batching", §8.8, and of the inference-stack
wiki's quantisation table); IEEE binary16 and bfloat16 follow their standards.
"""
import math
import struct

import numpy as np
import pytest

from oracle import pa_oracle_np as npo

# Values fixed by the E4M3 definition (bias 7, 3 mantissa bits, no infinities).
E4M3_KNOWN = {
    0x00: 0.0, 0x01: 2.0 ** -9, 0x07: 7 * 2.0 ** -9, 0x08: 2.0 ** -6, 0x30: 0.5,
    0x38: 1.0, 0x39: 1.125, 0x3F: 1.875, 0x40: 2.0, 0x77: 240.0, 0x78: 256.0,
    0x7E: 448.0, 0xB8: -1.0, 0xFE: -448.0, 0x81: -(2.0 ** -9),
}


def test_e4m3_decode_known_values(oracle):
    for b, v in E4M3_KNOWN.items():
        assert oracle.e4m3_to_double(b) == v, hex(b)
    assert math.isnan(oracle.e4m3_to_double(0x7F))
    assert math.isnan(oracle.e4m3_to_double(0xFF))
    neg0 = oracle.e4m3_to_double(0x80)
    assert neg0 == 0.0 and math.copysign(1.0, neg0) == -1.0


def test_e4m3_decode_all_bytes_structure(oracle):
    vals = [oracle.e4m3_to_double(b) for b in range(256)]
    pos = vals[:0x7F]
    # strictly increasing over the finite positive codes, negatives mirror
    assert all(a < b for a, b in zip(pos, pos[1:]))
    for b in range(0x7F):
        assert vals[b | 0x80] == -vals[b] or (b == 0 and vals[0x80] == 0.0)
    # spacing: 2^-9 in the subnormal/first binade, doubling each binade after
    for b in range(1, 0x7F):
        e = max((b - 1) >> 3, 1)
        assert pos[b] - pos[b - 1] == pytest.approx(2.0 ** (e - 10), rel=0, abs=0)
    # agrees with the independent NumPy twin for every byte
    tw = npo.e4m3_decode(np.arange(256, dtype=np.uint8))
    for b in range(256):
        if math.isnan(vals[b]):
            assert np.isnan(tw[b])
        else:
            assert tw[b] == vals[b]


def test_e4m3_encode_roundtrip_and_midpoints(oracle):
    for b in range(256):
        if b in (0x7F, 0xFF):
            continue
        assert oracle.e4m3_from_float(oracle.e4m3_to_double(b)) == b, hex(b)
    # midpoints between neighbours round to the even code
    for b in range(0x7E):
        lo, hi = oracle.e4m3_to_double(b), oracle.e4m3_to_double(b + 1)
        mid = (lo + hi) / 2
        if float(np.float32(mid)) != mid:
            continue
        want = b if b % 2 == 0 else b + 1
        assert oracle.e4m3_from_float(mid) == want, hex(b)
        assert oracle.e4m3_from_float(-mid) == want | 0x80
        # just off the midpoint goes to the nearer neighbour
        assert oracle.e4m3_from_float(float(np.nextafter(np.float32(mid), np.float32(0)))) == b
        assert oracle.e4m3_from_float(float(np.nextafter(np.float32(mid), np.float32(1e9)))) == b + 1


def test_e4m3_encode_saturation_and_specials(oracle):
    assert oracle.e4m3_from_float(448.0) == 0x7E
    assert oracle.e4m3_from_float(463.9) == 0x7E
    assert oracle.e4m3_from_float(1e30) == 0x7E
    assert oracle.e4m3_from_float(float("inf")) == 0x7E
    assert oracle.e4m3_from_float(-float("inf")) == 0xFE
    assert oracle.e4m3_from_float(float("nan")) == 0x7F
    assert oracle.e4m3_from_float(0.0) == 0x00
    assert oracle.e4m3_from_float(-0.0) == 0x80
    assert oracle.e4m3_from_float(2.0 ** -11) == 0x00     # a quarter of the smallest step
    assert oracle.e4m3_from_float(2.0 ** -10) == 0x00     # half way to 0x01: ties to even
    assert oracle.e4m3_from_float(3 * 2.0 ** -10) == 0x02  # half way 0x01/0x02: even


def test_e4m3_encode_matches_brute_force_nearest(oracle):
    """Against the definition: the nearest finite value, ties to even code."""
    rng = np.random.default_rng(5)
    table = [oracle.e4m3_to_double(b) for b in range(0x7F)]
    xs = np.concatenate([
        rng.standard_normal(3000).astype(np.float32) * 3,
        (np.exp2(rng.uniform(-12, 9.5, 3000)) * rng.choice([-1, 1], 3000)).astype(np.float32),
    ])
    twin = npo.e4m3_encode(xs)
    for x, tw in zip(xs.tolist(), twin.tolist()):
        a = abs(x)
        if a >= 448:
            want = 0x7E
        else:
            best = min(range(0x7F), key=lambda b: (abs(table[b] - a), b % 2))
            want = best
        if x < 0 or (x == 0 and math.copysign(1, x) < 0):
            want |= 0x80
        assert oracle.e4m3_from_float(x) == want, x
        assert tw == want, x


def test_f16_decode_known_values(oracle):
    assert oracle.f16_to_double(0x3C00) == 1.0
    assert oracle.f16_to_double(0xC000) == -2.0
    assert oracle.f16_to_double(0x7BFF) == 65504.0
    assert oracle.f16_to_double(0x0001) == 2.0 ** -24
    assert oracle.f16_to_double(0x0400) == 2.0 ** -14
    assert oracle.f16_to_double(0x3555) == (1 + 0x155 / 1024) * 2.0 ** -2
    assert math.isinf(oracle.f16_to_double(0x7C00))
    assert math.isnan(oracle.f16_to_double(0x7E00))


def test_f16_decode_matches_ieee_half_everywhere(oracle):
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ref = bits.view(np.float16).astype(np.float64)
    for b in range(0, 65536, 7):
        v = oracle.f16_to_double(b)
        if np.isnan(ref[b]):
            assert math.isnan(v)
        else:
            assert v == ref[b], hex(b)


def test_bf16_decode_is_upper_half_of_binary32(oracle):
    rng = np.random.default_rng(3)
    for b in rng.integers(0, 65536, 4000).tolist() + [0x3F80, 0xBF80, 0x0001, 0x7F7F]:
        want = struct.unpack("<f", struct.pack("<I", b << 16))[0]
        v = oracle.bf16_to_double(b)
        if math.isnan(want):
            assert math.isnan(v)
        else:
            assert v == want
    assert oracle.bf16_to_double(0x3F80) == 1.0
    assert oracle.bf16_to_double(0x4049) == 3.140625

