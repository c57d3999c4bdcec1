"""Pins for the oracle's INT4 quantiser, nibble packing and BF16 rounding."""
import os

import numpy as np
import pytest

import synthetic as S
from oracle import quant as Q

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _nibble_rows():
    rows = []
    with open(os.path.join(GOLDEN, "int4_nibbles.txt")) as f:
        for line in f:
            if line.strip() and not line.startswith("#"):
                a, b, h = line.split()
                rows.append((int(a), int(b), int(h, 16)))
    return rows


def test_golden_nibble_bytes_unpack():
    rows = _nibble_rows()
    packed = np.array([[r[2] for r in rows]], dtype=np.uint8)
    u = Q.unpack_nibbles(packed)
    codes = u.astype(int) - 8
    assert codes[0, 0::2].tolist() == [r[0] for r in rows]
    assert codes[0, 1::2].tolist() == [r[1] for r in rows]


def test_golden_nibble_bytes_quantise():
    # Build a one-group row whose codes are the fixture's, with scale 1/4 (exact
    # in fp16): w = code * s, plus one element of magnitude 7 s to fix the scale.
    rows = [r for r in _nibble_rows() if r[0] >= -7 and r[1] >= -7]
    codes = []
    for a, b, _ in rows:
        codes += [a, b]
    codes += [7, 0]
    s = 0.25
    w = np.array([codes], dtype=np.float64) * s
    packed, scale = Q.quantize_int4(w, group=len(codes))
    assert float(scale[0, 0]) == s
    assert packed[0, :len(rows)].tolist() == [r[2] for r in rows]


def test_roundtrip_and_error_bound():
    w = S.random_vectors((64, 256), seed=11, scale=0.02)
    for g in (32, 128):
        packed, s = Q.quantize_int4(w, g)
        wq = Q.dequantize_int4(packed, s, g)
        p2, s2 = Q.quantize_int4(wq, g)
        assert np.array_equal(p2, packed) and np.array_equal(s2, s)
        sg = np.repeat(s.astype(np.float64), g, axis=1)
        assert np.all(np.abs(w - wq) <= sg / 2 * (1 + 1e-12))
        # each group's largest |w| maps to |code| = 7
        u = Q.unpack_nibbles(packed).astype(int) - 8
        for n in range(w.shape[0]):
            for j in range(w.shape[1] // g):
                blk = w[n, j * g:(j + 1) * g]
                assert abs(u[n, j * g + int(np.argmax(np.abs(blk)))]) == 7
        assert u.min() >= -7 and u.max() <= 7


def test_scale_is_fp16_of_max_over_7():
    w = np.zeros((1, 32))
    w[0, 5] = -0.07
    packed, s = Q.quantize_int4(w, 32)
    assert s.dtype == np.float16
    # 0.01 is not representable in fp16; the nearest fp16 value is 0.01000213623046875
    assert float(s[0, 0]) == 0.01000213623046875
    assert Q.unpack_nibbles(packed)[0, 5] == 1  # code -7


def test_ties_round_to_even():
    # scale 0.25 exactly (max 1.75 / 7); w / s = 2.5, -2.5, 0.5, 1.5 are exact ties
    w = np.array([[0.625, -0.625, 0.125, 0.375, 1.75, 0.0, 0.0, 0.0]])
    packed, s = Q.quantize_int4(w, 8)
    assert float(s[0, 0]) == 0.25
    assert (Q.unpack_nibbles(packed)[0].astype(int) - 8).tolist() == [2, -2, 0, 2, 7, 0, 0, 0]


def test_zero_group():
    w = np.zeros((2, 64))
    w[1, 40] = 0.5
    packed, s = Q.quantize_int4(w, 32)
    assert float(s[0, 0]) == 0.0 and float(s[0, 1]) == 0.0 and float(s[1, 0]) == 0.0
    assert np.all(packed[0] == 0x88)
    assert np.all(Q.dequantize_int4(packed, s, 32)[0] == 0.0)


def test_dequant_matches_scalar_loops():
    rng = np.random.default_rng(3)
    N, K, g = 3, 16, 8
    packed = rng.integers(0, 256, (N, K // 2)).astype(np.uint8)
    s = rng.standard_normal((N, K // g)).astype(np.float16)
    ref = [[0.0] * K for _ in range(N)]
    for n in range(N):
        for k in range(K):
            byte = int(packed[n][k // 2])
            nib = (byte & 15) if k % 2 == 0 else (byte >> 4)
            ref[n][k] = (nib - 8) * float(s[n][k // g])
    assert np.array_equal(Q.dequantize_int4(packed, s, g), np.array(ref))


def test_rejects_bad_group():
    with pytest.raises(ValueError):
        Q.quantize_int4(np.zeros((1, 48)), 32)


def test_bf16_rounding_cases():
    one = 1.0
    # ties go to even
    assert Q.round_bf16(np.array([one + 2 ** -8]))[0] == one
    assert Q.round_bf16(np.array([one + 3 * 2 ** -8]))[0] == one + 2 ** -6
    # just above a tie rounds up even though float32 would first make it a tie
    assert Q.round_bf16(np.array([one + 2 ** -8 + 2 ** -40]))[0] == one + 2 ** -7
    assert Q.round_bf16(np.array([0.0, -0.0]))[0] == 0.0
    # smallest bf16 subnormal is 2^-133
    assert Q.round_bf16(np.array([2.0 ** -133 * 0.75]))[0] == 2.0 ** -133


def test_bf16_matches_float32_bit_rounding():
    # For inputs that are float32 values, round-to-nearest-even on the upper 16
    # bits of the float32 pattern is an independent route to the same result.
    x = S.random_vectors((4096,), seed=5, scale=0.02).astype(np.float32)
    b = x.view(np.uint32).astype(np.uint64)
    rounded = ((b + 0x7FFF + ((b >> 16) & 1)) >> 16).astype(np.uint16)
    assert np.array_equal(Q.bf16_bits(x.astype(np.float64)), rounded)
    assert np.array_equal(Q.bf16_from_bits(rounded), Q.round_bf16(x.astype(np.float64)))
