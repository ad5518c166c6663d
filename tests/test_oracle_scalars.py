"""Pins for the oracle's scalar formats: FP8 E4M3 and bf16 rounding (CPU only).

E4M3 is checked against torch's float8_e4m3fn conversion (an independent
implementation of the same OCP format); bf16 rounding against torch's
fp32->bf16 cast and, for float64 inputs, exact rational brute force.
"""
from fractions import Fraction
import math

import numpy as np
import torch

import oracle


def _torch_e4m3(x):
    return torch.from_numpy(np.asarray(x, np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def test_e4m3_decode_all_codes():
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8).view(torch.float8_e4m3fn)
    ref = codes.to(torch.float32).numpy().astype(np.float64)
    got = np.array([oracle.e4m3_decode(c) for c in range(256)])
    nan = np.isnan(ref)
    assert np.array_equal(nan, np.isnan(got))
    assert nan.sum() == 2                       # 0x7F and 0xFF
    assert np.array_equal(ref[~nan], got[~nan])
    assert got[0x7E] == 448.0 and got[0x01] == 2.0 ** -9


def test_e4m3_encode_matches_library_in_range():
    vals = np.array([oracle.e4m3_decode(c) for c in range(0x7F)], np.float64)
    pts = np.concatenate([vals, (vals[:-1] + vals[1:]) / 2]).astype(np.float32)
    # every float within 64 ulps of each code and each midpoint (ties)
    bits = pts.view(np.uint32).astype(np.int64)
    near = (bits[:, None] + np.arange(-64, 65)[None, :]).reshape(-1)
    near = near[(near >= 0) & (near <= np.float32(448.0).view(np.uint32))]
    x = near.astype(np.uint32).view(np.float32)
    rng = np.random.default_rng(7)
    x = np.concatenate([x, rng.uniform(0, 448, 1_000_000).astype(np.float32),
                        np.exp2(rng.uniform(-12, 8.8, 200_000)).astype(np.float32)])
    x = x[x <= 448]
    assert np.array_equal(oracle.e4m3_encode(x), _torch_e4m3(x))
    assert np.array_equal(oracle.e4m3_encode(-x), _torch_e4m3(-x))


def test_e4m3_encode_saturates_and_nan():
    big = np.array([448.0001, 464.0, 479.9, 480.0, 1e6, 3.4e38, np.inf], np.float32)
    assert np.all(oracle.e4m3_encode(big) == 0x7E)
    assert np.all(oracle.e4m3_encode(-big) == 0xFE)
    assert oracle.e4m3_encode(np.array([np.nan], np.float32))[0] == 0x7F


def test_bf16_decode_all_patterns():
    b = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ref = torch.from_numpy(b.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    got = oracle.bf16_to_f64(b)
    nan = np.isnan(ref)
    assert np.array_equal(nan, np.isnan(got))
    assert np.array_equal(ref[~nan], got[~nan])


def test_bf16_round_matches_library_on_fp32_inputs():
    rng = np.random.default_rng(11)
    u = rng.integers(0, 2 ** 32, 2_000_000, dtype=np.uint64).astype(np.uint32)
    # ties: low 16 bits exactly 0x8000; and neighbours of ties
    ties = (u & 0xFFFF0000) | 0x8000
    x = np.concatenate([u, ties, ties + 1, ties - 1]).view(np.float32)
    x = x[np.isfinite(x)]
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = oracle.bf16_round(x.astype(np.float64))
    assert np.array_equal(ref, got)


def _bf16_exact(b):
    return Fraction(float(oracle.bf16_to_f64(np.array([b], np.uint16))[0]))


def test_bf16_round_float64_inputs_brute_force():
    # a float64 just above/below a bf16 midpoint must not double-round
    rng = np.random.default_rng(5)
    for _ in range(2000):
        b = int(rng.integers(0x0080, 0x7F7F))
        lo, hi = _bf16_exact(b), _bf16_exact(b + 1)
        mid = (lo + hi) / 2
        for x in (float(mid), math.nextafter(float(mid), math.inf), math.nextafter(float(mid), -math.inf),
                  float(lo + (hi - lo) * Fraction(int(rng.integers(1, 1000)), 1000))):
            fx = Fraction(x)
            want = b if abs(fx - lo) < abs(hi - fx) else b + 1
            if abs(fx - lo) == abs(hi - fx):
                want = b if b % 2 == 0 else b + 1
            assert int(oracle.bf16_round(np.array([x]))[0]) == want
            assert int(oracle.bf16_round(np.array([-x]))[0]) == want | 0x8000
    assert oracle.bf16_round(np.array([1e39]))[0] == 0x7F80
    assert oracle.bf16_round(np.array([-0.0]))[0] == 0x8000
