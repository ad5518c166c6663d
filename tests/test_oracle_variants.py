"""Pins for the oracle's format variants, its FP16 compute type and its LoRA
merge (CPU only).

  - fp16 rounding and decoding against numpy's float16 (an independent
    implementation of IEEE binary16) and exact rational brute force;
  - the INT4 table by its closed form (the 16 integers [-8, 7] of "QLoRA
    原理精讲" §2.1, evenly spaced), nearest-code search on it by rational brute
    force;
  - each first-level-constant format by an exact round trip on inputs built
    so that the stored constants are exact, and by the bits per weight the
    pages print ("QLoRA 原理精讲" §2.2);
  - the default format through the variant entry points equals the pinned
    default functions bit for bit;
  - dequantization into fp16 equals torch's fp32 multiply then fp16 cast;
  - the LoRA merge: A = 0 or s = 0 gives back Wd, and the merged weight
    reproduces the unmerged forward exactly on integer problems with
    non-square shapes (a transposed operand or a dropped term fails it);
  - the linear layer in FP16: the same exact identities as in bf16.
"""
from fractions import Fraction
import os

import numpy as np
import pytest
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "pages_numbers.txt")


def _golden():
    out = {}
    for line in open(GOLDEN, encoding="utf-8"):
        line = line.split("#", 1)[0].strip()
        if line:
            k, v = line.split("=")
            out[k.strip()] = float(v)
    return out


def _bf16_bits(x):
    return torch.from_numpy(np.asarray(x, np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def _f32(bits):
    return (np.asarray(bits, np.uint32) << 16).view(np.float32)


# ------------------------------------------------------------------ fp16
def test_f16_decode_all_patterns():
    h = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ref = h.view(np.float16).astype(np.float64)
    got = oracle.f16_to_f64(h)
    nan = np.isnan(ref)
    assert np.array_equal(nan, np.isnan(got))
    assert np.array_equal(ref[~nan], got[~nan])


def test_f16_round_matches_numpy_and_brute_force():
    rng = np.random.default_rng(5)
    # every fp16 value, every midpoint between neighbours, and their float64 neighbours
    v = np.arange(0, 0x7C00, dtype=np.uint16).view(np.float16).astype(np.float64)
    mids = (v[:-1] + v[1:]) / 2
    pts = np.concatenate([v, mids, np.nextafter(mids, np.inf), np.nextafter(mids, -np.inf),
                          rng.uniform(0, 70000, 200_000), np.exp2(rng.uniform(-30, 16, 200_000)),
                          [65504.0, 65519.999, 65520.0, 1e6, 2.0 ** -25, 2.0 ** -24 * 1.5]])
    x = np.concatenate([pts, -pts])
    got = oracle.f16_round(x)
    with np.errstate(over="ignore"):
        ref = x.astype(np.float16).view(np.uint16)
    assert np.array_equal(got, ref)
    # brute force on a sample: the nearest fp16 value, ties to an even significand
    vals = np.arange(0, 0x7C00, dtype=np.uint16)
    fv = [Fraction(float(t)) for t in vals.view(np.float16).astype(np.float64)]
    for xv in rng.choice(pts[pts < 65504], 300):
        X = Fraction(float(xv))
        i = int(np.searchsorted(vals.view(np.float16).astype(np.float64), xv))
        cands = [j for j in (i - 1, i) if 0 <= j < len(vals)]
        best = min(cands, key=lambda j: (abs(fv[j] - X), int(vals[j]) & 1))
        assert oracle.f16_round(np.array([xv]))[0] == vals[best]


# ------------------------------------------------------------------ INT4 table
def test_int4_codebook_closed_form():
    c = oracle.codebook_int4()
    assert np.array_equal(c.astype(np.float64), (np.arange(16) - 8) / 8.0)
    assert np.all(np.diff(c) == np.float32(0.125)) and c[8] == 0.0 and c[0] == -1.0


def test_int4_nearest_code_brute_force():
    codes = oracle.codebook_int4()
    rng = np.random.default_rng(8)
    w, a = [], []
    for _ in range(3000):
        av = np.float32(np.exp2(rng.uniform(-20, 20)))
        a.append(_f32(_bf16_bits(av)))
        w.append(_f32(_bf16_bits(np.float32(rng.uniform(-1, 1)) * a[-1])))
    for i in range(15):                        # exact ties and their neighbours
        mid = np.float32((float(codes[i]) + float(codes[i + 1])) / 2)
        for k in range(-2, 3):
            w.append(np.float32(np.nextafter(mid, np.float32(np.inf * np.sign(k))) if k else mid))
            a.append(np.float32(1.0))
    w = np.array(w, np.float32).reshape(-1)
    a = np.array(a, np.float32).reshape(-1)

    def brute(wi, ai):
        if ai == 0:
            return 8
        x = Fraction(float(wi)) / Fraction(float(ai))
        return min(range(16), key=lambda k: (abs(x - Fraction(float(codes[k]))), k))

    got = oracle.nearest_code_fmt(oracle.QUANT_INT4, w, a)
    assert np.array_equal(got, np.array([brute(wi, ai) for wi, ai in zip(w, a)]))


def test_int4_zero_block_and_round_trip():
    codes = oracle.codebook_int4()
    rng = np.random.default_rng(12)
    nb = 256 * 2
    q = rng.integers(0, 16, (nb, 64))
    q[:, 3] = 0                                # every block holds -1: absmax = its scale
    S = np.exp2(rng.integers(-20, -2, nb)).astype(np.float32)
    vals = (codes[q] * S[:, None]).astype(np.float32)     # exact: k/8 * 2^e
    vals[7] = 0.0                              # an all-zero block
    q[7] = 8
    W = _bf16_bits(vals).reshape(-1)
    for dq in (oracle.DQ_NONE, oracle.DQ_E4M3, oracle.DQ_U8):
        packed, c1, c2, bad = oracle.quantize_fmt(W, oracle.QUANT_INT4, dq)
        assert not bad
        got_q = np.empty(W.size, np.int64)
        got_q[0::2] = packed & 0xF
        got_q[1::2] = packed >> 4
        assert np.array_equal(got_q, q.reshape(-1))
        if dq == oracle.DQ_NONE:                # FP32 scale1 is exact: the round trip is too
            assert np.array_equal(oracle.dequant_fmt(packed, c1, c2, W.size, oracle.QUANT_INT4, dq), W)


# ------------------------------------------------------------------ first-level constants
def test_default_format_through_variant_entry_points():
    rng = np.random.default_rng(4)
    for n in (1, 63, 64 * 256 + 65, 3 * 16384):
        W = _bf16_bits(rng.standard_normal(n).astype(np.float32) * 0.02)
        a = oracle.quantize(W)
        b = oracle.quantize_fmt(W, oracle.QUANT_NF4, oracle.DQ_E4M3)
        for x, y in zip(a[:3], b[:3]):
            assert np.array_equal(x.view(np.uint8), y.view(np.uint8))
        assert np.array_equal(oracle.dequant(*a[:3], n), oracle.dequant_fmt(*b[:3], n))


def test_fp32_scale1_is_the_block_absmax_and_round_trips():
    codes = oracle.codebook()
    rng = np.random.default_rng(6)
    nb = 300                                    # ragged last group
    q = rng.integers(0, 16, (nb, 64))
    q[:, 9] = rng.choice([0, 15], nb)
    S = np.exp2(rng.integers(-30, 10, nb)).astype(np.float32)   # any power of two per block
    vals = (codes[q].astype(np.float32) * S[:, None]).astype(np.float32)
    W = _bf16_bits(vals).reshape(-1)
    packed, c1, c2, bad = oracle.quantize_fmt(W, oracle.QUANT_NF4, oracle.DQ_NONE)
    assert not bad and c1.dtype == np.float32 and c2.size == 0
    assert np.array_equal(c1, np.abs(_f32(W)).reshape(nb, 64).max(1))
    assert np.array_equal(oracle.dequant_fmt(packed, c1, c2, W.size, oracle.QUANT_NF4, oracle.DQ_NONE), W)


def test_u8_scale1_round_trip():
    """scale1_b = m_b * 2^-k with integers m_b <= 255, one m_b = 255 per group,
    every block holding a +-1 code: scale2 = 255 * 2^-k / 255 = 2^-k exactly,
    the 8-bit codes are the m_b, and dequantization returns the input."""
    codes = oracle.codebook()
    rng = np.random.default_rng(10)
    nb = 256 * 2 + 17
    m = rng.integers(1, 256, nb)
    m[0] = m[256] = m[512] = 255
    k = 14
    S = (m * 2.0 ** -k).astype(np.float32)
    q = rng.integers(0, 16, (nb, 64))
    q[:, 2] = rng.choice([0, 15], nb)
    vals = (codes[q].astype(np.float32) * S[:, None]).astype(np.float32)
    W = _bf16_bits(vals).reshape(-1)
    packed, c1, c2, bad = oracle.quantize_fmt(W, oracle.QUANT_NF4, oracle.DQ_U8)
    assert not bad
    assert np.all(c2 == np.float32(2.0 ** -k))
    assert np.array_equal(c1.astype(np.int64), m)
    assert np.array_equal(oracle.dequant_fmt(packed, c1, c2, W.size, oracle.QUANT_NF4, oracle.DQ_U8), W)


def test_u8_codes_order_and_zero_group():
    rng = np.random.default_rng(11)
    x = rng.standard_normal(64 * 256).astype(np.float32) * 0.02
    x[:64] = 0.0
    W = _bf16_bits(np.concatenate([x, np.zeros(64 * 256, np.float32)]))
    packed, c1, c2, _ = oracle.quantize_fmt(W, oracle.QUANT_NF4, oracle.DQ_U8)
    a = np.abs(_f32(W[:64 * 256])).reshape(256, 64).max(1)
    order = np.argsort(a, kind="stable")
    assert np.all(np.diff(c1[:256][order].astype(np.int64)) >= 0)     # monotone in scale1
    assert c1[0] == 0 and c1[:256].max() == 255
    assert c2[1] == 0 and np.all(c1[256:] == 0)                       # an all-zero group
    assert np.all(packed[64 * 128:] == 0x77)


def test_bits_per_weight_of_the_variants():
    g = _golden()
    n = 4096 * 4096
    nb, ng = oracle.nblocks(n), oracle.ngroups(n)
    W = np.zeros(n, np.uint16)
    for dq, expect, tol in ((oracle.DQ_NONE, g["dq_off_bits_per_weight"], 0.0),
                            (oracle.DQ_E4M3, g["dq_on_bits_per_weight"], 5e-4),
                            (oracle.DQ_U8, g["dq_on_bits_per_weight"], 5e-4)):
        _, c1, c2, _ = oracle.quantize_fmt(W[:64 * 256 * 2], oracle.QUANT_NF4, dq)
        per_block = c1.itemsize * 8
        bits = (nb * per_block + (ng * 32 if c2.size else 0)) / n
        assert abs(bits - expect) <= tol, (dq, bits)


def test_dequant_to_f16_is_fp32_multiply_then_f16_round():
    codes = oracle.codebook()
    c2 = np.array([np.float32(0.0123)], np.float32)
    c1q = np.arange(0x7F, dtype=np.uint8)[: 255]
    nb = c1q.size
    q = np.tile(np.arange(16), 4 * nb)[: nb * 64]
    packed = (q[0::2] | (q[1::2] << 4)).astype(np.uint8)
    d = oracle.dequant_fmt(packed, c1q, c2, nb * 64, dtype=oracle.F16)
    s1 = torch.tensor([oracle.e4m3_decode(c) for c in c1q], dtype=torch.float32) * float(c2[0])
    ref = (torch.from_numpy(codes)[torch.from_numpy(q.reshape(nb, 64))] * s1[:, None]).to(torch.float16)
    assert np.array_equal(d, ref.view(torch.int16).numpy().view(np.uint16).reshape(-1))


# ------------------------------------------------------------------ LoRA merge
def _ints(rng, shape, lo=-3, hi=4):
    return rng.integers(lo, hi, shape).astype(np.float64)


@pytest.mark.parametrize("dtype", [oracle.BF16, oracle.F16])
def test_merge_identities(dtype):
    rnd = oracle.f16_round if dtype == oracle.F16 else oracle.bf16_round
    rng = np.random.default_rng(13)
    N, K, r = 7, 9, 3
    Wd = rnd(rng.standard_normal((N, K)) * 0.02)
    A, B = rnd(rng.standard_normal((K, r)) * 0.01), rnd(rng.standard_normal((r, N)) * 0.01)
    Wm, _ = oracle.lora_merge(Wd, rnd(np.zeros((K, r))), B, 0.5, dtype)
    assert np.array_equal(Wm, Wd)
    Wm, _ = oracle.lora_merge(Wd, A, B, 0.0, dtype)
    assert np.array_equal(Wm, Wd)


@pytest.mark.parametrize("dtype", [oracle.BF16, oracle.F16])
def test_merged_weight_reproduces_the_unmerged_forward(dtype):
    """X W'^T = X Wd^T + s (X A) B exactly when nothing rounds: integer inputs
    small enough that T and the merged weight are exact in the compute type."""
    rnd = oracle.f16_round if dtype == oracle.F16 else oracle.bf16_round
    rng = np.random.default_rng(14)
    M, N, K, r = 5, 7, 9, 3
    X, W, A, B = _ints(rng, (M, K)), _ints(rng, (N, K)), _ints(rng, (K, r), -2, 3), _ints(rng, (r, N), -2, 3)
    for s in (1.0, 0.5, 2.0):
        Wm, exact = oracle.lora_merge(rnd(W), rnd(A), rnd(B), s, dtype)
        assert np.array_equal(oracle._f64(Wm, dtype), exact)            # exact in the compute type
        Y, _ = oracle.qlora_fwd(rnd(X), rnd(W), rnd(A), rnd(B), s, dtype=dtype)
        assert np.array_equal(X @ exact.T, Y)


def test_merge_rounds_once():
    rng = np.random.default_rng(15)
    N, K, r = 16, 24, 8
    Wd = oracle.bf16_round(rng.standard_normal((N, K)) * 0.02)
    A = oracle.bf16_round(rng.standard_normal((K, r)) * 0.01)
    B = oracle.bf16_round(rng.standard_normal((r, N)) * 0.01)
    Wm, exact = oracle.lora_merge(Wd, A, B, 0.25)
    assert np.array_equal(Wm, oracle.bf16_round(exact))
    d = np.abs(oracle.bf16_to_f64(Wm) - exact)
    assert np.all(d <= np.abs(exact) * 2.0 ** -8)                     # within half a bf16 spacing


# ------------------------------------------------------------------ linear layer in fp16
def test_f16_linear_identities():
    rnd = oracle.f16_round
    rng = np.random.default_rng(16)
    M, N, K, R = 5, 7, 9, 3
    X, W, A, B = _ints(rng, (M, K)), _ints(rng, (N, K)), _ints(rng, (K, R), -2, 3), _ints(rng, (R, N))
    dY = _ints(rng, (M, N))
    s = 0.25
    Y0, _ = oracle.qlora_fwd(rnd(X), rnd(np.zeros((N, K))), rnd(A), rnd(B), s, dtype=oracle.F16)
    assert np.array_equal(Y0, s * (X @ A) @ B)
    Y1, T = oracle.qlora_fwd(rnd(X), rnd(W), rnd(np.zeros((K, R))), rnd(B), s, dtype=oracle.F16)
    assert np.array_equal(Y1, X @ W.T)

    def f(X_, A_, B_):
        Y, _ = oracle.qlora_fwd(rnd(X_), rnd(W), rnd(A_), rnd(B_), s, dtype=oracle.F16)
        return np.sum(dY * Y)

    _, T = oracle.qlora_fwd(rnd(X), rnd(W), rnd(A), rnd(B), s, dtype=oracle.F16)
    dX, dA, dB = oracle.qlora_bwd(rnd(dY), rnd(X), rnd(W), rnd(A), rnd(B), s, T, dtype=oracle.F16)
    base = f(X, A, B)
    for _ in range(4):
        V = _ints(rng, (M, K), -1, 2)
        assert f(X + V, A, B) - base == np.sum(dX * V)
        Va = _ints(rng, (K, R), -1, 2)
        assert f(X, A + Va, B) - base == np.sum(dA * Va)
        Vb = _ints(rng, (R, N), -1, 2)
        assert f(X, A, B + Vb) - base == np.sum(dB * Vb)
