"""Pins for the oracle's quantize / double-quantize / dequantize (CPU only).

  - nearest-code search against exact rational brute force (Fraction);
  - the cheap fp32 reading used on the GPU (x = w * fp32(1/absmax), compare
    with fp32 midpoints rounded down) gives the same code as the exact
    quotient for every bf16 pair -- enumerated, so the kernel's arithmetic is
    a valid implementation of the oracle's definition;
  - byte layout, ragged tails, all-zero blocks, non-finite flag;
  - an exact round trip on codebook-valued inputs;
  - the bits-per-weight figures the pages print ("QLoRA 原理精讲" §2.2, §2.4).
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


@pytest.fixture(scope="module")
def codes():
    return oracle.codebook()


def _brute_nearest(codes, w, a):
    if a == 0:
        return 7
    x = Fraction(float(w)) / Fraction(float(a))
    d = [abs(x - Fraction(float(c))) for c in codes]
    return min(range(16), key=lambda k: (d[k], k))


def test_nearest_code_brute_force(codes):
    rng = np.random.default_rng(3)
    w, a = [], []
    # random bf16 pairs with |w| <= absmax
    for _ in range(3000):
        av = np.float32(np.exp2(rng.uniform(-20, 20)))
        a.append(_f32(_bf16_bits(av)))
        w.append(_f32(_bf16_bits(np.float32(rng.uniform(-1, 1)) * a[-1])))
    # fp32 values straddling every midpoint (absmax 1 and absmax 3)
    for i in range(15):
        mid = (np.float64(codes[i]) + np.float64(codes[i + 1])) / 2
        for scale in (1.0, 3.0):
            m = np.float32(mid * scale)
            for k in range(-3, 4):
                w.append(np.float32(np.nextafter(m, np.float32(np.inf * np.sign(k))) if k else m))
                a.append(np.float32(scale))
    w = np.array(w, np.float32).reshape(-1)
    a = np.array(a, np.float32).reshape(-1)
    got = oracle.nearest_code(w, a)
    want = np.array([_brute_nearest(codes, wi, ai) for wi, ai in zip(w, a)])
    assert np.array_equal(got, want)


def test_nearest_code_ties_go_low(codes):
    hit = 0
    for i in range(15):
        mid = (np.float64(codes[i]) + np.float64(codes[i + 1])) / 2
        if np.float64(np.float32(mid)) == mid:        # representable: an exact tie
            assert oracle.nearest_code(np.array([mid], np.float32), np.float32(1))[0] == i
            hit += 1
    # build ties with absmax != 1: w = mid * a exactly representable
    for i in range(15):
        mid = Fraction(float(codes[i])) + Fraction(float(codes[i + 1]))
        mid /= 2
        for a in (0.5, 2.0, 0.25):
            w = float(mid * Fraction(a))
            if Fraction(float(np.float32(w))) == mid * Fraction(a):
                assert oracle.nearest_code(np.array([w], np.float32), np.float32(a))[0] == i
                hit += 1
    assert hit >= 1


def test_fp32_reciprocal_reading_equals_exact_for_all_bf16_pairs(codes):
    """Every normal bf16 absmax significand (exponent fixed: only w/absmax
    matters) against every bf16 w with |w| <= absmax."""
    mids = (codes[:-1].astype(np.float64) + codes[1:].astype(np.float64)) / 2
    T = mids.astype(np.float32)
    T = np.where(T.astype(np.float64) > mids, np.nextafter(T, np.float32(-np.inf)), T)
    wb = np.arange(0, 0x7F80, dtype=np.uint32)
    wabs = _f32(wb)
    for m in range(128):
        a = _f32(np.array([(127 << 7) | m]))[0]           # absmax in [1, 2)
        w = wabs[wabs <= a]
        w = np.concatenate([w, -w]).astype(np.float32)
        inv = np.float32(1.0) / a
        x = w * inv                                          # float32 RN
        q_fast = np.searchsorted(T, x, side="left").astype(np.int32)   # #{T_i < x}
        q_exact = oracle.nearest_code(w, a)
        assert np.array_equal(q_fast, q_exact), m


def test_packing_layout_and_constants(codes):
    # element e = code[e % 16] exactly: every block has absmax 1
    n = 64 * 256 * 2
    W = _bf16_bits(codes[np.arange(n) % 16])
    packed, c1q, c2, bad = oracle.quantize(W)
    assert not bad
    assert packed.size == n // 2 and c1q.size == n // 64 and c2.size == 2
    q = _f32(W)
    exp_q = np.array([oracle.nearest_code(np.array([v], np.float32), np.float32(1))[0] for v in q[:16]])
    # codes that are not bf16-exact still land on their own index
    assert np.array_equal(exp_q, np.arange(16))
    assert np.all(packed[:8] == np.array([0x10, 0x32, 0x54, 0x76, 0x98, 0xBA, 0xDC, 0xFE], np.uint8))
    # absmax 1 everywhere: scale2 = 1/448, scale1 code = E4M3(1/(1/448)) = 448
    assert np.all(c2 == np.float32(1.0) / np.float32(448.0))
    assert np.all(c1q == 0x7E)


def test_ragged_tail_and_zero_blocks():
    rng = np.random.default_rng(9)
    n = 64 * 256 + 64 + 1                       # 2 groups; last block of 1 element
    x = rng.standard_normal(n).astype(np.float32) * 0.02
    x[64:128] = 0.0                             # an all-zero block
    x[128:192] = -0.0
    W = _bf16_bits(x)
    packed, c1q, c2, bad = oracle.quantize(W)
    assert not bad
    assert packed.size == (n + 1) // 2 and c1q.size == 258 and c2.size == 2
    assert packed[-1] >> 4 == 0                 # pad nibble
    assert c1q[1] == 0 and c1q[2] == 0
    assert np.all(packed[32:96] == 0x77)        # zero blocks -> code of 0.0
    # the one-element final block: its absmax is |w|, so its code is +-1
    last = _f32(W[-1:])[0]
    assert (packed[-1] & 0xF) == (15 if last > 0 else 0)
    # second group holds 2 blocks: scale2 from their absmax
    a = np.abs(_f32(W[64 * 256:]))
    assert c2[1] == np.float32(max(a[:64].max(), a[64:].max())) / np.float32(448)
    d = oracle.dequant(packed, c1q, c2, n)
    assert np.all(_f32(d[64:192]) == 0)


def test_nonfinite_flag():
    for bad in (np.nan, np.inf, -np.inf):
        x = np.zeros(300, np.float32)
        x[200] = bad
        *_, flag = oracle.quantize(_bf16_bits(x))
        assert flag
    *_, flag = oracle.quantize(_bf16_bits(np.ones(300, np.float32)))
    assert not flag


def test_round_trip_exact_on_codebook_values(codes):
    """scale1_b = e_b * 2^-k with e_b an E4M3 value, one e_b = 448 per group,
    every block holding a +-1 code: scale2 = 2^-k and scale1 codes e_b are
    exact, the codes come back, and dequantization returns the input bits."""
    rng = np.random.default_rng(21)
    e4m3_vals = np.array([oracle.e4m3_decode(c) for c in range(0x08, 0x7F)], np.float64)
    nb = 256 * 3
    e = rng.choice(e4m3_vals, nb)
    e[0] = e[256] = e[512] = 448.0
    k = 12
    S = (e * 2.0 ** -k).astype(np.float32)
    q = rng.integers(0, 16, (nb, 64))
    q[:, 5] = rng.choice([0, 15], nb)
    vals = (codes[q].astype(np.float32) * S[:, None]).astype(np.float32)   # fp32 RN product
    W = _bf16_bits(vals).reshape(-1)
    packed, c1q, c2, bad = oracle.quantize(W)
    assert not bad
    assert np.all(c2 == np.float32(2.0 ** -k))
    assert np.array_equal(np.array([oracle.e4m3_decode(c) for c in c1q]), e)
    got_q = np.empty(nb * 64, np.int64)
    got_q[0::2] = packed & 0xF
    got_q[1::2] = packed >> 4
    assert np.array_equal(got_q, q.reshape(-1))
    assert np.array_equal(oracle.dequant(packed, c1q, c2, W.size), W)


def test_dequant_is_fp32_multiply_then_bf16_round(codes):
    # reduces to a library routine: torch fp32 multiply then cast to bf16
    c2 = np.array([np.float32(0.0123)], np.float32)
    c1q = np.arange(256, dtype=np.uint8)
    c1q = c1q[(c1q & 0x7F) != 0x7F][:255]            # drop NaN codes
    c1q = c1q[c1q < 0x80]                            # non-negative scales only
    nb = c1q.size
    q = np.tile(np.arange(16), 4 * nb)[: nb * 64]
    packed = (q[0::2] | (q[1::2] << 4)).astype(np.uint8)
    # one group per block: pad c1q to a full group is unnecessary (nb <= 256)
    d = oracle.dequant(packed, c1q, c2, nb * 64)
    s1 = torch.tensor([oracle.e4m3_decode(c) for c in c1q], dtype=torch.float32) * float(c2[0])
    ref = (torch.from_numpy(codes)[torch.from_numpy(q.reshape(nb, 64))] * s1[:, None]).to(torch.bfloat16)
    assert np.array_equal(d, ref.view(torch.int16).numpy().view(np.uint16).reshape(-1))


def test_quantization_error_bound(codes):
    rng = np.random.default_rng(2)
    x = rng.standard_normal(64 * 256 * 4).astype(np.float32) * 0.02
    W = _bf16_bits(x)
    packed, c1q, c2, _ = oracle.quantize(W)
    d = _f32(oracle.dequant(packed, c1q, c2, W.size)).astype(np.float64)
    w = _f32(W).astype(np.float64)
    a = np.abs(w).reshape(-1, 64).max(1)
    half_gap = np.max(np.diff(codes.astype(np.float64))) / 2
    # nearest-code error + E4M3 scale error (3 mantissa bits: <= 2^-4) + bf16 rounding
    bound = a * (half_gap + 2.0 ** -4 * (1 + half_gap)) + a * 2.0 ** -8
    assert np.all(np.abs(d - w).reshape(-1, 64) <= bound[:, None])


def test_bits_per_weight_match_pages():
    g = _golden()
    assert g["block_size"] == oracle.BLOCK and g["group_size"] == oracle.GROUP
    assert oracle.codebook().size == g["codebook_size"]
    n = 4096 * 4096
    assert oracle.nblocks(n) * 32 / n == g["dq_off_bits_per_weight"]
    dq = (oracle.nblocks(n) * 8 + oracle.ngroups(n) * 32) / n
    assert abs(dq - g["dq_on_bits_per_weight"]) < 5e-4            # 0.126953
    assert abs(70e9 * 0.5 / 8 / 1e9 - g["dq_off_70b_gb"]) < 0.05
    assert abs(70e9 * (0.5 - dq) / 8 / 1e9 - g["dq_saved_70b_gb"]) < 0.05
    # the 70B-shaped layer set: 80 layers of the LLaMA-70B matrices
    from bit_nf4_quantized_12_b200.workloads import LLAMA70B
    total = 0
    for _, N, K in LLAMA70B:
        numel = N * K
        total += oracle.packed_bytes(numel) + oracle.nblocks(numel) + 4 * oracle.ngroups(numel)
    total *= 80
    params = 80 * sum(N * K for _, N, K in LLAMA70B)
    assert abs(total / 1e9 - g["nf4_base_70b_gb"]) < 1.0            # 35.31 GB
    assert abs(params * 2 / 1e9 - g["bf16_base_70b_gb"]) < 5.0       # 136.9 GB
