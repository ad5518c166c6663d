"""Host-side launch planning of the linear layer (CPU only, no device).

qlora_linear_plan reports the path, tiles and reduction splits the library
picks for a call.  These tests sweep shapes and SM counts and check what the
kernels rely on:
  - the path: generic exactly when r % 8 is nonzero (ragged K and N run on
    the tensor cores); the decode kernel exactly for a forward with 1 to 16
    tokens and K % 64 == 0; its persistent CTAs take every (tile, column
    chunk) unit once;
  - the tile grid covers the output exactly once and fits the launch limits;
  - a split reduction is used only when the tiles leave SMs idle, fits one
    cluster (<= 8 CTAs) and gives every CTA at least one step of the
    contiguous partition ceil(steps / splits) the kernels use (an empty
    split would add an unwritten accumulator);
  - sizes the calls reject are rejected by the plan query with the same code.
"""
import ctypes
import itertools

import pytest

from bit_nf4_quantized_12_b200 import binding


def cdiv(a, b):
    return -(-a // b)


def nonempty(steps, s):
    return s == 1 or (s - 1) * cdiv(steps, s) < steps


LOWRANK_STEPS = {  # 64-wide reduction steps of T, G, dA (hi and lo passes), dB
    0: lambda M, N, K: cdiv(K, 64),
    1: lambda M, N, K: cdiv(N, 64),
    2: lambda M, N, K: 2 * cdiv(M, 64),
    3: lambda M, N, K: cdiv(M, 64),
}


def check_plan(M, N, K, r, backward, sms):
    p = binding.plan(M, N, K, r, backward=backward, num_sms=sms)
    generic = r % 8 != 0
    if generic:
        assert p["path"] == binding.PATH_GENERIC
        assert p["lowrank_splits"] == [0, 0, 0, 0]
        return p
    if not backward and M <= 16 and K % 64 == 0:
        assert p["path"] == binding.PATH_DECODE
    if p["path"] == binding.PATH_DECODE:
        assert not backward and M <= 16 and K % 64 == 0
        assert p["tiles_w"] == cdiv(N, 256) and p["main_steps"] == cdiv(K, 256) and p["tiles_t"] == 1
        units = p["tiles_w"] * p["main_steps"]
        ctas = p["splits"]
        assert 1 <= ctas <= min(units, sms)
        # the stream-K ranges [p U / P, (p+1) U / P) tile the units, none empty
        begins = [q * units // ctas for q in range(ctas + 1)]
        assert begins[0] == 0 and begins[-1] == units and all(b1 > b0 for b0, b1 in zip(begins, begins[1:]))
    else:
        assert p["path"] == binding.PATH_FUSED
        bt = p["token_tile"]
        assert bt == (32 if M <= 32 else 64 if M <= 64 else 128 if M <= 128 else 256)
        assert p["tiles_t"] == cdiv(M, bt) and (p["tiles_t"] - 1) * bt < M <= p["tiles_t"] * bt
        assert p["tiles_t"] <= 65535
        assert p["tiles_w"] == cdiv(K if backward else N, 128)
        steps = cdiv(N, 64) if backward else cdiv(K, 64)
        assert p["main_steps"] == steps
        assert p["lora_steps"] == 2 * cdiv(r, 64)
        s = p["splits"]
        assert s in (1, 2, 4, 8)
        if s > 1:
            tiles = p["tiles_w"] * p["tiles_t"]
            assert tiles < sms and tiles * s <= sms
            assert steps // s >= 4 and nonempty(steps, s)
    kinds = (0, 1, 2, 3) if (backward and p["path"] == binding.PATH_FUSED) else (0,)
    for kind in range(4):
        s = p["lowrank_splits"][kind]
        if kind not in kinds:
            assert s == 0
            continue
        assert s in (1, 2, 4, 8)
        # beside a fused GEMM that fills the SMs unsplit: dA and dB unsplit, T at
        # most 2 ways while a partial stays within 128 steps
        gp = binding.plan(M, N, K, 64, backward=kind != 0, num_sms=sms)
        fills = M > 16 and gp["splits"] == 1
        if fills and kind >= 2:
            assert s == 1, (kind, s)
        if fills and kind == 1 and gp["tiles_w"] * gp["tiles_t"] < sms:
            assert s <= 2, s   # G beside a dX GEMM of less than one wave
        if fills and kind == 0 and cdiv(LOWRANK_STEPS[0](M, N, K), 2) <= 128:
            assert s <= 2, s
        if s > 1:
            assert nonempty(LOWRANK_STEPS[kind](M, N, K), s), (kind, s)
    return p


MS = [1, 2, 16, 31, 32, 33, 64, 65, 127, 128, 129, 256, 257, 512, 2047, 2048, 4096, 16384]
NS = [8, 64, 128, 136, 640, 1024, 4096, 11008, 28672]
KS = [64, 128, 192, 256, 1024, 4096, 8192, 28672]
RS = [8, 16, 64, 72, 128, 256]


@pytest.mark.parametrize("sms", [148, 132, 16, 1])
@pytest.mark.parametrize("backward", [0, 1])
def test_fused_plans_sweep(sms, backward):
    for M, N, K, r in itertools.product(MS, NS, KS, RS):
        check_plan(M, N, K, r, backward, sms)


def test_every_split_count_is_exercised():
    """The sweep reaches splits of 2, 4 and 8 for the fused product and of 2,
    4 and 8 for the low-rank kernels (4 and 8 only beside the decode kernel,
    at 1-16 tokens), so the invariants above are not vacuous."""
    seen_main, seen_low = set(), set()
    for M, N, K, r in itertools.product(MS, NS, KS, RS[:3]):
        for backward in (0, 1):
            p = check_plan(M, N, K, r, backward, 148)
            if p["path"] == binding.PATH_FUSED:
                seen_main.add(p["splits"])
            seen_low.update(p["lowrank_splits"])
    assert {1, 2, 4, 8} <= seen_main
    assert {1, 2, 4, 8} <= seen_low


@pytest.mark.parametrize("M,N,K,r", [(33, 40, 1000, 12), (1, 96, 130, 4), (1, 4096, 4096, 12), (5, 24, 100, 3)])
def test_ranks_off_the_granule_take_the_generic_path(M, N, K, r):
    for backward in (0, 1):
        assert check_plan(M, N, K, r, backward, 148)["path"] == binding.PATH_GENERIC


@pytest.mark.parametrize("M,N,K,r", [(5, 24, 100, 8), (17, 13, 64, 8), (4096, 4095, 11007, 8), (4, 4095, 4096, 8),
                                     (1, 8, 4100, 16), (2048, 11008, 4095, 64)])
def test_ragged_shapes_take_the_tensor_cores(M, N, K, r):
    """K % 64 != 0 (rows not starting on an NF4 block) and N % 8 != 0 run on
    the tensor cores: the fused GEMM, or the decode kernel for a forward with
    up to 16 tokens whose rows start on blocks."""
    for backward in (0, 1):
        p = check_plan(M, N, K, r, backward, 148)
        want = binding.PATH_DECODE if (not backward and M <= 16 and K % 64 == 0) else binding.PATH_FUSED
        assert p["path"] == want
        assert binding.workspace_bytes(M, N, K, r) < N * K * 2 or M * (K + N) * 2 >= N * K  # no copy of Wd


def test_plans_match_the_calls_limits():
    L = binding.lib()
    out = binding.QloraPlan()
    max_fused = 65535 * 256
    cases = [
        ((max_fused, 4096, 64, 8), 0),
        ((max_fused + 1, 4096, 64, 8), 3),       # token tiles beyond grid.y
        ((max_fused + 1, 4096, 100, 8), 3),      # ragged K runs on the fused grid too
        ((max_fused + 1, 4096, 100, 12), 0),     # the generic path walks its tiles
        ((1 << 31, 8, 64, 8), 3),
        ((1 << 31, 8, 100, 12), 0),
        (((1 << 31) + 1, 8, 100, 12), 3),
        ((16, 1 << 31, 1 << 31, 12), 3),         # Wd copy beyond 2^40 elements
        ((0, 64, 64, 8), 1),
        ((16, 64, 64, 0), 1),
        ((16, 64, 64, 257), 1),
    ]
    for (M, N, K, r), code in cases:
        for backward in (0, 1):
            assert L.qlora_linear_plan(M, N, K, r, backward, 148, ctypes.byref(out)) == code, (M, N, K, r)
        assert (L.qlora_workspace_bytes(M, N, K, r) == 0) == (code != 0)
    assert L.qlora_linear_plan(16, 64, 64, 8, 0, 148, None) == 1


def test_fused_call_rejects_too_many_tokens_before_launch():
    """The forward and backward return NF4_ERR_UNSUPPORTED on the host for a
    token count the fused grid cannot hold (fake pointers: nothing is read)."""
    L = binding.lib()
    fake = ctypes.c_void_p(0x10000)
    w = binding.NF4Weight(0x10000, 0x10000, 0x10000, 4096, 64)
    M = 65535 * 256 + 1
    assert L.qlora_linear_fwd(fake, M, w, fake, fake, 8, 1.0, fake, None, fake, 1 << 62, None) == 3
    assert L.qlora_linear_bwd(fake, fake, M, w, fake, fake, 8, 1.0, None, fake, fake, fake, fake, 1 << 62,
                              None) == 3

