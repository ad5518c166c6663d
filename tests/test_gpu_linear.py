"""GPU parity of the QLoRA linear layer (forward, backward, decode shapes)
against the float64 oracle, with the layer's stated tolerance:
relative Frobenius <= 2e-3, elementwise relative <= 1e-2 (denominator
floored at 1e-2 x rms of the reference)."""
import numpy as np
import pytest
import torch

import oracle
from bit_nf4_quantized_12_b200 import binding, workloads
from gpu_helpers import (bf16_rounded, bits, f64, gpu_quantize, oracle_dequant_full, oracle_dequant_rows,
                         tol_check)

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _problem(M, N, K, r, seed, w_std=0.02, kind="normal"):
    W = workloads.weight(N, K, w_std, seed=seed, device=DEV, kind=kind)
    io = workloads.layer_inputs(M, N, K, r, seed=seed, device=DEV)
    return W, io


def _run(M, N, K, r, s, seed, rows=None, check_bwd=True, W=None, io=None):
    """Forward on the GPU against the oracle; backward on the GPU fed the
    oracle's T (T is an input of the backward: its bf16 rounding is a
    floating-point decision, so both sides take the same T)."""
    if W is None:
        W, io = _problem(M, N, K, r, seed)
    qw, st = gpu_quantize(W)
    assert st == 0
    ws = binding.workspace(M, N, K, r, DEV)
    Y, T = binding.linear_fwd(io["X"], qw, io["A"], io["B"], s, ws=ws)
    torch.cuda.synchronize()
    assert binding.workspace_status(ws) == 0
    Wd = oracle_dequant_full(bits(W).reshape(-1)).reshape(N, K)
    X, A, B, dY = (bits(io[k]) for k in ("X", "A", "B", "dY"))
    Yr, Tr = oracle.qlora_fwd(X, Wd, A, B, s, rows=rows)
    Yg = f64(Y) if rows is None else f64(Y)[rows]
    Tg = f64(T) if rows is None else f64(T)[rows]
    tol_check(Yg, Yr, "Y", bf16_rounded)
    tol_check(Tg, oracle.bf16_to_f64(Tr), "T")
    # T is rounded to bf16: where the fp32 sum X A lands next to a rounding
    # midpoint (or, after cancellation, within a few bf16 steps of a small T)
    # the two sides may round apart; such elements must be rare (their values
    # are within the tolerance checked above)
    Tb = bits(T if rows is None else T[torch.as_tensor(rows, device=DEV)])
    assert np.sum(Tb != Tr) <= max(1, 0.01 * Tr.size)
    if check_bwd:
        _, Tfull = oracle.qlora_fwd(X, Wd, A, B, s)
        T_in = workloads.from_bits(Tfull, DEV)
        dX, dA, dB = binding.linear_bwd(io["dY"], io["X"], qw, io["A"], io["B"], s, T=T_in, ws=ws)
        torch.cuda.synchronize()
        assert binding.workspace_status(ws) == 0
        dXr, dAr, dBr = oracle.qlora_bwd(dY, X, Wd, A, B, s, Tfull, dx_rows=rows)
        tol_check(f64(dX) if rows is None else f64(dX)[rows], dXr, "dX", bf16_rounded)
        tol_check(f64(dA), dAr, "dA")
        tol_check(f64(dB), dBr, "dB")


def test_pr1():
    wl = workloads.WORKLOADS["pr1"]
    _run(32, 1024, 1024, 16, wl.s, seed=0)


@pytest.mark.parametrize("M,N,K,r,s", [(1, 256, 512, 16, 1.0), (37, 520, 640, 8, 4.0), (300, 384, 1024, 64, 0.25),
                                       (129, 1024, 192, 32, 0.7), (256, 512, 512, 128, 0.125),
                                       (64, 136, 256, 256, 0.0625)])
def test_small_shapes(M, N, K, r, s):
    _run(M, N, K, r, s, seed=M + N)


def test_special_cases():
    M, N, K, r = 96, 256, 512, 16
    W, io = _problem(M, N, K, r, seed=11)
    _run(M, N, K, r, 1.0, seed=0, W=torch.zeros_like(W), io=io)           # low-rank path alone
    io0 = dict(io, A=torch.zeros_like(io["A"]))
    _run(M, N, K, r, 2.0, seed=0, W=W, io=io0)                           # frozen path alone
    io1 = dict(io, B=torch.zeros_like(io["B"]))
    _run(M, N, K, r, 2.0, seed=0, W=W, io=io1)
    _run(M, N, K, r, 0.0, seed=0, W=W, io=io)                            # s = 0


def test_recomputed_T_matches():
    M, N, K, r = 128, 256, 512, 64
    W, io = _problem(M, N, K, r, seed=4)
    qw, _ = gpu_quantize(W)
    ws = binding.workspace(M, N, K, r, DEV)
    Y, T = binding.linear_fwd(io["X"], qw, io["A"], io["B"], 0.25, ws=ws)
    g1 = binding.linear_bwd(io["dY"], io["X"], qw, io["A"], io["B"], 0.25, T=T, ws=ws)
    g1 = [g.clone() for g in g1]
    g2 = binding.linear_bwd(io["dY"], io["X"], qw, io["A"], io["B"], 0.25, T=None, ws=ws)
    torch.cuda.synchronize()
    for a, b in zip(g1, g2):
        assert torch.equal(a, b)


@pytest.mark.parametrize("idx", [0, 4, 6])
def test_llama7b_layer_sampled_rows(idx):
    """The 7B matrices at the bench's full size (2048 tokens, r=64), 192
    sampled token rows for Y and dX, full dA and dB."""
    wl = workloads.WORKLOADS["llama7b"]
    name, N, K = wl.mats[idx]
    seed = workloads.matrix_seed("llama7b", 0, idx)
    W = workloads.weight(N, K, wl.w_std, seed=seed, device=DEV)
    io = workloads.layer_inputs(wl.tokens, N, K, wl.r, seed=seed, device=DEV)
    rows = np.sort(np.random.default_rng(idx).choice(wl.tokens, 192, replace=False))
    _run(wl.tokens, N, K, wl.r, wl.s, seed=seed, rows=rows, W=W, io=io)


@pytest.mark.parametrize("M,N,K,r,s", [(5, 24, 100, 8, 2.0), (33, 40, 1000, 12, 0.5), (17, 13, 64, 8, 1.0),
                                       (1, 96, 130, 4, 4.0), (70, 100, 257, 3, 1.5), (40, 8, 4095, 16, 0.25),
                                       (2, 13, 4100, 8, 1.0), (300, 520, 11007, 16, 0.5), (129, 4095, 1000, 8, 4.0),
                                       (64, 1001, 129, 64, 0.25), (16, 1024, 3001, 8, 1.0)])
def test_ragged_shapes(M, N, K, r, s):
    """K % 64 != 0 (rows of W do not start on an NF4 block, nibble phase odd
    or even, segments straddling two blocks), N % 8 != 0 (ragged output rows),
    one or two tokens, split reductions: the fused GEMM's ragged mode.  A rank
    off the 8-element granule (r = 12, 4, 3): the generic path."""
    _run(M, N, K, r, s, seed=M + N + K)


def test_robust_weight_layer_sampled_rows():
    """The 4095 x 11007 Student-t weight with outliers at 4096 tokens, r = 8,
    alpha = 32 (K = 11007 is not a multiple of the block): 128 sampled token
    rows for Y and dX, full dA and dB, on the tensor cores (ragged mode)."""
    wl = workloads.WORKLOADS["robust"]
    _, N, K = wl.mats[0]
    assert binding.plan(wl.tokens, N, K, wl.r)["path"] == binding.PATH_FUSED
    W = workloads.weight(N, K, wl.w_std, seed=0, device=DEV, kind=wl.w_kind)
    io = workloads.layer_inputs(wl.tokens, N, K, wl.r, seed=0, device=DEV)
    rows = np.sort(np.random.default_rng(5).choice(wl.tokens, 128, replace=False))
    _run(wl.tokens, N, K, wl.r, wl.s, seed=0, rows=rows, W=W, io=io)


@pytest.mark.parametrize("M,N,K,r", [(2, 8, 4096, 8), (100, 256, 512, 72), (33, 1032, 2112, 16),
                                     (257, 384, 1024, 24), (1576, 2560, 1024, 24), (1100, 256, 64, 8)])
def test_tile_and_split_edges(M, N, K, r):
    """A single W tile split 8 ways, padding inside the rank (r = 72 of 128),
    33 blocks per row with a ragged W tile, a last token tile of one token,
    and large token counts whose last token tile is mostly empty (40 of its
    tokens present; a single reduction step)."""
    _run(M, N, K, r, 0.75, seed=M * 7 + N)


@pytest.mark.parametrize("M,N,K,r", [(1, 104, 2112, 8), (1, 4104, 64, 16), (1, 8, 64, 8), (1, 520, 4096, 64),
                                     (1, 2056, 640, 256), (2, 256, 512, 16), (3, 1024, 1024, 72), (7, 264, 320, 8),
                                     (8, 1024, 1024, 16), (9, 1032, 2112, 24), (12, 776, 768, 32),
                                     (16, 4096, 4096, 64), (16, 8, 256, 8), (5, 20480, 192, 16)])
def test_decode_kernel_edges(M, N, K, r):
    """1-16 tokens take the decode kernel: a last 256-row tile of 8 rows
    (N = 4104), a last column chunk of one NF4 block (K = 2112, 33 blocks),
    a single block per row, tiles split between CTAs (stream-K) and whole,
    one and two 8-token MMA tiles, the largest rank."""
    _run(M, N, K, r, 0.5, seed=N + K + M)


@pytest.mark.parametrize("M,N,K", [(16, 4104, 2112), (1, 1024, 4096), (7, 520, 640), (64, 1032, 2112),
                                   (300, 384, 1024), (40, 1001, 1000), (3, 13, 4099), (257, 4095, 1007)])
def test_one_hot_tokens_give_the_dequantized_weight_bitwise(M, N, K):
    """Token m = the unit vector e_{k_m} and A = 0: Y[m, n] = Wd[n, k_m], a
    single exact product, so Y must equal the oracle's dequantized weight
    bit for bit.  Likewise dY = e_{n_m}, B = 0: dX[m, k] = Wd[n_m, k].  This
    pins the on-chip dequantization of the decode kernel (M <= 16) and of the
    fused GEMM (forward and backward, aligned and ragged K) to the
    fp32-multiply-then-round rule."""
    r = 16
    W = workloads.weight(N, K, 0.02, seed=N + K, device=DEV)
    qw, st = gpu_quantize(W)
    assert st == 0
    Wd = oracle_dequant_full(bits(W).reshape(-1)).reshape(N, K)
    rng = np.random.default_rng(M)
    ks = rng.choice(K, M, replace=M > K)
    ns = rng.choice(N, M, replace=M > N)
    X = torch.zeros(M, K, dtype=torch.bfloat16, device=DEV)
    X[torch.arange(M), torch.as_tensor(ks, device=DEV)] = 1.0
    dY = torch.zeros(M, N, dtype=torch.bfloat16, device=DEV)
    dY[torch.arange(M), torch.as_tensor(ns, device=DEV)] = 1.0
    A = torch.zeros(K, r, dtype=torch.bfloat16, device=DEV)
    B = torch.zeros(r, N, dtype=torch.bfloat16, device=DEV)
    ws = binding.workspace(M, N, K, r, DEV)
    Y, _ = binding.linear_fwd(X, qw, A, B, 1.0, ws=ws)
    dX, _, _ = binding.linear_bwd(dY, X, qw, A, B, 1.0, ws=ws)
    torch.cuda.synchronize()
    assert binding.workspace_status(ws) == 0
    assert np.array_equal(bits(Y), Wd[:, ks].T)
    assert np.array_equal(bits(dX), Wd[ns, :])


def test_decode_is_deterministic():
    """Split tiles are summed in a fixed order: two calls give the same bits."""
    M, N, K, r = 16, 28672, 8192, 16
    W, io = _problem(M, N, K, r, seed=13)
    qw, _ = gpu_quantize(W)
    ws = binding.workspace(M, N, K, r, DEV)
    assert binding.plan(M, N, K, r)["path"] == binding.PATH_DECODE
    outs = []
    for _ in range(3):
        Y, T = binding.linear_fwd(io["X"], qw, io["A"], io["B"], 1.0, ws=ws)
        outs.append(Y.clone())
    torch.cuda.synchronize()
    assert binding.workspace_status(ws) == 0
    assert torch.equal(outs[0], outs[1]) and torch.equal(outs[0], outs[2])


@pytest.mark.parametrize("M", [1, 4, 16])
@pytest.mark.parametrize("shape", [(28672, 8192), (8192, 28672)])
def test_decode_shapes_sampled_columns(M, shape):
    """Decode: full-size weight, every token, 64 sampled output features
    (the decode kernel: stream-K over 3584 units on all SMs)."""
    wl = workloads.WORKLOADS["decode"]
    N, K = shape
    W = workloads.weight(N, K, wl.w_std, seed=0, device=DEV)
    io = workloads.layer_inputs(M, N, K, wl.r, seed=1, device=DEV)
    qw, st = gpu_quantize(W)
    assert st == 0
    ws = binding.workspace(M, N, K, wl.r, DEV)
    Y, T = binding.linear_fwd(io["X"], qw, io["A"], io["B"], wl.s, ws=ws)
    torch.cuda.synchronize()
    cols = np.sort(np.random.default_rng(M).choice(N, 64, replace=False))
    Wd = oracle_dequant_rows(bits(W), cols)
    X, A, B = bits(io["X"]), bits(io["A"]), bits(io["B"])
    Yr, Tr = oracle.qlora_fwd(X, Wd, A, B[:, cols], wl.s)
    tol_check(f64(Y)[:, cols], Yr, "Y")
    tol_check(f64(T), oracle.bf16_to_f64(Tr), "T")


def test_70b_kv_shape_uses_split_reduction():
    wl = workloads.WORKLOADS["llama70b"]
    name, N, K = wl.mats[1]   # k: 1024 x 8192
    seed = workloads.matrix_seed("llama70b", 0, 1)
    W = workloads.weight(N, K, wl.w_std, seed=seed, device=DEV)
    io = workloads.layer_inputs(wl.tokens, N, K, wl.r, seed=seed, device=DEV)
    rows = np.sort(np.random.default_rng(7).choice(wl.tokens, 96, replace=False))
    _run(wl.tokens, N, K, wl.r, wl.s, seed=seed, rows=rows, W=W, io=io)


@pytest.mark.parametrize("idx", [4, 6])
def test_70b_large_shapes_sampled_rows(idx):
    """The 70B gate (28672 x 8192) and down (8192 x 28672) matrices at 512
    tokens, r = 64: 48 sampled token rows for Y and dX, full dA and dB."""
    wl = workloads.WORKLOADS["llama70b"]
    name, N, K = wl.mats[idx]
    seed = workloads.matrix_seed("llama70b", 0, idx)
    W = workloads.weight(N, K, wl.w_std, seed=seed, device=DEV)
    io = workloads.layer_inputs(wl.tokens, N, K, wl.r, seed=seed, device=DEV)
    rows = np.sort(np.random.default_rng(idx).choice(wl.tokens, 48, replace=False))
    _run(wl.tokens, N, K, wl.r, wl.s, seed=seed, rows=rows, W=W, io=io)


def test_deterministic_outputs():
    M, N, K, r = 512, 1024, 8192, 64
    W, io = _problem(M, N, K, r, seed=9)
    qw, _ = gpu_quantize(W)
    ws = binding.workspace(M, N, K, r, DEV)
    outs = []
    for _ in range(2):
        Y, T = binding.linear_fwd(io["X"], qw, io["A"], io["B"], 0.25, ws=ws)
        g = binding.linear_bwd(io["dY"], io["X"], qw, io["A"], io["B"], 0.25, T=T, ws=ws)
        outs.append([Y.clone(), T.clone()] + [x.clone() for x in g])
    torch.cuda.synchronize()
    for a, b in zip(*outs):
        assert torch.equal(a, b)
