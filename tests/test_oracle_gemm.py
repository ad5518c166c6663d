"""Pins for the oracle's QLoRA linear layer (CPU only).

Small integer-valued inputs make every product and every bf16 rounding exact,
so the checks are exact equalities:
  - special cases that reduce to plain indexing or to hand-summed loops
    (W = 0 leaves only the low-rank path; A = 0 leaves only the frozen path,
    here a permutation, so Y is a column shuffle of X);
  - the backward pass is the adjoint of the forward pass: directional
    derivatives in X, A and B computed from the forward map must equal the
    inner products with dX, dA, dB;
  - non-square shapes (M, N, K, r all different) catch a transposed operand.
"""
import numpy as np

import oracle


def _bits(a):
    return oracle.bf16_round(np.asarray(a, np.float64))


def _ints(rng, shape, lo=-3, hi=4):
    return rng.integers(lo, hi, shape).astype(np.float64)


M, N, K, R = 5, 7, 9, 3


def test_lora_only_when_weight_is_zero():
    rng = np.random.default_rng(0)
    X, A, B = _ints(rng, (M, K)), _ints(rng, (K, R)), _ints(rng, (R, N))
    Y, T = oracle.qlora_fwd(_bits(X), _bits(np.zeros((N, K))), _bits(A), _bits(B), 0.5)
    for m in range(M):
        for n in range(N):
            t = [sum(X[m, k] * A[k, j] for k in range(K)) for j in range(R)]
            assert Y[m, n] == 0.5 * sum(t[j] * B[j, n] for j in range(R))
    assert np.array_equal(oracle.bf16_to_f64(T), np.array(
        [[sum(X[m, k] * A[k, j] for k in range(K)) for j in range(R)] for m in range(M)]))


def test_frozen_only_when_lora_is_zero_is_a_column_shuffle():
    rng = np.random.default_rng(1)
    X = _ints(rng, (M, K))
    perm = rng.permutation(K)[:N]               # Wd[n, perm[n]] = 1
    Wd = np.zeros((N, K))
    Wd[np.arange(N), perm] = 1.0
    for s in (0.0, 1.0, 7.5):
        Y, _ = oracle.qlora_fwd(_bits(X), _bits(Wd), _bits(np.zeros((K, R))), _bits(_ints(rng, (R, N))), s)
        assert np.array_equal(Y, X[:, perm])


def test_scale_multiplies_only_the_low_rank_term():
    rng = np.random.default_rng(2)
    X, W, A, B = _ints(rng, (M, K)), _ints(rng, (N, K)), _ints(rng, (K, R)), _ints(rng, (R, N))
    Y0, _ = oracle.qlora_fwd(_bits(X), _bits(W), _bits(A), _bits(B), 0.0)
    Y1, _ = oracle.qlora_fwd(_bits(X), _bits(W), _bits(A), _bits(B), 1.0)
    Y3, _ = oracle.qlora_fwd(_bits(X), _bits(W), _bits(A), _bits(B), 3.0)
    assert np.array_equal(Y3 - Y0, 3.0 * (Y1 - Y0))
    Yw, _ = oracle.qlora_fwd(_bits(X), _bits(np.zeros((N, K))), _bits(A), _bits(B), 1.0)
    assert np.array_equal(Y1 - Y0, Yw)


def test_backward_is_adjoint_of_forward():
    rng = np.random.default_rng(3)
    X, W, A, B = _ints(rng, (M, K)), _ints(rng, (N, K)), _ints(rng, (K, R), -2, 3), _ints(rng, (R, N))
    dY = _ints(rng, (M, N))
    s = 0.25

    def f(X_, A_, B_):
        Y, _ = oracle.qlora_fwd(_bits(X_), _bits(W), _bits(A_), _bits(B_), s)
        return np.sum(dY * Y)

    _, T = oracle.qlora_fwd(_bits(X), _bits(W), _bits(A), _bits(B), s)
    dX, dA, dB = oracle.qlora_bwd(_bits(dY), _bits(X), _bits(W), _bits(A), _bits(B), s, T)
    assert dX.shape == (M, K) and dA.shape == (K, R) and dB.shape == (R, N)
    base = f(X, A, B)
    for _ in range(5):
        V = _ints(rng, (M, K), -1, 2)
        assert f(X + V, A, B) - base == np.sum(dX * V)      # f is linear in X here
        Va = _ints(rng, (K, R), -1, 2)
        assert f(X, A + Va, B) - base == np.sum(dA * Va)
        Vb = _ints(rng, (R, N), -1, 2)
        assert f(X, A, B + Vb) - base == np.sum(dB * Vb)


def test_row_sampling_matches_full():
    rng = np.random.default_rng(4)
    X, W, A, B = (rng.standard_normal(s) for s in ((M, K), (N, K), (K, R), (R, N)))
    dY = rng.standard_normal((M, N))
    args = [_bits(v) for v in (X, W, A, B)]
    Y, T = oracle.qlora_fwd(*args, 2.0)
    rows = np.array([4, 1])
    Yr, Tr = oracle.qlora_fwd(*args, 2.0, rows=rows)
    assert np.array_equal(Yr, Y[rows]) and np.array_equal(Tr, T[rows])
    dX, dA, dB = oracle.qlora_bwd(_bits(dY), *args, 2.0, T)
    dXr, dAr, dBr = oracle.qlora_bwd(_bits(dY), *args, 2.0, T, dx_rows=rows)
    assert np.array_equal(dXr, dX[rows]) and np.array_equal(dAr, dA) and np.array_equal(dBr, dB)
