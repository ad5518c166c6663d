"""GPU parity of NF4 quantize / double quantize / dequantize: bit-exact
against the oracle on the workloads' weights and on edge cases."""
import numpy as np
import pytest
import torch

import oracle
from bit_nf4_quantized_12_b200 import binding, workloads
from gpu_helpers import bits, gpu_quantize

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _compare_full(W, name=""):
    qw, st = gpu_quantize(W)
    wb = bits(W).reshape(-1)
    p, c1q, c2, bad = oracle.quantize(wb)
    assert st == (1 if bad else 0), name
    if bad:
        return
    assert np.array_equal(qw.packed.cpu().numpy(), p), name + " packed"
    assert np.array_equal(qw.c1q.cpu().numpy(), c1q), name + " c1q"
    assert np.array_equal(qw.c2.cpu().numpy().view(np.uint32), c2.view(np.uint32)), name + " c2"
    d = binding.dequant(qw)
    torch.cuda.synchronize()
    ref = oracle.dequant(p, c1q, c2, wb.size)
    assert np.array_equal(bits(d).reshape(-1), ref), name + " dequant"


def _compare_groups(W, groups, name=""):
    """Full-size tensor, sampled 16384-element groups compared bit for bit."""
    qw, st = gpu_quantize(W)
    assert st == 0
    d = binding.dequant(qw)
    torch.cuda.synchronize()
    wb = bits(W).reshape(-1)
    db = bits(d).reshape(-1)
    G = 16384
    pk, c1q, c2 = qw.packed.cpu().numpy(), qw.c1q.cpu().numpy(), qw.c2.cpu().numpy()
    for g in groups:
        sl = wb[g * G:(g + 1) * G]
        p, q1, q2, _ = oracle.quantize(sl)
        assert np.array_equal(pk[g * G // 2: g * G // 2 + p.size], p), (name, g)
        assert np.array_equal(c1q[g * 256: g * 256 + q1.size], q1), (name, g)
        assert c2[g].view(np.uint32) == q2[0].view(np.uint32), (name, g)
        assert np.array_equal(db[g * G: g * G + sl.size], oracle.dequant(p, q1, q2, sl.size)), (name, g)


def test_pr1_weight():
    _compare_full(workloads.weight(1024, 1024, 0.02, seed=0, device=DEV), "pr1")


@pytest.mark.parametrize("shape", [(1, 1), (1, 2), (3, 5), (1, 63), (1, 64), (1, 65), (2, 8192), (1, 16385),
                                   (257, 63), (7, 4099), (33, 16383), (64, 16449)])
def test_ragged_shapes(shape):
    _compare_full(workloads.weight(*shape, 0.02, seed=sum(shape), device=DEV), str(shape))


def test_llama7b_q_full_and_other_matrices_sampled():
    W = workloads.weight(4096, 4096, 0.02, seed=workloads.matrix_seed("llama7b", 0, 0), device=DEV)
    _compare_full(W, "q")
    rng = np.random.default_rng(0)
    for idx, (name, N, K) in enumerate(workloads.LLAMA7B[4:], start=4):
        W = workloads.weight(N, K, 0.02, seed=workloads.matrix_seed("llama7b", 0, idx), device=DEV)
        ng = (N * K + 16383) // 16384
        _compare_groups(W, sorted(set(rng.integers(0, ng, 48).tolist()) | {0, ng - 1}), name)


@pytest.mark.parametrize("layer", [0, 79])
def test_llama70b_matrices_sampled_groups(layer):
    """Every 70B layer shape at full size, with the seeds of the first and the
    last layer: sampled groups bit for bit, first and last group included."""
    rng = np.random.default_rng(3 + layer)
    wl = workloads.WORKLOADS["llama70b"]
    for idx, (name, N, K) in enumerate(wl.mats):
        W = workloads.weight(N, K, wl.w_std, seed=workloads.matrix_seed("llama70b", layer, idx), device=DEV)
        ng = (N * K + 16383) // 16384
        _compare_groups(W, sorted(set(rng.integers(0, ng, 24).tolist()) | {0, ng - 1}), f"{name}@{layer}")
        del W


def test_robustness_weight_full():
    W = workloads.weight(4095, 11007, 0.02, seed=0, device=DEV, kind="student_t_outliers")
    _compare_full(W, "robust")


def test_zero_and_extreme_magnitudes():
    rng = np.random.default_rng(1)
    x = rng.standard_normal(64 * 256 * 3).astype(np.float32)
    scales = np.exp2(rng.choice([-140.0, -133.0, -127.0, -126.0, -100.0, 0.0, 100.0, 125.0, 126.0, 127.0],
                                size=x.size // 64)).astype(np.float32)
    x = (x.reshape(-1, 64) * scales[:, None]).reshape(-1)
    x[:64] = 0.0
    x[64:128] = -0.0
    x[200] = 3.3e38
    W = torch.from_numpy(x).to(torch.bfloat16).reshape(3 * 64, 256).to(DEV)
    _compare_full(W, "extremes")


def test_every_bf16_pair_on_device():
    """Blocks [absmax, w_1..w_63] enumerating every bf16 |w| <= absmax, for all
    128 absmax significands at exponent 0 and a few other exponents."""
    allw = np.arange(0, 0x7F80, dtype=np.uint32)
    blocks = []
    for e in (127, 1, 0, 250, 254):
        for m in range(128):
            if e == 0 and m == 0:
                continue
            c = (e << 7) | m
            w = allw[allw <= c]
            w = np.concatenate([w, w | 0x8000]).astype(np.uint16)
            pad = (-w.size) % 63
            w = np.concatenate([w, np.zeros(pad, np.uint16)]).reshape(-1, 63)
            blk = np.concatenate([np.full((w.shape[0], 1), c, np.uint16), w], axis=1)
            blocks.append(blk)
    allb = np.concatenate(blocks).reshape(-1)
    W = workloads.from_bits(allb, DEV).reshape(-1, 64)
    _compare_full(W, "pairs")


@pytest.mark.parametrize("bad", [float("nan"), float("inf"), float("-inf")])
def test_nonfinite_flag(bad):
    W = workloads.weight(300, 1000, 0.02, seed=5, device=DEV)
    W[123, 456] = bad
    _, st = gpu_quantize(W)
    assert st & 1


def test_deterministic():
    W = workloads.weight(2048, 1024, 0.02, seed=3, device=DEV)
    a, _ = gpu_quantize(W)
    b, _ = gpu_quantize(W)
    assert torch.equal(a.packed, b.packed) and torch.equal(a.c1q, b.c1q) and torch.equal(a.c2, b.c2)
