"""GPU parity of the storage-format variants, the FP16 compute type and the
LoRA merge against the oracle.

  - quantize: every (table, first-level constant format) pair bit-exact:
    packed codes, 8-bit codes or FP32 scale1, FP32 scale2;
  - dequantize: bit-exact into bf16 and into fp16 ("QLoRA 原理精讲" §三 误区4);
  - LoRA merge ("QLoRA 原理精讲" §2.5, §三 误区3): bit-exact except where the
    kernel's fp32 arithmetic (accumulation of the rank-r product, the fused
    add) may round the other way: near rounding ties, or where the merged
    value cancels to far below its inputs; every such element must lie within
    that arithmetic's error bound of the exact value, and they must be rare;
  - the QLoRA linear layer in FP16, and in bf16 on the variant formats,
    within the linear layer's stated tolerance (relative Frobenius 2e-3, elementwise
    1e-2 with the denominator floored at 1e-2 x rms)."""
import numpy as np
import pytest
import torch

import oracle
from bit_nf4_quantized_12_b200 import binding, workloads
from gpu_helpers import bf16_rounded, bits, f16_rounded, f64, tol_check

pytestmark = pytest.mark.gpu
DEV = "cuda"
FORMATS = [(q, d) for q in (oracle.QUANT_NF4, oracle.QUANT_INT4) for d in (oracle.DQ_E4M3, oracle.DQ_NONE, oracle.DQ_U8)]


def _quantize(W, qt, dq):
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    qw = binding.quantize(W, status=status, quant_type=qt, double_quant=dq)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    return qw


def _oracle_storage(W, qt, dq):
    return oracle.quantize_fmt(bits(W).reshape(-1), qt, dq)


def _assert_storage_equal(qw, ref):
    p, c1, c2, bad = ref
    assert not bad
    assert np.array_equal(qw.packed.cpu().numpy(), p)
    assert np.array_equal(qw.c1q.cpu().numpy().view(np.uint8), c1.view(np.uint8))
    assert np.array_equal(qw.c2.cpu().numpy().view(np.uint32), c2.view(np.uint32))


@pytest.mark.parametrize("qt,dq", FORMATS)
@pytest.mark.parametrize("shape,kind", [((1024, 1024), "normal"), ((37, 4095), "student_t_outliers"),
                                        ((4096, 4096), "normal")])
def test_quantize_and_dequant_formats_bit_exact(qt, dq, shape, kind):
    N, K = shape
    W = workloads.weight(N, K, 0.02, seed=N + qt * 7 + dq, device=DEV, kind=kind)
    qw = _quantize(W, qt, dq)
    ref = _oracle_storage(W, qt, dq)
    _assert_storage_equal(qw, ref)
    for dt, code in ((torch.bfloat16, oracle.BF16), (torch.float16, oracle.F16)):
        d = binding.dequant(qw, dtype=dt)
        torch.cuda.synchronize()
        want = oracle.dequant_fmt(ref[0], ref[1], ref[2], N * K, qt, dq, code)
        assert np.array_equal(d.view(torch.int16).cpu().numpy().view(np.uint16).reshape(-1), want)


def test_int4_zero_and_extreme_blocks():
    x = torch.zeros(3, 4096, dtype=torch.float32)
    x[1, :64] = 1e-30                      # tiny absmax
    x[1, 64:128] = 3e37                    # huge absmax
    x[2] = torch.linspace(-1, 1, 4096)
    W = x.to(torch.bfloat16).to(DEV)
    for dq in (oracle.DQ_E4M3, oracle.DQ_NONE, oracle.DQ_U8):
        qw = _quantize(W, oracle.QUANT_INT4, dq)
        _assert_storage_equal(qw, _oracle_storage(W, oracle.QUANT_INT4, dq))
    assert np.all(qw.packed.cpu().numpy()[:2048] == 0x88)    # all-zero row: the 0.0 code of INT4


# ------------------------------------------------------------------ LoRA merge
def _ulp(v, dtype):
    """Spacing of the compute type at each value (bf16: 8 significant bits,
    fp16: 11; subnormal spacing below the smallest normal)."""
    a = np.abs(v)
    if dtype == oracle.F16:
        e = np.floor(np.log2(np.maximum(a, 2.0 ** -14)))
        return 2.0 ** (e - 10)
    e = np.floor(np.log2(np.maximum(a, 2.0 ** -126)))
    return 2.0 ** (e - 7)


def _merge_check(got, Wd, A, B, s, dtype):
    """got: uint16 bits [N,K]; Wd, A, B: oracle-side bits.  Every element
    that differs from the oracle's correctly rounded value must lie within
    the kernel's arithmetic error of the exact value: the fp32 accumulation
    of the r products (at most r units of 2^-23 relative to sum |a b|, twice
    the fp32 unit roundoff per step, scaled by |s|), the fp32 rounding of the
    sum, and half a step of the compute type at the result.  Such elements
    (near-ties, and values that cancel to far below their inputs) must be
    rare."""
    ref, exact = oracle.lora_merge(Wd, A, B, s, dtype)
    dec = oracle.f16_to_f64 if dtype == oracle.F16 else oracle.bf16_to_f64
    bad = got != ref
    if bad.any():
        r = A.shape[1]
        g = dec(got[bad])
        absp = (np.abs(dec(A)) @ np.abs(dec(B))).T[bad]
        u = 2.0 ** -23
        bound = abs(s) * r * u * absp + u * (abs(s) * absp + np.abs(exact[bad])) + 0.5 * _ulp(g, dtype) * (1 + 1e-6)
        far = np.abs(g - exact[bad]) > bound
        idx = np.argwhere(bad)
        worst = [(tuple(idx[i]), int(got[bad][i]), int(ref[bad][i]), float(exact[bad][i]), float(bound[i]))
                 for i in np.nonzero(far)[0][:8]]
        assert not far.any(), f"outside the arithmetic's error bound: {worst}"
    assert bad.mean() < 1e-3, bad.mean()
    return int(bad.sum())


@pytest.mark.parametrize("cfg", ["pr1", "llama7b_q", "robust"])
def test_merge_bf16(cfg):
    if cfg == "pr1":
        N, K, r, s, kind = 1024, 1024, 16, 1.0, "normal"
    elif cfg == "llama7b_q":
        N, K, r, s, kind = 4096, 4096, 64, 0.25, "normal"
    else:
        N, K, r, s, kind = 4095, 11007, 8, 4.0, "student_t_outliers"
    W = workloads.weight(N, K, 0.02, seed=3, device=DEV, kind=kind)
    io = workloads.layer_inputs(1, N, K, r, seed=3, device=DEV)
    qw = _quantize(W, 0, 0)
    out = binding.lora_merge(qw, io["A"], io["B"], s)
    torch.cuda.synchronize()
    p, c1, c2, _ = _oracle_storage(W, 0, 0)
    Wd = oracle.dequant(p, c1, c2, N * K).reshape(N, K)
    _merge_check(bits(out), Wd, bits(io["A"]), bits(io["B"]), s, oracle.BF16)


@pytest.mark.parametrize("qt,dq", [(0, 0), (1, 1), (0, 2)])
@pytest.mark.parametrize("N,K,r,s", [(1024, 1024, 16, 1.0), (520, 640, 72, 0.5), (136, 576, 8, 1.5),
                                     (13, 100, 3, 2.0)])
def test_merge_f16_and_formats(qt, dq, N, K, r, s):
    W = workloads.weight(N, K, 0.02, seed=N + r, device=DEV)
    io = workloads.layer_inputs(1, N, K, r, seed=N + r, device=DEV)
    qw = _quantize(W, qt, dq)
    p, c1, c2, _ = _oracle_storage(W, qt, dq)
    for dt, code in ((torch.bfloat16, oracle.BF16), (torch.float16, oracle.F16)):
        A, B = io["A"].to(dt), io["B"].to(dt)
        out = binding.lora_merge(qw, A, B, s)
        torch.cuda.synchronize()
        Wd = oracle.dequant_fmt(p, c1, c2, N * K, qt, dq, code).reshape(N, K)
        _merge_check(bits(out), Wd, bits(A), bits(B), s, code)


def test_merge_zero_adapter_is_dequant():
    N, K, r = 512, 768, 16
    W = workloads.weight(N, K, 0.02, seed=5, device=DEV)
    qw = _quantize(W, 0, 0)
    A = torch.zeros(K, r, dtype=torch.bfloat16, device=DEV)
    B = workloads.normal((r, N), 0.01, seed=6, device=DEV)
    out = binding.lora_merge(qw, A, B, 3.0)
    torch.cuda.synchronize()
    assert torch.equal(out, binding.dequant(qw))


# ------------------------------------------------------------------ linear layer
def _run_linear(M, N, K, r, s, seed, dt, qt=0, dq=0, rows=None, kind="normal"):
    code = oracle.F16 if dt == torch.float16 else oracle.BF16
    W = workloads.weight(N, K, 0.02, seed=seed, device=DEV, kind=kind)
    io = {k: v.to(dt) for k, v in workloads.layer_inputs(M, N, K, r, seed=seed, device=DEV).items()}
    qw = _quantize(W, qt, dq)
    p, c1, c2, _ = _oracle_storage(W, qt, dq)
    Wd = oracle.dequant_fmt(p, c1, c2, N * K, qt, dq, code).reshape(N, K)
    h = lambda t: t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)
    X, A, B, dY = (h(io[k]) for k in ("X", "A", "B", "dY"))
    ws = binding.workspace(M, N, K, r, DEV)
    Y, T = binding.linear_fwd(io["X"], qw, io["A"], io["B"], s, ws=ws)
    torch.cuda.synchronize()
    assert binding.workspace_status(ws) == 0
    Yr, Tr = oracle.qlora_fwd(X, Wd, A, B, s, rows=rows, dtype=code)
    dec = oracle.f16_to_f64 if code == oracle.F16 else oracle.bf16_to_f64
    rnd = f16_rounded if code == oracle.F16 else bf16_rounded
    tol_check(f64(Y) if rows is None else f64(Y)[rows], Yr, "Y", rnd)
    tol_check(f64(T) if rows is None else f64(T)[rows], dec(Tr), "T")
    _, Tfull = oracle.qlora_fwd(X, Wd, A, B, s, dtype=code)
    T_in = torch.from_numpy(Tfull.view(np.int16)).view(dt).to(DEV)
    dX, dA, dB = binding.linear_bwd(io["dY"], io["X"], qw, io["A"], io["B"], s, T=T_in, ws=ws)
    torch.cuda.synchronize()
    assert binding.workspace_status(ws) == 0
    dXr, dAr, dBr = oracle.qlora_bwd(dY, X, Wd, A, B, s, Tfull, dx_rows=rows, dtype=code)
    tol_check(f64(dX) if rows is None else f64(dX)[rows], dXr, "dX", rnd)
    tol_check(f64(dA), dAr, "dA")
    tol_check(f64(dB), dBr, "dB")


@pytest.mark.parametrize("M,N,K,r,s", [(32, 1024, 1024, 16, 1.0), (300, 384, 1024, 64, 0.25), (1, 520, 4096, 64, 0.5),
                                       (129, 1024, 192, 32, 0.7), (5, 24, 100, 8, 2.0), (4, 1024, 8192, 16, 1.0)])
def test_linear_f16(M, N, K, r, s):
    _run_linear(M, N, K, r, s, seed=M + N, dt=torch.float16)


def test_linear_f16_llama7b_gate_sampled_rows():
    rows = np.sort(np.random.default_rng(3).choice(2048, 96, replace=False))
    _run_linear(2048, 11008, 4096, 64, 0.25, seed=4, dt=torch.float16, rows=rows)


@pytest.mark.parametrize("qt,dq", [(1, 0), (0, 1), (0, 2), (1, 2)])
@pytest.mark.parametrize("M,N,K,r,s", [(32, 1024, 1024, 16, 1.0), (1, 1024, 2048, 16, 1.0), (37, 520, 640, 8, 4.0),
                                       (17, 13, 64, 8, 1.0)])
def test_linear_formats(qt, dq, M, N, K, r, s):
    _run_linear(M, N, K, r, s, seed=M + N + K, dt=torch.bfloat16, qt=qt, dq=dq)


def test_linear_f16_int4_fp32_scales():
    _run_linear(64, 512, 1024, 32, 0.5, seed=21, dt=torch.float16, qt=1, dq=1)
