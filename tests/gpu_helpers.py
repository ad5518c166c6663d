"""Helpers shared by the -m gpu parity tests: tolerance checks and oracle
evaluation of sampled rows.  The oracle always quantizes W itself from the
same seeded bf16 bits the GPU got; nothing the GPU produced feeds it."""
import numpy as np
import torch

import oracle
from bit_nf4_quantized_12_b200 import binding, workloads

REL_FRO = 2e-3    # relative Frobenius error bound (GEMM outputs and gradients)
ELEM = 1e-2       # elementwise relative bound, denominator floored at 1e-2 * rms


def rounding_floor(ref, out_round):
    """Relative Frobenius error of the exact values rounded once to the
    output type: what the best possible implementation of an output in that
    type reaches.  On a handful of outputs it alone can exceed REL_FRO (a
    bf16 value carries up to 2^-8 relative rounding error)."""
    if out_round is None or ref.size == 0:
        return 0.0
    nref = np.linalg.norm(ref)
    return np.linalg.norm(out_round(ref) - ref) / nref if nref > 0 else 0.0


def tol_check(got, ref, name="", out_round=None):
    """got against the exact reference: relative Frobenius <= REL_FRO (or
    1.5 x the correctly rounded result's own error, when the output is
    rounded to a 16-bit type and so small that the rounding alone reaches
    REL_FRO), elementwise <= ELEM.  out_round: exact -> rounded value of the
    output type (None for fp32 outputs)."""
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    assert got.shape == ref.shape, (name, got.shape, ref.shape)
    assert np.all(np.isfinite(got)), name
    nref = np.linalg.norm(ref)
    rel = np.linalg.norm(got - ref) / nref if nref > 0 else np.linalg.norm(got)
    floor = 1e-2 * np.sqrt(np.mean(ref * ref)) if nref > 0 else 1e-30
    elem = np.max(np.abs(got - ref) / np.maximum(np.abs(ref), floor)) if ref.size else 0.0
    bound = max(REL_FRO, 1.5 * rounding_floor(ref, out_round))
    assert rel <= bound, f"{name}: rel Frobenius {rel:.3e} > {bound:.3e} (elementwise {elem:.3e})"
    assert elem <= ELEM, f"{name}: elementwise {elem:.3e} > {ELEM}"
    return rel, elem


def bf16_rounded(x):
    """Exact values -> their nearest bf16, as float64 (the oracle's rounding)."""
    return oracle.bf16_to_f64(oracle.bf16_round(x))


def f16_rounded(x):
    return oracle.f16_to_f64(oracle.f16_round(x))


def f64(t):
    """bf16 / fp32 torch tensor -> float64 numpy (exact)."""
    return t.detach().float().cpu().numpy().astype(np.float64)


def bits(t):
    return workloads.bits(t)


def oracle_dequant_full(W_bits):
    """Oracle Wd (uint16 bits, flat) of a whole weight."""
    packed, c1q, c2, _ = oracle.quantize(W_bits)
    return oracle.dequant(packed, c1q, c2, W_bits.size)


def oracle_dequant_rows(W_bits_2d, rows):
    """Oracle Wd rows (uint16 [len(rows), K]) quantizing only the 16384-element
    groups that cover each row (groups are independent)."""
    N, K = W_bits_2d.shape
    flat = W_bits_2d.reshape(-1)
    G = oracle.BLOCK * oracle.GROUP
    out = np.empty((len(rows), K), np.uint16)
    for i, n in enumerate(rows):
        e0, e1 = n * K, (n + 1) * K
        g0, g1 = e0 // G, (e1 + G - 1) // G
        sl = flat[g0 * G: min(g1 * G, flat.size)]
        d = oracle_dequant_full(sl)
        out[i] = d[e0 - g0 * G: e1 - g0 * G]
    return out


def gpu_quantize(W):
    status = torch.zeros(1, dtype=torch.int32, device=W.device)
    qw = binding.quantize(W, status=status)
    torch.cuda.synchronize()
    return qw, int(status.item())
