"""Plain, slow CPU oracle for NF4 + double quantization + the QLoRA linear layer.

TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and the
cpu_baseline / reference legs of bench.py may import this package.  It shares
no code with the CUDA library in bit_nf4_quantized_12_b200/ and imports
nothing from it.

Quantization and dequantization are plain C loops (nf4_oracle.c, built with
-ffp-contract=off so each float operation is one IEEE round-to-nearest-even
step).  The linear layer is its definition written out in float64 numpy, with
numpy's matmul as the only library step.

bf16 and fp16 tensors cross this interface as numpy uint16 bit patterns.

Beyond the method's default format (NF4 codes, FP8 E4M3 scale1, FP32 scale2,
BF16 compute) the oracle also defines the variants the pages contrast with
it -- a uniform INT4 table, FP32 or unsigned 8-bit first-level constants, the
FP16 compute type -- and the LoRA merge for serving.  Each function is pinned
by a -m "not gpu" test (tests/test_oracle_*.py); none is "parity unpinned".
"""
import ctypes
import numpy as np

from . import build as _build

_lib = None


def _L():
    global _lib
    if _lib is None:
        path = _build.build()
        lib = ctypes.CDLL(path)
        i64, p = ctypes.c_int64, ctypes.c_void_p
        lib.oracle_codebook.argtypes = [p]
        lib.oracle_quantize.argtypes = [p, i64, p, p, p]
        lib.oracle_quantize.restype = ctypes.c_int
        lib.oracle_dequant.argtypes = [p, p, p, i64, p]
        lib.oracle_bf16_round_array.argtypes = [p, i64, p]
        lib.oracle_bf16_decode_array.argtypes = [p, i64, p]
        lib.oracle_e4m3_encode_array.argtypes = [p, i64, p]
        lib.oracle_e4m3_decode.argtypes = [ctypes.c_uint8]
        lib.oracle_e4m3_decode.restype = ctypes.c_double
        lib.oracle_classify_array.argtypes = [p, p, i64, p]
        lib.oracle_f16_round_array.argtypes = [p, i64, p]
        lib.oracle_f16_decode_array.argtypes = [p, i64, p]
        lib.oracle_codebook_int4.argtypes = [p]
        lib.oracle_quantize_fmt.argtypes = [p, i64, ctypes.c_int, ctypes.c_int, p, p, p]
        lib.oracle_quantize_fmt.restype = ctypes.c_int
        lib.oracle_dequant_fmt.argtypes = [p, p, p, i64, ctypes.c_int, ctypes.c_int, ctypes.c_int, p]
        lib.oracle_classify_fmt_array.argtypes = [ctypes.c_int, p, p, i64, p]
        for f in ("oracle_nblocks", "oracle_ngroups", "oracle_packed_bytes"):
            getattr(lib, f).argtypes = [i64]
            getattr(lib, f).restype = i64
        _lib = lib
    return _lib


def _ptr(a):
    return a.ctypes.data_as(ctypes.c_void_p)


# ----------------------------------------------------------------- format
BLOCK = 64    # weights per first-level block ("QLoRA 原理精讲" §2.1/§2.2)
GROUP = 256   # first-level scales per second-level group ("QLoRA 原理精讲" §2.2)


def nblocks(numel):
    return int(_L().oracle_nblocks(int(numel)))


def ngroups(numel):
    return int(_L().oracle_ngroups(int(numel)))


def packed_bytes(numel):
    return int(_L().oracle_packed_bytes(int(numel)))


def codebook():
    """The 16 NF4 values, ascending, fp32."""
    out = np.zeros(16, np.float32)
    _L().oracle_codebook(_ptr(out))
    return out


# ----------------------------------------------------------------- scalars
def bf16_round(x):
    """Nearest bf16 (ties to even) of each float64 value -> uint16 bits."""
    x = np.ascontiguousarray(x, np.float64)
    out = np.empty(x.shape, np.uint16)
    _L().oracle_bf16_round_array(_ptr(x), x.size, _ptr(out))
    return out


def bf16_to_f64(b):
    b = np.ascontiguousarray(b, np.uint16)
    out = np.empty(b.shape, np.float64)
    _L().oracle_bf16_decode_array(_ptr(b), b.size, _ptr(out))
    return out


def e4m3_encode(x):
    x = np.ascontiguousarray(x, np.float32)
    out = np.empty(x.shape, np.uint8)
    _L().oracle_e4m3_encode_array(_ptr(x), x.size, _ptr(out))
    return out


def e4m3_decode(c):
    return float(_L().oracle_e4m3_decode(int(c)))


def nearest_code(w, absmax):
    """Index of the NF4 code nearest to the exact quotient w/absmax (ties low)."""
    w = np.ascontiguousarray(w, np.float32)
    a = np.ascontiguousarray(np.broadcast_to(absmax, w.shape), np.float32)
    out = np.empty(w.shape, np.int32)
    _L().oracle_classify_array(_ptr(w), _ptr(a), w.size, _ptr(out))
    return out


# ----------------------------------------------------------------- quantize
def quantize(W_bits):
    """NF4 quantize + double quantization of a bf16 tensor (any shape; blocks
    run over the row-major flattening).  Returns (packed u8, c1q u8, c2 f32,
    nonfinite flag)."""
    W = np.ascontiguousarray(W_bits, np.uint16).reshape(-1)
    n = W.size
    packed = np.zeros(packed_bytes(n), np.uint8)
    c1q = np.zeros(nblocks(n), np.uint8)
    c2 = np.zeros(ngroups(n), np.float32)
    flag = _L().oracle_quantize(_ptr(W), n, _ptr(packed), _ptr(c1q), _ptr(c2))
    return packed, c1q, c2, bool(flag)


def dequant(packed, c1q, c2, numel):
    """Double dequantization to bf16 bits (flat array of numel)."""
    packed = np.ascontiguousarray(packed, np.uint8)
    c1q = np.ascontiguousarray(c1q, np.uint8)
    c2 = np.ascontiguousarray(c2, np.float32)
    out = np.empty(int(numel), np.uint16)
    _L().oracle_dequant(_ptr(packed), _ptr(c1q), _ptr(c2), int(numel), _ptr(out))
    return out


# ----------------------------------------------------------------- format variants
# quant_type: NF4 (the method) or a uniform INT4 table ("QLoRA 原理精讲" §2.1
# contrasts the two).  double_quant: E4M3 scale1 + FP32 scale2 (the method,
# §2.2), none (FP32 scale1 per block, §2.2 工程动机), or an unsigned 8-bit
# linear scale1 + FP32 scale2 (an integer reading of the "8 bit" of
# "LoRA、Q-LoRA 与 PortLLM" §3.2).  The pages' flags for these are
# bnb_4bit_quant_type and bnb_4bit_use_double_quant (§三 误区5).
QUANT_NF4, QUANT_INT4 = 0, 1
DQ_E4M3, DQ_NONE, DQ_U8 = 0, 1, 2
BF16, F16 = 0, 1


def f16_round(x):
    """Nearest IEEE binary16 (ties to even) of each float64 value -> uint16 bits."""
    x = np.ascontiguousarray(x, np.float64)
    out = np.empty(x.shape, np.uint16)
    _L().oracle_f16_round_array(_ptr(x), x.size, _ptr(out))
    return out


def f16_to_f64(h):
    h = np.ascontiguousarray(h, np.uint16)
    out = np.empty(h.shape, np.float64)
    _L().oracle_f16_decode_array(_ptr(h), h.size, _ptr(out))
    return out


def codebook_int4():
    out = np.zeros(16, np.float32)
    _L().oracle_codebook_int4(_ptr(out))
    return out


def nearest_code_fmt(quant_type, w, absmax):
    w = np.ascontiguousarray(w, np.float32)
    a = np.ascontiguousarray(np.broadcast_to(absmax, w.shape), np.float32)
    out = np.empty(w.shape, np.int32)
    _L().oracle_classify_fmt_array(int(quant_type), _ptr(w), _ptr(a), w.size, _ptr(out))
    return out


def quantize_fmt(W_bits, quant_type=QUANT_NF4, double_quant=DQ_E4M3):
    """quantize() with a chosen table and first-level-constant format.
    Returns (packed u8, c1 (u8 codes, or f32 for DQ_NONE), c2 f32 (empty for
    DQ_NONE), nonfinite flag)."""
    W = np.ascontiguousarray(W_bits, np.uint16).reshape(-1)
    n = W.size
    packed = np.zeros(packed_bytes(n), np.uint8)
    c1 = np.zeros(nblocks(n), np.float32 if double_quant == DQ_NONE else np.uint8)
    c2 = np.zeros(0 if double_quant == DQ_NONE else ngroups(n), np.float32)
    flag = _L().oracle_quantize_fmt(_ptr(W), n, int(quant_type), int(double_quant), _ptr(packed), _ptr(c1),
                                    _ptr(c2) if c2.size else None)
    return packed, c1, c2, bool(flag)


def dequant_fmt(packed, c1, c2, numel, quant_type=QUANT_NF4, double_quant=DQ_E4M3, dtype=BF16):
    """Double dequantization of any format into bf16 (dtype BF16) or fp16
    (dtype F16) bits."""
    packed = np.ascontiguousarray(packed, np.uint8)
    c1 = np.ascontiguousarray(c1, np.float32 if double_quant == DQ_NONE else np.uint8)
    c2 = np.ascontiguousarray(c2, np.float32)
    out = np.empty(int(numel), np.uint16)
    _L().oracle_dequant_fmt(_ptr(packed), _ptr(c1), _ptr(c2) if c2.size else None, int(numel), int(quant_type),
                            int(double_quant), int(dtype), _ptr(out))
    return out


# ----------------------------------------------------------------- linear layer
def _f64(b, dtype=BF16):
    return f16_to_f64(b) if dtype == F16 else bf16_to_f64(b)


def _round(x, dtype=BF16):
    return f16_round(x) if dtype == F16 else bf16_round(x)


def lora_merge(Wd, A, B, s, dtype=BF16):
    """Merge the adapter into the frozen weight for serving ("QLoRA 原理精讲"
    §2.5: after merging, the weights go back to BF16; §三 误区3, path ②):
        W' = round(Wd + s (A B)^T)
    with Wd [N,K] the dequantized weight and A [K,r], B [r,N] the LoRA factors,
    all in the compute type (bits), computed in float64 (each product exact,
    the sums rounded far below the compute type's spacing) and rounded once to
    the compute type.  Returns (W' bits [N,K], the unrounded float64 value)."""
    exact = _f64(Wd, dtype) + float(s) * (_f64(A, dtype) @ _f64(B, dtype)).T
    return _round(exact, dtype), exact


def qlora_fwd(X, Wd, A, B, s, rows=None, dtype=BF16):
    """QLoRA linear forward, exact in float64 from bf16 inputs.

    Y = X Wd^T + s * T B with T = bf16(X A): the frozen weight Wd is the
    dequantized BF16 tensor, the LoRA factors A [K,r], B [r,N] stay BF16 and
    the low-rank product X A is held in the BF16 compute type ("从LoRA到QLoRA"
    §3.1; LoRA adapters in BF16: "QLoRA 原理精讲" §三 误区1).  Y is returned
    unrounded (float64).  `rows` restricts the computation to those rows of X.

    X [M,K], Wd [N,K], A [K,r], B [r,N] as uint16 bits of the compute type:
    bf16 (dtype BF16), or fp16 (dtype F16, the pages' choice for GPUs without
    BF16, "QLoRA 原理精讲" §三 误区4), in which T is held too.
    Returns (Y float64 [m,N], T uint16 [m,r]).
    """
    Xf = _f64(X if rows is None else np.asarray(X)[rows], dtype)
    Wf, Af, Bf = _f64(Wd, dtype), _f64(A, dtype), _f64(B, dtype)
    T = _round(Xf @ Af, dtype)
    Y = Xf @ Wf.T + float(s) * (_f64(T, dtype) @ Bf)
    return Y, T


def qlora_bwd(dY, X, Wd, A, B, s, T, dx_rows=None, dtype=BF16):
    """QLoRA linear backward, exact in float64.  Only the LoRA factors and the
    input receive gradients; the frozen NF4 weight gets none ("从LoRA到QLoRA"
    §3.1).  With G = s dY B^T:
        dX = dY Wd + G A^T,  dA = X^T G,  dB = s T^T dY.
    T is the bf16 [M,r] tensor of the forward.  `dx_rows` restricts dX to
    those rows.  All tensors are bits of the compute type (dtype as in
    qlora_fwd).  Returns (dX, dA, dB) as float64."""
    dYf, Xf, Wf, Af, Bf, Tf = (_f64(t, dtype) for t in (dY, X, Wd, A, B, T))
    G = float(s) * (dYf @ Bf.T)
    dA = Xf.T @ G
    dB = float(s) * (Tf.T @ dYf)
    if dx_rows is None:
        dX = dYf @ Wf + G @ Af.T
    else:
        dX = dYf[dx_rows] @ Wf + G[dx_rows] @ Af.T
    return dX, dA, dB
