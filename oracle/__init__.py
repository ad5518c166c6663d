"""Plain, slow CPU oracle for NF4 + double quantization + the QLoRA linear layer.

TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and the
cpu_baseline / reference legs of bench.py may import this package.  It shares
no code with the CUDA library in bit_nf4_quantized_12_b200/ and imports
nothing from it.

Quantization and dequantization are plain C loops (nf4_oracle.c, built with
-ffp-contract=off so each float operation is one IEEE round-to-nearest-even
step).  The linear layer is its definition written out in float64 numpy, with
numpy's matmul as the only library step.

bf16 tensors cross this interface as numpy uint16 bit patterns.
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


# ----------------------------------------------------------------- linear layer
def _f64(b):
    return bf16_to_f64(b)


def qlora_fwd(X, Wd, A, B, s, rows=None):
    """QLoRA linear forward, exact in float64 from bf16 inputs.

    Y = X Wd^T + s * T B with T = bf16(X A): the frozen weight Wd is the
    dequantized BF16 tensor, the LoRA factors A [K,r], B [r,N] stay BF16 and
    the low-rank product X A is held in the BF16 compute type ("从LoRA到QLoRA"
    §3.1; LoRA adapters in BF16: "QLoRA 原理精讲" §三 误区1).  Y is returned
    unrounded (float64).  `rows` restricts the computation to those rows of X.

    X [M,K], Wd [N,K], A [K,r], B [r,N] as uint16 bf16 bits.
    Returns (Y float64 [m,N], T uint16 [m,r]).
    """
    Xf = _f64(X if rows is None else np.asarray(X)[rows])
    Wf, Af, Bf = _f64(Wd), _f64(A), _f64(B)
    T = bf16_round(Xf @ Af)
    Y = Xf @ Wf.T + float(s) * (_f64(T) @ Bf)
    return Y, T


def qlora_bwd(dY, X, Wd, A, B, s, T, dx_rows=None):
    """QLoRA linear backward, exact in float64.  Only the LoRA factors and the
    input receive gradients; the frozen NF4 weight gets none ("从LoRA到QLoRA"
    §3.1).  With G = s dY B^T:
        dX = dY Wd + G A^T,  dA = X^T G,  dB = s T^T dY.
    T is the bf16 [M,r] tensor of the forward.  `dx_rows` restricts dX to
    those rows.  Returns (dX, dA, dB) as float64."""
    dYf, Xf, Wf, Af, Bf, Tf = _f64(dY), _f64(X), _f64(Wd), _f64(A), _f64(B), _f64(T)
    G = float(s) * (dYf @ Bf.T)
    dA = Xf.T @ G
    dB = float(s) * (Tf.T @ dYf)
    if dx_rows is None:
        dX = dYf @ Wf + G @ Af.T
    else:
        dX = dYf[dx_rows] @ Wf + G[dx_rows] @ Af.T
    return dX, dA, dB
