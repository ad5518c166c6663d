"""Thin Python binding of libqlora_nf4.so (include/qlora_nf4.h).

Argument marshalling only: torch tensors supply device memory and the current
CUDA stream; every step of the computation runs in the library's kernels.
There is no fallback: a missing library or a CPU tensor raises.
"""
import ctypes
import os
from dataclasses import dataclass

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libqlora_nf4.so")

NF4_OK = 0
STATUS_NONFINITE = 1
STATUS_TIMEOUT = 2

_lib = None


class NF4Error(RuntimeError):
    pass


class NF4Weight(ctypes.Structure):
    _fields_ = [("packed", ctypes.c_void_p), ("c1q", ctypes.c_void_p), ("c2", ctypes.c_void_p),
                ("rows", ctypes.c_int64), ("cols", ctypes.c_int64), ("quant_type", ctypes.c_int32),
                ("double_quant", ctypes.c_int32)]


# storage formats and compute types (include/qlora_nf4.h)
QUANT_NF4, QUANT_INT4 = 0, 1
DQ_E4M3, DQ_NONE, DQ_U8 = 0, 1, 2
_DTYPES = {torch.bfloat16: 0, torch.float16: 1}


class QloraPlan(ctypes.Structure):
    _fields_ = [("path", ctypes.c_int32), ("token_tile", ctypes.c_int32), ("splits", ctypes.c_int32),
                ("lora_steps", ctypes.c_int32), ("tiles_w", ctypes.c_int64), ("tiles_t", ctypes.c_int64),
                ("main_steps", ctypes.c_int64), ("lowrank_splits", ctypes.c_int32 * 4)]


PATH_FUSED, PATH_DECODE, PATH_GENERIC = 0, 1, 2

# (name, restype, argtypes) for every symbol of include/qlora_nf4.h
_P, _I64, _I32, _F, _SZ = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_float, ctypes.c_size_t
SIGNATURES = {
    "nf4_build_codebook": (ctypes.c_int, [_P, _P]),
    "nf4_sizes": (ctypes.c_int, [_I64, _P, _P, _P]),
    "nf4_quantize_dq": (ctypes.c_int, [_P, _I64, _I64, _P, _P, _P, _P, _P]),
    "nf4_quantize": (ctypes.c_int, [_P, _I64, _I64, _I32, _I32, _P, _P, _P, _P, _P]),
    "nf4_dequant_bf16": (ctypes.c_int, [NF4Weight, _P, _P]),
    "nf4_dequant": (ctypes.c_int, [NF4Weight, _I32, _P, _P]),
    "nf4_lora_merge": (ctypes.c_int, [NF4Weight, _P, _P, _I32, _F, _I32, _P, _P]),
    "qlora_workspace_bytes": (_SZ, [_I64, _I64, _I64, _I32]),
    "qlora_linear_fwd": (ctypes.c_int, [_P, _I64, NF4Weight, _P, _P, _I32, _F, _P, _P, _P, _SZ, _P]),
    "qlora_linear_bwd": (ctypes.c_int, [_P, _P, _I64, NF4Weight, _P, _P, _I32, _F, _P, _P, _P, _P, _P,
                                        _SZ, _P]),
    "qlora_linear_fwd_ex": (ctypes.c_int, [_I32, _P, _I64, NF4Weight, _P, _P, _I32, _F, _P, _P, _P, _SZ, _P]),
    "qlora_linear_bwd_ex": (ctypes.c_int, [_I32, _P, _P, _I64, NF4Weight, _P, _P, _I32, _F, _P, _P, _P, _P, _P,
                                           _SZ, _P]),
    "qlora_linear_fwd_noalloc": (ctypes.c_int, [_P, _I64, NF4Weight, _P, _P, _I32, _F, _P, _P, _P]),
    "qlora_linear_fwd_noalloc_info": (ctypes.c_int, [_P, _P]),
    "qlora_linear_plan": (ctypes.c_int, [_I64, _I64, _I64, _I32, _I32, _I32, _P]),
    "nf4_wait_selftest": (ctypes.c_int, [_P, _I64, _P]),
    "nf4_status_str": (ctypes.c_char_p, [ctypes.c_int]),
}


def lib():
    """Load the library (raises NF4Error when it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise NF4Error(f"{LIB_PATH} not found: run `python -m bit_nf4_quantized_12_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def _check(code):
    if code != NF4_OK:
        raise NF4Error(lib().nf4_status_str(code).decode())


def _dev(t, dtype, name):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise NF4Error(f"{name} must be a CUDA tensor (no CPU path exists)")
    if t.dtype != dtype:
        raise NF4Error(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise NF4Error(f"{name} must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _dtype(t):
    """Compute-type code of a bf16 / fp16 tensor."""
    if t.dtype not in _DTYPES:
        raise NF4Error(f"compute type must be bf16 or fp16, got {t.dtype}")
    return _DTYPES[t.dtype]


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


# ---------------------------------------------------------------- format
def build_codebook():
    codes = np.zeros(16, np.float32)
    thr = np.zeros(15, np.float32)
    _check(lib().nf4_build_codebook(codes.ctypes.data_as(_P), thr.ctypes.data_as(_P)))
    return codes, thr


def sizes(numel):
    pb, nb, ng = ctypes.c_size_t(), ctypes.c_int64(), ctypes.c_int64()
    _check(lib().nf4_sizes(int(numel), ctypes.byref(pb), ctypes.byref(nb), ctypes.byref(ng)))
    return pb.value, nb.value, ng.value


@dataclass
class QuantizedWeight:
    packed: torch.Tensor   # uint8 [ceil(numel/2)]
    c1q: torch.Tensor      # uint8 [nblocks] (float32 [nblocks] for DQ_NONE)
    c2: torch.Tensor       # float32 [ngroups] (empty for DQ_NONE)
    rows: int
    cols: int
    quant_type: int = QUANT_NF4
    double_quant: int = DQ_E4M3

    def abi(self):
        return NF4Weight(self.packed.data_ptr(), self.c1q.data_ptr(),
                         self.c2.data_ptr() if self.c2.numel() else None, self.rows, self.cols, self.quant_type,
                         self.double_quant)


def empty_quantized(rows, cols, device, quant_type=QUANT_NF4, double_quant=DQ_E4M3):
    pb, nb, ng = sizes(rows * cols)
    # packed is padded to 16 bytes so its size is a multiple of the vector width
    packed = torch.zeros(((pb + 15) // 16) * 16, dtype=torch.uint8, device=device)[:pb]
    c1 = torch.zeros(nb, dtype=torch.float32 if double_quant == DQ_NONE else torch.uint8, device=device)
    c2 = torch.zeros(0 if double_quant == DQ_NONE else ng, dtype=torch.float32, device=device)
    return QuantizedWeight(packed, c1, c2, rows, cols, quant_type, double_quant)


def quantize(W, out: QuantizedWeight = None, status: torch.Tensor = None, quant_type=QUANT_NF4,
             double_quant=DQ_E4M3):
    """4-bit quantization of a bf16 CUDA tensor [rows, cols]: NF4 with double
    quantization by default; a QUANT_* table and DQ_* constant format
    otherwise (taken from `out` when it is given)."""
    rows, cols = W.shape
    if out is None:
        out = empty_quantized(rows, cols, W.device, quant_type, double_quant)
    _check(lib().nf4_quantize(_dev(W, torch.bfloat16, "W"), rows, cols, out.quant_type, out.double_quant,
                              ctypes.c_void_p(out.packed.data_ptr()), ctypes.c_void_p(out.c1q.data_ptr()),
                              ctypes.c_void_p(out.c2.data_ptr()) if out.c2.numel() else None,
                              None if status is None else _dev(status, torch.int32, "status"), _stream()))
    return out


def dequant(qw: QuantizedWeight, out: torch.Tensor = None, dtype=torch.bfloat16):
    """Wd in the compute type (bf16, or fp16)."""
    if out is None:
        out = torch.empty(qw.rows, qw.cols, dtype=dtype, device=qw.packed.device)
    _check(lib().nf4_dequant(qw.abi(), _dtype(out), _dev(out, out.dtype, "out"), _stream()))
    return out


def lora_merge(qw: QuantizedWeight, A, B, s, out: torch.Tensor = None):
    """W' = round(Wd + s (A B)^T) in the compute type of A and B; [rows, cols]."""
    if out is None:
        out = torch.empty(qw.rows, qw.cols, dtype=A.dtype, device=A.device)
    dt = _dtype(A)
    _check(lib().nf4_lora_merge(qw.abi(), _dev(A, A.dtype, "A"), _dev(B, A.dtype, "B"), A.shape[1], float(s), dt,
                                _dev(out, A.dtype, "out"), _stream()))
    return out


# ---------------------------------------------------------------- linear layer
def workspace_bytes(M, N, K, r):
    return int(lib().qlora_workspace_bytes(int(M), int(N), int(K), int(r)))


def plan(M, N, K, r, backward=False, num_sms=0):
    """Launch plan the library picks for a linear call of these sizes (host
    only).  Returns a dict of the qlora_plan fields."""
    out = QloraPlan()
    _check(lib().qlora_linear_plan(int(M), int(N), int(K), int(r), int(bool(backward)), int(num_sms),
                                   ctypes.byref(out)))
    d = {name: getattr(out, name) for name, _ in QloraPlan._fields_}
    d["lowrank_splits"] = list(out.lowrank_splits)
    return d


def workspace(M, N, K, r, device):
    return torch.zeros(workspace_bytes(M, N, K, r), dtype=torch.uint8, device=device)


def linear_fwd(X, qw: QuantizedWeight, A, B, s, ws=None, Y=None, T=None, want_T=True):
    """Y = X Wd^T + s (X A) B in the compute type of X (bf16 or fp16);
    returns (Y, T)."""
    M, K = X.shape
    r = A.shape[1]
    dt, ty = _dtype(X), X.dtype
    if ws is None:
        ws = workspace(M, qw.rows, K, r, X.device)
    if Y is None:
        Y = torch.empty(M, qw.rows, dtype=ty, device=X.device)
    if T is None and want_T:
        T = torch.empty(M, r, dtype=ty, device=X.device)
    _check(lib().qlora_linear_fwd_ex(dt, _dev(X, ty, "X"), M, qw.abi(), _dev(A, ty, "A"), _dev(B, ty, "B"), r,
                                     float(s), _dev(Y, ty, "Y"), None if T is None else _dev(T, ty, "T"),
                                     _dev(ws, torch.uint8, "ws"), ws.numel(), _stream()))
    return Y, T


def linear_fwd_noalloc(X, qw: QuantizedWeight, A, B, s, Y=None, T=None, want_T=True):
    """linear_fwd with the library's fixed scratch array instead of a workspace;
    returns (Y, T).  Y and T are allocated here unless given."""
    M, K = X.shape
    r = A.shape[1]
    if Y is None:
        Y = torch.empty(M, qw.rows, dtype=torch.bfloat16, device=X.device)
    if T is None and want_T:
        T = torch.empty(M, r, dtype=torch.bfloat16, device=X.device)
    _check(lib().qlora_linear_fwd_noalloc(_dev(X, torch.bfloat16, "X"), M, qw.abi(), _dev(A, torch.bfloat16, "A"),
                                          _dev(B, torch.bfloat16, "B"), r, float(s), _dev(Y, torch.bfloat16, "Y"),
                                          None if T is None else _dev(T, torch.bfloat16, "T"), _stream()))
    return Y, T


class _DeviceWord:
    """A view of one int32 at a raw device address (no allocation), for torch."""

    def __init__(self, ptr):
        self.__cuda_array_interface__ = {"shape": (1,), "typestr": "<i4", "data": (int(ptr), False),
                                         "version": 3}


def wait_selftest(status: torch.Tensor, limit_cycles: int):
    """Run the bounded device wait on a barrier nothing arrives at (see
    nf4_wait_selftest); status: int32 CUDA tensor of one element."""
    _check(lib().nf4_wait_selftest(_dev(status, torch.int32, "status"), int(limit_cycles), _stream()))


def noalloc_info():
    """(device address of the no-allocation status word on the current
    device, size of the fixed scratch array in bytes)."""
    ptr, nbytes = ctypes.c_void_p(), ctypes.c_size_t()
    _check(lib().qlora_linear_fwd_noalloc_info(ctypes.byref(ptr), ctypes.byref(nbytes)))
    return ptr.value, nbytes.value


def noalloc_status():
    """Status word of the last qlora_linear_fwd_noalloc call on the current
    device (read after the stream synchronizes)."""
    ptr, _ = noalloc_info()
    return int(torch.as_tensor(_DeviceWord(ptr), device="cuda").item())


def linear_bwd(dY, X, qw: QuantizedWeight, A, B, s, T=None, ws=None, dX=None, dA=None, dB=None):
    """Returns (dX [M,K] in the compute type of X, dA fp32 [K,r], dB fp32 [r,N])."""
    M, K = X.shape
    r = A.shape[1]
    N = qw.rows
    dt, ty = _dtype(X), X.dtype
    if ws is None:
        ws = workspace(M, N, K, r, X.device)
    if dX is None:
        dX = torch.empty(M, K, dtype=ty, device=X.device)
    if dA is None:
        dA = torch.empty(K, r, dtype=torch.float32, device=X.device)
    if dB is None:
        dB = torch.empty(r, N, dtype=torch.float32, device=X.device)
    _check(lib().qlora_linear_bwd_ex(dt, _dev(dY, ty, "dY"), _dev(X, ty, "X"), M, qw.abi(), _dev(A, ty, "A"),
                                     _dev(B, ty, "B"), r, float(s), None if T is None else _dev(T, ty, "T"),
                                     _dev(dX, ty, "dX"), _dev(dA, torch.float32, "dA"),
                                     _dev(dB, torch.float32, "dB"), _dev(ws, torch.uint8, "ws"), ws.numel(),
                                     _stream()))
    return dX, dA, dB


def workspace_status(ws):
    """The status word a linear call leaves in its workspace (read after sync)."""
    return int(ws[:4].view(torch.int32).item())
