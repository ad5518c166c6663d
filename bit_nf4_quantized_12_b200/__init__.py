"""NF4 + double quantization + QLoRA linear layer for NVIDIA B200 (sm_100a).

The compute lives in the C-ABI library libqlora_nf4.so (hand-written CUDA in
csrc/); `binding` marshals torch tensors into it.  There is no CPU fallback:
every call raises if the library or a CUDA device is missing.
"""
from . import workloads  # noqa: F401  (pure Python, no CUDA needed)

__all__ = ["workloads", "binding"]


def __getattr__(name):
    if name == "binding":
        from . import binding
        return binding
    raise AttributeError(name)
