"""NF4 + double quantization + QLoRA linear layer for NVIDIA B200 (sm_100a).

The compute lives in the C-ABI library libqlora_nf4.so (hand-written CUDA in
csrc/); `bit_nf4_quantized_12_b200.binding` marshals torch tensors into it.
There is no CPU fallback: every call raises if the library or a CUDA device
is missing.  `workloads` holds the seeded synthetic inputs (no arithmetic of
the method).
"""
__all__ = ["binding", "workloads"]
