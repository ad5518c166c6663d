"""The C-ABI library loads on a machine without a GPU, exports every symbol
its header declares, and validates arguments on the host before any launch.
No compute call reaches the GPU here."""
import ctypes
import os
import re

import numpy as np
import pytest

import oracle
from bit_nf4_quantized_12_b200 import binding

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "qlora_nf4.h")


def _declared():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_]*\s*\*?\s*([a-z][a-z0-9_]*)\s*\(", text, flags=re.M)
    return sorted(set(names))


def test_exports_every_declared_symbol():
    names = _declared()
    assert set(names) == set(binding.SIGNATURES), names
    L = binding.lib()
    for n in names:
        assert hasattr(L, n), n


def test_codebook_matches_oracle_bitwise():
    codes, thr = binding.build_codebook()
    ref = oracle.codebook()
    assert np.array_equal(codes.view(np.uint32), ref.view(np.uint32))
    mids = (ref[:-1].astype(np.float64) + ref[1:].astype(np.float64)) / 2
    assert np.all(thr.astype(np.float64) <= mids)
    assert np.all(np.nextafter(thr, np.float32(np.inf)).astype(np.float64) > mids)


@pytest.mark.parametrize("numel", [1, 2, 63, 64, 65, 16384, 16385, 4095 * 11007, 28672 * 8192])
def test_sizes_match_oracle(numel):
    pb, nb, ng = binding.sizes(numel)
    assert (pb, nb, ng) == (oracle.packed_bytes(numel), oracle.nblocks(numel), oracle.ngroups(numel))


def test_host_validation_before_launch():
    L = binding.lib()
    P = ctypes.c_void_p
    fake = P(0x10000)          # never dereferenced: validation fails first
    odd = P(0x10001)
    assert L.nf4_sizes(0, None, None, None) == 1
    assert L.nf4_quantize_dq(None, 4, 4, fake, fake, fake, None, None) == 1
    assert L.nf4_quantize_dq(fake, 0, 4, fake, fake, fake, None, None) == 1
    assert L.nf4_quantize_dq(odd, 4, 4, fake, fake, fake, None, None) == 2
    w = binding.NF4Weight(0x10000, 0x10000, 0x10000, 64, 128)
    assert L.nf4_dequant_bf16(w, odd, None) == 2
    assert L.nf4_dequant_bf16(binding.NF4Weight(0, 0x10000, 0x10000, 64, 128), fake, None) == 1
    # linear layer: rank bounds, workspace
    assert L.qlora_linear_fwd(fake, 16, w, fake, fake, 0, 1.0, fake, None, fake, 1 << 30, None) == 1
    assert L.qlora_linear_fwd(fake, 16, w, fake, fake, 300, 1.0, fake, None, fake, 1 << 30, None) == 1
    # a rank off the 8-element granule takes the generic path, whose workspace
    # also holds the dequantized W; ragged K and N stay on the tensor cores,
    # with X (K % 8 != 0), dY and B (N % 8 != 0) re-pitched instead
    w_rag = binding.NF4Weight(0x10000, 0x10000, 0x10000, 64, 100)      # K % 64 != 0
    need = L.qlora_workspace_bytes(16, 64, 100, 12)
    assert need >= 256 + 64 * 100 * 2 + 16 * 12 * 2 + 16 * 12 * 4
    assert L.qlora_linear_fwd(fake, 16, w_rag, fake, fake, 12, 1.0, fake, None, fake, need - 1, None) == 4
    need = L.qlora_workspace_bytes(16, 64, 100, 16)
    assert 16 * 104 * 2 <= need < 64 * 100 * 2 + 16 * 104 * 2                     # X re-pitched, no Wd copy
    assert L.qlora_linear_fwd(fake, 16, w_rag, fake, fake, 16, 1.0, fake, None, fake, need - 1, None) == 4
    assert L.qlora_workspace_bytes(16, 64, 128, 12) >= 256 + 64 * 128 * 2          # r % 8 != 0
    assert L.qlora_workspace_bytes(64, 60, 128, 16) >= 256 + 2 * 64 * 64 * 2        # N % 8: dY, B re-pitched
    assert L.qlora_workspace_bytes(32, 64, 128, 16) < 64 * 128 * 2                 # fused: no Wd copy
    assert L.qlora_linear_fwd(fake, 16, w, fake, fake, 12, 1.0, fake, None, fake, 16, None) == 4
    assert L.qlora_workspace_bytes(16, 1 << 31, 1 << 31, 12) == 0                  # Wd copy too large
    assert L.qlora_linear_fwd(fake, 16, w, fake, fake, 16, 1.0, fake, None, fake, 16, None) == 4
    assert L.qlora_linear_fwd(odd, 16, w, fake, fake, 16, 1.0, fake, None, fake, 1 << 30, None) == 2
    assert L.qlora_linear_bwd(fake, fake, 16, w, fake, fake, 16, 1.0, None, fake, fake, None, fake, 1 << 30,
                              None) == 1
    assert L.qlora_workspace_bytes(0, 64, 64, 16) == 0
    assert L.qlora_workspace_bytes(2048, 4096, 4096, 64) > 2048 * 128 * 2
    for code in range(7):
        assert L.nf4_status_str(code).startswith(b"NF4_")


def test_noalloc_entry_point_validates_on_host():
    """The allocation-free forward checks its scratch limit and its arguments
    before any set-up or launch: no device is touched here."""
    L = binding.lib()
    fake = ctypes.c_void_p(0x10000)
    w = binding.NF4Weight(0x10000, 0x10000, 0x10000, 256, 512)
    nbytes = ctypes.c_size_t()
    assert L.qlora_linear_fwd_noalloc_info(None, ctypes.byref(nbytes)) == 0   # size only: no device needed
    limit = nbytes.value
    assert limit == 4 << 20                      # the size the header states
    big_m = 12000                                # needs more than the fixed scratch at r = 64
    assert L.qlora_workspace_bytes(big_m, 256, 512, 64) > limit
    assert L.qlora_linear_fwd_noalloc(fake, big_m, w, fake, fake, 64, 1.0, fake, None, None) == 4   # WORKSPACE
    assert L.qlora_linear_fwd_noalloc(fake, 16, w, fake, fake, 0, 1.0, fake, None, None) == 1       # r out of range
    assert L.qlora_linear_fwd_noalloc(fake, 0, w, fake, fake, 16, 1.0, fake, None, None) == 1       # no tokens


def test_binding_refuses_cpu_tensors():
    import torch
    with pytest.raises(binding.NF4Error):
        binding.quantize(torch.zeros(4, 64, dtype=torch.bfloat16))
