"""qlora_linear_fwd_noalloc (scratch from the library's fixed device array)
against qlora_linear_fwd (caller workspace), through the C ABI, on two calls
in a row for each of several shapes, plus the rejection of a request larger than the
fixed array.

The entry point exists for callers that cannot allocate device memory when
they run the layer, such as a C decode loop with a memory budget fixed at
start-up.  So the test also checks that the calls leave both torch's
allocator and the device's free memory unchanged, and that the status word
the calls write (read through qlora_linear_fwd_noalloc_info) is 0 after each.
Kept last in collection order so that it also runs after every other test has
used the library in the same process."""
import pytest
import torch

from bit_nf4_quantized_12_b200 import binding, workloads
from gpu_helpers import f64, gpu_quantize, tol_check

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _layer(M, N, K, r, seed):
    W = workloads.weight(N, K, 0.02, seed=seed, device=DEV)
    io = workloads.layer_inputs(M, N, K, r, seed=seed, device=DEV)
    qw, st = gpu_quantize(W)
    assert st == 0
    return qw, io


def test_noalloc_matches_workspace_entry_point_two_calls():
    _, scratch_bytes = binding.noalloc_info()
    # the second call has a different shape and rank, so a stale status word
    # or stale scratch from the first would show
    # (the last two take the decode kernel and the generic path for a ragged K)
    cases = [(300, 384, 1024, 64, 0.25, 3), (37, 520, 640, 8, 4.0, 5), (1, 1024, 1024, 16, 1.0, 11),
             (5, 24, 100, 8, 2.0, 9)]
    for M, N, K, r, s, seed in cases:
        assert binding.workspace_bytes(M, N, K, r) <= scratch_bytes
        qw, io = _layer(M, N, K, r, seed)
        ws = binding.workspace(M, N, K, r, DEV)
        Yw, Tw = binding.linear_fwd(io["X"], qw, io["A"], io["B"], s, ws=ws)
        torch.cuda.synchronize()
        assert binding.workspace_status(ws) == 0
        outs = [(torch.empty(M, N, dtype=torch.bfloat16, device=DEV), torch.empty(M, r, dtype=torch.bfloat16, device=DEV))
                for _ in range(2)]
        for call, (Yn, Tn) in enumerate(outs):
            # The first launch of a kernel in a fresh process can make the
            # driver load its code into device memory, so the free-memory
            # check brackets the second of the two calls.
            torch.cuda.synchronize()
            before = (torch.cuda.memory_allocated(), torch.cuda.mem_get_info()[0])
            binding.linear_fwd_noalloc(io["X"], qw, io["A"], io["B"], s, Y=Yn, T=Tn)
            torch.cuda.synchronize()
            after = (torch.cuda.memory_allocated(), torch.cuda.mem_get_info()[0])
            if call == 1:
                assert after == before, (before, after)
            assert binding.noalloc_status() == 0
            tol_check(f64(Yn), f64(Yw), f"Y {M}x{N}x{K} r{r} call {call}")
            tol_check(f64(Tn), f64(Tw), f"T {M}x{N}x{K} r{r} call {call}")
            # same kernels, same launch plan: the results are the same bits
            assert torch.equal(Yn, Yw) and torch.equal(Tn, Tw)


def test_noalloc_rejects_oversize_request():
    _, scratch_bytes = binding.noalloc_info()
    M, N, K, r = 12000, 256, 512, 64
    assert binding.workspace_bytes(M, N, K, r) > scratch_bytes
    qw, io = _layer(M, N, K, r, 7)
    with pytest.raises(binding.NF4Error, match="NF4_ERR_WORKSPACE"):
        binding.linear_fwd_noalloc(io["X"], qw, io["A"], io["B"], 1.0)
