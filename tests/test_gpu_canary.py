"""Out-of-bounds write checks by canary bytes: guard regions around every
buffer a kernel writes stand in for a device memory checker.

Every buffer a kernel writes -- quantized weight, dequantized weight, Y, T,
dX, dA, dB and the workspace, sized exactly as the C ABI states -- sits
between two 4 KB guard regions filled with a pattern.  After the calls the
guards must be intact.  The shapes reach every kernel: quantize/dequant with
ragged tails, the fused GEMM with and without a split reduction and with
ragged tiles, the decode kernel (1-16 tokens, whole and split tiles), and
the generic path for ragged shapes.
"""
import pytest
import torch

from bit_nf4_quantized_12_b200 import binding, workloads

pytestmark = pytest.mark.gpu
DEV = "cuda"
GUARD = 4096          # bytes on each side (a multiple of 16: the ABI's pointer alignment)
PATTERN = 0xA5


class Guarded:
    """A tensor placed between two guard regions of one allocation."""

    def __init__(self, shape, dtype):
        n = 1
        for d in shape:
            n *= d
        self.nbytes = n * torch.empty((), dtype=dtype).element_size()
        self.buf = torch.full((GUARD + self.nbytes + GUARD,), PATTERN, dtype=torch.uint8, device=DEV)
        self.t = self.buf[GUARD:GUARD + self.nbytes].view(dtype).view(shape)

    def intact(self):
        head = self.buf[:GUARD]
        tail = self.buf[GUARD + self.nbytes:]
        return bool((head == PATTERN).all().item()) and bool((tail == PATTERN).all().item())


def guarded_weight(rows, cols):
    pb, nb, ng = binding.sizes(rows * cols)
    parts = [Guarded((pb,), torch.uint8), Guarded((nb,), torch.uint8), Guarded((ng,), torch.float32)]
    return binding.QuantizedWeight(parts[0].t, parts[1].t, parts[2].t, rows, cols), parts


@pytest.mark.parametrize("shape", [(1024, 1024), (7, 4099), (33, 16383), (257, 63)])
def test_quantize_and_dequant_stay_in_bounds(shape):
    rows, cols = shape
    W = workloads.weight(rows, cols, 0.02, seed=rows + cols, device=DEV)
    qw, parts = guarded_weight(rows, cols)
    binding.quantize(W, out=qw)
    out = Guarded((rows, cols), torch.bfloat16)
    binding.dequant(qw, out=out.t)
    torch.cuda.synchronize()
    for name, g in zip(("packed", "c1q", "c2", "dequant"), parts + [out]):
        assert g.intact(), (shape, name)


@pytest.mark.parametrize("M,N,K,r", [(32, 1024, 1024, 16),     # fused, no split
                                     (2, 8, 4096, 8),          # one W tile, 8-way split
                                     (257, 384, 1024, 24),     # ragged token and W tiles
                                     (1, 1024, 1024, 16),      # decode kernel (forward), split tiles
                                     (16, 4104, 4096, 64),     # decode: ragged last 256-row tile
                                     (9, 512, 1088, 8),        # decode: ragged last column chunk
                                     (5, 24, 100, 8),          # generic path: K % 64 != 0
                                     (17, 13, 64, 12)])        # generic path: N % 8, r % 8
def test_linear_layer_stays_in_bounds(M, N, K, r):
    W = workloads.weight(N, K, 0.02, seed=M + N, device=DEV)
    io = workloads.layer_inputs(M, N, K, r, seed=M + N, device=DEV)
    qw = binding.quantize(W)
    ws = Guarded((binding.workspace_bytes(M, N, K, r),), torch.uint8)
    ws.t.zero_()
    Y, T = Guarded((M, N), torch.bfloat16), Guarded((M, r), torch.bfloat16)
    binding.linear_fwd(io["X"], qw, io["A"], io["B"], 0.5, ws=ws.t, Y=Y.t, T=T.t)
    dX, dA, dB = Guarded((M, K), torch.bfloat16), Guarded((K, r), torch.float32), Guarded((r, N), torch.float32)
    binding.linear_bwd(io["dY"], io["X"], qw, io["A"], io["B"], 0.5, T=T.t, ws=ws.t, dX=dX.t, dA=dA.t, dB=dB.t)
    # the backward again with T recomputed into the workspace
    binding.linear_bwd(io["dY"], io["X"], qw, io["A"], io["B"], 0.5, T=None, ws=ws.t, dX=dX.t, dA=dA.t, dB=dB.t)
    torch.cuda.synchronize()
    assert binding.workspace_status(ws.t) == 0
    for name, g in (("workspace", ws), ("Y", Y), ("T", T), ("dX", dX), ("dA", dA), ("dB", dB)):
        assert g.intact(), ((M, N, K, r), name)
