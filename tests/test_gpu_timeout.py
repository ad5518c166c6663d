"""The bounded device wait gives up instead of hanging.

Every kernel waits on shared-memory barriers through one bounded wait; when
an arrival never comes, the wait sets the timeout bit (bit 1) of the call's
status word and the kernel returns.  Here that wait runs on a barrier nothing
arrives at, with a limit of about 1 ms of SM cycles: the call must finish,
report the timeout bit, and leave the device usable for a normal call."""
import time

import pytest
import torch

from bit_nf4_quantized_12_b200 import binding, workloads
from gpu_helpers import gpu_quantize

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.mark.parametrize("limit", [2_000, 2_000_000])
def test_wait_with_no_arrival_sets_the_timeout_bit(limit):
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    t0 = time.perf_counter()
    binding.wait_selftest(status, limit)
    torch.cuda.synchronize()
    elapsed = time.perf_counter() - t0
    assert int(status.item()) == binding.STATUS_TIMEOUT
    assert elapsed < 5.0                       # gave up; did not wait for the 2 s default
    # the device still runs a normal call, and its own status word stays clean
    M, N, K, r = 32, 256, 512, 16
    W = workloads.weight(N, K, 0.02, seed=1, device=DEV)
    io = workloads.layer_inputs(M, N, K, r, seed=1, device=DEV)
    qw, st = gpu_quantize(W)
    assert st == 0
    ws = binding.workspace(M, N, K, r, DEV)
    binding.linear_fwd(io["X"], qw, io["A"], io["B"], 1.0, ws=ws)
    torch.cuda.synchronize()
    assert binding.workspace_status(ws) == 0


def test_selftest_validates_its_limit_on_the_host():
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    for bad in (0, -5, (1 << 40) + 1):
        with pytest.raises(binding.NF4Error, match="INVALID_ARG"):
            binding.wait_selftest(status, bad)
