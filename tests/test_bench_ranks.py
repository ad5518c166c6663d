"""The multi-rank host logic of bench.py on CPU: two gloo ranks agree on the
slowest rank's time and on the whole-job throughput, and the reference arm
runs on rank 0 alone."""
import multiprocessing as mp
import os
import socket
import sys
from types import SimpleNamespace

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    own_ms = [10.0, 25.0][rank]
    ms = bench.max_over_ranks(own_ms, dist, torch.device("cpu"))
    value = bench.whole_job_tflops(world, 1.0e12, 4, ms)
    dist.barrier()
    dist.destroy_process_group()
    out.put((rank, ms, value))


def test_two_gloo_ranks_take_the_slowest_time():
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    got = sorted(out.get(timeout=10) for _ in range(2))
    for rank, ms, value in got:
        assert ms == 25.0
        # 2 replicas x 4 steps x 1e12 flop in 25 ms
        assert value == pytest.approx(2 * 4 * 1.0e12 / 0.025 / 1e12)


def test_reference_arm_runs_on_rank_zero_only(monkeypatch, capsys):
    import bench
    from bit_nf4_quantized_12_b200 import workloads

    def boom(*a, **k):
        raise AssertionError("rank 1 must not run the oracle")

    monkeypatch.setattr(bench, "oracle_sample_step", boom)
    args = SimpleNamespace(steps=2, warmup=1)
    assert bench.run_reference(args, workloads.WORKLOADS["llama7b"], rank=1, world=2) is None
    assert capsys.readouterr().out == ""


def test_single_rank_max_is_identity():
    import bench
    assert bench.max_over_ranks(12.5, None, None) == 12.5
