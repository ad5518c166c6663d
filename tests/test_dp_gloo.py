"""Data-parallel replicas of the QLoRA linear layer on CPU with two gloo
ranks: each rank takes its slice of the tokens, computes its partial LoRA
gradients (here with the oracle: the host logic is what is under test), and
the one all-reduce of the shared gradient bucket yields the full-batch dA
and dB.  Also: the token slices cover the batch exactly once, and a single
rank calls no collective."""
import multiprocessing as mp
import os
import socket
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

from bit_nf4_quantized_12_b200 import dp  # noqa: E402

SHAPES = [(48, 40, 8), (32, 24, 4)]      # (K, N, r) of two layers
M = 13                                   # tokens: not a multiple of the world size


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _problem(K, N, r, seed):
    rng = np.random.default_rng(seed)
    bf = lambda a: __import__("oracle").bf16_round(a)
    return dict(X=bf(rng.standard_normal((M, K))), dY=bf(rng.standard_normal((M, N))),
                W=bf(rng.standard_normal((N, K)) * 0.02), A=bf(rng.standard_normal((K, r)) * 0.01),
                B=bf(rng.standard_normal((r, N)) * 0.01))


def _grads(p, s, lo, hi):
    import oracle
    _, T = oracle.qlora_fwd(p["X"], p["W"], p["A"], p["B"], s)
    _, dA, dB = oracle.qlora_bwd(p["dY"][lo:hi], p["X"][lo:hi], p["W"], p["A"], p["B"], s, T[lo:hi])
    return dA, dB


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    lo, hi = dp.token_shard(M, world, rank)
    bucket = dp.GradBucket.for_layers(SHAPES, "cpu")
    for li, (K, N, r) in enumerate(SHAPES):
        dA, dB = _grads(_problem(K, N, r, li), 0.5, lo, hi)
        bucket.views[li][0].copy_(torch.from_numpy(dA))
        bucket.views[li][1].copy_(torch.from_numpy(dB))
    works = dp.allreduce_lora_grads([bucket.flat], async_op=True)
    for w in works:
        w.wait()
    dist.barrier()
    dist.destroy_process_group()
    out.put((rank, (lo, hi), [(a.numpy().copy(), b.numpy().copy()) for a, b in bucket.views]))


def test_two_ranks_sum_to_the_full_batch_gradients():
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    got = sorted((out.get(timeout=120) for _ in range(2)), key=lambda x: x[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [g[1] for g in got] == [(0, 7), (7, 13)]
    for li, (K, N, r) in enumerate(SHAPES):
        dA, dB = _grads(_problem(K, N, r, li), 0.5, 0, M)
        for rank in range(2):
            gA, gB = got[rank][2][li]
            np.testing.assert_allclose(gA, dA, rtol=1e-5, atol=1e-7)
            np.testing.assert_allclose(gB, dB, rtol=1e-5, atol=1e-7)
        # both ranks hold the same bits after the reduction
        assert np.array_equal(got[0][2][li][0], got[1][2][li][0])


@pytest.mark.parametrize("M_,world", [(13, 2), (2048, 8), (7, 7), (3, 4), (0, 3)])
def test_token_shards_cover_the_batch_once(M_, world):
    spans = [dp.token_shard(M_, world, r) for r in range(world)]
    assert spans[0][0] == 0 and spans[-1][1] == M_
    assert all(a[1] == b[0] for a, b in zip(spans, spans[1:]))
    sizes = [b - a for a, b in spans]
    assert max(sizes) - min(sizes) <= 1


def test_single_rank_calls_no_collective():
    import torch
    assert dp.allreduce_lora_grads([torch.zeros(4)]) == []


def test_bucket_views_are_disjoint_and_cover_the_buffer():
    b = dp.GradBucket.for_layers(SHAPES, "cpu")
    total = 0
    for (dA, dB), (K, N, r) in zip(b.views, SHAPES):
        assert dA.shape == (K, r) and dB.shape == (r, N)
        total += dA.numel() + dB.numel()
        dA.fill_(1.0)
        dB.fill_(2.0)
    assert total == b.flat.numel() and bool((b.flat > 0).all())
