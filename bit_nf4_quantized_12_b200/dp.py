"""Data-parallel replicas of the QLoRA linear layer.

Each rank holds the whole frozen NF4 weight (4-bit storage makes a replica
cheap: "QLoRA 原理精讲" §2.4) and its own LoRA factors A, B, identical on every
rank, and runs the layer on its own slice of the batch's tokens.  Y and dX
belong to the rank's tokens and need no exchange.  dA = X^T G and dB =
s T^T dY are sums over tokens, so the global gradients are the sums of the
ranks' partial gradients: one all-reduce of dA and dB per layer is the path's
only exchange step, (K + N) * r * 4 bytes ("QLoRA 原理精讲" §三 误区4 ties
multi-GPU training to the NVLink between the cards).

The reduction uses torch.distributed (NCCL over NVLink / NVSwitch on GPUs,
gloo on the host); no kernel of this package reads another GPU's memory.
Gradients of several layers can share one flat fp32 bucket (GradBucket), so
that a step issues one all-reduce per bucket, started as soon as the bucket's
last backward call has been queued and awaited before the optimizer reads it.
"""
from dataclasses import dataclass

import torch
import torch.distributed as dist


def token_shard(M, world, rank):
    """[start, stop) of the tokens rank `rank` of `world` takes from a batch
    of M: contiguous slices whose sizes differ by at most one."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError(f"rank {rank} of world {world}")
    base, extra = divmod(int(M), int(world))
    start = rank * base + min(rank, extra)
    return start, start + base + (1 if rank < extra else 0)


@dataclass
class GradBucket:
    """One flat fp32 buffer holding dA [K, r] and dB [r, N] of several layers,
    exposed as views, so that one collective reduces them all."""
    flat: torch.Tensor
    views: list

    @staticmethod
    def for_layers(shapes, device):
        """shapes: [(K, N, r)] per layer -> bucket whose views are
        [(dA_0, dB_0), (dA_1, dB_1), ...]."""
        total = sum(K * r + r * N for K, N, r in shapes)
        flat = torch.zeros(total, dtype=torch.float32, device=device)
        views, off = [], 0
        for K, N, r in shapes:
            dA = flat[off:off + K * r].view(K, r)
            off += K * r
            dB = flat[off:off + r * N].view(r, N)
            off += r * N
            views.append((dA, dB))
        return GradBucket(flat, views)


def allreduce_lora_grads(tensors, group=None, async_op=False):
    """Sum the ranks' partial LoRA gradients in place (dA, dB, or a bucket's
    flat buffer).  With one rank (or no process group) there is nothing to
    exchange and nothing is called.  Returns the pending works when async_op."""
    if not dist.is_available() or not dist.is_initialized() or dist.get_world_size(group) == 1:
        return []
    works = [dist.all_reduce(t, op=dist.ReduceOp.SUM, group=group, async_op=async_op) for t in tensors]
    return [w for w in works if w is not None]


def data_parallel_backward(binding, dY, X, qw, A, B, s, T, ws, dA, dB, dX=None, group=None, async_op=False):
    """The layer's backward on this rank's tokens followed by the gradient
    exchange: returns (dX of the local tokens, pending works).  dA and dB end
    up holding the global gradients once the works complete."""
    dX, _, _ = binding.linear_bwd(dY, X, qw, A, B, s, T=T, ws=ws, dX=dX, dA=dA, dB=dB)
    return dX, allreduce_lora_grads([dA, dB], group=group, async_op=async_op)
