"""Context-parallel attention across ranks ("NVIDIA FlashDreams Is the
Open-Source Inference Engine Robotics World Models Needed", Multi-GPU Context
Parallelism: one rollout's inference sharded across ranks started by torchrun).

Rank r of a group of N holds its rollouts' caches as shard r of N
(``binding.make_desc(w, shards=N, shard=r)``): ring slots s with s mod N == r.
Every rank receives the same q/k/v of each call and commits the same k/v (each
shard keeps only its own slots).  A call computes the shard's rows and
log-sum-exps (``fd_block_attention``; shard 0 also attends to the block's own
keys), all-gathers them over the process group (NCCL over NVLink / NVSwitch on
GPUs) and merges them on every rank (``fd_attention_combine``).  This module is
host orchestration only: every step of the computation runs in the library's
kernels.
"""
from __future__ import annotations

from typing import Callable, Optional


class ShardedBlockAttention:
    """Attention of one shard cache per rank, gathered and combined.

    attn_fn(layer, n_rollouts, q, k, v, out, lse) and combine_fn(outs, lses,
    out, lse) default to the library's entry points; they are parameters so
    that the collective logic can run on CPU tensors (tests).
    """

    def __init__(self, cache, world: int, rank: int, group=None,
                 attn_fn: Optional[Callable] = None, combine_fn: Optional[Callable] = None):
        self.cache, self.world, self.rank, self.group = cache, world, rank, group
        if attn_fn is None or combine_fn is None:
            from . import binding as fd
            attn_fn = attn_fn or (lambda l, n, q, k, v, o, s: fd.fd_block_attention(
                cache, l, n, q, k, v, o, s))
            combine_fn = combine_fn or fd.fd_attention_combine
        self.attn_fn, self.combine_fn = attn_fn, combine_fn

    def __call__(self, layer: int, n_rollouts: int, q, k, v, out, lse=None):
        import torch
        import torch.distributed as dist
        R, Mq, H = out.shape[0], out.shape[1], out.shape[2]
        part = torch.empty_like(out)
        part_lse = torch.empty((R, H, Mq), dtype=torch.float32, device=out.device)
        self.attn_fn(layer, n_rollouts, q, k, v, part, part_lse)
        if self.world == 1:
            parts, lses = [part], [part_lse]
        else:
            parts = [torch.empty_like(part) for _ in range(self.world)]
            lses = [torch.empty_like(part_lse) for _ in range(self.world)]
            # the same two collectives, in the same order, on every rank
            dist.all_gather(parts, part, group=self.group)
            dist.all_gather(lses, part_lse, group=self.group)
        self.combine_fn(parts, lses, out, lse)
        return out
