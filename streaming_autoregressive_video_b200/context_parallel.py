"""Context-parallel attention across ranks ("NVIDIA FlashDreams Is the
Open-Source Inference Engine Robotics World Models Needed", Multi-GPU Context
Parallelism: one rollout's inference sharded across ranks started by torchrun).

Rank r of a group of N holds its rollouts' caches as shard r of N
(``binding.make_desc(w, shards=N, shard=r)``): ring slots s with s mod N == r.
Every rank receives the same q/k/v of each call and commits the same k/v (each
shard keeps only its own slots).  A call computes the shard's rows and
log-sum-exps over all query rows (``fd_block_attention``; shard 0 also attends
to the block's own keys).  The query rows are then cut into N chunks and chunk
j of every rank's result goes to rank j (one gather per chunk, over NCCL on
NVLink / NVSwitch on GPUs), so each rank receives (N-1)/N of a call's rows
instead of the N-1 whole results an all-gather would bring.  Rank j merges
the N parts of its chunk (``fd_attention_combine``): that is where a
row-sharded next layer would continue.  When every rank needs every row, the
merged chunks are all-gathered once more, (N-1)/N of the rows again.  This
module is host orchestration only: every step of the computation runs in the
library's kernels.
"""
from __future__ import annotations

from typing import Callable, List, Optional, Tuple


def row_chunks(rows: int, world: int) -> List[Tuple[int, int]]:
    """[begin, end) of each rank's query rows: N contiguous chunks whose
    sizes differ by at most one."""
    return [(j * rows // world, (j + 1) * rows // world) for j in range(world)]


class ShardedBlockAttention:
    """Attention of one shard cache per rank, exchanged by row chunk and
    combined.

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

    def __call__(self, layer: int, n_rollouts: int, q, k, v, out, lse=None,
                 rows_only: bool = False):
        """Whole-key-set attention rows into `out` [R][Mq][H][d] (and `lse`
        [R][H][Mq]).  With rows_only, only this rank's chunk of query rows
        (row_chunks(Mq, N)[rank]) is written and its bounds are returned;
        otherwise every row is written on every rank."""
        import torch
        import torch.distributed as dist
        R, Mq, H = out.shape[0], out.shape[1], out.shape[2]
        N, me = self.world, self.rank
        part = torch.empty_like(out)
        part_lse = torch.empty((R, H, Mq), dtype=torch.float32, device=out.device)
        self.attn_fn(layer, n_rollouts, q, k, v, part, part_lse)
        if N == 1:
            self.combine_fn([part], [part_lse], out, lse)
            return (0, Mq)
        chunks = row_chunks(Mq, N)
        q0, q1 = chunks[me]
        mine, mine_lse = [], []
        # the same collectives, in the same order, on every rank: chunk j of
        # every rank's result (rows, then log-sum-exps) is gathered on rank j
        for j, (a, b) in enumerate(chunks):
            send = part[:, a:b].contiguous()
            send_lse = part_lse[:, :, a:b].contiguous()
            if j == me:
                mine = [torch.empty_like(send) for _ in range(N)]
                mine_lse = [torch.empty_like(send_lse) for _ in range(N)]
            dist.gather(send, mine if j == me else None, dst=j, group=self.group)
            dist.gather(send_lse, mine_lse if j == me else None, dst=j, group=self.group)
        rows = torch.empty((R, q1 - q0) + tuple(out.shape[2:]), dtype=out.dtype,
                           device=out.device)
        rows_lse = torch.empty((R, H, q1 - q0), dtype=torch.float32, device=out.device)
        self.combine_fn(mine, mine_lse, rows, rows_lse)
        if rows_only:
            out[:, q0:q1] = rows
            if lse is not None:
                lse[:, :, q0:q1] = rows_lse
            return (q0, q1)
        # every rank needs every row: gather the merged chunks (padded to the
        # largest chunk, as all_gather takes equal sizes)
        c = max(b - a for a, b in chunks)
        pad = torch.zeros((R, c) + tuple(out.shape[2:]), dtype=out.dtype, device=out.device)
        pad[:, :q1 - q0] = rows
        pad_lse = torch.zeros((R, H, c), dtype=torch.float32, device=out.device)
        pad_lse[:, :, :q1 - q0] = rows_lse
        got = [torch.empty_like(pad) for _ in range(N)]
        got_lse = [torch.empty_like(pad_lse) for _ in range(N)]
        dist.all_gather(got, pad, group=self.group)
        dist.all_gather(got_lse, pad_lse, group=self.group)
        for (a, b), t, tl in zip(chunks, got, got_lse):
            out[:, a:b] = t[:, :b - a]
            if lse is not None:
                lse[:, :, a:b] = tl[:, :, :b - a]
        return (0, Mq)
