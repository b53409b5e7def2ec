"""The N > 1 path of bench.py on the CPU: two ranks over gloo.

The hot path has no exchange step (every (rollout, head) unit lives on one GPU),
so N GPUs run N independent replicas; what the ranks share is host logic: every
rank takes the same collective steps in the same order, the job time is the
maximum over ranks, the job throughput counts the work of all ranks, each
replica draws its own inputs, and only rank 0 prints (also for the reference
arm, whose other ranks exit without work)."""
import contextlib
import io
import json
import os
import socket
import sys
import types

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

WORLD = 2


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime

    import bench
    from streaming_autoregressive_video_b200.workloads import Workload

    dist.init_process_group("gloo", rank=rank, world_size=WORLD,
                            timeout=datetime.timedelta(seconds=60))
    try:
        res = {}
        # rank-dependent local timings: every rank must see the slowest
        res["max"] = bench.max_over_ranks([1.0 + rank, 5.0 - rank, 3.0], WORLD)
        # a second reduction in the same order on every rank
        res["max2"] = bench.max_over_ranks([10.0 * (rank + 1)], WORLD)
        res["rate"] = bench.job_rate(100.0, WORLD, res["max"][0])
        res["seed"] = bench.replica_seed_base(rank)
        # the reference arm: rank 0 alone runs and prints, the others return
        w = Workload("gloo-tiny", layers=1, rollouts=1, heads=2, head_dim=16, grid_h=3,
                     grid_w=4, action_tokens=0, block_frames=1, sink_frames=1,
                     window_frames=2, steps=1, blocks=1, dtype="bf16")
        args = types.SimpleNamespace(steps=1, warmup=0, gpus=WORLD)
        buf = io.StringIO()
        with contextlib.redirect_stdout(buf):
            bench.run_reference(args, w, rank)
        res["printed"] = buf.getvalue()
        dist.barrier()
    finally:
        dist.destroy_process_group()
    with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
        json.dump(res, f)


def test_two_replicas_over_gloo(tmp_path):
    mp.start_processes(_rank_main, args=(_free_port(), str(tmp_path)), nprocs=WORLD,
                       join=True, start_method="spawn")
    res = [json.load(open(tmp_path / f"rank{r}.json")) for r in range(WORLD)]
    for r in res:
        assert r["max"] == [2.0, 5.0, 3.0]
        assert r["max2"] == [20.0]
        # 100 units per rank, 2 ranks, slowest rank 2 ms -> 1e5 units/s
        assert r["rate"] == pytest.approx(100.0 * WORLD / 2e-3)
    assert res[0]["seed"] != res[1]["seed"]
    # only rank 0 prints the reference arm's JSON line
    assert res[1]["printed"] == ""
    line = json.loads(res[0]["printed"].strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["n_gpus"] == WORLD
    assert line["value"] > 0 and line["unit"] == "TFLOP/s"
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["cpu_baseline"]["kind"] == "oracle"


def _cp_rank_main(rank, port, out_dir, world, commits):
    """One rank of a context-parallel attention call over gloo: the rank's part
    of the key set (oracle, standing in for the shard's kernel), the exchange
    of row chunks, the combination of this rank's chunk (oracle) and, for the
    full output, the gather of the merged chunks."""
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime

    import numpy as np
    import torch

    import oracle
    from streaming_autoregressive_video_b200.context_parallel import (ShardedBlockAttention,
                                                                      row_chunks)

    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        rng = np.random.default_rng(71)   # the same inputs on every rank
        S, W, F, T, H, d = 1, 4, 2, 6, 2, 12
        c = oracle.RolloutCache(S, W, T, H, d, "f32")
        for _ in range(commits):
            c.commit(rng.standard_normal((F, T, H, d)).astype(np.float32),
                     rng.standard_normal((F, T, H, d)).astype(np.float32))
        q = rng.standard_normal((F * T, H, d)).astype(np.float32)
        k = rng.standard_normal((F * T, H, d)).astype(np.float32)
        v = rng.standard_normal((F * T, H, d)).astype(np.float32)
        kw = dict(tokens=T, grid_w=3, theta=1.0e4)

        def attn(layer, n, q_, k_, v_, out, lse):
            o, l = oracle.block_attention(c, q_[0], k_[0], v_[0], slot_part=(world, rank),
                                          include_block=(rank == 0), **kw)
            out[0] = torch.from_numpy(o)
            lse[0] = torch.from_numpy(l)

        def combine(outs, lses, out, lse):
            o, l = oracle.combine_partials([x[0].numpy() for x in outs],
                                           [x[0].numpy() for x in lses])
            out[0] = torch.from_numpy(o)
            if lse is not None:
                lse[0] = torch.from_numpy(l)

        cp = ShardedBlockAttention(None, world, rank, attn_fn=attn, combine_fn=combine)
        full, full_lse = oracle.block_attention(c, q, k, v, **kw)
        out = torch.zeros((1, F * T, H, d), dtype=torch.float64)
        lse = torch.zeros((1, H, F * T), dtype=torch.float64)
        assert cp(0, 1, q[None], k[None], v[None], out, lse) == (0, F * T)
        err = float(np.abs(out[0].numpy() - full).max())
        err_lse = float(np.abs(lse[0].numpy() - full_lse).max())
        # only this rank's chunk of rows
        out2 = torch.zeros_like(out)
        lse2 = torch.zeros_like(lse)
        q0, q1 = cp(0, 1, q[None], k[None], v[None], out2, lse2, rows_only=True)
        assert (q0, q1) == row_chunks(F * T, world)[rank]
        err_rows = float(np.abs(out2[0, q0:q1].numpy() - full[q0:q1]).max())
        untouched = bool((out2[0, :q0] == 0).all() and (out2[0, q1:] == 0).all())
        with open(os.path.join(out_dir, f"cp{rank}.json"), "w") as f:
            json.dump({"err": err, "err_lse": err_lse, "err_rows": err_rows,
                       "untouched": untouched}, f)
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,commits", [(2, 3), (3, 3), (3, 0), (5, 3)])
def test_context_parallel_gather_and_combine_over_gloo(tmp_path, world, commits):
    """N ranks, rank r holding the cache slots s with s mod N == r (the block's
    keys on rank 0): after the exchange of row chunks and the combination
    every rank has the attention over the whole key set for its chunk of
    query rows (rows_only) or, after the gather of the merged chunks, for
    every row.  With an empty cache (no commit) every rank but 0 holds no
    key: its part weighs nothing.  Five ranks over 12 rows give unequal
    chunks (the padded gather)."""
    mp.start_processes(_cp_rank_main, args=(_free_port(), str(tmp_path), world, commits),
                       nprocs=world, join=True, start_method="spawn")
    # the parts' log-sum-exps travel as fp32 (the library's type), hence the
    # fp32-level bound on an fp64 computation
    for r in range(world):
        res = json.load(open(tmp_path / f"cp{r}.json"))
        assert res["err"] < 1e-6 and res["err_rows"] < 1e-6 and res["err_lse"] < 1e-6
        assert res["untouched"]
