"""GPU parity at the full workload sizes, in the launch configuration the bench
times (one attention call = block-key rotation pass + tensor-core kernel over
the whole grid of query tiles).  The oracle evaluates sampled query rows of
every head (rows spread over all query tiles, including the ragged last tile);
each row's softmax still runs over the rollout's whole key set.  Inputs are
seeded; the oracle's cache is rebuilt from the same seeds, never read back
from the GPU."""
import numpy as np
import pytest
import torch

import oracle
from streaming_autoregressive_video_b200 import binding as fd
from streaming_autoregressive_video_b200 import synth
from streaming_autoregressive_video_b200.workloads import (BATCHED_RAGGED, GQA_480P,
                                                           LARGE_ACTIONS, LONG_ROLLOUT,
                                                           MULTIVIEW_4, SINGLE_480P)

from support import Lockstep, block_inputs, compare, new_cache, out_values, to_device, \
    to_host, views

pytestmark = pytest.mark.gpu


def sample_rows(Mq, n=192, seed=0):
    """Rows spread over every 128-row tile plus the first and last rows."""
    rng = np.random.default_rng(seed)
    rows = set(rng.integers(0, Mq, size=n).tolist())
    rows |= {0, 1, 127, 128, Mq - 1, Mq - 2, (Mq // 128) * 128}
    return np.array(sorted(r for r in rows if r < Mq))


def prefill_and_call(w, layers_used, seed, n_prefill=None, frames_fn=None):
    ls = Lockstep(w)
    n_prefill = n_prefill if n_prefill is not None else -(-w.slots // w.block_frames) + 1
    for b in range(n_prefill):
        frames = frames_fn(b) if frames_fn else None
        ks, vs = [], []
        for l in range(w.layers):
            _, k, v = block_inputs(w, (seed, b, l, 5), w.rollouts)
            ks.append(k)
            vs.append(v)
        ls.commit(list(range(w.layers)), ks, vs, frames=frames)
    ls.check_cache_exact()
    errs = []
    for l in layers_used:
        q, k, v = block_inputs(w, (seed, 99, l), w.rollouts)
        rows = sample_rows(w.queries, seed=l)
        _, e = ls.attention(l, q, k, v, rows=rows, what=f"{w.name} layer {l}")
        errs += e
    assert fd.fd_get_device_error(ls.cache) == 0
    return errs


def test_single_480p_full_cache():
    """30x52 grid, 1 sink + 6-frame window (full), 12 heads: 4680 queries x 15600 keys."""
    w = SINGLE_480P.scaled(layers=2)
    prefill_and_call(w, [0, 1], seed=21)


def test_large_model_with_action_tokens():
    """40 heads, 1 sink + 12-frame window (full), 4 action tokens per frame
    (Tf = 1564): 4680 queries x 25024 keys, values N(0,1)*0.5."""
    w = LARGE_ACTIONS.scaled(layers=1)
    prefill_and_call(w, [0], seed=22)


def test_multiview_four_cameras_704x1280():
    """4 views of 44x80 per frame (14080 tokens), 16 heads, 1 sink + 3-frame
    window (full): 14080 queries x 70400 keys."""
    w = MULTIVIEW_4.scaled(layers=1)
    prefill_and_call(w, [0], seed=25)


def test_grouped_query_attention_480p():
    """12 query heads over 4 key/value heads at the 480p shape."""
    w = GQA_480P.scaled(layers=1)
    prefill_and_call(w, [0], seed=26)


def test_batched_ragged_rollouts():
    """16 rollouts, 24 heads, 16x20 grid, window fill w_r ~ U{3..12} per rollout."""
    w = BATCHED_RAGGED
    fill = synth.ragged_fill(synth.seed_of(23, 0), w.rollouts, *w.ragged_window)
    left = fill.copy()
    F = w.block_frames
    steps = []
    while left.max() > 0:
        fr = np.minimum(left, F)
        steps.append([int(x) for x in fr])
        left -= fr
    prefill_and_call(w, [0], seed=23, n_prefill=len(steps), frames_fn=lambda b: steps[b])


def _frame_kv(w, seed, m, dev):
    """K/V of frame m of the long rollout, drawn on the device from its seed."""
    shape = (1, w.frame_tokens, w.heads, w.head_dim)
    k = synth.normal_device(synth.seed_of(seed, m, 1), shape, "bf16", dev).view(torch.int16)
    v = synth.normal_device(synth.seed_of(seed, m, 2), shape, "bf16", dev).view(torch.int16)
    return k, v


def _check_block(w, cache, seed, b, q, k, v, out, pos_v):
    dev = q.device
    S, W, T, Tf = w.sink_frames, w.window_frames, w.tokens, w.frame_tokens
    torch.cuda.synchronize()
    oc = oracle.RolloutCache(S, W, Tf, w.heads, w.head_dim, "bf16")
    for m in list(range(min(b, S))) + list(range(max(S, b - W), b)):
        km, vm = _frame_kv(w, seed, m, dev)   # rebuild the cache from the frames' seeds
        oc.k[oracle.slot_of(m, S, W)] = to_host(km)[0]
        oc.v[oracle.slot_of(m, S, W)] = to_host(vm)[0]
        oc.pos[oracle.slot_of(m, S, W)] = m
    oc.n = b
    rows = sample_rows(w.queries, n=96, seed=b)
    want, _ = oracle.block_attention(oc, to_host(q)[0], to_host(k)[0], to_host(v)[0],
                                     tokens=T, grid_w=w.grid_w, theta=w.theta, rows=rows)
    got = out_values(out)[0]
    compare(got[rows], want[rows], "bf16", f"block {b}")
    assert np.array_equal(to_host(pos_v)[0, 0], oc.pos), b


def _run_block(w, cache, seed, b, out, check, pos_v):
    dev = out.device
    qshape = (1, w.queries, w.heads, w.head_dim)
    for step in range(w.steps):
        q = synth.normal_device(synth.seed_of(seed, b, step, 0), qshape, "bf16", dev).view(torch.int16)
        if step == w.steps - 1:
            k, v = _frame_kv(w, seed, b, dev)   # the frame that gets committed
        else:
            k, v = _frame_kv(w, seed + 1, b * 10 + step, dev)
        fd.fd_block_attention(cache, 0, 1, q, k, v, out)
        if check and step == w.steps - 1:
            _check_block(w, cache, seed, b, q, k, v, out, pos_v)
    fd.fd_cache_commit(cache, 0, 1, 1, [k], [v])


def test_long_rollout_10k_blocks_memory_constant():
    """10,000 one-frame blocks through a 1-sink + 8-frame ring, 2 denoising
    steps each; device memory constant; slot map and counters checked against
    the closed form; attention checked against the oracle at sampled blocks
    (first blocks, around ring wraps, the last)."""
    w = LONG_ROLLOUT
    dev = torch.device("cuda")
    cache = new_cache(w)
    seed = 24
    S, W = w.sink_frames, w.window_frames
    out = torch.empty((1, w.queries, w.heads, w.head_dim), dtype=torch.int16, device=dev)
    check_at = set(range(10)) | {15, 16, 17, 100, 1001, 5002, w.blocks - 1}
    _, _, pos_v, count_v = views(cache, w)
    mem0 = free0 = None
    for b in range(w.blocks):
        if b == 20:
            # every code path of the loop has run once (including the oracle
            # checks, whose first launches may grow the driver's per-thread
            # local-memory pool); from here on device memory must not move.
            # torch's caching allocator is emptied so only live allocations count.
            torch.cuda.synchronize()
            torch.cuda.empty_cache()
            mem0 = torch.cuda.memory_allocated()
            free0 = torch.cuda.mem_get_info()[0]
        _run_block(w, cache, seed, b, out, b in check_at, pos_v)
        if b % 997 == 0:
            torch.cuda.synchronize()
            n = b + 1
            assert int(count_v[0, 0]) == n
            want_pos = np.full(S + W, -1, np.int32)
            for m in list(range(min(n, S))) + list(range(max(S, n - W), n)):
                want_pos[oracle.slot_of(m, S, W)] = m
            assert np.array_equal(to_host(pos_v)[0, 0], want_pos), b
    torch.cuda.synchronize()
    assert int(count_v[0, 0]) == w.blocks
    assert fd.fd_cache_frames(cache, 0, 0) == w.blocks
    assert torch.cuda.memory_allocated() == mem0
    torch.cuda.empty_cache()
    assert abs(torch.cuda.mem_get_info()[0] - free0) < (8 << 20)
    assert fd.fd_get_device_error(cache) == 0
