"""Calls on several CUDA streams.

* finalize() in the background ("NVIDIA FlashDreams ...", Hot-Path Generation,
  Background State Updates): each layer's commit runs on a second stream as
  soon as that layer's last denoising-step attention is done, while the
  attention of the following layers goes on.  The ordering that makes it safe
  is two events per layer: the commit waits for the layer's last attention
  call (it overwrites a slot that call reads once the ring is full, and it
  rebuilds the layer's counter and t table), and the next block's first
  attention call on the layer waits for the commit.  Nothing else is shared:
  a commit writes only its own layer's slots, positions, counter and t table;
  attention on other layers reads only theirs and writes the call's work set.
  Outputs and cache must be bit-identical to the serial order, which itself
  is checked against the oracle, over a rollout through the ring's
  wraparound.
* work sets: with two work sets, attention calls on two layers issued on two
  streams at once give exactly the results of the same calls in sequence.
"""
import numpy as np
import pytest
import torch

from streaming_autoregressive_video_b200 import binding as fd
from streaming_autoregressive_video_b200.workloads import Workload

from support import (Lockstep, block_inputs, krot_view, new_cache, out_values, to_device,
                     views)

pytestmark = pytest.mark.gpu

W = Workload("streams-bf16", layers=3, rollouts=2, heads=2, head_dim=128, grid_h=12,
             grid_w=13, action_tokens=2, block_frames=2, sink_frames=1, window_frames=3,
             steps=2, blocks=7, dtype="bf16")


def _empty_out(w):
    return torch.empty((w.rollouts, w.queries, w.heads, w.head_dim), dtype=torch.int16,
                       device="cuda")


def test_commit_on_a_side_stream_matches_serial_order_and_oracle():
    w = W
    serial = Lockstep(w)             # one stream, every call checked against the oracle
    side = new_cache(w)              # commits on a second stream
    main = torch.cuda.current_stream()
    aux = torch.cuda.Stream()
    attn_done = [torch.cuda.Event() for _ in range(w.layers)]
    commit_done = [torch.cuda.Event() for _ in range(w.layers)]
    for blk in range(w.blocks):      # 1 sink + 3 window slots, 2 frames a block: wraps
        host = {(s, l): block_inputs(w, (91, blk, s, l), w.rollouts)
                for s in range(w.steps) for l in range(w.layers)}
        dev = {key: tuple(to_device(a) for a in val) for key, val in host.items()}
        outs = {key: _empty_out(w) for key in host}
        for s in range(w.steps):
            for l in range(w.layers):
                if s == 0 and blk > 0:
                    main.wait_event(commit_done[l])   # the layer's cache is final
                q, k, v = dev[(s, l)]
                fd.fd_block_attention(side, l, w.rollouts, q, k, v, outs[(s, l)],
                                      stream=main)
                if s == w.steps - 1:
                    attn_done[l].record(main)
                    aux.wait_event(attn_done[l])      # its last reader is done
                    fd.fd_cache_commit(side, l, l + 1, w.rollouts, [k], [v], stream=aux)
                    commit_done[l].record(aux)
        torch.cuda.synchronize()
        # the serial path (each call checked against the oracle) gives the
        # same output values, bit for bit
        for s in range(w.steps):
            for l in range(w.layers):
                q, k, v = host[(s, l)]
                want, _ = serial.attention(l, q, k, v, what=f"blk {blk} step {s} layer {l}")
                assert np.array_equal(out_values(outs[(s, l)]), want), (blk, s, l)
        last = w.steps - 1
        serial.commit(list(range(w.layers)), [host[(last, l)][1] for l in range(w.layers)],
                      [host[(last, l)][2] for l in range(w.layers)])
        serial.check_cache_exact()
        for a, b in zip(views(serial.cache, w), views(side, w)):
            assert torch.equal(a, b), blk
        assert torch.equal(krot_view(serial.cache, w), krot_view(side, w)), blk
    assert fd.fd_get_device_error(side) == 0
    assert fd.fd_get_device_error(serial.cache) == 0


def test_two_work_sets_let_two_layers_run_at_once():
    w = W.scaled(layers=2, blocks=1)
    cache = new_cache(w, work_sets=2)
    for b in range(3):
        ks, vs = [], []
        for l in range(w.layers):
            _, k, v = block_inputs(w, (93, b, l), w.rollouts)
            ks.append(to_device(k))
            vs.append(to_device(v))
        fd.fd_cache_commit(cache, 0, w.layers, w.rollouts, ks, vs)
    inputs = [tuple(to_device(a) for a in block_inputs(w, (94, l), w.rollouts))
              for l in range(w.layers)]
    want = [_empty_out(w) for _ in range(w.layers)]
    for l in range(w.layers):
        fd.fd_block_attention(cache, l, w.rollouts, *inputs[l], want[l])
    torch.cuda.synchronize()
    streams = [torch.cuda.Stream() for _ in range(w.layers)]
    ready = torch.cuda.Event()
    ready.record(torch.cuda.current_stream())
    for rep in range(3):
        got = [_empty_out(w) for _ in range(w.layers)]
        for l in range(w.layers):
            streams[l].wait_event(ready)
            fd.fd_block_attention(cache, l, w.rollouts, *inputs[l], got[l], stream=streams[l])
        torch.cuda.synchronize()
        for l in range(w.layers):
            assert torch.equal(got[l], want[l]), (rep, l)
    assert fd.fd_get_device_error(cache) == 0
