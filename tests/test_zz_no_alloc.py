"""fd_block_attention_static: the attention call for callers that cannot set
device memory aside for the per-layer work area in the cache storage (storage
from someone else's pool or arena, or a process that may not call cudaMalloc
because it can synchronise the device).  Its work area is a static device
array of the library, so it allocates nothing.

Checked here: two calls in a row through the C ABI give the same results as
the regular entry point within the bf16 tolerance of the parity tests, and a
request larger than the static area is refused before any launch.  This file
is collected last; it passes alone in a fresh process (the first call looks
up the array's device address) and after the other tests."""
import numpy as np
import pytest
import torch

from streaming_autoregressive_video_b200 import binding as fd
from streaming_autoregressive_video_b200.workloads import Workload

from support import TOL_BF16_MAX, TOL_BF16_MEAN, block_inputs, new_cache, out_values, \
    to_device

pytestmark = pytest.mark.gpu

W = Workload("static-work-bf16", layers=2, rollouts=2, heads=4, head_dim=128,
             grid_h=12, grid_w=26, action_tokens=4, block_frames=3, sink_frames=1,
             window_frames=4, steps=2, blocks=1, dtype="bf16")


def _call(entry, cache, layer, q, k, v):
    out = torch.empty(q.shape, dtype=torch.int16, device="cuda")
    lse = torch.empty((q.shape[0], W.heads, W.queries), dtype=torch.float32, device="cuda")
    entry(cache, layer, W.rollouts, q, k, v, out, lse)
    torch.cuda.synchronize()
    return out_values(out), lse.cpu().numpy()


def test_static_work_area_matches_regular_entry_point_twice():
    cache = new_cache(W)
    for b in range(3):   # sink + part of the window
        ks, vs = [], []
        for l in range(W.layers):
            _, k, v = block_inputs(W, (71, b, l), W.rollouts)
            ks.append(to_device(k))
            vs.append(to_device(v))
        fd.fd_cache_commit(cache, 0, W.layers, W.rollouts, ks, vs)
    for call in range(2):   # two calls in a row, different layers and inputs
        layer = call % W.layers
        q, k, v = (to_device(a) for a in block_inputs(W, (72, call), W.rollouts))
        want, want_lse = _call(fd.fd_block_attention, cache, layer, q, k, v)
        got, got_lse = _call(fd.fd_block_attention_static, cache, layer, q, k, v)
        err = np.abs(got - want)
        assert err.max() <= TOL_BF16_MAX and err.mean() <= TOL_BF16_MEAN, call
        assert np.abs(got_lse - want_lse).max() <= 1e-2, call
    assert fd.fd_get_device_error(cache) == 0


def test_static_work_area_refuses_oversized_calls():
    # 40 heads x 3 frames x 1564 tokens x 128 x 2 bytes = 48 MB of rotated keys
    big = Workload("static-work-too-big", layers=1, rollouts=1, heads=40, head_dim=128,
                   grid_h=30, grid_w=52, action_tokens=4, block_frames=3, sink_frames=0,
                   window_frames=3, steps=1, blocks=1, dtype="bf16")
    assert big.block_frames * big.frame_tokens * big.heads * big.head_dim * 2 > \
        fd.STATIC_WORK_BYTES
    cache = new_cache(big)
    q = torch.zeros((1, big.queries, big.heads, big.head_dim), dtype=torch.int16, device="cuda")
    kv = torch.zeros((1, big.block_frames * big.frame_tokens, big.heads, big.head_dim),
                     dtype=torch.int16, device="cuda")
    launches = fd.fd_launch_count()
    with pytest.raises(fd.FdError) as e:
        fd.fd_block_attention_static(cache, 0, 1, q, kv, kv, torch.empty_like(q))
    assert e.value.status == 4   # FD_ERR_CAPACITY
    assert fd.fd_launch_count() == launches
