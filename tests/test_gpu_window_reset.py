"""The window-boundary policy ("Single-GPU inference for DreamZero", Sequential
requests; reading R12 of the oracle) driven through the C ABI: before each
block, fd_cache_window_full says which rollouts' windows cannot take it; those
are released with fd_cache_reset and given their re-encoded conditioning frame
with fd_cache_commit, then the block runs.  Every attention call is checked
against the oracle, the cache bytes, positions and counters bit for bit, and
the library's decision against the oracle's."""
import numpy as np
import pytest

import oracle
from streaming_autoregressive_video_b200 import binding as fd
from streaming_autoregressive_video_b200.workloads import Workload

from support import Lockstep, block_inputs

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_window_reset_policy_through_the_library(dtype):
    w = Workload(f"window-reset-{dtype}", layers=2, rollouts=2, heads=2,
                 head_dim=128 if dtype == "bf16" else 64, grid_h=6, grid_w=13,
                 action_tokens=2, block_frames=2, sink_frames=1, window_frames=4,
                 steps=2, blocks=8, dtype=dtype)
    ls = Lockstep(w)
    F, S, W = w.block_frames, w.sink_frames, w.window_frames
    layers = list(range(w.layers))

    def start_window(ids, seed):
        """Release the listed rollouts' frames and commit one conditioning
        frame each (position 0)."""
        ls.reset(ids)
        ks, vs = [], []
        for l in layers:
            _, k, v = block_inputs(w, (seed, l), w.rollouts)
            ks.append(k)
            vs.append(v)
        ls.commit(layers, ks, vs, frames=[1 if r in ids else 0 for r in range(w.rollouts)])

    start_window(list(range(w.rollouts)), 500)      # a new sequence
    restarts = 0
    for blk in range(w.blocks):
        ids = [r for r in range(w.rollouts) if fd.fd_cache_window_full(ls.cache, 0, r, F)]
        want_ids = [r for r in range(w.rollouts)
                    if oracle.window_boundary_reached(ls.orc[0][r].n, F, S, W)]
        assert ids == want_ids, blk
        if ids:
            start_window(ids, 600 + blk)
            restarts += len(ids)
        for l in layers:
            assert all(ls.orc[l][r].n + F <= S + W for r in range(w.rollouts))
        for s in range(w.steps):
            for l in layers:
                q, k, v = block_inputs(w, (700, blk, s, l), w.rollouts)
                ls.attention(l, q, k, v, what=f"blk {blk} step {s} layer {l}")
        # rollout 1 commits one frame at block 2, so the two rollouts' windows
        # restart at different blocks
        frames = [F, 1] if blk == 2 else None
        ls.commit(layers, [block_inputs(w, (700, blk, w.steps - 1, l), w.rollouts)[1]
                           for l in layers],
                  [block_inputs(w, (700, blk, w.steps - 1, l), w.rollouts)[2] for l in layers],
                  frames=frames)
        ls.check_cache_exact()
        # inside a window the ring never wraps: positions are the slot indices
        for l in layers:
            for r in range(w.rollouts):
                o = ls.orc[l][r]
                assert np.array_equal(o.pos[:o.valid_slots()], np.arange(o.valid_slots()))
    assert restarts >= 3
    assert fd.fd_get_device_error(ls.cache) == 0


def test_window_full_rejects_bad_arguments():
    w = Workload("window-reset-args", layers=1, rollouts=1, heads=1, head_dim=64, grid_h=2,
                 grid_w=2, action_tokens=0, block_frames=2, sink_frames=0, window_frames=3,
                 steps=1, blocks=1, dtype="f32")
    ls = Lockstep(w)
    for layer, rollout, frames in [(1, 0, 1), (0, 1, 1), (0, 0, 0), (0, 0, 3)]:
        with pytest.raises(fd.FdError) as e:
            fd.fd_cache_window_full(ls.cache, layer, rollout, frames)
        assert e.value.status == 1
    assert not fd.fd_cache_window_full(ls.cache, 0, 0, 2)
