"""fd_block_attention_static: the attention call for callers that cannot set
device memory aside for the per-layer work area in the cache storage (storage
from someone else's pool or arena, or a process that may not call cudaMalloc
because it can synchronise the device).  Its work area is a static device
array of the library, so it allocates nothing.

Checked here: two calls in a row through the C ABI give exactly the results of
the regular entry point (the same kernels on the same inputs; only the work
area's address differs, so outputs and log-sum-exps must be bit-identical), on
the tensor-core path (multi-head and grouped-query; the area holds the
block's rotated keys and queries) and on the CUDA-core path (fp32, which needs
no area); and a request larger than the static area is refused before any
launch.  This file is collected last; it passes alone in a fresh process (the
first call looks up the array's device address) and after the other tests."""
import pytest
import torch

from streaming_autoregressive_video_b200 import binding as fd
from streaming_autoregressive_video_b200.workloads import TINY_F32, Workload

from support import block_inputs, new_cache, to_device

pytestmark = pytest.mark.gpu

BF16 = Workload("static-work-bf16", layers=2, rollouts=2, heads=4, head_dim=128,
                grid_h=12, grid_w=26, action_tokens=4, block_frames=3, sink_frames=1,
                window_frames=4, steps=2, blocks=1, dtype="bf16")
CASES = {
    "bf16-mha": BF16,
    # grouped-query: the rotated-block-key map of the static area has Hkv rows
    "bf16-gqa": BF16.scaled(name="static-work-bf16-gqa", kv_heads=2),
    # fp32: the CUDA-core kernel rotates as it stages and uses no work area
    "f32-tiny": TINY_F32.scaled(layers=2),
}


def _call(entry, w, cache, layer, q, k, v):
    dt = torch.int16 if w.dtype == "bf16" else torch.float32
    out = torch.empty(q.shape, dtype=dt, device="cuda")
    lse = torch.empty((q.shape[0], w.heads, w.queries), dtype=torch.float32, device="cuda")
    entry(cache, layer, w.rollouts, q, k, v, out, lse)
    torch.cuda.synchronize()
    return out.cpu(), lse.cpu()


@pytest.mark.parametrize("case", sorted(CASES))
def test_static_work_area_matches_regular_entry_point_twice(case):
    w = CASES[case]
    cache = new_cache(w)
    for b in range(3):   # sink + part of the window
        ks, vs = [], []
        for l in range(w.layers):
            _, k, v = block_inputs(w, (71, b, l), w.rollouts)
            ks.append(to_device(k))
            vs.append(to_device(v))
        fd.fd_cache_commit(cache, 0, w.layers, w.rollouts, ks, vs)
    for call in range(2):   # two calls in a row, different layers and inputs
        layer = call % w.layers
        q, k, v = (to_device(a) for a in block_inputs(w, (72, call), w.rollouts))
        want, want_lse = _call(fd.fd_block_attention, w, cache, layer, q, k, v)
        got, got_lse = _call(fd.fd_block_attention_static, w, cache, layer, q, k, v)
        assert torch.equal(got, want), (case, call)
        assert torch.equal(got_lse, want_lse), (case, call)
    assert fd.fd_get_device_error(cache) == 0


def test_static_work_area_refuses_oversized_calls():
    # a tensor-core call's area holds the block's rotated keys (Hkv heads) and
    # rotated queries (H heads): 3 frames x (1564 x 4 + 1560 x 8) tokens x
    # heads x 128 x 2 bytes = 14.4 MB per rollout, so two rollouts fit in the
    # 32 MiB area and three do not
    big = Workload("static-work-too-big", layers=1, rollouts=3, heads=8, head_dim=128,
                   grid_h=30, grid_w=52, action_tokens=4, block_frames=3, sink_frames=0,
                   window_frames=3, steps=1, blocks=1, dtype="bf16", kv_heads=4)
    g = fd._Geom(fd.make_desc(big))
    need = g.kv + g.q                                # bytes of one rollout
    assert g.kv == big.block_frames * big.frame_tokens * big.hkv * big.head_dim * 2
    assert g.q == big.queries * big.heads * big.head_dim * 2
    assert 2 * need <= fd.STATIC_WORK_BYTES < 3 * need
    cache = new_cache(big)
    q = torch.zeros((3, big.queries, big.heads, big.head_dim), dtype=torch.int16,
                    device="cuda")
    kv = torch.zeros((3, big.block_frames * big.frame_tokens, big.hkv, big.head_dim),
                     dtype=torch.int16, device="cuda")
    out = torch.empty_like(q)
    # two rollouts fit and run
    fd.fd_block_attention_static(cache, 0, 2, q, kv, kv, out)
    torch.cuda.synchronize()
    launches = fd.fd_launch_count()
    with pytest.raises(fd.FdError) as e:
        fd.fd_block_attention_static(cache, 0, 3, q, kv, kv, out)
    assert e.value.status == 4   # FD_ERR_CAPACITY
    assert fd.fd_launch_count() == launches
    assert fd.fd_get_device_error(cache) == 0
