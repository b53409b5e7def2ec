"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle on the
same seeded bytes.  Cache contents, slot positions and counters bit-exact;
bf16 outputs max abs <= 2e-2 and mean abs <= 2e-3; fp32 outputs max abs
<= 1e-4.  Sizes span several 128-row / 128-key tiles with ragged tails."""
import numpy as np
import pytest
import torch

import oracle
from streaming_autoregressive_video_b200 import binding as fd
from streaming_autoregressive_video_b200 import synth
from streaming_autoregressive_video_b200.workloads import TINY_F32, Workload

from support import (Lockstep, block_inputs, compare, rotated_bound, to_device, to_host,
                     views)

pytestmark = pytest.mark.gpu

SMALL = Workload("small-bf16", layers=2, rollouts=3, heads=2, head_dim=128,
                 grid_h=12, grid_w=13, action_tokens=0, block_frames=2,
                 sink_frames=1, window_frames=3, steps=2, blocks=6, dtype="bf16")


def _commit_block(ls, w, seed, layers=None, frames=None):
    layers = layers or list(range(w.layers))
    ks, vs = [], []
    for l in layers:
        _, k, v = block_inputs(w, (seed, l, 77), w.rollouts)
        ks.append(k)
        vs.append(v)
    ls.commit(layers, ks, vs, frames=frames)


@pytest.mark.parametrize("dtype,kv_heads,views", [("bf16", 0, 1), ("f32", 0, 1),
                                                  ("bf16", 1, 1), ("bf16", 0, 2)])
def test_commit_and_reset_bit_exact(dtype, kv_heads, views):
    w = SMALL.scaled(dtype=dtype, grid_h=3, grid_w=5, action_tokens=2, kv_heads=kv_heads,
                     views=views)
    ls = Lockstep(w)
    ls.check_cache_exact()
    rng = np.random.default_rng(5)
    for blk in range(9):
        frames = None if blk % 2 else [int(x) for x in rng.integers(0, w.block_frames + 1, w.rollouts)]
        _commit_block(ls, w, 100 + blk, frames=frames)
        ls.check_cache_exact()
        ls.check_rotated_keys()
        if blk == 5:
            ls.reset([1])
            ls.check_cache_exact()
            ls.check_rotated_keys()
    assert fd.fd_get_device_error(ls.cache) == 0


@pytest.mark.parametrize("dtype,tokens", [("bf16", "T"), ("bf16", "Tf"), ("f32", "Tf")])
def test_rope3d_matches_oracle(dtype, tokens):
    # keys carry Hkv = 1 head, queries H = 2; two camera views per frame
    w = SMALL.scaled(dtype=dtype, grid_h=5, grid_w=7, action_tokens=3, window_frames=4,
                     kv_heads=1, views=2)
    ls = Lockstep(w)
    for blk in range(3):
        _commit_block(ls, w, 200 + blk)
    Tx = w.tokens if tokens == "T" else w.frame_tokens
    heads = w.heads if tokens == "T" else w.hkv
    x = synth.normal(synth.seed_of(9, Tx), (w.rollouts, w.block_frames, Tx, heads, w.head_dim), dtype)
    xd = to_device(x)
    fd.fd_rope3d(ls.cache, 1, w.rollouts, xd, Tx, heads)
    torch.cuda.synchronize()
    got = oracle.values_f64(to_host(xd), dtype)
    h, ww = oracle.token_coords(Tx, w.tokens, w.grid_w, w.view_tokens)
    for r in range(w.rollouts):
        n = ls.orc[1][r].n
        t = (n + np.arange(w.block_frames))[:, None]
        ang = oracle.rope_angles(t, h[None, :], ww[None, :], w.head_dim, w.theta)[:, :, None, :]
        raw = oracle.values_f64(x[r], dtype)
        want = oracle.rope_rotate(raw, ang)
        err = np.abs(got[r] - want)
        if dtype == "bf16":
            # one bf16 rounding of the fp32 rotation
            assert np.all(err <= rotated_bound(want, raw, dtype))
        else:
            assert err.max() <= 1e-5


@pytest.mark.parametrize("kv_heads,views", [(0, 1), (1, 1), (0, 2)])
def test_attention_f32_tiny_rollout(kv_heads, views):
    """Tiny fp32 rollout: 20 blocks x 2 steps through a 3-frame window (and
    the same with grouped-query attention, one key/value head, and with two
    camera views per frame)."""
    w = TINY_F32.scaled(kv_heads=kv_heads, views=views)
    ls = Lockstep(w)
    for blk in range(w.blocks):
        for step in range(w.steps):
            q, k, v = block_inputs(w, (1, blk, step), w.rollouts)
            ls.attention(0, q, k, v, what=f"blk {blk} step {step}")
        ls.commit([0], [k], [v])
        ls.check_cache_exact()
    assert fd.fd_get_device_error(ls.cache) == 0


@pytest.mark.parametrize("d,shape", [
    (64, dict()),                                           # Tf=156, Mq=312
    (64, dict(heads=4, kv_heads=2, action_tokens=4, views=2)),  # GQA, actions, 2 views
    (32, dict(rollouts=2, sink_frames=2, window_frames=2)),     # sinks straddled
    (96, dict(grid_h=5, grid_w=7, action_tokens=1)),        # d/2 = 48 pairs: t/h/w = 16/16/16
])
def test_attention_bf16_head_sizes(d, shape):
    """bf16 caches with d = 64 run on the tensor-core kernel's 64-column
    instance, d = 32 and 96 on the CUDA-core kernel (fp32 arithmetic on the
    stored bf16 values): a rollout through empty, partial, full and wrapped
    cache states against the oracle at the bf16 tolerance."""
    w = SMALL.scaled(head_dim=d, blocks=5, **shape)
    ls = Lockstep(w)
    for blk in range(w.blocks):
        for l in range(w.layers):
            q, k, v = block_inputs(w, (8, blk, l), w.rollouts)
            ls.attention(l, q, k, v, what=f"d {d} blk {blk} layer {l}")
        _commit_block(ls, w, 700 + blk)
        ls.check_cache_exact()
        ls.check_rotated_keys()
    assert fd.fd_get_device_error(ls.cache) == 0


def test_attention_bf16_d64_tensor_cores_480p_shape():
    """The d = 64 tensor-core instance at the 480p frame shape (30x52 grid,
    3-frame blocks, 1 sink + 6 window frames, cache full): many query-tile
    pairs per head, split between CTAs, against the oracle on sampled rows of
    every head (rows from every query tile, the ragged last one included)."""
    from streaming_autoregressive_video_b200.workloads import SINGLE_480P
    w = SINGLE_480P.scaled(name="480p-d64", head_dim=64, heads=4, layers=1)
    ls = Lockstep(w)
    for blk in range(3):
        _commit_block(ls, w, 900 + blk)
    ls.check_cache_exact()
    ls.check_rotated_keys()
    rows = np.unique(np.concatenate([np.arange(0, w.queries, 37), [w.queries - 1]]))
    for step in range(2):
        q, k, v = block_inputs(w, (901, step), 1)
        ls.attention(0, q, k, v, rows=rows, what=f"480p d64 step {step}")
    assert fd.fd_get_device_error(ls.cache) == 0


def test_unsupported_bf16_head_dim_is_refused_cleanly():
    """A head size that no attention kernel takes (d = 48: a multiple of 8, so
    the cache accepts it, but not of 32): the cache commits and rotates, but
    attention returns FD_ERR_UNSUPPORTED without launching anything, and the
    context stays usable."""
    w = Workload("bf16-d48", layers=1, rollouts=1, heads=2, head_dim=48, grid_h=3, grid_w=4,
                 action_tokens=0, block_frames=1, sink_frames=0, window_frames=2, steps=1,
                 blocks=1, dtype="bf16")
    ls = Lockstep(w)
    q, k, v = block_inputs(w, (7, 0), 1)
    _commit_block(ls, w, 500)
    ls.check_cache_exact()
    ls.check_rotated_keys()
    out = torch.empty((1, w.queries, w.heads, w.head_dim), dtype=torch.int16, device="cuda")
    before = fd.fd_launch_count()
    with pytest.raises(fd.FdError) as e:
        fd.fd_block_attention(ls.cache, 0, 1, to_device(q), to_device(k), to_device(v), out)
    assert e.value.status == 7
    assert fd.fd_launch_count() == before
    assert fd.fd_get_device_error(ls.cache) == 0


def test_single_key_returns_value_exactly_bf16():
    w = Workload("one-key", layers=1, rollouts=1, heads=3, head_dim=128, grid_h=1, grid_w=1,
                 action_tokens=0, block_frames=1, sink_frames=0, window_frames=1, steps=1,
                 blocks=1, dtype="bf16")
    ls = Lockstep(w)
    q, k, v = block_inputs(w, (3, 0), 1)
    got, _ = ls.attention(0, q, k, v, what="one key")
    assert np.array_equal(got[0], oracle.values_f64(v[0], "bf16"))


@pytest.mark.parametrize("shape", [
    dict(),                                            # Tf=156, Mq=312
    dict(action_tokens=4),                             # Tf=160 with action tokens
    dict(grid_h=16, grid_w=20, block_frames=3, window_frames=3, sink_frames=0),  # F = W
    dict(rollouts=4, sink_frames=2, window_frames=4),  # sinks straddled
    dict(heads=4, kv_heads=2, action_tokens=4),        # grouped-query attention
    dict(heads=3, kv_heads=1, rollouts=2),             # one key/value head
    dict(views=3, grid_h=4, grid_w=5, action_tokens=2),  # three camera views
])
def test_attention_bf16_rollout(shape):
    """Rollout through empty, partial, full and wrapped cache states."""
    w = SMALL.scaled(**shape)
    ls = Lockstep(w)
    for blk in range(w.blocks):
        for step in range(w.steps):
            for l in range(w.layers):
                q, k, v = block_inputs(w, (2, blk, step, l), w.rollouts)
                ls.attention(l, q, k, v, what=f"blk {blk} step {step} layer {l}")
        _commit_block(ls, w, 300 + blk)
        ls.check_cache_exact()
    assert fd.fd_get_device_error(ls.cache) == 0


def test_attention_bf16_ragged_rollouts():
    """Rollouts with different cache fill in one call."""
    w = SMALL.scaled(rollouts=5, window_frames=6, sink_frames=0, block_frames=3, layers=1)
    ls = Lockstep(w)
    rng = np.random.default_rng(11)
    for blk in range(4):
        frames = [int(x) for x in rng.integers(0, 4, w.rollouts)]
        _commit_block(ls, w, 400 + blk, frames=frames)
    ls.check_cache_exact()
    q, k, v = block_inputs(w, (4,), w.rollouts)
    ls.attention(0, q, k, v, what="ragged")
    # fewer active rollouts than the cache holds
    ls.attention(0, q[:2], k[:2], v[:2], n_rollouts=2, what="ragged n=2")


def test_attention_bf16_many_rollouts():
    """More rollouts than the fold kernel keeps iteration offsets for in
    shared memory (64), with ragged fills so the rollouts' units differ in
    length: 70 single-tile units on at most 148 CTAs, every one split between
    CTAs and folded, the offsets of rollouts 64-69 recomputed."""
    w = Workload("many-rollouts-bf16", layers=1, rollouts=70, heads=1, head_dim=128,
                 grid_h=3, grid_w=4, action_tokens=0, block_frames=2, sink_frames=1,
                 window_frames=4, steps=1, blocks=1, dtype="bf16")
    ls = Lockstep(w)
    rng = np.random.default_rng(5)
    for blk in range(3):
        frames = [int(x) for x in rng.integers(0, w.block_frames + 1, w.rollouts)]
        _commit_block(ls, w, 500 + blk, frames=frames)
    ls.check_cache_exact()
    q, k, v = block_inputs(w, (5,), w.rollouts)
    ls.attention(0, q, k, v, what="70 rollouts")
    assert fd.fd_get_device_error(ls.cache) == 0


def test_softmax_exp2_against_exp2f():
    """The FMA-pipe exponential used for part of the softmax weights agrees
    with CUDA's exp2f (and the exact 2^x) to the fitted polynomial's bound."""
    g = torch.Generator().manual_seed(5)
    x = torch.cat([torch.linspace(-126.0, 8.0, 1 << 20),
                   torch.rand(1 << 18, generator=g) * 134.0 - 126.0]).float()
    y = torch.empty(3 * x.numel(), dtype=torch.float32, device="cuda")
    xd = x.cuda()
    fd.fd_exp2_selfcheck(xd, y)
    torch.cuda.synchronize()
    poly, hw, ref = y.view(-1, 3).cpu().double().T
    exact = torch.exp2(x.double())
    # the cubic's own bound is 7.5e-5; fp32 evaluation adds a few ulp
    assert float(((poly - ref).abs() / ref).max()) <= 2.0e-4
    assert float(((poly - exact).abs() / exact).max()) <= 2.0e-4
    assert float(((hw - exact).abs() / exact).max()) <= 1.0e-5


def test_device_wait_gives_up_and_reports():
    """A device-side wait on a barrier nothing completes gives up after its
    limit, sets the error word (timeout, site 5) and leaves the context usable."""
    w = TINY_F32
    ls = Lockstep(w)
    assert fd.fd_get_device_error(ls.cache) == 0
    fd.fd_selftest_bounded_wait(ls.cache, 50)
    torch.cuda.synchronize()
    assert fd.fd_get_device_error(ls.cache) == (5 << 8) | 1
    assert fd.fd_get_device_error(ls.cache) == 0       # read clears it
    q, k, v = block_inputs(w, (6, 0), 1)               # the context still works
    ls.attention(0, q, k, v, what="after self-test")
    assert fd.fd_get_device_error(ls.cache) == 0


def test_block_captured_in_cuda_graph_matches_eager():
    """One block (denoising steps x layers + commit) captured once in a CUDA
    graph and replayed for three blocks gives bit-identical outputs and cache
    contents to eager calls (no host synchronisation inside the calls; the
    device counters drive the positions)."""
    w = SMALL.scaled(rollouts=2)
    eager, graphed = Lockstep(w), Lockstep(w)
    shape_q = (w.rollouts, w.queries, w.heads, w.head_dim)
    shape_k = (w.rollouts, w.block_frames * w.frame_tokens, w.heads, w.head_dim)
    sq = [[torch.empty(shape_q, dtype=torch.int16, device="cuda") for _ in range(w.layers)]
          for _ in range(w.steps)]
    sk = [[torch.empty(shape_k, dtype=torch.int16, device="cuda") for _ in range(w.layers)]
          for _ in range(w.steps)]
    sv = [[torch.empty(shape_k, dtype=torch.int16, device="cuda") for _ in range(w.layers)]
          for _ in range(w.steps)]
    outs = [[torch.empty(shape_q, dtype=torch.int16, device="cuda") for _ in range(w.layers)]
            for _ in range(w.steps)]

    def block(cache):
        for s in range(w.steps):
            for l in range(w.layers):
                fd.fd_block_attention(cache, l, w.rollouts, sq[s][l], sk[s][l], sv[s][l],
                                      outs[s][l])
        fd.fd_cache_commit(cache, 0, w.layers, w.rollouts, sk[-1], sv[-1])

    def fill(blk):
        for s in range(w.steps):
            for l in range(w.layers):
                q, k, v = block_inputs(w, (8, blk, s, l), w.rollouts)
                sq[s][l].copy_(to_device(q))
                sk[s][l].copy_(to_device(k))
                sv[s][l].copy_(to_device(v))

    # warm-up launch outside capture (first-call set-up happens here)
    fill(0)
    block(eager.cache)
    want0 = [[o.clone() for o in row] for row in outs]
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        block(graphed.cache)
    for blk in range(3):
        fill(blk)
        g.replay()
        torch.cuda.synchronize()
        got = [[o.clone() for o in row] for row in outs]
        if blk > 0:
            block(eager.cache)
            torch.cuda.synchronize()
            want = [[o.clone() for o in row] for row in outs]
        else:
            want = want0
        for s in range(w.steps):
            for l in range(w.layers):
                assert torch.equal(got[s][l], want[s][l]), (blk, s, l)
    ke, ve, pe, ce = views(eager.cache, w)
    kg, vg, pg, cg = views(graphed.cache, w)
    assert torch.equal(pe, pg) and torch.equal(ce, cg)
    assert torch.equal(ke, kg) and torch.equal(ve, vg)
    assert fd.fd_get_device_error(graphed.cache) == 0


@pytest.mark.parametrize("seed", range(10))
def test_random_shapes_rollout(seed):
    """Seeded random geometries (heads and key/value heads, grid, views, action
    tokens, block / sink / window sizes, rollouts, dtype and head size), a
    short rollout with ragged commits through the cache, every call against
    the oracle and the cache bit-exact."""
    rng = np.random.default_rng(1000 + seed)
    heads = int(rng.integers(1, 5))
    kv = int(rng.choice([h for h in range(1, heads + 1) if heads % h == 0]))
    F = int(rng.integers(1, 4))
    dtype = "f32" if seed % 4 == 3 else "bf16"
    d = int(rng.choice([32, 64])) if dtype == "f32" else 128
    w = Workload(f"random-{seed}", layers=1, rollouts=int(rng.integers(1, 4)), heads=heads,
                 head_dim=d, grid_h=int(rng.integers(1, 7)), grid_w=int(rng.integers(1, 10)),
                 action_tokens=int(rng.choice([0, 1, 3])), block_frames=F,
                 sink_frames=int(rng.integers(0, 3)), window_frames=F + int(rng.integers(0, 3)),
                 steps=1, blocks=int(rng.integers(3, 6)), dtype=dtype,
                 kv_heads=kv if kv != heads else 0, views=int(rng.choice([1, 1, 2])))
    ls = Lockstep(w)
    for blk in range(w.blocks):
        q, k, v = block_inputs(w, (71, seed, blk), w.rollouts)
        ls.attention(0, q, k, v, what=f"{w} blk {blk}")
        frames = [int(x) for x in rng.integers(0, F + 1, w.rollouts)]
        ls.commit([0], [k], [v], frames=frames)
        ls.check_cache_exact()
    assert fd.fd_get_device_error(ls.cache) == 0
