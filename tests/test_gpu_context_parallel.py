"""Context parallelism on one GPU: the key set of every call split over N
shard caches (the shards N GPUs would hold), each shard's attention rows and
log-sum-exp recombined by fd_attention_combine, checked against the oracle's
attention over the whole key set.  Shard r stores ring slots s with
s mod N == r at local index s div N (bit-exact against the oracle's slots);
the block's own keys belong to shard 0, so at the first block every other
shard has no key at all."""
import numpy as np
import pytest
import torch

import oracle
from streaming_autoregressive_video_b200 import binding as fd
from streaming_autoregressive_video_b200 import synth
from streaming_autoregressive_video_b200.workloads import Workload

from support import block_inputs, compare, new_cache, out_values, to_device, to_host

pytestmark = pytest.mark.gpu

BASE = Workload("cp-small", layers=2, rollouts=2, heads=2, head_dim=128, grid_h=6,
                grid_w=13, action_tokens=2, block_frames=2, sink_frames=1, window_frames=4,
                steps=2, blocks=6, dtype="bf16")


def shard_views(cache, w, N, r):
    """Local K, V, positions and counter of one shard's storage."""
    lay = cache.layout
    esz = 2 if w.dtype == "bf16" else 4
    ls = -(-w.slots // N)
    n_kv = w.layers * w.rollouts * ls * w.frame_tokens * w.hkv * w.head_dim
    dt = torch.int16 if esz == 2 else torch.float32
    shape = (w.layers, w.rollouts, ls, w.frame_tokens, w.hkv, w.head_dim)
    st = cache.storage
    k = st[lay.k:lay.k + n_kv * esz].view(dt).view(shape)
    v = st[lay.v:lay.v + n_kv * esz].view(dt).view(shape)
    pos = st[lay.pos:lay.pos + w.layers * w.rollouts * ls * 4].view(torch.int32)
    pos = pos.view(w.layers, w.rollouts, ls)
    cnt = st[lay.count:lay.count + w.layers * w.rollouts * 4].view(torch.int32)
    return k, v, pos, cnt.view(w.layers, w.rollouts)


@pytest.mark.parametrize("N,dtype,extra", [(2, "bf16", {}), (3, "bf16", {"kv_heads": 1}),
                                           (2, "f32", {"head_dim": 64}),
                                           (5, "bf16", {"window_frames": 4})])
def test_shards_recombine_to_whole_key_set(N, dtype, extra):
    w = BASE.scaled(dtype=dtype, **extra)
    caches = [new_cache(w, shards=N, shard=r) for r in range(N)]
    orc = [[oracle.RolloutCache(w.sink_frames, w.window_frames, w.frame_tokens, w.hkv,
                                w.head_dim, dtype) for _ in range(w.rollouts)]
           for _ in range(w.layers)]
    dev = "cuda"
    qshape = (w.rollouts, w.queries, w.heads, w.head_dim)
    lshape = (w.rollouts, w.heads, w.queries)
    tdt = torch.int16 if dtype == "bf16" else torch.float32
    for blk in range(w.blocks):
        for step in range(w.steps):
            for l in range(w.layers):
                q, k, v = block_inputs(w, (61, blk, step, l), w.rollouts)
                qd, kd, vd = to_device(q), to_device(k), to_device(v)
                outs = [torch.empty(qshape, dtype=tdt, device=dev) for _ in range(N)]
                lses = [torch.empty(lshape, dtype=torch.float32, device=dev) for _ in range(N)]
                for r in range(N):
                    fd.fd_block_attention(caches[r], l, w.rollouts, qd, kd, vd, outs[r], lses[r])
                out = torch.empty(qshape, dtype=tdt, device=dev)
                lse = torch.empty(lshape, dtype=torch.float32, device=dev)
                fd.fd_attention_combine(outs, lses, out, lse)
                torch.cuda.synchronize()
                got = out_values(out)
                for ro in range(w.rollouts):
                    want, want_lse = oracle.block_attention(
                        orc[l][ro], q[ro], k[ro], v[ro], tokens=w.tokens, grid_w=w.grid_w,
                        theta=w.theta)
                    compare(got[ro], want, dtype, f"N={N} blk {blk} step {step} l {l} r {ro}")
                    lse_err = np.abs(lse[ro].cpu().numpy() - want_lse).max()
                    assert lse_err <= (1e-2 if dtype == "bf16" else 1e-4), lse_err
                if blk == 0:
                    # before any commit only shard 0 (the block's keys) has keys
                    for r in range(1, N):
                        assert torch.all(outs[r] == 0)
                        assert torch.all(torch.isneginf(lses[r]))
        # commit the last step's keys/values to every shard and the oracle
        ks, vs = [], []
        for l in range(w.layers):
            _, k, v = block_inputs(w, (62, blk, l), w.rollouts)
            ks.append(to_device(k))
            vs.append(to_device(v))
            for ro in range(w.rollouts):
                F, Tf = w.block_frames, w.frame_tokens
                orc[l][ro].commit(k[ro].reshape(F, Tf, w.hkv, w.head_dim),
                                  v[ro].reshape(F, Tf, w.hkv, w.head_dim))
        for r in range(N):
            fd.fd_cache_commit(caches[r], 0, w.layers, w.rollouts, ks, vs)
        torch.cuda.synchronize()
        # each shard holds exactly its slots, bit for bit
        for r in range(N):
            kk, vv, pos, cnt = shard_views(caches[r], w, N, r)
            kk, vv, pos, cnt = to_host(kk), to_host(vv), to_host(pos), to_host(cnt)
            for l in range(w.layers):
                for ro in range(w.rollouts):
                    o = orc[l][ro]
                    assert cnt[l, ro] == o.n
                    for s in range(r, o.valid_slots(), N):
                        assert np.array_equal(kk[l, ro, s // N], o.k[s]), (r, l, ro, s)
                        assert np.array_equal(vv[l, ro, s // N], o.v[s]), (r, l, ro, s)
                        assert pos[l, ro, s // N] == o.pos[s]
    for c in caches:
        assert fd.fd_get_device_error(c) == 0


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_combine_matches_oracle(dtype):
    R, Mq, H, d, N = 2, 37, 3, 96, 4
    g = torch.Generator().manual_seed(9)
    outs, lses = [], []
    for i in range(N):
        o = torch.randn((R, Mq, H, d), generator=g)
        lse = torch.randn((R, H, Mq), generator=g) * 4
        if i == 2:
            lse[0] = -float("inf")          # a part without keys for rollout 0
        outs.append(o.to(torch.bfloat16) if dtype == "bf16" else o)
        lses.append(lse)
    lses[0][1, 1, :5] = -float("inf")       # rows with no key in any part
    lses[1][1, 1, :5] = -float("inf")
    lses[2][1, 1, :5] = -float("inf")
    lses[3][1, 1, :5] = -float("inf")
    dev = "cuda"
    out = torch.empty((R, Mq, H, d), dtype=outs[0].dtype, device=dev)
    lse = torch.empty((R, H, Mq), dtype=torch.float32, device=dev)
    fd.fd_attention_combine([o.to(dev) for o in outs], [x.to(dev) for x in lses], out, lse)
    torch.cuda.synchronize()
    # the oracle states the combination per rollout: [Mq][H][d] rows, [H][Mq] lse
    per = [oracle.combine_partials([o[r].double().numpy() for o in outs],
                                   [x[r].double().numpy() for x in lses]) for r in range(R)]
    want = np.stack([p[0] for p in per])
    want_lse = np.stack([p[1] for p in per])
    got = out.double().cpu().numpy()
    compare(got, want, dtype, "combine")
    gl = lse.cpu().numpy()
    fin = np.isfinite(want_lse)
    assert np.all(np.isneginf(gl[~fin]))
    assert np.abs(gl[fin] - want_lse[fin]).max() <= 1e-5


def test_shard_without_lse_is_refused():
    w = BASE.scaled(layers=1, rollouts=1)
    c = new_cache(w, shards=2, shard=1)
    q, k, v = block_inputs(w, (63,), 1)
    out = torch.empty((1, w.queries, w.heads, w.head_dim), dtype=torch.int16, device="cuda")
    with pytest.raises(fd.FdError) as e:
        fd.fd_block_attention(c, 0, 1, to_device(q), to_device(k), to_device(v), out, None)
    assert e.value.status == 1
