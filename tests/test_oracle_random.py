"""Randomised pins of the oracle's attention against masked full-history
attention written as pure-Python loops.

Hypothesis draws the ring geometry (sinks, window, block size), the frame
grid, action tokens, query and key/value heads, camera views, and a rollout
of ragged commits (each commit stores 1..F frames).  At every block the
oracle's answer over its rolling cache must equal attention over every frame
ever committed, masked to the sinks (frames 0..S-1), the last W non-sink
frames and the block itself ("NVIDIA FlashDreams Is the Open-Source Inference
Engine Robotics World Models Needed", Bounded Memory for Infinite Rollouts;
readings: sinks first, then a W-slot ring; query head h reads key/value head
h div (H/Hkv); views share t and repeat (h, w))."""
import math

import numpy as np
from hypothesis import HealthCheck, given, settings
from hypothesis import strategies as st

from oracle import RolloutCache, block_attention, rope_angles, rope_rotate


def _coords(j, T, Tv, gw):
    if j >= T:                        # action token
        return 0, 0
    tv = j % Tv
    return tv // gw, tv % gw


def _masked_full_history(history, n, S, W, q, k, v, T, Tv, gw, theta):
    """history: frames 0..n-1 as (k [Tf][Hkv][d], v), fp64.  Pure loops."""
    Mq, H, d = q.shape
    F = Mq // T
    Tf = k.shape[0] // F
    Hkv = k.shape[1]
    keys = []
    for m in range(n):
        if m < S or (m >= S and m >= n - W):
            keys += [(m, j, history[m][0][j], history[m][1][j]) for j in range(Tf)]
    for f in range(F):
        keys += [(n + f, j, k[f * Tf + j], v[f * Tf + j]) for j in range(Tf)]
    out = np.zeros((Mq, H, d))
    lse = np.zeros((H, Mq))
    for i in range(Mq):
        hq, wq = _coords(i % T, T, Tv, gw)
        for hh in range(H):
            g = hh // (H // Hkv)
            qr = rope_rotate(q[i, hh], rope_angles(n + i // T, hq, wq, d, theta))
            scores = []
            for (tk, j, kvec, _) in keys:
                hk, wk = _coords(j, T, Tv, gw)
                kr = rope_rotate(kvec[g], rope_angles(tk, hk, wk, d, theta))
                scores.append(sum(float(a) * float(b) for a, b in zip(qr, kr)) / math.sqrt(d))
            mx = max(scores)
            ex = [math.exp(s - mx) for s in scores]
            tot = sum(ex)
            for e_, (_, _, _, vvec) in zip(ex, keys):
                out[i, hh] += (e_ / tot) * vvec[g]
            lse[hh, i] = mx + math.log(tot)
    return out, lse


@st.composite
def rollouts(draw):
    S = draw(st.integers(0, 2))
    W = draw(st.integers(1, 4))
    F = draw(st.integers(1, min(W, 2)))
    views = draw(st.integers(1, 2))
    gh, gw = draw(st.integers(1, 2)), draw(st.integers(1, 3))
    A = draw(st.integers(0, 2))
    Hkv = draw(st.integers(1, 2))
    H = Hkv * draw(st.integers(1, 2))
    commits = draw(st.lists(st.integers(1, F), min_size=0, max_size=6))
    seed = draw(st.integers(0, 2 ** 31 - 1))
    return S, W, F, views, gh, gw, A, H, Hkv, commits, seed


@settings(max_examples=30, deadline=None, suppress_health_check=[HealthCheck.too_slow])
@given(rollouts())
def test_rolling_cache_equals_masked_full_history_random(case):
    S, W, F, views, gh, gw, A, H, Hkv, commits, seed = case
    rng = np.random.default_rng(seed)
    d, theta = 6 * int(rng.integers(1, 3)), 1.0e4
    Tv = gh * gw
    T = views * Tv
    Tf = T + A
    cache = RolloutCache(S, W, Tf, Hkv, d, "f32")
    history = []
    for nf in commits + [None]:       # attention after every commit, then one more
        q = rng.standard_normal((F * T, H, d)).astype(np.float32)
        k = rng.standard_normal((F * Tf, Hkv, d)).astype(np.float32)
        v = rng.standard_normal((F * Tf, Hkv, d)).astype(np.float32)
        out, lse = block_attention(cache, q, k, v, tokens=T, grid_w=gw, theta=theta,
                                   view_tokens=Tv if views > 1 else 0)
        hist = [(hk.astype(np.float64), hv.astype(np.float64)) for hk, hv in history]
        ref, ref_lse = _masked_full_history(hist, cache.n, S, W, q.astype(np.float64),
                                            k.astype(np.float64), v.astype(np.float64),
                                            T, Tv, gw, theta)
        np.testing.assert_allclose(out, ref, rtol=0, atol=1e-12)
        np.testing.assert_allclose(lse, ref_lse, rtol=0, atol=1e-12)
        if nf is None:
            break
        kf = k.reshape(F, Tf, Hkv, d)[:nf]
        vf = v.reshape(F, Tf, Hkv, d)[:nf]
        cache.commit(kf, vf)
        history += [(kf[f], vf[f]) for f in range(nf)]


@settings(max_examples=30, deadline=None, suppress_health_check=[HealthCheck.too_slow])
@given(rollouts(), st.integers(1, 5))
def test_key_set_parts_recombine_random(case, N):
    """Context parallelism ("NVIDIA FlashDreams ...", Multi-GPU Context
    Parallelism; reading: cache slot s belongs to part s mod N, the block's
    keys to part 0): the parts' rows merged by their log-sum-exps equal the
    attention over the whole key set, for any fill of the ring."""
    from oracle import combine_partials
    S, W, F, views, gh, gw, A, H, Hkv, commits, seed = case
    rng = np.random.default_rng(seed)
    d, theta = 12, 1.0e4
    Tv = gh * gw
    T = views * Tv
    Tf = T + A
    vt = Tv if views > 1 else 0
    cache = RolloutCache(S, W, Tf, Hkv, d, "f32")
    for nf in commits:
        cache.commit(rng.standard_normal((nf, Tf, Hkv, d)).astype(np.float32),
                     rng.standard_normal((nf, Tf, Hkv, d)).astype(np.float32))
    q = rng.standard_normal((F * T, H, d)).astype(np.float32)
    k = rng.standard_normal((F * Tf, Hkv, d)).astype(np.float32)
    v = rng.standard_normal((F * Tf, Hkv, d)).astype(np.float32)
    kw = dict(tokens=T, grid_w=gw, theta=theta, view_tokens=vt)
    whole, whole_lse = block_attention(cache, q, k, v, **kw)
    outs, lses = [], []
    for part in range(N):
        o, l = block_attention(cache, q, k, v, slot_part=(N, part),
                               include_block=(part == 0), **kw)
        outs.append(o)
        lses.append(l)
    got, got_lse = combine_partials(outs, lses)
    np.testing.assert_allclose(got, whole, rtol=0, atol=1e-12)
    np.testing.assert_allclose(got_lse, whole_lse, rtol=0, atol=1e-12)
