"""The oracle against the hand-derived fixtures under tests/golden/.

Each fixture states its source passage and the reading it follows, and was
written by hand from them (no program produced its numbers).  They pin the
ring's slot map, the RoPE section split and frequencies, the token
coordinates of multi-view frames with action tokens, and one worked attention
call through sink, window eviction and the block."""
import json
import math
import os

import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _rows(name):
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                head, _, tail = line.partition("|")
                yield head.split(), tail


def test_ring_slots_fixture():
    n = 0
    for head, tail in _rows("ring_slots.txt"):
        kind, S, W = head[0], int(head[1]), int(head[2])
        want = [int(x) for x in tail.split()]
        if kind == "slot":
            assert [oracle.slot_of(m, S, W) for m in range(len(want))] == want, (S, W)
        else:
            assert [oracle.valid_slot_count(k, S, W) for k in range(len(want))] == want, (S, W)
        n += 1
    assert n == 11


def test_ring_cache_follows_the_slot_fixture():
    """The oracle's cache object stores frame m in the fixture's slot."""
    for head, tail in _rows("ring_slots.txt"):
        if head[0] != "slot":
            continue
        S, W = int(head[1]), int(head[2])
        want = [int(x) for x in tail.split()]
        c = oracle.RolloutCache(S, W, 1, 1, 2, "f32")
        for m, slot in enumerate(want):
            c.commit(np.full((1, 1, 1, 2), m, np.float32), np.full((1, 1, 1, 2), -m, np.float32))
            assert c.pos[slot] == m and c.k[slot, 0, 0, 0] == m and c.v[slot, 0, 0, 0] == -m


def test_rope_sections_and_frequencies_fixture():
    n = 0
    for head, tail in _rows("rope_sections.txt"):
        vals = tail.split()
        if head[0] == "sections":
            assert oracle.rope_sections(int(head[1])) == tuple(int(x) for x in vals)
        else:
            d, theta = int(head[1]), float(head[2])
            p_t, p_h, p_w = oracle.rope_sections(d)
            got = np.concatenate([oracle.rope_inv_freq(p, theta) for p in (p_t, p_h, p_w)])
            want = np.array([float(x) for x in vals])
            assert got.shape == want.shape
            assert np.allclose(got, want, rtol=1e-14, atol=0)
            # the angles of a token at (t, h, w) = (1, 1, 1) are the frequencies
            assert np.allclose(oracle.rope_angles(1.0, 1.0, 1.0, d, theta), want,
                               rtol=1e-14, atol=0)
        n += 1
    assert n == 14


def test_token_coords_fixture():
    n = 0
    for head, tail in _rows("token_coords.txt"):
        Tf, T, gw, vt = (int(x) for x in head[1:5])
        hs, ws = tail.split(";")
        h, w = oracle.token_coords(Tf, T, gw, vt)
        assert list(h) == [int(x) for x in hs.split()], head
        assert list(w) == [int(x) for x in ws.split()], head
        n += 1
    assert n == 4


def test_worked_attention_fixture():
    with open(os.path.join(GOLDEN, "attention_sink_window.json")) as f:
        g = json.load(f)
    d, H = g["head_dim"], g["heads"]
    T = g["grid_h"] * g["grid_w"]
    c = oracle.RolloutCache(g["sink_frames"], g["window_frames"], T, H, d, "f32")
    for k, v in zip(g["commits_k"], g["commits_v"]):
        c.commit(np.array(k, np.float32).reshape(1, T, H, d),
                 np.array(v, np.float32).reshape(1, T, H, d))
    assert c.valid_slots() == g["want_valid_slots"]
    assert list(c.pos[:c.valid_slots()]) == g["want_pos"]
    q = np.array(g["block_q"], np.float32).reshape(T, H, d)
    k = np.array(g["block_k"], np.float32).reshape(T, H, d)
    v = np.array(g["block_v"], np.float32).reshape(T, H, d)
    out, lse = oracle.block_attention(c, q, k, v, tokens=T, grid_w=g["grid_w"],
                                      theta=g["theta"])
    assert np.allclose(out.reshape(-1), g["want_out"], rtol=0, atol=1e-12)
    want_lse = g["want_score_dot"] / math.sqrt(d) + math.log(g["want_keys"])
    assert abs(float(lse.reshape(-1)[0]) - want_lse) <= 1e-12


@pytest.mark.parametrize("mistake", ["none", "t_on_h_pair", "evicted_frame_kept",
                                     "no_block_key"])
def test_worked_attention_fixture_catches_mistakes(mistake):
    """The fixture's numbers follow from its inputs by hand arithmetic, and
    each mistake it is meant to catch moves the result away from them
    (scores rebuilt here pair by pair, without the oracle)."""
    with open(os.path.join(GOLDEN, "attention_sink_window.json")) as f:
        g = json.load(f)
    d = g["head_dim"]
    q = np.array(g["block_q"], dtype=np.float64)
    keys = [np.array(x, dtype=np.float64) for x in g["commits_k"]]
    vals = [np.array(x, dtype=np.float64) for x in g["commits_v"]]
    frames = [0, 2, 3]                   # the fixture's key set (cache part)
    if mistake == "evicted_frame_kept":
        frames = [0, 1, 2, 3]
    ks = [keys[m] for m in frames]
    vs = [vals[m] for m in frames]
    ts = list(frames)
    if mistake != "no_block_key":
        ks.append(np.array(g["block_k"], dtype=np.float64))
        vs.append(np.array(g["block_v"], dtype=np.float64))
        ts.append(4)

    def turn(x, pair, ang):
        y = x.copy()
        c, s = math.cos(ang), math.sin(ang)
        y[2 * pair] = x[2 * pair] * c - x[2 * pair + 1] * s
        y[2 * pair + 1] = x[2 * pair] * s + x[2 * pair + 1] * c
        return y

    # the t rotation applied to the h pair (pair 1) instead of pair 0
    rot_pair = 1 if mistake == "t_on_h_pair" else 0
    qr = turn(q, rot_pair, 4.0)
    s = np.array([turn(kk, rot_pair, float(t)) @ qr for kk, t in zip(ks, ts)]) / math.sqrt(d)
    p = np.exp(s - s.max())
    out = (p[:, None] * np.array(vs)).sum(0) / p.sum()
    if mistake == "none":
        assert np.allclose(out, g["want_out"], rtol=0, atol=1e-12)
    else:
        assert not np.allclose(out, g["want_out"], rtol=0, atol=1e-6)


def test_window_reset_fixture():
    """The window-boundary policy (R12) follows the hand-worked sequences:
    when the window restarts, which positions the block gets, which slots its
    attention sees and the counter after its commit."""
    caches, n_rows = {}, 0
    for head, tail in _rows("window_reset.txt"):
        S, W, F, c, blk = (int(x) for x in head)
        n0, restart, n1, t_blk, seen, n2 = tail.split()
        if (S, W, F, c) not in caches:
            cache = oracle.RolloutCache(S, W, 1, 1, 2, "f32")
            cond = np.zeros((c, 1, 1, 2), np.float32)
            oracle.start_window(cache, cond, cond)          # a new sequence
            caches[(S, W, F, c)] = cache
        cache = caches[(S, W, F, c)]
        assert cache.n == int(n0), (S, W, F, c, blk)
        hit = oracle.window_boundary_reached(cache.n, F, S, W)
        assert hit == bool(int(restart)), (S, W, F, c, blk)
        if hit:
            cond = np.zeros((c, 1, 1, 2), np.float32)
            oracle.start_window(cache, cond, cond)
        assert cache.n == int(n1)
        assert [cache.n + f for f in range(F)] == [int(x) for x in t_blk.split(",")]
        nv = cache.valid_slots()
        assert [f"{s}:{cache.pos[s]}" for s in range(nv)] == seen.split(","), (S, W, blk)
        frames = np.full((F, 1, 1, 2), 7, np.float32)
        cache.commit(frames, frames)
        assert cache.n == int(n2)
        n_rows += 1
    assert n_rows == 14
