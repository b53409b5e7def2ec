"""Pins of the CPU oracle against closed forms, invariants and brute force.

Each test checks the oracle against something other than itself: a value
derived by hand from the stated reading, an identity the mathematics fixes, or
an independent pure-Python brute force on tiny inputs (full-history attention
with an explicit sink + window + block mask instead of the ring buffer).
"""
import math

import numpy as np
import pytest

import oracle
from oracle import (RolloutCache, block_attention, bf16_bits_to_f64,
                    rope_angles, rope_rotate, rope_sections, slot_of,
                    valid_slot_count, token_coords)


# --------------------------------------------------------------------------
# number format
# --------------------------------------------------------------------------
def test_bf16_decode_closed_forms():
    bits = np.array([0x3F80, 0xC000, 0x0000, 0x8000, 0x7F80, 0x0001, 0x3F81,
                     0x4049], dtype=np.uint16)
    got = bf16_bits_to_f64(bits)
    want = [1.0, -2.0, 0.0, -0.0, math.inf, 2.0 ** -133, 1.0 + 2.0 ** -7,
            3.140625]
    assert list(got) == want
    assert math.copysign(1.0, got[3]) == -1.0


# --------------------------------------------------------------------------
# 3D RoPE
# --------------------------------------------------------------------------
def test_rope_sections():
    assert rope_sections(128) == (22, 21, 21)
    assert rope_sections(64) == (12, 10, 10)
    assert rope_sections(6) == (1, 1, 1)
    assert rope_sections(12) == (2, 2, 2)
    for d in range(6, 258, 2):
        assert sum(rope_sections(d)) == d // 2


def _complex_rotate(x, angles):
    z = x[..., 0::2] + 1j * x[..., 1::2]
    z = z * np.exp(1j * angles)
    out = np.empty_like(x)
    out[..., 0::2] = z.real
    out[..., 1::2] = z.imag
    return out


def test_rope_d6_closed_form():
    # d = 6: one pair per axis, frequency theta^0 = 1: pair 0 turns by t,
    # pair 1 by h, pair 2 by w radians, counter-clockwise in (x[2i], x[2i+1]).
    rng = np.random.default_rng(0)
    x = rng.standard_normal(6)
    t, h, w = 5.0, 2.0, 3.0
    got = rope_rotate(x, rope_angles(t, h, w, 6, 1.0e4))
    want = _complex_rotate(x, np.array([t, h, w]))
    np.testing.assert_allclose(got, want, rtol=0, atol=1e-15)
    # explicit: unit vector e0 lands on (cos t, sin t)
    e0 = np.array([1.0, 0, 0, 0, 0, 0])
    r = rope_rotate(e0, rope_angles(t, h, w, 6, 1.0e4))
    assert r[0] == math.cos(t) and r[1] == math.sin(t)


def test_rope_d12_second_frequency():
    # d = 12: two pairs per axis; with theta = 1e4 the second pair of each
    # axis turns at theta^(-1/2) = 1/100 rad per unit coordinate.
    t, h, w = 100.0, 3.0, 7.0
    ang = rope_angles(t, h, w, 12, 1.0e4)
    want = np.array([t, t / 100, h, h / 100, w, w / 100])
    np.testing.assert_allclose(ang, want, rtol=1e-15, atol=0)
    rng = np.random.default_rng(1)
    x = rng.standard_normal(12)
    np.testing.assert_allclose(rope_rotate(x, ang), _complex_rotate(x, want),
                               rtol=0, atol=1e-13)


def test_rope_axis_structure_d128():
    # moving along one axis turns only that axis' pairs: t -> pairs [0,22),
    # h -> [22,43), w -> [43,64); the first pair of each section turns at 1.
    base = rope_angles(4.0, 5.0, 6.0, 128, 1.0e4)
    dt = rope_angles(5.0, 5.0, 6.0, 128, 1.0e4) - base
    dh = rope_angles(4.0, 6.0, 6.0, 128, 1.0e4) - base
    dw = rope_angles(4.0, 5.0, 7.0, 128, 1.0e4) - base
    assert np.all(dt[:22] > 0) and np.all(dt[22:] == 0)
    assert np.all(dh[22:43] > 0) and np.all(dh[:22] == 0) and np.all(dh[43:] == 0)
    assert np.all(dw[43:] > 0) and np.all(dw[:43] == 0)
    assert dt[0] == 1.0 and dh[22] == 1.0 and dw[43] == 1.0
    # geometric decay inside a section, ending above theta^-1
    for sec in (dt[:22], dh[22:43], dw[43:]):
        ratio = sec[1:] / sec[:-1]
        np.testing.assert_allclose(ratio, ratio[0], rtol=1e-12)
        assert sec[-1] > 1.0e-4


def test_rope_preserves_norm_and_is_identity_at_origin():
    rng = np.random.default_rng(2)
    x = rng.standard_normal((50, 128))
    coords = rng.integers(0, 10000, size=(50, 3)).astype(np.float64)
    y = rope_rotate(x, rope_angles(coords[:, 0], coords[:, 1], coords[:, 2], 128, 1.0e4))
    np.testing.assert_allclose(np.linalg.norm(y, axis=1), np.linalg.norm(x, axis=1),
                               rtol=1e-12)
    z = rope_rotate(x, rope_angles(0.0, 0.0, 0.0, 128, 1.0e4))
    assert np.array_equal(z, x)


def test_rope_depends_only_on_relative_position():
    rng = np.random.default_rng(3)
    for _ in range(20):
        q = rng.standard_normal(128)
        k = rng.standard_normal(128)
        p1 = rng.integers(0, 200, size=3).astype(np.float64)
        p2 = rng.integers(0, 200, size=3).astype(np.float64)
        delta = rng.integers(0, 5000, size=3).astype(np.float64)
        a = rope_rotate(q, rope_angles(*p1, 128, 1.0e4)) @ rope_rotate(k, rope_angles(*p2, 128, 1.0e4))
        b = rope_rotate(q, rope_angles(*(p1 + delta), 128, 1.0e4)) @ \
            rope_rotate(k, rope_angles(*(p2 + delta), 128, 1.0e4))
        assert abs(a - b) <= 1e-9 * (1 + abs(a))


def test_token_coords_row_major_and_actions_at_origin():
    h, w = token_coords(3 * 5 + 4, 15, 5)
    assert list(h[:15]) == [i // 5 for i in range(15)]
    assert list(w[:15]) == [i % 5 for i in range(15)]
    assert list(h[15:]) == [0] * 4 and list(w[15:]) == [0] * 4


# --------------------------------------------------------------------------
# ring buffer
# --------------------------------------------------------------------------
def test_slot_map_closed_form_tables():
    assert [slot_of(m, 1, 3) for m in range(9)] == [0, 1, 2, 3, 1, 2, 3, 1, 2]
    assert [slot_of(m, 0, 3) for m in range(7)] == [0, 1, 2, 0, 1, 2, 0]
    assert [slot_of(m, 2, 1) for m in range(5)] == [0, 1, 2, 2, 2]
    assert [valid_slot_count(n, 1, 6) for n in range(10)] == [0, 1, 2, 3, 4, 5, 6, 7, 7, 7]


@pytest.mark.parametrize("S,W,F", [(0, 3, 1), (1, 6, 3), (1, 8, 1), (0, 12, 3),
                                   (2, 5, 5), (3, 4, 2), (1, 12, 3)])
def test_ring_keeps_sinks_and_last_window_frames(S, W, F):
    rng = np.random.default_rng(S * 100 + W * 10 + F)
    c = RolloutCache(S, W, 2, 1, 2, "f32")
    committed = {}
    for blk in range(60):
        nf = int(rng.integers(0, F + 1)) if blk % 3 == 0 else F
        frames = np.arange(c.n, c.n + nf, dtype=np.float32)
        kf = np.broadcast_to(frames[:, None, None, None], (nf, 2, 1, 2)).copy()
        c.commit(kf, -kf)
        for m in frames:
            committed[int(m)] = m
        n = c.n
        nv = c.valid_slots()
        # valid slots are a prefix; the rest are empty
        assert np.all(c.pos[:nv] >= 0) and np.all(c.pos[nv:] == -1)
        want = set(range(min(n, S))) | set(range(max(S, n - W), n))
        assert set(int(p) for p in c.pos[:nv]) == want
        # each valid slot holds exactly the frame its position names
        for s in range(nv):
            assert np.all(c.k[s] == c.pos[s]) and np.all(c.v[s] == -c.pos[s])
            assert slot_of(int(c.pos[s]), S, W) == s


def test_ring_rejects_commit_larger_than_window():
    c = RolloutCache(1, 3, 2, 1, 2, "f32")
    with pytest.raises(ValueError):
        c.commit(np.zeros((4, 2, 1, 2), np.float32), np.zeros((4, 2, 1, 2), np.float32))


def test_ten_thousand_blocks_memory_constant_and_positions():
    c = RolloutCache(1, 8, 1, 1, 2, "f32")
    nbytes = c.k.nbytes + c.v.nbytes + c.pos.nbytes
    for blk in range(10000):
        f = np.full((1, 1, 1, 2), blk, np.float32)
        c.commit(f, f)
    assert c.k.nbytes + c.v.nbytes + c.pos.nbytes == nbytes
    assert c.n == 10000
    assert int(c.pos[0]) == 0
    assert sorted(int(p) for p in c.pos[1:]) == list(range(9992, 10000))


def test_reset_starts_a_new_sequence():
    c = RolloutCache(1, 3, 2, 1, 2, "f32")
    for _ in range(5):
        c.commit(np.ones((2, 2, 1, 2), np.float32), np.ones((2, 2, 1, 2), np.float32))
    c.reset()
    assert c.n == 0 and np.all(c.pos == -1) and c.valid_slots() == 0


# --------------------------------------------------------------------------
# attention
# --------------------------------------------------------------------------
def _brute_force_block(history, n, S, W, q, k, v, T, Tf, grid_w, theta):
    """Full-history attention with an explicit mask, pure Python loops.

    history: list of (k_frame, v_frame) for frames 0..n-1, fp64 [Tf][H][d].
    A key of frame m is visible to the block iff m < S (sink), or
    max(S, n - W) <= m < n (window), or m belongs to the block itself.
    """
    F = q.shape[0] // T
    H, d = q.shape[1], q.shape[2]
    keys = []        # (t, token, k_vec per head, v_vec per head)
    for m in range(n):
        if m < S or (S <= m and n - W <= m):
            keys += [(m, j, history[m][0][j], history[m][1][j]) for j in range(Tf)]
    for f in range(F):
        keys += [(n + f, j, k[f * Tf + j], v[f * Tf + j]) for j in range(Tf)]
    out = np.zeros(q.shape)
    lse = np.zeros((H, q.shape[0]))
    for i in range(q.shape[0]):
        tq, tok = n + i // T, i % T
        for hh in range(H):
            qr = rope_rotate(q[i, hh], rope_angles(tq, tok // grid_w, tok % grid_w, d, theta))
            scores = []
            for (tk, j, kvec, _) in keys:
                hk, wk = (j // grid_w, j % grid_w) if j < T else (0, 0)
                kr = rope_rotate(kvec[hh], rope_angles(tk, hk, wk, d, theta))
                scores.append(sum(float(a) * float(b) for a, b in zip(qr, kr)) / math.sqrt(d))
            mx = max(scores)
            ex = [math.exp(s - mx) for s in scores]
            tot = sum(ex)
            for e_, (_, _, _, vvec) in zip(ex, keys):
                out[i, hh] += (e_ / tot) * vvec[hh]
            lse[hh, i] = mx + math.log(tot)
    return out, lse


@pytest.mark.parametrize("S,W,F,A", [(1, 3, 2, 1), (0, 3, 1, 0), (2, 2, 2, 0)])
def test_rolling_cache_equals_masked_full_history(S, W, F, A):
    rng = np.random.default_rng(10 + S + W + F + A)
    gh, gw, H, d, theta = 2, 2, 2, 12, 1.0e4
    T = gh * gw
    Tf = T + A
    cache = RolloutCache(S, W, Tf, H, d, "f32")
    history = []
    for blk in range(6):
        n = cache.n
        for step in range(2):
            q = rng.standard_normal((F * T, H, d)).astype(np.float32)
            k = rng.standard_normal((F * Tf, H, d)).astype(np.float32)
            v = rng.standard_normal((F * Tf, H, d)).astype(np.float32)
            out, lse = block_attention(cache, q, k, v, tokens=T, grid_w=gw, theta=theta)
            hist = [(hk.astype(np.float64), hv.astype(np.float64)) for hk, hv in history]
            ref, ref_lse = _brute_force_block(hist, n, S, W, q.astype(np.float64),
                                              k.astype(np.float64), v.astype(np.float64),
                                              T, Tf, gw, theta)
            np.testing.assert_allclose(out, ref, rtol=0, atol=1e-12)
            np.testing.assert_allclose(lse, ref_lse, rtol=0, atol=1e-12)
        kf = k.reshape(F, Tf, H, d)
        vf = v.reshape(F, Tf, H, d)
        cache.commit(kf, vf)
        history += [(kf[f], vf[f]) for f in range(F)]


def test_softmax_rows_sum_to_one():
    rng = np.random.default_rng(20)
    c = RolloutCache(1, 4, 6, 2, 16, "bf16")
    for _ in range(3):
        c.commit(rng.integers(0, 2 ** 16, (2, 6, 2, 16), dtype=np.uint16) & 0xBFFF,
                 rng.integers(0, 2 ** 16, (2, 6, 2, 16), dtype=np.uint16) & 0xBFFF)
    q = (rng.standard_normal((12, 2, 16)).astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)
    k = (rng.standard_normal((12, 2, 16)).astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)
    _, _, probs = block_attention(c, q, k, k, tokens=6, grid_w=3, theta=1.0e4,
                                  return_probs=True)
    for p in probs.values():
        np.testing.assert_allclose(p.sum(axis=1), 1.0, rtol=0, atol=1e-12)
        assert np.all(p >= 0)


def test_single_key_returns_value_exactly():
    rng = np.random.default_rng(21)
    c = RolloutCache(0, 1, 1, 3, 64, "f32")
    q = rng.standard_normal((1, 3, 64)).astype(np.float32)
    k = rng.standard_normal((1, 3, 64)).astype(np.float32)
    v = rng.standard_normal((1, 3, 64)).astype(np.float32)
    out, lse = block_attention(c, q, k, v, tokens=1, grid_w=1, theta=1.0e4)
    assert np.array_equal(out, v.astype(np.float64))


def test_uniform_attention_gives_mean_of_values():
    # zero queries, or zero keys everywhere, make every score 0: the output is
    # the plain mean of V over the key set and the LSE is log(#keys).
    rng = np.random.default_rng(22)
    S, W, T, A, H, d = 1, 3, 4, 2, 2, 16
    Tf = T + A
    caches = {"q0": RolloutCache(S, W, Tf, H, d, "f32"),
              "k0": RolloutCache(S, W, Tf, H, d, "f32")}
    hist_v = []
    for _ in range(3):
        kf = rng.standard_normal((2, Tf, H, d)).astype(np.float32)
        vf = rng.standard_normal((2, Tf, H, d)).astype(np.float32)
        caches["q0"].commit(kf, vf)
        caches["k0"].commit(np.zeros_like(kf), vf)
        hist_v.append(vf)
    v = rng.standard_normal((2 * Tf, H, d)).astype(np.float32)
    # frames 0..5 committed: sink frame 0 and window frames 3, 4, 5 remain
    kept = np.concatenate([hist_v[0][0:1], hist_v[1][1:2], hist_v[2]], axis=0)
    want = np.concatenate([kept.reshape(-1, H, d), v]).astype(np.float64).mean(axis=0)
    cases = {"q0": (np.zeros((2 * T, H, d), np.float32),
                    rng.standard_normal((2 * Tf, H, d)).astype(np.float32)),
             "k0": (rng.standard_normal((2 * T, H, d)).astype(np.float32),
                    np.zeros((2 * Tf, H, d), np.float32))}
    for name, (q, k) in cases.items():
        out, lse = block_attention(caches[name], q, k, v, tokens=T, grid_w=2, theta=1.0e4)
        np.testing.assert_allclose(out, np.broadcast_to(want, out.shape), rtol=0, atol=1e-12)
        np.testing.assert_allclose(lse, math.log((4 + 2) * Tf), rtol=0, atol=1e-12)


def test_two_keys_closed_form():
    # one query token and one frame of two tokens (T=1, A=1), empty cache, d=6,
    # vectors chosen so RoPE leaves them alone (coordinates all zero).
    c = RolloutCache(0, 1, 2, 1, 6, "f32")
    q = np.array([[[1.0, 0, 0, 0, 0, 0]]], np.float32)
    k = np.array([[[2.0, 0, 0, 0, 0, 0]], [[-1.0, 0, 0, 0, 0, 0]]], np.float32)
    v = np.array([[[1.0, 2, 3, 4, 5, 6]], [[-1.0, 0, 1, 0, -1, 0]]], np.float32)
    out, lse = block_attention(c, q, k, v, tokens=1, grid_w=1, theta=1.0e4)
    s0, s1 = 2.0 / math.sqrt(6), -1.0 / math.sqrt(6)
    p0 = 1.0 / (1.0 + math.exp(s1 - s0))
    want = p0 * v[0, 0].astype(np.float64) + (1 - p0) * v[1, 0].astype(np.float64)
    np.testing.assert_allclose(out[0, 0], want, rtol=0, atol=1e-15)
    assert abs(lse[0, 0] - (s0 + math.log(1 + math.exp(s1 - s0)))) < 1e-15


def test_attention_invariant_to_slot_permutation():
    rng = np.random.default_rng(23)
    S, W, T, H, d = 1, 4, 4, 2, 12
    c = RolloutCache(S, W, T, H, d, "f32")
    for _ in range(7):
        c.commit(rng.standard_normal((1, T, H, d)).astype(np.float32),
                 rng.standard_normal((1, T, H, d)).astype(np.float32))
    q = rng.standard_normal((T, H, d)).astype(np.float32)
    k = rng.standard_normal((T, H, d)).astype(np.float32)
    v = rng.standard_normal((T, H, d)).astype(np.float32)
    out, lse = block_attention(c, q, k, v, tokens=T, grid_w=2, theta=1.0e4)
    perm = np.array([0, 3, 1, 4, 2])
    c2 = RolloutCache(S, W, T, H, d, "f32")
    c2.k[:] = c.k[perm]
    c2.v[:] = c.v[perm]
    c2.pos[:] = c.pos[perm]
    c2.n = c.n
    out2, lse2 = block_attention(c2, q, k, v, tokens=T, grid_w=2, theta=1.0e4)
    np.testing.assert_allclose(out2, out, rtol=0, atol=1e-13)
    np.testing.assert_allclose(lse2, lse, rtol=0, atol=1e-13)


def test_uniform_shift_of_all_positions_leaves_attention_unchanged():
    # relativity at the attention level: a rollout that was reset and one that
    # started 1000 frames earlier see the same outputs for the same content.
    rng = np.random.default_rng(24)
    S, W, T, H, d = 0, 3, 4, 1, 12
    data = [(rng.standard_normal((1, T, H, d)).astype(np.float32),
             rng.standard_normal((1, T, H, d)).astype(np.float32)) for _ in range(3)]
    a = RolloutCache(S, W, T, H, d, "f32")
    b = RolloutCache(S, W, T, H, d, "f32")
    for _ in range(1000):
        z = np.zeros((1, T, H, d), np.float32)
        b.commit(z, z)
    for kf, vf in data:
        a.commit(kf, vf)
        b.commit(kf, vf)
    q = rng.standard_normal((T, H, d)).astype(np.float32)
    k = rng.standard_normal((T, H, d)).astype(np.float32)
    v = rng.standard_normal((T, H, d)).astype(np.float32)
    oa, _ = block_attention(a, q, k, v, tokens=T, grid_w=2, theta=1.0e4)
    ob, _ = block_attention(b, q, k, v, tokens=T, grid_w=2, theta=1.0e4)
    np.testing.assert_allclose(ob, oa, rtol=0, atol=1e-10)


# --------------------------------------------------------------------------
# grouped-query attention (reading R9)
# --------------------------------------------------------------------------
@pytest.mark.parametrize("H,Hkv", [(4, 2), (6, 1), (6, 3)])
def test_grouped_query_attention_equals_repeated_key_value_heads(H, Hkv):
    # GQA with Hkv key/value heads is multi-head attention on key/value heads
    # repeated so that query heads h*G .. h*G+G-1 see key/value head h
    # (np.repeat along the head axis, an independent statement of the map)
    rng = np.random.default_rng(31)
    S, W, F, T, d = 1, 3, 2, 6, 12
    G = H // Hkv
    gqa = RolloutCache(S, W, T, Hkv, d, "f32")
    mha = RolloutCache(S, W, T, H, d, "f32")
    for _ in range(4):
        kf = rng.standard_normal((F, T, Hkv, d)).astype(np.float32)
        vf = rng.standard_normal((F, T, Hkv, d)).astype(np.float32)
        gqa.commit(kf, vf)
        mha.commit(np.repeat(kf, G, axis=2), np.repeat(vf, G, axis=2))
    q = rng.standard_normal((F * T, H, d)).astype(np.float32)
    k = rng.standard_normal((F * T, Hkv, d)).astype(np.float32)
    v = rng.standard_normal((F * T, Hkv, d)).astype(np.float32)
    og, lg = block_attention(gqa, q, k, v, tokens=T, grid_w=3, theta=1.0e4)
    om, lm = block_attention(mha, q, np.repeat(k, G, axis=1), np.repeat(v, G, axis=1),
                             tokens=T, grid_w=3, theta=1.0e4)
    np.testing.assert_array_equal(og, om)
    np.testing.assert_array_equal(lg, lm)
    # and the map is not interleaved: with G > 1 the first two query heads
    # share a key/value head (identical queries give identical rows)
    if G > 1:
        q2 = q.copy()
        q2[:, 1] = q2[:, 0]
        o2, _ = block_attention(gqa, q2, k, v, tokens=T, grid_w=3, theta=1.0e4)
        np.testing.assert_array_equal(o2[:, 0], o2[:, 1])


def test_grouped_query_attention_rejects_non_dividing_heads():
    c = RolloutCache(0, 2, 4, 2, 12, "f32")
    q = np.zeros((4, 3, 12), np.float32)
    kv = np.zeros((4, 2, 12), np.float32)
    with pytest.raises(ValueError):
        block_attention(c, q, kv, kv, tokens=4, grid_w=2, theta=1.0e4)


# --------------------------------------------------------------------------
# multi-view frames (reading R10)
# --------------------------------------------------------------------------
def test_multiview_token_coords_repeat_per_view():
    # 3 views of a 2 x 4 grid + 2 action tokens, enumerated by hand
    gh, gw, V, A = 2, 4, 3, 2
    h, w = token_coords(V * gh * gw + A, V * gh * gw, gw, gh * gw)
    want_h = [0, 0, 0, 0, 1, 1, 1, 1] * V + [0] * A
    want_w = [0, 1, 2, 3, 0, 1, 2, 3] * V + [0] * A
    assert list(h) == want_h and list(w) == want_w


def test_multiview_attention_is_equivariant_to_swapping_views():
    # swapping two views in the cache, the block keys/values and the queries
    # swaps the corresponding output rows: positions do not depend on the view
    rng = np.random.default_rng(41)
    S, W, F, gh, gw, V, A, H, d = 1, 2, 1, 2, 3, 2, 1, 2, 12
    Tv = gh * gw
    T, Tf = V * Tv, V * Tv + A
    perm = np.concatenate([np.arange(Tv, 2 * Tv), np.arange(Tv), np.arange(2 * Tv, Tf)])
    a = RolloutCache(S, W, Tf, H, d, "f32")
    b = RolloutCache(S, W, Tf, H, d, "f32")
    for _ in range(3):
        kf = rng.standard_normal((F, Tf, H, d)).astype(np.float32)
        vf = rng.standard_normal((F, Tf, H, d)).astype(np.float32)
        a.commit(kf, vf)
        b.commit(kf[:, perm], vf[:, perm])
    q = rng.standard_normal((F * T, H, d)).astype(np.float32)
    k = rng.standard_normal((F * Tf, H, d)).astype(np.float32)
    v = rng.standard_normal((F * Tf, H, d)).astype(np.float32)
    oa, la = block_attention(a, q, k, v, tokens=T, grid_w=gw, theta=1.0e4, view_tokens=Tv)
    ob, lb = block_attention(b, q[perm[:T]], k[perm], v[perm], tokens=T, grid_w=gw,
                             theta=1.0e4, view_tokens=Tv)
    np.testing.assert_allclose(ob, oa[perm[:T]], rtol=0, atol=1e-12)
    np.testing.assert_allclose(lb, la[:, perm[:T]], rtol=0, atol=1e-12)
    # with views read as extra grid rows the swap would change the result
    oc, _ = block_attention(b, q[perm[:T]], k[perm], v[perm], tokens=T, grid_w=gw,
                            theta=1.0e4)
    assert np.abs(oc - oa[perm[:T]]).max() > 1e-3


# --------------------------------------------------------------------------
# context parallelism (reading R11)
# --------------------------------------------------------------------------
@pytest.mark.parametrize("N", [2, 3, 4])
def test_parts_recombine_to_the_whole_key_set(N):
    # cache slots split round-robin over N parts, the block's keys in part 0:
    # recombining the parts' normalised outputs by their log-sum-exps gives the
    # attention over the whole key set (an identity of the softmax)
    rng = np.random.default_rng(51 + N)
    S, W, F, T, H, d = 1, 4, 2, 6, 2, 12
    c = RolloutCache(S, W, T, H, d, "f32")
    for _ in range(4):
        c.commit(rng.standard_normal((F, T, H, d)).astype(np.float32),
                 rng.standard_normal((F, T, H, d)).astype(np.float32))
    q = rng.standard_normal((F * T, H, d)).astype(np.float32)
    k = rng.standard_normal((F * T, H, d)).astype(np.float32)
    v = rng.standard_normal((F * T, H, d)).astype(np.float32)
    kw = dict(tokens=T, grid_w=3, theta=1.0e4)
    full, full_lse = block_attention(c, q, k, v, **kw)
    parts = [block_attention(c, q, k, v, slot_part=(N, r), include_block=(r == 0), **kw)
             for r in range(N)]
    out, lse = oracle.combine_partials([p[0] for p in parts], [p[1] for p in parts])
    np.testing.assert_allclose(out, full, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, full_lse, rtol=0, atol=1e-12)


def test_empty_part_has_no_weight():
    rng = np.random.default_rng(57)
    S, W, T, H, d = 0, 2, 4, 1, 12
    c = RolloutCache(S, W, T, H, d, "f32")
    c.commit(rng.standard_normal((1, T, H, d)).astype(np.float32),
             rng.standard_normal((1, T, H, d)).astype(np.float32))
    q = rng.standard_normal((T, H, d)).astype(np.float32)
    k = rng.standard_normal((T, H, d)).astype(np.float32)
    v = rng.standard_normal((T, H, d)).astype(np.float32)
    kw = dict(tokens=T, grid_w=2, theta=1.0e4)
    # one valid slot (slot 0): part 1 of 2 holds nothing and no block keys
    o1, l1 = block_attention(c, q, k, v, slot_part=(2, 1), include_block=False, **kw)
    assert np.all(o1 == 0) and np.all(np.isneginf(l1))
    o0, l0 = block_attention(c, q, k, v, slot_part=(2, 0), include_block=True, **kw)
    out, lse = oracle.combine_partials([o0, o1], [l0, l1])
    np.testing.assert_array_equal(out, o0)
    np.testing.assert_array_equal(lse, l0)
    # no keys anywhere: zero rows, -inf
    out, lse = oracle.combine_partials([o1, o1], [l1, l1])
    assert np.all(out == 0) and np.all(np.isneginf(lse))


@pytest.mark.parametrize("S,W,F,c", [(1, 4, 2, 1), (0, 3, 1, 2), (2, 3, 1, 1)])
def test_window_reset_equals_attention_over_the_current_window(S, W, F, c):
    """R12: with the window-boundary policy every attention call equals the
    brute-force attention over the frames committed since the window's start
    (conditioning at t = 0 .. c-1, then the blocks), positions counted from
    that start: earlier windows leave no trace."""
    from oracle import start_window, window_boundary_reached
    rng = np.random.default_rng(40 + S + W + F + c)
    gh, gw, H, d, theta = 2, 2, 2, 12, 1.0e4
    T = gh * gw
    Tf = T
    cache = RolloutCache(S, W, Tf, H, d, "f32")
    window = []                       # (k, v) of the frames of the current window

    def new_window():
        ck = rng.standard_normal((c, Tf, H, d)).astype(np.float32)
        cv = rng.standard_normal((c, Tf, H, d)).astype(np.float32)
        start_window(cache, ck, cv)
        window[:] = [(ck[f].astype(np.float64), cv[f].astype(np.float64)) for f in range(c)]

    new_window()
    restarts = 0
    for blk in range(7):
        if window_boundary_reached(cache.n, F, S, W):
            new_window()
            restarts += 1
        n = cache.n
        assert n == len(window)
        q = rng.standard_normal((F * T, H, d)).astype(np.float32)
        k = rng.standard_normal((F * Tf, H, d)).astype(np.float32)
        v = rng.standard_normal((F * Tf, H, d)).astype(np.float32)
        out, lse = block_attention(cache, q, k, v, tokens=T, grid_w=gw, theta=theta)
        # every frame of the window is visible: a sink + window mask as wide
        # as the whole window
        ref, ref_lse = _brute_force_block(window, n, n, 0, q.astype(np.float64),
                                          k.astype(np.float64), v.astype(np.float64),
                                          T, Tf, gw, theta)
        np.testing.assert_allclose(out, ref, rtol=0, atol=1e-12)
        np.testing.assert_allclose(lse, ref_lse, rtol=0, atol=1e-12)
        kf, vf = k.reshape(F, Tf, H, d), v.reshape(F, Tf, H, d)
        cache.commit(kf, vf)
        window += [(kf[f].astype(np.float64), vf[f].astype(np.float64)) for f in range(F)]
        assert cache.n <= S + W   # the ring never wraps under this policy
    assert restarts >= 1
