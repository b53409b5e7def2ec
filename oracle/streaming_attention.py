"""fp64 CPU statement of block-causal chunk attention over a streaming KV cache.

TEST INFRASTRUCTURE (see the package docstring): plain numpy, one obvious step
per line, no blocking or fusion beyond processing independent query rows in
chunks to bound memory.

What the pages fix (behaviour only, no formulas are printed):

* "NVIDIA FlashDreams Is the Open-Source Inference Engine Robotics World Models
  Needed", section Bounded Memory for Infinite Rollouts: each rollout keeps a
  cache of bounded size and evicts old state, so a 10,000-step rollout does not
  grow memory.  Section Hot-Path Generation, Background State Updates: the
  denoising pass (generate) and the cache update (finalize) are separate.
* "Cosmos3-H-Dreams" model card, Model Architecture: a block-causal, few-step
  student with a KV cache; the conditioning frame is prefilled into the cache
  once; each later latent frame consumes the next 4 action vectors.  Section
  Software Integration: the KV cache has a static shape.
* AlpaDreams GTC 2026 write-up, section VII: the causal DiT produces the next
  frame from historical clean frames and the current noisy frame through a KV
  cache.
* "Single-GPU inference for DreamZero", Sequential requests: frame positions
  and KV carry over between requests and are reset explicitly.

Readings taken where the pages are silent:

R1  scores are q.k / sqrt(d); softmax over the whole key set, no bias, no
    softcap, no mask inside the key set.
R2  the key set of every query of the current block is all valid cache tokens
    plus all tokens of the current block (bidirectional inside the block; the
    whole cache lies in the past of the block).
R3  the first S frames committed to a rollout are sinks, never evicted; later
    frames fill a ring of W window slots: slot_of(m) = m for m < S and
    S + ((m - S) mod W) otherwise.  A commit of F <= W frames therefore evicts
    the oldest window frames once the ring is full, and the valid slots are
    always the prefix [0, min(n,S) + min(max(n-S,0), W)).
R4  3D RoPE: the d/2 rotation pairs split into contiguous sections for t, h, w
    of p_h = p_w = floor(d/6) pairs and p_t = d/2 - 2 floor(d/6) pairs; pair j
    of a section of n_s pairs rotates the adjacent elements (2i, 2i+1) by the
    angle coord * theta^(-j/n_s).
R5  video token i of a frame sits at (h, w) = (i div Gw, i mod Gw); the action
    tokens of a frame sit at (0, 0); every token of frame m has t = m.
R6  t is the absolute frame index since the rollout's start (or last reset);
    eviction never renumbers frames.
R7  the cache keeps K/V exactly as committed (before RoPE) plus one int32 frame
    position per slot (-1 = empty) and the committed-frame counter n; RoPE is
    applied to cached keys when they are used.
R8  the block being denoised has frames n .. n+F-1; its K/V are committed after
    the last denoising step (whatever K/V the caller passes).
R9  grouped-query attention (a variant of the cache semantics, not on the
    pages): keys and values carry Hkv heads, queries H = G * Hkv heads, and
    query head h reads key/value head h div G (consecutive query heads share
    a key/value head, as in Ainslie et al., "GQA: Training Generalized
    Multi-Query Transformer Models from Multi-Head Checkpoints", 2023).
    Hkv = H is plain multi-head attention.
R10 multi-view frames (a shape variant; the pages show four-camera models
    attending across views without saying how positions are assigned): a
    frame holds V views of Gh x Gw video tokens, view-major, so T = V*Gh*Gw;
    video token i sits at (h, w) of its position inside its view, i mod
    (Gh*Gw), and all views of a frame share t.  Views therefore differ only by
    content (any learned view embedding belongs to the model, before the
    attention).  V = 1 is R5.
R12 window-boundary reset ("Single-GPU inference for DreamZero", Sequential
    requests; a second cache policy next to the ring of R3): the cache's
    S + W slots hold one local-attention window of consecutive frames that
    is never evicted frame by frame.  Before a block of F frames, if the
    window cannot take it (n + F > S + W), the old frames are released
    (reset: n = 0, every slot empty), the conditioning is re-encoded and
    committed first at positions 0 .. c-1, and the block follows at t = c.
    Inside a window no slot is ever reused, so the ring of R3 never wraps
    and every attention call sees exactly the frames committed since the
    last reset.
R11 context parallelism (a way to compute the same attention on N devices,
    named by the pages without formulas): the key set splits into disjoint
    parts; part i yields the softmax-normalised output O_i and log-sum-exp
    lse_i over its own keys; the whole-set result is
    O = sum_i exp(lse_i - M) O_i / sum_i exp(lse_i - M) and
    lse = M + log sum_i exp(lse_i - M), M = max_i lse_i (a part with no keys
    has lse = -inf and weight 0).  Parts here: cache slot s belongs to part
    s mod N; the block's own keys belong to part 0.
"""
from __future__ import annotations

import math

import numpy as np


# --------------------------------------------------------------------------
# number formats
# --------------------------------------------------------------------------
def bf16_bits_to_f64(bits) -> np.ndarray:
    """Exact value of bfloat16 bit patterns.

    A bfloat16 is the upper 16 bits of an IEEE-754 binary32, so placing the
    pattern in the high half of a 32-bit word gives the same value exactly.
    """
    b = np.asarray(bits, dtype=np.uint16)
    return (b.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)


def values_f64(x, dtype: str) -> np.ndarray:
    """Stored inputs ("bf16" bit patterns or "f32" floats) as exact fp64 values."""
    if dtype == "bf16":
        return bf16_bits_to_f64(x)
    if dtype == "f32":
        return np.asarray(x, dtype=np.float32).astype(np.float64)
    raise ValueError(f"unknown dtype {dtype!r}")


# --------------------------------------------------------------------------
# 3D RoPE (readings R4, R5)
# --------------------------------------------------------------------------
def rope_sections(d: int):
    """(p_t, p_h, p_w): rotation pairs given to the t, h and w axes (R4)."""
    if d <= 0 or d % 2:
        raise ValueError("head_dim must be a positive even number")
    p_hw = d // 6
    return d // 2 - 2 * p_hw, p_hw, p_hw


def rope_inv_freq(n_pairs: int, theta: float) -> np.ndarray:
    """Angular frequency of each pair of one section: theta^(-j/n_pairs) (R4)."""
    j = np.arange(n_pairs, dtype=np.float64)
    return np.power(float(theta), -j / n_pairs)


def rope_angles(t, h, w, d: int, theta: float) -> np.ndarray:
    """Rotation angle of every pair for tokens at coordinates (t, h, w).

    t, h, w broadcast against each other; the result has one more trailing
    axis of length d/2 ordered [t section | h section | w section].
    """
    p_t, p_h, p_w = rope_sections(d)
    t = np.asarray(t, dtype=np.float64)[..., None]
    h = np.asarray(h, dtype=np.float64)[..., None]
    w = np.asarray(w, dtype=np.float64)[..., None]
    a_t = t * rope_inv_freq(p_t, theta)
    a_h = h * rope_inv_freq(p_h, theta)
    a_w = w * rope_inv_freq(p_w, theta)
    shape = np.broadcast_shapes(a_t.shape[:-1], a_h.shape[:-1], a_w.shape[:-1])
    return np.concatenate([np.broadcast_to(a_t, shape + (p_t,)),
                           np.broadcast_to(a_h, shape + (p_h,)),
                           np.broadcast_to(a_w, shape + (p_w,))], axis=-1)


def rope_rotate(x: np.ndarray, angles: np.ndarray) -> np.ndarray:
    """Rotate adjacent pairs (x[2i], x[2i+1]) of the last axis by angles[..., i]."""
    x = np.asarray(x, dtype=np.float64)
    c = np.cos(angles)
    s = np.sin(angles)
    x0 = x[..., 0::2]
    x1 = x[..., 1::2]
    out = np.empty(np.broadcast_shapes(x.shape, c.shape[:-1] + (x.shape[-1],)),
                   dtype=np.float64)
    out[..., 0::2] = x0 * c - x1 * s
    out[..., 1::2] = x0 * s + x1 * c
    return out


def token_coords(n_tokens: int, T: int, grid_w: int, view_tokens: int = 0):
    """(h, w) of the tokens of one frame (R5, R10): video tokens row-major
    inside their view (view_tokens = Gh*Gw per view; 0 = a single view of T
    tokens), actions at 0."""
    i = np.arange(n_tokens)
    iv = i % (view_tokens or T)
    h = np.where(i < T, iv // grid_w, 0)
    w = np.where(i < T, iv % grid_w, 0)
    return h, w


# --------------------------------------------------------------------------
# bounded streaming cache (readings R3, R6, R7)
# --------------------------------------------------------------------------
def slot_of(m: int, S: int, W: int) -> int:
    """Cache slot of frame m of a rollout (R3)."""
    if m < S:
        return m
    return S + (m - S) % W


def valid_slot_count(n: int, S: int, W: int) -> int:
    """Number of valid slots after n committed frames; they form a prefix (R3)."""
    return min(n, S) + min(max(n - S, 0), W)


class RolloutCache:
    """Cache of one (rollout, layer): raw K/V per slot, positions and counter."""

    def __init__(self, S: int, W: int, frame_tokens: int, heads: int,
                 head_dim: int, dtype: str):
        if W < 1 or S < 0:
            raise ValueError("need W >= 1 and S >= 0")
        self.S, self.W, self.dtype = S, W, dtype
        store = np.uint16 if dtype == "bf16" else np.float32
        shape = (S + W, frame_tokens, heads, head_dim)
        self.k = np.zeros(shape, dtype=store)
        self.v = np.zeros(shape, dtype=store)
        self.pos = np.full(S + W, -1, dtype=np.int32)
        self.n = 0

    def reset(self) -> None:
        """Start a new sequence: no valid frame, positions restart at 0."""
        self.k[...] = 0
        self.v[...] = 0
        self.pos[:] = -1
        self.n = 0

    def commit(self, k_frames: np.ndarray, v_frames: np.ndarray) -> None:
        """Write frames n, n+1, ... into their slots (R3, R8); n grows by their count.

        k_frames, v_frames: [frames][Tf][H][d] in storage form, pre-RoPE.
        """
        nf = k_frames.shape[0]
        if nf > self.W:
            raise ValueError("a commit may not hold more frames than the window")
        for f in range(nf):
            s = slot_of(self.n + f, self.S, self.W)
            self.k[s] = k_frames[f]
            self.v[s] = v_frames[f]
            self.pos[s] = self.n + f
        self.n += nf

    def valid_slots(self) -> int:
        return valid_slot_count(self.n, self.S, self.W)


def window_boundary_reached(n: int, frames: int, S: int, W: int) -> bool:
    """R12: the next block of `frames` frames does not fit in the window of
    S + W slots after n committed frames, so the window restarts."""
    return n + frames > S + W


def start_window(cache: "RolloutCache", cond_k: np.ndarray, cond_v: np.ndarray) -> None:
    """R12: release the window's frames and commit the re-encoded conditioning
    frames ([c][Tf][H][d], storage form) at positions 0 .. c-1."""
    cache.reset()
    cache.commit(cond_k, cond_v)


# --------------------------------------------------------------------------
# one attention call (readings R1, R2, R4-R8)
# --------------------------------------------------------------------------
def block_attention(cache: RolloutCache, q, k, v, *, tokens: int, grid_w: int,
                    theta: float, heads=None, rows=None, row_chunk: int = 512,
                    return_probs: bool = False, view_tokens: int = 0,
                    slot_part=None, include_block: bool = True):
    """Attention of the current block's queries of one (rollout, layer).

    q:    [F*T][H][d]    queries of the block, storage form, pre-RoPE
    k, v: [F*Tf][Hkv][d] keys / values of the block, storage form, pre-RoPE
          (Hkv divides H; query head h reads key/value head h div (H/Hkv))
    cache: the rollout's cache for this layer (not modified)
    heads: optional subset of head indices to evaluate (others are left 0)
    rows:  optional subset of query rows to evaluate (others are left 0);
           every row's softmax still runs over the whole key set
    view_tokens: video tokens per view of a multi-view frame (R10; 0 = one
           view of all `tokens`)
    slot_part, include_block: attention over a part of the key set (R11):
           only valid cache slots s with s mod N == r for slot_part = (N, r),
           and the block's keys only if include_block; rows with no key get
           out = 0 and lse = -inf

    Returns (out [F*T][H][d] fp64, lse [H][F*T] fp64 natural-log sum of exp of
    the scaled scores) and, with return_probs, a dict head -> P [F*T][Nk].
    """
    dtype = cache.dtype
    T = tokens
    Mq, H, d = q.shape
    F = Mq // T
    if F * T != Mq or k.shape[0] % F:
        raise ValueError("q rows must be F*T and k rows F*Tf")
    Tf = k.shape[0] // F
    Hkv = k.shape[1]
    if H % Hkv or cache.k.shape[2] != Hkv:
        raise ValueError("key/value heads must divide the query heads and match the cache")
    group = H // Hkv
    n = cache.n
    nv = cache.valid_slots()

    # the key set's slots (R11: possibly one part of it)
    slots = np.arange(nv)
    if slot_part is not None:
        n_parts, part = slot_part
        slots = slots[slots % n_parts == part]
    nf_block = F if include_block else 0
    ns = len(slots)

    # coordinates of every key: the slots in slot order, then the block
    h_tok, w_tok = token_coords(Tf, T, grid_w, view_tokens)
    t_cache = np.repeat(cache.pos[slots].astype(np.float64), Tf)
    t_block = np.repeat(np.arange(n, n + nf_block, dtype=np.float64), Tf)
    t_key = np.concatenate([t_cache, t_block])
    h_key = np.tile(h_tok, ns + nf_block)
    w_key = np.tile(w_tok, ns + nf_block)
    ang_k = rope_angles(t_key, h_key, w_key, d, theta)          # [Nk][d/2]

    # coordinates of the evaluated queries (video tokens only)
    rows = np.arange(Mq) if rows is None else np.asarray(rows, dtype=np.int64)
    tok_q = (rows % T) % (view_tokens or T)
    ang_q = rope_angles(n + rows // T, tok_q // grid_w, tok_q % grid_w, d, theta)

    scale = 1.0 / math.sqrt(d)
    out = np.zeros((Mq, H, d), dtype=np.float64)
    lse = np.zeros((H, Mq), dtype=np.float64)
    probs = {}
    if ns + nf_block == 0:  # no key at all (R11)
        lse[:] = -np.inf
        return (out, lse, probs) if return_probs else (out, lse)
    for hh in (range(H) if heads is None else heads):
        g = hh // group  # key/value head of this query head (R9)
        qh = rope_rotate(values_f64(q[rows, hh, :], dtype), ang_q)
        kc = values_f64(cache.k[slots, :, g, :], dtype).reshape(ns * Tf, d)
        vc = values_f64(cache.v[slots, :, g, :], dtype).reshape(ns * Tf, d)
        kb = values_f64(k[:, g, :], dtype)[:nf_block * Tf]
        vb = values_f64(v[:, g, :], dtype)[:nf_block * Tf]
        kh = rope_rotate(np.concatenate([kc, kb]), ang_k)
        vh = np.concatenate([vc, vb])
        if return_probs:
            probs[hh] = np.zeros((Mq, kh.shape[0]), dtype=np.float64)
        for c0 in range(0, len(rows), row_chunk):
            sel = rows[c0:c0 + row_chunk]
            s = (qh[c0:c0 + row_chunk] @ kh.T) * scale
            m = s.max(axis=1, keepdims=True)
            e = np.exp(s - m)
            l = e.sum(axis=1, keepdims=True)
            out[sel, hh, :] = (e @ vh) / l
            lse[hh, sel] = (m + np.log(l))[:, 0]
            if return_probs:
                probs[hh][sel] = e / l
    if return_probs:
        return out, lse, probs
    return out, lse


# --------------------------------------------------------------------------
# context parallelism (reading R11)
# --------------------------------------------------------------------------
def combine_partials(outs, lses):
    """Whole-key-set attention from per-part results (R11).

    outs: list of [Mq][H][d] fp64 outputs, each normalised over its part
    lses: list of [H][Mq] fp64 log-sum-exp of the same parts (-inf: no keys)
    Returns (out [Mq][H][d], lse [H][Mq]).
    """
    L = np.stack([np.asarray(x, dtype=np.float64) for x in lses])       # [N][H][Mq]
    M = L.max(axis=0)                                                  # [H][Mq]
    Msafe = np.where(np.isfinite(M), M, 0.0)
    w = np.where(np.isfinite(L), np.exp(L - Msafe[None]), 0.0)          # [N][H][Mq]
    tot = w.sum(axis=0)                                                # [H][Mq]
    out = np.zeros_like(np.asarray(outs[0], dtype=np.float64))
    for wi, oi in zip(w, outs):
        out += np.asarray(oi, dtype=np.float64) * wi.T[:, :, None]
    has = tot > 0
    out = np.where(has.T[:, :, None], out / np.where(has, tot, 1.0).T[:, :, None], 0.0)
    lse = np.where(has, Msafe + np.log(np.where(has, tot, 1.0)), -np.inf)
    return out, lse
