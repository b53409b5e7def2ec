"""Shared helpers of the GPU tests: cache set-up, host<->device marshalling,
and lockstep drivers that feed identical seeded bytes to the CUDA path (through
the C ABI) and to the CPU oracle."""
from __future__ import annotations

import numpy as np
import torch

import oracle
from streaming_autoregressive_video_b200 import binding as fd
from streaming_autoregressive_video_b200 import synth

TOL_BF16_MAX = 2e-2
TOL_BF16_MEAN = 2e-3
TOL_F32_MAX = 1e-4


def new_cache(w, device="cuda", shards=1, shard=0, work_sets=1):
    desc = fd.make_desc(w, shards=shards, shard=shard, work_sets=work_sets)
    nbytes = fd.fd_cache_bytes(desc)
    assert nbytes > 0
    storage = torch.empty(nbytes + 1024, dtype=torch.uint8, device=device)
    off = (-storage.data_ptr()) % 1024
    storage = storage[off:off + nbytes]
    return fd.fd_cache_create(desc, storage)


def views(cache, w):
    """torch views of the cache regions inside the caller-owned storage."""
    lay = cache.layout
    st = cache.storage
    L, R, slots = w.layers, w.rollouts, w.slots
    esz = 2 if w.dtype == "bf16" else 4
    n_kv = L * R * slots * w.frame_tokens * w.hkv * w.head_dim
    kv_dt = torch.int16 if esz == 2 else torch.float32
    shape = (L, R, slots, w.frame_tokens, w.hkv, w.head_dim)
    k = st[lay.k:lay.k + n_kv * esz].view(kv_dt).view(shape)
    v = st[lay.v:lay.v + n_kv * esz].view(kv_dt).view(shape)
    pos = st[lay.pos:lay.pos + L * R * slots * 4].view(torch.int32).view(L, R, slots)
    count = st[lay.count:lay.count + L * R * 4].view(torch.int32).view(L, R)
    return k, v, pos, count


def krot_view(cache, w):
    """The cache's committed keys rotated to their frame positions."""
    lay = cache.layout
    esz = 2 if w.dtype == "bf16" else 4
    n_kv = w.layers * w.rollouts * w.slots * w.frame_tokens * w.hkv * w.head_dim
    kv_dt = torch.int16 if esz == 2 else torch.float32
    shape = (w.layers, w.rollouts, w.slots, w.frame_tokens, w.hkv, w.head_dim)
    return cache.storage[lay.krot:lay.krot + n_kv * esz].view(kv_dt).view(shape)


def rotated_bound(want: np.ndarray, raw: np.ndarray, dtype: str) -> np.ndarray:
    """Error bound of a stored rotated value against the fp64 rotation.

    The kernels rotate in fp32 with cos/sin rounded once to fp32: the value
    before storage is off by at most about 3 * 2^-24 * (|x0| + |x1|) of its
    input pair (x0, x1), which matters where the rotation cancels.  A bf16
    value is then rounded once more (half an ulp, at most 2^-8 of the value).
    The bound takes 2^-21 * (|x0| + |x1|) for the fp32 part (a factor 2
    over the estimate)."""
    x = np.abs(np.asarray(raw, dtype=np.float64))
    pair = np.repeat(x[..., 0::2] + x[..., 1::2], 2, axis=-1)
    if dtype == "bf16":
        return np.abs(want) * 2.0 ** -8 + pair * 2.0 ** -21
    return np.abs(want) * 1e-6 + 1e-6


def check_rotated(got_storage: np.ndarray, raw: np.ndarray, t, w, what=""):
    """got = RoPE(raw) at frame positions t (one entry per frame), within one
    rounding to the storage dtype of the fp32 rotation (rotated_bound)."""
    h, ww = oracle.token_coords(w.frame_tokens, w.tokens, w.grid_w, w.view_tokens)
    t = np.asarray(t, dtype=np.float64)[:, None]
    ang = oracle.rope_angles(t, h[None, :], ww[None, :], w.head_dim, w.theta)[:, :, None, :]
    raw64 = oracle.values_f64(raw, w.dtype)
    want = oracle.rope_rotate(raw64, ang)
    got = oracle.values_f64(got_storage, w.dtype)
    err = np.abs(got - want)
    bound = rotated_bound(want, raw64, w.dtype)
    assert np.all(err <= bound), f"{what}: rotated keys off by {float(err.max()):.3g}"


def to_device(a: np.ndarray, device="cuda") -> torch.Tensor:
    if a.dtype == np.uint16:
        return torch.from_numpy(a.view(np.int16).copy()).to(device)
    return torch.from_numpy(np.ascontiguousarray(a)).to(device)


def to_host(t: torch.Tensor) -> np.ndarray:
    a = t.detach().cpu().numpy()
    return a.view(np.uint16) if a.dtype == np.int16 else a


def out_values(t: torch.Tensor) -> np.ndarray:
    if t.dtype == torch.int16:
        return oracle.bf16_bits_to_f64(to_host(t))
    return t.detach().cpu().numpy().astype(np.float64)


def empty_like_q(w, n_rollouts, device="cuda"):
    shape = (n_rollouts, w.queries, w.heads, w.head_dim)
    dt = torch.int16 if w.dtype == "bf16" else torch.float32
    return torch.empty(shape, dtype=dt, device=device)


def block_inputs(w, seed_parts, n_rollouts):
    """Seeded q, k, v of one attention call, storage form (numpy)."""
    qs = (n_rollouts, w.queries, w.heads, w.head_dim)
    ks = (n_rollouts, w.block_frames * w.frame_tokens, w.hkv, w.head_dim)
    q = synth.normal(synth.seed_of(*seed_parts, 0), qs, w.dtype, w.value_scale)
    k = synth.normal(synth.seed_of(*seed_parts, 1), ks, w.dtype, w.value_scale)
    v = synth.normal(synth.seed_of(*seed_parts, 2), ks, w.dtype, w.value_scale)
    return q, k, v


def compare(got: np.ndarray, want: np.ndarray, dtype: str, what: str = ""):
    err = np.abs(got - want)
    mx, mean = float(err.max()), float(err.mean())
    if dtype == "bf16":
        assert mx <= TOL_BF16_MAX and mean <= TOL_BF16_MEAN, \
            f"{what}: max abs {mx:.3g} mean abs {mean:.3g}"
    else:
        assert mx <= TOL_F32_MAX, f"{what}: max abs {mx:.3g}"
    return mx, mean


class Lockstep:
    """Drives the GPU cache and per-(rollout, layer) oracle caches together."""

    def __init__(self, w, device="cuda"):
        self.w = w
        self.cache = new_cache(w, device)
        self.device = device
        self.orc = [[oracle.RolloutCache(w.sink_frames, w.window_frames, w.frame_tokens,
                                         w.hkv, w.head_dim, w.dtype)
                     for _ in range(w.rollouts)] for _ in range(w.layers)]

    def attention(self, layer, q, k, v, n_rollouts=None, rows=None, with_lse=True,
                  check=True, what=""):
        w = self.w
        nr = n_rollouts or w.rollouts
        out = empty_like_q(w, nr, self.device)
        lse = torch.empty((nr, w.heads, w.queries), dtype=torch.float32,
                          device=self.device) if with_lse else None
        qd, kd, vd = to_device(q, self.device), to_device(k, self.device), to_device(v, self.device)
        fd.fd_block_attention(self.cache, layer, nr, qd, kd, vd, out, lse)
        torch.cuda.synchronize()
        got = out_values(out)
        errs = []
        if check:
            for r in range(nr):
                want, want_lse = oracle.block_attention(
                    self.orc[layer][r], q[r], k[r], v[r], tokens=w.tokens,
                    grid_w=w.grid_w, theta=w.theta, rows=rows, view_tokens=w.view_tokens)
                sel = slice(None) if rows is None else np.asarray(rows)
                errs.append(compare(got[r][sel], want[sel], w.dtype, f"{what} r={r}"))
                if with_lse:
                    lse_got = lse[r].cpu().numpy().astype(np.float64)
                    d_lse = np.abs(lse_got[:, sel] - want_lse[:, sel]).max()
                    assert d_lse <= (1e-2 if w.dtype == "bf16" else 1e-4), \
                        f"{what} r={r}: lse max abs {d_lse:.3g}"
        return got, errs

    def commit(self, layers, k_list, v_list, n_rollouts=None, frames=None):
        """k_list[i]: numpy [nr][F*Tf][H][d] for layer layers[0]+i."""
        w = self.w
        nr = n_rollouts or w.rollouts
        kd = [to_device(a, self.device) for a in k_list]
        vd = [to_device(a, self.device) for a in v_list]
        fd.fd_cache_commit(self.cache, layers[0], layers[-1] + 1, nr, kd, vd, frames)
        F, Tf = w.block_frames, w.frame_tokens
        for i, l in enumerate(layers):
            for r in range(nr):
                nf = F if frames is None else int(frames[r])
                kf = k_list[i][r].reshape(F, Tf, w.hkv, w.head_dim)[:nf]
                vf = v_list[i][r].reshape(F, Tf, w.hkv, w.head_dim)[:nf]
                self.orc[l][r].commit(kf, vf)
        torch.cuda.synchronize()

    def reset(self, ids):
        fd.fd_cache_reset(self.cache, ids)
        for l in range(self.w.layers):
            for r in ids:
                self.orc[l][r].reset()
        torch.cuda.synchronize()

    def check_cache_exact(self):
        """Slot positions, counters and every valid slot's bytes, bit for bit."""
        w = self.w
        k, v, pos, count = views(self.cache, w)
        k, v, pos, count = to_host(k), to_host(v), to_host(pos), to_host(count)
        for l in range(w.layers):
            for r in range(w.rollouts):
                o = self.orc[l][r]
                assert count[l, r] == o.n, (l, r, count[l, r], o.n)
                assert np.array_equal(pos[l, r], o.pos), (l, r, pos[l, r], o.pos)
                nv = o.valid_slots()
                assert np.array_equal(k[l, r, :nv], o.k[:nv]), ("K", l, r)
                assert np.array_equal(v[l, r, :nv], o.v[:nv]), ("V", l, r)
                assert fd.fd_cache_frames(self.cache, l, r) == o.n

    def check_rotated_keys(self):
        """The rotated-key region holds every valid slot's keys at its frame position."""
        w = self.w
        kr = to_host(krot_view(self.cache, w))
        for l in range(w.layers):
            for r in range(w.rollouts):
                o = self.orc[l][r]
                nv = o.valid_slots()
                if nv:
                    check_rotated(kr[l, r, :nv], o.k[:nv], o.pos[:nv], w, f"krot l={l} r={r}")
