"""The bound the GPU tests hold stored rotated keys to (support.rotated_bound),
checked on the CPU against a model of the kernels' arithmetic: fp64 angles,
cos/sin rounded to fp32, the rotation in fp32, one round-to-nearest-even to
bf16.  Such values must pass at every head size; a plausible mistake (a
position off by one, the h and w sections swapped) must not."""
import numpy as np
import pytest

import oracle
from streaming_autoregressive_video_b200 import synth

from support import rotated_bound


def _bf16_rne(x32: np.ndarray) -> np.ndarray:
    u = x32.astype(np.float32).view(np.uint32).astype(np.uint64)
    r = ((u + 0x7FFF + ((u >> 16) & 1)) >> 16) & 0xFFFF
    return (r.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def _fp32_rotation(raw: np.ndarray, t, h, w, d, theta):
    """raw [tokens][heads][d] rotated as the kernels do it (fp32 tables and
    products), rounded to bf16."""
    p_t, p_h, p_w = oracle.rope_sections(d)

    def tab(pos, p):
        a = np.asarray(pos, dtype=np.float64)[:, None] * np.power(theta, -np.arange(p) / p)
        return np.cos(a).astype(np.float32), np.sin(a).astype(np.float32)

    ct, st = tab(np.broadcast_to(t, h.shape), p_t)
    ch, sh = tab(h, p_h)
    cw, sw = tab(w, p_w)
    c = np.concatenate([ct, ch, cw], 1)[:, None, :]
    s = np.concatenate([st, sh, sw], 1)[:, None, :]
    x = raw.astype(np.float32)
    a, b = x[..., 0::2], x[..., 1::2]
    o = np.empty_like(x)
    o[..., 0::2] = a * c - b * s
    o[..., 1::2] = a * s + b * c
    return _bf16_rne(o)


@pytest.mark.parametrize("d", [32, 64, 96, 128])
def test_fp32_rotation_within_bound_and_mistakes_outside(d):
    gh, gw, heads, t = 12, 13, 2, 5
    h, w = oracle.token_coords(gh * gw, gh * gw, gw)
    raw = oracle.values_f64(synth.normal(synth.seed_of(31, d), (gh * gw, heads, d), "bf16"),
                            "bf16")
    want = oracle.rope_rotate(raw, oracle.rope_angles(float(t), h, w, d, 1.0e4)[:, None, :])
    bound = rotated_bound(want, raw, "bf16")
    got = _fp32_rotation(raw, float(t), h.astype(np.float64), w.astype(np.float64), d, 1.0e4)
    assert np.all(np.abs(got - want) <= bound)
    # mistakes the bound must catch
    off_t = _fp32_rotation(raw, float(t + 1), h.astype(np.float64), w.astype(np.float64), d,
                           1.0e4)
    assert np.any(np.abs(off_t - want) > bound)
    swapped = _fp32_rotation(raw, float(t), w.astype(np.float64), h.astype(np.float64), d,
                             1.0e4)
    assert np.any(np.abs(swapped - want) > bound)
