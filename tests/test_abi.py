"""The C ABI on the host: the library loads without a GPU, exports every symbol
include/fd.h declares, and rejects bad arguments before touching the device."""
import ctypes
import os
import re

import pytest

from streaming_autoregressive_video_b200 import binding as fd
from streaming_autoregressive_video_b200.workloads import ALL, SINGLE_480P

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_symbols():
    src = open(os.path.join(ROOT, "include", "fd.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(fd_[a-z0-9_]+)\s*\(", src)))


def test_library_exports_every_declared_symbol():
    lib = fd.load()
    syms = declared_symbols()
    assert len(syms) >= 14
    for s in syms:
        assert hasattr(lib, s), s
    assert sorted(fd.EXPORTS) == syms


def test_cache_bytes_and_layout():
    for w in ALL:
        desc = fd.make_desc(w)
        n = fd.fd_cache_bytes(desc)
        lay = fd.fd_cache_get_layout(desc)
        assert n == lay.total > 0
        esz = 2 if w.dtype == "bf16" else 4
        kv = w.layers * w.rollouts * w.slots * w.frame_tokens * w.hkv * w.head_dim * esz
        assert lay.layer_kv_bytes * w.layers == kv
        regions = [lay.k, lay.v, lay.krot, lay.kblk, lay.qblk, lay.part, lay.pos,
                   lay.count,
                   lay.ttab, lay.htab, lay.wtab, lay.err]
        assert regions == sorted(regions) and all(r % 1024 == 0 for r in regions)
        assert lay.v - lay.k >= kv and lay.krot - lay.v >= kv and lay.kblk - lay.krot >= kv
        # one work set by default: the block's rotated keys, the split-pair
        # partial results (148 CTAs x 2 slots, fp32 O [256][128] + max + sum)
        # and their counters, for one call at a time; none of the latter two
        # for fp32 caches
        blk = w.rollouts * w.block_frames * w.frame_tokens * w.hkv * w.head_dim * esz
        assert blk <= lay.qblk - lay.kblk < blk + 1024
        # the block's rotated queries (bf16 caches: the tensor-core calls)
        qb = w.rollouts * w.queries * w.heads * w.head_dim * esz if w.dtype == "bf16" else 0
        assert qb <= lay.part - lay.qblk < qb + 1024
        part = 148 * 2 * (256 * 128 + 512) * 4 if w.dtype == "bf16" else 0
        assert part <= lay.pos - lay.part < part + 1024
        # one work set per layer multiplies the three by L and nothing else
        lay_l = fd.fd_cache_get_layout(fd.make_desc(w, work_sets=w.layers))
        assert lay_l.qblk - lay_l.kblk >= w.layers * blk
        assert lay_l.part - lay_l.qblk >= w.layers * qb
        assert lay_l.pos - lay_l.part >= w.layers * part
        assert (lay_l.total - lay.total) - (w.layers - 1) * (blk + qb + part) < 4 * 1024
        assert (lay.rope_pairs_t, lay.rope_pairs_h, lay.rope_pairs_w) == \
            (w.head_dim // 2 - 2 * (w.head_dim // 6), w.head_dim // 6, w.head_dim // 6)


def test_single_480p_cache_is_about_3_gb():
    n = fd.fd_cache_bytes(fd.make_desc(SINGLE_480P))
    # 30 layers x 7 slots x 1560 tokens x 12 heads x 128 x 2 B x (K, V, rotated K)
    # + one work area for the block's rotated keys and queries (3 frames each)
    # + one set of partial-result slots of the attention kernel
    part = 148 * 2 * (256 * 128 + 512) * 4
    assert abs(n - (30 * 7 * 3 + 3 + 3) * 1560 * 12 * 128 * 2 - part) < 1 << 20
    assert n <= 3.1e9
    # K and V as the method keeps them: 2.01 GB
    assert 30 * 7 * 2 * 1560 * 12 * 128 * 2 == 2012774400


def test_large_model_cache_holds_little_beyond_its_keys_and_values():
    from streaming_autoregressive_video_b200.workloads import LARGE_ACTIONS as w
    n = fd.fd_cache_bytes(fd.make_desc(w))
    kv = 2 * w.layers * w.slots * w.frame_tokens * w.heads * w.head_dim * 2  # K and V
    # K and V, the rotated keys (half of that again) and one work set
    assert n <= 1.5 * kv + 0.2e9 and n <= 25.5e9


@pytest.mark.parametrize("sets", [-1, 31])
def test_work_sets_outside_one_to_layers_rejected(sets):
    desc = fd.make_desc(SINGLE_480P, work_sets=sets)
    assert fd.fd_cache_bytes(desc) == 0


@pytest.mark.parametrize("field,value,status", [
    ("block_frames", 0, 2), ("window_frames", 0, 2), ("head_dim", 12, 2),
    ("num_heads", 0, 2), ("dtype", 7, 3), ("sink_frames", -1, 2),
    ("action_tokens", -2, 2), ("rope_theta", float("nan"), 2)])
def test_bad_descriptors_rejected(field, value, status):
    desc = fd.make_desc(SINGLE_480P)
    setattr(desc, field, value)
    assert fd.fd_cache_bytes(desc) == 0
    lay = fd.CacheLayout()
    assert fd.load().fd_cache_get_layout(ctypes.byref(desc), ctypes.byref(lay)) == status


def test_block_larger_than_window_rejected():
    desc = fd.make_desc(SINGLE_480P)
    desc.block_frames = 7
    assert fd.fd_cache_bytes(desc) == 0


def test_host_errors_before_any_device_call():
    lib = fd.load()
    desc = fd.make_desc(SINGLE_480P)
    h = ctypes.c_void_p()
    # null storage: rejected after validation, before any CUDA call
    assert lib.fd_cache_create(ctypes.byref(desc), None, 1 << 40, ctypes.byref(h)) == 1
    assert lib.fd_cache_create(ctypes.byref(desc), 1024, 16, ctypes.byref(h)) == 4
    assert lib.fd_cache_create(ctypes.byref(desc), 1000, 1 << 40, ctypes.byref(h)) == 8
    assert lib.fd_block_attention(None, 0, 1, 16, 16, 16, 16, None, None) == 1
    assert lib.fd_cache_commit(None, 0, 1, 1, None, None, None, None) == 1
    assert lib.fd_cache_reset(None, None, 1, None) == 1
    assert lib.fd_rope3d(None, 0, 1, 16, 4, 1, None) == 1
    code = ctypes.c_int32()
    assert lib.fd_get_device_error(None, ctypes.byref(code)) == 1
    assert lib.fd_cache_destroy(None) == 1
    assert fd.fd_status_string(6) == "device-side wait gave up"
    assert fd.fd_launch_count() >= 0


@pytest.mark.parametrize("heads,kv_heads,status", [(4, 3, 2), (4, 8, 2), (4, -1, 2),
                                                   (4, 2, 0), (6, 1, 0), (4, 0, 0)])
def test_grouped_query_heads_validated(heads, kv_heads, status):
    w = SINGLE_480P.scaled(heads=heads, kv_heads=kv_heads, layers=1)
    desc = fd.make_desc(w)
    lay = fd.CacheLayout()
    assert fd.load().fd_cache_get_layout(ctypes.byref(desc), ctypes.byref(lay)) == status
    if status == 0:
        # K and V regions hold Hkv heads
        hkv = kv_heads or heads
        kv = w.slots * w.frame_tokens * hkv * w.head_dim * 2
        assert lay.layer_kv_bytes == kv


@pytest.mark.parametrize("shards,shard,status", [(2, 0, 0), (2, 1, 0), (7, 6, 0), (8, 0, 2),
                                                 (2, 2, 2), (2, -1, 2), (0, 0, 0)])
def test_shard_descriptor_validated(shards, shard, status):
    # 480p ring: 1 sink + 6 window slots -> at most 7 shards
    desc = fd.make_desc(SINGLE_480P.scaled(layers=1), shards=shards, shard=shard)
    lay = fd.CacheLayout()
    assert fd.load().fd_cache_get_layout(ctypes.byref(desc), ctypes.byref(lay)) == status
    if status == 0:
        n = max(shards, 1)
        local = -(-7 // n)
        assert lay.layer_kv_bytes == local * 1560 * 12 * 128 * 2


def test_combine_host_errors():
    lib = fd.load()
    vp = ctypes.c_void_p
    one = (vp * 1)(16)
    assert lib.fd_attention_combine(0, one, one, 1, 1, 1, 8, 0, 16, None, None) == 2
    assert lib.fd_attention_combine(17, one, one, 1, 1, 1, 8, 0, 16, None, None) == 2
    assert lib.fd_attention_combine(1, one, one, 1, 1, 1, 8, 9, 16, None, None) == 3
    assert lib.fd_attention_combine(1, None, one, 1, 1, 1, 8, 0, 16, None, None) == 1
    assert lib.fd_attention_combine(1, one, one, 1, 1, 1, 8, 0, 17, None, None) == 8


def test_layout_regions_cannot_wrap_the_total():
    """A geometry whose K region alone is 2^63 bytes (a 4096x4096 grid, 4096
    heads of 256 fp32, 64 window slots, 1024 rollouts, 2 layers) is refused
    with FD_ERR_CAPACITY: summed with V and the rotated keys it would wrap a
    64-bit size and report a small storage requirement."""
    desc = fd.CacheDesc(2, 1024, 4096, 256, 4096, 4096, 0, 1, 0, 64, 1.0e4, fd.FD_F32,
                        0, 1, 1, 0)
    lay = fd.CacheLayout()
    assert fd.load().fd_cache_get_layout(ctypes.byref(desc), ctypes.byref(lay)) == 4
    assert fd.fd_cache_bytes(desc) == 0
    # one layer of one rollout of the same frame size still lays out
    small = fd.CacheDesc(1, 1, 4, 256, 64, 64, 0, 1, 0, 64, 1.0e4, fd.FD_F32, 0, 1, 1, 0)
    assert fd.load().fd_cache_get_layout(ctypes.byref(small), ctypes.byref(lay)) == 0
    assert lay.total == fd.fd_cache_bytes(small) > 3 * lay.layer_kv_bytes
