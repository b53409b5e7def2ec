"""ctypes binding of libfd.so: argument marshalling and argument checks only.

Every function here has the name of a C entry point in include/fd.h, checks
that each tensor argument is a contiguous CUDA tensor (on the cache's device)
holding at least the bytes the call reads or writes, converts Python / torch
arguments into plain pointers and sizes, calls the library and raises FdError
on a non-OK status.  No step of the computation runs here; if the library
cannot be loaded the call fails loudly.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libfd.so")

FD_BF16, FD_F32 = 0, 1
STATUS = {0: "FD_OK", 1: "FD_ERR_INVALID_ARG", 2: "FD_ERR_SHAPE", 3: "FD_ERR_DTYPE",
          4: "FD_ERR_CAPACITY", 5: "FD_ERR_CUDA", 6: "FD_ERR_DEVICE_TIMEOUT",
          7: "FD_ERR_UNSUPPORTED", 8: "FD_ERR_ALIGNMENT"}

# every symbol include/fd.h declares
EXPORTS = ["fd_cache_bytes", "fd_cache_get_layout", "fd_cache_create",
           "fd_cache_destroy", "fd_cache_get_desc", "fd_cache_layout_of",
           "fd_cache_reset", "fd_rope3d", "fd_block_attention",
           "fd_block_attention_static",
           "fd_cache_commit", "fd_cache_frames", "fd_cache_window_full",
           "fd_get_device_error",
           "fd_exp2_selfcheck", "fd_selftest_bounded_wait", "fd_attention_combine",
           "fd_launch_count", "fd_status_string"]


class FdError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {STATUS.get(status, status)}")


class CacheDesc(ctypes.Structure):
    _fields_ = [("num_layers", ctypes.c_int32), ("max_rollouts", ctypes.c_int32),
                ("num_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
                ("grid_h", ctypes.c_int32), ("grid_w", ctypes.c_int32),
                ("action_tokens", ctypes.c_int32), ("block_frames", ctypes.c_int32),
                ("sink_frames", ctypes.c_int32), ("window_frames", ctypes.c_int32),
                ("rope_theta", ctypes.c_float), ("dtype", ctypes.c_int32),
                ("num_kv_heads", ctypes.c_int32), ("num_views", ctypes.c_int32),
                ("num_shards", ctypes.c_int32), ("shard_index", ctypes.c_int32),
                ("num_work_sets", ctypes.c_int32)]


class CacheLayout(ctypes.Structure):
    _fields_ = [("k", ctypes.c_size_t), ("v", ctypes.c_size_t), ("krot", ctypes.c_size_t),
                ("kblk", ctypes.c_size_t), ("qblk", ctypes.c_size_t),
                ("part", ctypes.c_size_t),
                ("pos", ctypes.c_size_t),
                ("count", ctypes.c_size_t), ("ttab", ctypes.c_size_t),
                ("htab", ctypes.c_size_t), ("wtab", ctypes.c_size_t),
                ("err", ctypes.c_size_t), ("total", ctypes.c_size_t),
                ("layer_kv_bytes", ctypes.c_size_t), ("rope_pairs_t", ctypes.c_int32),
                ("rope_pairs_h", ctypes.c_int32), ("rope_pairs_w", ctypes.c_int32)]


_lib = None


def load(path: Optional[str] = None, build_if_missing: bool = True) -> ctypes.CDLL:
    """Load libfd.so (building it in-tree first when it is missing or stale)."""
    global _lib
    if _lib is not None:
        return _lib
    path = path or LIB_PATH
    if build_if_missing and path == LIB_PATH:
        from . import build as _build
        if not _build.up_to_date():
            _build.build()
    if not os.path.exists(path):
        raise FdError(-1, f"libfd.so not found at {path}")
    lib = ctypes.CDLL(path)
    vp, i32, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_size_t
    lib.fd_cache_bytes.argtypes = [ctypes.POINTER(CacheDesc)]
    lib.fd_cache_bytes.restype = sz
    lib.fd_cache_get_layout.argtypes = [ctypes.POINTER(CacheDesc), ctypes.POINTER(CacheLayout)]
    lib.fd_cache_create.argtypes = [ctypes.POINTER(CacheDesc), vp, sz, ctypes.POINTER(vp)]
    lib.fd_cache_destroy.argtypes = [vp]
    lib.fd_cache_get_desc.argtypes = [vp, ctypes.POINTER(CacheDesc)]
    lib.fd_cache_layout_of.argtypes = [vp, ctypes.POINTER(CacheLayout)]
    lib.fd_cache_reset.argtypes = [vp, ctypes.POINTER(i32), i32, vp]
    lib.fd_rope3d.argtypes = [vp, i32, i32, vp, i32, i32, vp]
    lib.fd_block_attention.argtypes = [vp, i32, i32, vp, vp, vp, vp, vp, vp]
    lib.fd_block_attention_static.argtypes = [vp, i32, i32, vp, vp, vp, vp, vp, vp]
    lib.fd_cache_commit.argtypes = [vp, i32, i32, i32, ctypes.POINTER(i32),
                                    ctypes.POINTER(vp), ctypes.POINTER(vp), vp]
    lib.fd_cache_frames.argtypes = [vp, i32, i32, ctypes.POINTER(ctypes.c_int64)]
    lib.fd_cache_window_full.argtypes = [vp, i32, i32, i32, ctypes.POINTER(i32)]
    lib.fd_get_device_error.argtypes = [vp, ctypes.POINTER(i32)]
    lib.fd_exp2_selfcheck.argtypes = [vp, vp, ctypes.c_int64, vp]
    lib.fd_selftest_bounded_wait.argtypes = [vp, i32, vp]
    lib.fd_attention_combine.argtypes = [i32, ctypes.POINTER(vp), ctypes.POINTER(vp), i32, i32,
                                         i32, i32, i32, vp, vp, vp]
    lib.fd_launch_count.argtypes = []
    lib.fd_launch_count.restype = ctypes.c_uint64
    lib.fd_status_string.argtypes = [i32]
    lib.fd_status_string.restype = ctypes.c_char_p
    for name in EXPORTS:
        f = getattr(lib, name)
        if f.restype is ctypes.c_int:  # default: status-returning functions
            f.restype = ctypes.c_int32
    _lib = lib
    return lib


def _check(status: int, where: str) -> None:
    if status != 0:
        raise FdError(status, where)


def _ptr(t) -> Optional[int]:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _dev_ptr(t, nbytes: int, where: str, name: str, device=None) -> Optional[int]:
    """Address of the tensor argument `name` after checking that the kernels
    may read or write `nbytes` bytes there: a contiguous CUDA tensor (on
    `device` when given) of at least that many bytes.  The C entry points take
    bare addresses and cannot check this themselves; a host or short buffer
    would otherwise reach a kernel.  Raw integer addresses pass unchecked (the
    caller vouches for them), None stays None."""
    if t is None or isinstance(t, int):
        return t
    if not getattr(t, "is_cuda", False):
        raise FdError(1, f"{where}: {name} is not a CUDA tensor")
    if device is not None and t.device != device:
        raise FdError(1, f"{where}: {name} is on {t.device}, the cache on {device}")
    if not t.is_contiguous():
        raise FdError(1, f"{where}: {name} is not contiguous")
    have = t.numel() * t.element_size()
    if have < nbytes:
        raise FdError(2, f"{where}: {name} holds {have} bytes, needs {nbytes}")
    return t.data_ptr()


class _Geom:
    """Per-call tensor sizes of a cache's geometry (bytes per rollout)."""

    def __init__(self, desc: "CacheDesc"):
        self.esz = 2 if desc.dtype == FD_BF16 else 4
        views = desc.num_views or 1
        self.T = views * desc.grid_h * desc.grid_w
        self.Tf = self.T + desc.action_tokens
        self.F = desc.block_frames
        self.H = desc.num_heads
        self.Hkv = desc.num_kv_heads or desc.num_heads
        self.d = desc.head_dim
        self.q = self.F * self.T * self.H * self.d * self.esz      # q and out
        self.kv = self.F * self.Tf * self.Hkv * self.d * self.esz  # block k and v
        self.lse = self.H * self.F * self.T * 4


def _device_of(cache: "Cache"):
    return getattr(cache.storage, "device", None)


def _stream(stream) -> Optional[int]:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def make_desc(w, dtype: Optional[str] = None, shards: int = 1, shard: int = 0,
              work_sets: int = 1) -> CacheDesc:
    """CacheDesc of a workload (see workloads.Workload); `shards`/`shard`
    select one context-parallel shard of its key set; `work_sets` is the
    number of per-call work areas (attention calls whose layers differ modulo
    it may run at the same time)."""
    dt = dtype or w.dtype
    return CacheDesc(w.layers, w.rollouts, w.heads, w.head_dim, w.grid_h, w.grid_w,
                     w.action_tokens, w.block_frames, w.sink_frames, w.window_frames,
                     float(w.theta), FD_BF16 if dt == "bf16" else FD_F32,
                     getattr(w, "kv_heads", 0), getattr(w, "views", 1), shards, shard,
                     work_sets)


def fd_cache_bytes(desc: CacheDesc) -> int:
    return load().fd_cache_bytes(ctypes.byref(desc))


def fd_cache_get_layout(desc: CacheDesc) -> CacheLayout:
    lay = CacheLayout()
    _check(load().fd_cache_get_layout(ctypes.byref(desc), ctypes.byref(lay)),
           "fd_cache_get_layout")
    return lay


def fd_status_string(status: int) -> str:
    return load().fd_status_string(status).decode()


def fd_launch_count() -> int:
    return int(load().fd_launch_count())


class Cache:
    """Host handle of a cache bound to caller-owned device storage."""

    def __init__(self, desc: CacheDesc, storage):
        self.desc = desc
        self.storage = storage          # keeps the caller's buffer alive
        self.layout = fd_cache_get_layout(desc)
        h = ctypes.c_void_p()
        _check(load().fd_cache_create(ctypes.byref(desc), _ptr(storage),
                                      storage.numel() * storage.element_size(),
                                      ctypes.byref(h)), "fd_cache_create")
        self.handle = h

    def close(self) -> None:
        if self.handle:
            _check(load().fd_cache_destroy(self.handle), "fd_cache_destroy")
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def fd_cache_create(desc: CacheDesc, storage) -> Cache:
    """Bind a cache to `storage` (a uint8 CUDA tensor of fd_cache_bytes bytes)."""
    return Cache(desc, storage)


def fd_cache_reset(cache: Cache, rollout_ids: Sequence[int], stream=None) -> None:
    ids = (ctypes.c_int32 * len(rollout_ids))(*rollout_ids)
    _check(load().fd_cache_reset(cache.handle, ids, len(rollout_ids), _stream(stream)),
           "fd_cache_reset")


def fd_rope3d(cache: Cache, layer: int, n_rollouts: int, x, tokens_per_frame: int,
              heads: int, stream=None) -> None:
    g = _Geom(cache.desc)
    n = max(n_rollouts, 0) * g.F * max(tokens_per_frame, 0) * max(heads, 0) * g.d * g.esz
    xp = _dev_ptr(x, n, "fd_rope3d", "x", _device_of(cache))
    _check(load().fd_rope3d(cache.handle, layer, n_rollouts, xp, tokens_per_frame,
                            heads, _stream(stream)), "fd_rope3d")


def _attention_ptrs(cache: Cache, n_rollouts: int, q, k, v, out, lse, where: str):
    g = _Geom(cache.desc)
    n = max(n_rollouts, 0)
    dev = _device_of(cache)
    return (_dev_ptr(q, n * g.q, where, "q", dev), _dev_ptr(k, n * g.kv, where, "k", dev),
            _dev_ptr(v, n * g.kv, where, "v", dev), _dev_ptr(out, n * g.q, where, "out", dev),
            _dev_ptr(lse, n * g.lse, where, "lse", dev))


def fd_block_attention(cache: Cache, layer: int, n_rollouts: int, q, k, v, out,
                       lse=None, stream=None) -> None:
    ptrs = _attention_ptrs(cache, n_rollouts, q, k, v, out, lse, "fd_block_attention")
    _check(load().fd_block_attention(cache.handle, layer, n_rollouts, *ptrs, _stream(stream)),
           "fd_block_attention")


# FD_STATIC_WORK_BYTES of include/fd.h
STATIC_WORK_BYTES = 32 << 20


def fd_block_attention_static(cache: Cache, layer: int, n_rollouts: int, q, k, v, out,
                              lse=None, stream=None) -> None:
    """fd_block_attention with its work area in the library's static array."""
    ptrs = _attention_ptrs(cache, n_rollouts, q, k, v, out, lse, "fd_block_attention_static")
    _check(load().fd_block_attention_static(cache.handle, layer, n_rollouts, *ptrs,
                                            _stream(stream)),
           "fd_block_attention_static")


def fd_cache_commit(cache: Cache, layer_begin: int, layer_end: int, n_rollouts: int,
                    k_list, v_list, frames: Optional[Sequence[int]] = None,
                    stream=None) -> None:
    nl = layer_end - layer_begin
    if nl < 1 or len(k_list) != nl or len(v_list) != nl:
        raise FdError(1, f"fd_cache_commit: {len(k_list)} k and {len(v_list)} v tensors "
                         f"for {nl} layers")
    if frames is not None and len(frames) != n_rollouts:
        raise FdError(1, f"fd_cache_commit: {len(frames)} frame counts for {n_rollouts} "
                         "rollouts")
    g = _Geom(cache.desc)
    nb = max(n_rollouts, 0) * g.kv
    dev = _device_of(cache)
    kp = (ctypes.c_void_p * nl)(*[_dev_ptr(t, nb, "fd_cache_commit", f"k[{i}]", dev)
                                  for i, t in enumerate(k_list)])
    vp = (ctypes.c_void_p * nl)(*[_dev_ptr(t, nb, "fd_cache_commit", f"v[{i}]", dev)
                                  for i, t in enumerate(v_list)])
    fr = None if frames is None else (ctypes.c_int32 * n_rollouts)(*frames)
    _check(load().fd_cache_commit(cache.handle, layer_begin, layer_end, n_rollouts, fr,
                                  kp, vp, _stream(stream)), "fd_cache_commit")


def fd_cache_frames(cache: Cache, layer: int, rollout: int) -> int:
    n = ctypes.c_int64()
    _check(load().fd_cache_frames(cache.handle, layer, rollout, ctypes.byref(n)),
           "fd_cache_frames")
    return n.value


def fd_cache_window_full(cache: Cache, layer: int, rollout: int, frames: int) -> bool:
    """Whether the next block of `frames` frames restarts the rollout's window
    (the window-boundary policy)."""
    r = ctypes.c_int32()
    _check(load().fd_cache_window_full(cache.handle, layer, rollout, frames, ctypes.byref(r)),
           "fd_cache_window_full")
    return bool(r.value)


def fd_exp2_selfcheck(x, y, stream=None) -> None:
    xp = _dev_ptr(x, x.numel() * 4, "fd_exp2_selfcheck", "x")
    yp = _dev_ptr(y, 3 * x.numel() * 4, "fd_exp2_selfcheck", "y", x.device)
    _check(load().fd_exp2_selfcheck(xp, yp, x.numel(), _stream(stream)),
           "fd_exp2_selfcheck")


def fd_selftest_bounded_wait(cache: Cache, limit_ms: int, stream=None) -> None:
    _check(load().fd_selftest_bounded_wait(cache.handle, limit_ms, _stream(stream)),
           "fd_selftest_bounded_wait")


def fd_attention_combine(outs, lses, out, lse=None, stream=None) -> None:
    """out (and lse) = log-sum-exp combination of per-part rows `outs` [R][Mq][H][d]
    with their log-sum-exps `lses` [R][H][Mq] (device tensors)."""
    n = len(outs)
    if len(lses) != n:
        raise FdError(1, f"fd_attention_combine: {n} row tensors, {len(lses)} lse tensors")
    R, Mq, H, d = out.shape
    dt = FD_BF16 if out.element_size() == 2 else FD_F32
    rows = R * Mq * H * d * out.element_size()
    lse_bytes = R * H * Mq * 4
    w = "fd_attention_combine"
    dev = getattr(out, "device", None)
    op = (ctypes.c_void_p * n)(*[_dev_ptr(t, rows, w, f"outs[{i}]", dev)
                                 for i, t in enumerate(outs)])
    lp = (ctypes.c_void_p * n)(*[_dev_ptr(t, lse_bytes, w, f"lses[{i}]", dev)
                                 for i, t in enumerate(lses)])
    _dev_ptr(out, rows, w, "out")
    _dev_ptr(lse, lse_bytes, w, "lse", dev)
    _check(load().fd_attention_combine(n, op, lp, R, Mq, H, d, dt, _ptr(out), _ptr(lse),
                                       _stream(stream)), "fd_attention_combine")


def fd_get_device_error(cache: Cache) -> int:
    code = ctypes.c_int32()
    st = load().fd_get_device_error(cache.handle, ctypes.byref(code))
    if st not in (0, 6):
        raise FdError(st, "fd_get_device_error")
    return code.value
