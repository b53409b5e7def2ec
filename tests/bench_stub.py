"""Runs bench.run_fd on the CPU with CUDA and the library replaced by
stand-ins, and prints its JSON line.  The numbers mean nothing; the point is
that every line of the GPU arm's host code runs and the line it prints keeps
the bench contract.  Used by tests/test_bench_contract.py in a subprocess
(the stand-ins patch torch process-wide).

    python tests/bench_stub.py <workload> [layers]
"""
import contextlib
import json
import os
import sys
import types

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

import bench  # noqa: E402
from streaming_autoregressive_video_b200 import binding as fd  # noqa: E402
from streaming_autoregressive_video_b200 import synth  # noqa: E402

_device = torch.device
torch.device = lambda *a, **k: _device("cpu")
torch.cuda.set_device = lambda *a: None
torch.cuda.synchronize = lambda *a: None


class _Event:
    def __init__(self, *a, **k):
        pass

    def record(self, *a):
        pass

    def elapsed_time(self, other):
        return 1.0


class _Stream:
    cuda_stream = 0

    def __init__(self, *a, **k):
        pass

    def wait_event(self, e):
        pass


torch.cuda.empty_cache = lambda: None


torch.cuda.Event = _Event
torch.cuda.Stream = _Stream
torch.cuda.current_stream = lambda *a: _Stream()
torch.cuda.stream = lambda s: contextlib.nullcontext()
torch.Tensor.pin_memory = lambda self: self
synth.normal_device = lambda seed, shape, dtype, dev, scale=1.0: torch.zeros(
    shape, dtype=torch.bfloat16 if dtype == "bf16" else torch.float32)

_state = {"n": None, "launches": 0, "fills": []}


class _Cache:
    def __init__(self, desc, storage):
        self.desc, self.storage = desc, storage
        _state["n"] = [[0] * desc.max_rollouts for _ in range(desc.num_layers)]


def _commit(cache, l0, l1, R, ks, vs, frames=None, stream=None):
    assert len(ks) == l1 - l0 == len(vs)
    g = fd._Geom(cache.desc)
    for t in list(ks) + list(vs):
        assert t.numel() * t.element_size() == R * g.kv
    for l in range(l0, l1):
        for r in range(R):
            _state["n"][l][r] += cache.desc.block_frames if frames is None else frames[r]
    _state["launches"] += 2


def _attention(cache, l, R, q, k, v, out, lse=None, stream=None):
    _state["fills"].append(list(_state["n"][l][:R]))  # frames each rollout's call sees
    g = fd._Geom(cache.desc)
    assert q.numel() * q.element_size() == R * g.q
    assert k.numel() * k.element_size() == R * g.kv == v.numel() * v.element_size()
    assert out.numel() * out.element_size() == R * g.q
    _state["launches"] += 2


def _reset(cache, rollout_ids, stream=None):
    for row in _state["n"]:
        for r in rollout_ids:
            row[r] = 0
    _state["launches"] += 1


fd.fd_cache_create = _Cache
fd.fd_cache_commit = _commit
fd.fd_cache_reset = _reset
fd.fd_cache_frames = lambda cache, l, r: _state["n"][l][r]
fd.fd_block_attention = _attention
fd.fd_launch_count = lambda: _state["launches"]
fd.fd_get_device_error = lambda cache: 0


class _Sampler:
    def __init__(self, i):
        pass

    def start(self):
        pass

    def stop(self):
        return {"sm_mhz": 1.0, "sm_max_mhz": 1.0, "reasons": []}


bench.ClockSampler = _Sampler

if __name__ == "__main__":
    w = bench.workloads()[sys.argv[1]]
    layers = int(sys.argv[2]) if len(sys.argv) > 2 else 2
    w = w.scaled(layers=min(w.layers, layers))
    args = types.SimpleNamespace(steps=2, warmup=3, no_e2e=False, no_cpu_baseline=True,
                                 gpus=1, no_extra=False, workload=sys.argv[1])
    bench.run_fd(args, w, 0, 1, 0)
    # the frame counts every attention call saw, for the tests to check
    print("FILLS " + json.dumps(_state["fills"]), file=sys.stderr)
