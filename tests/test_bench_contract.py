"""bench.py's JSON line on the CPU: the GPU arm's host code runs with CUDA
and the library replaced by stand-ins (tests/bench_stub.py, in a subprocess),
and the line it prints carries every key of the bench contract.  The
reference arm runs for real (the oracle on the host)."""
import json
import os
import subprocess
import sys
import types

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from streaming_autoregressive_video_b200.workloads import Workload  # noqa: E402


def _stub_run(workload):
    res = subprocess.run([sys.executable, os.path.join(ROOT, "tests", "bench_stub.py"),
                          workload], capture_output=True, text=True, timeout=600)
    assert res.returncode == 0, res.stderr[-2000:]
    fills = [json.loads(x[len("FILLS "):]) for x in res.stderr.splitlines()
             if x.startswith("FILLS ")]
    return json.loads(res.stdout.strip().splitlines()[-1]), fills[-1]


def _stub_line(workload):
    return _stub_run(workload)[0]


def test_ragged_calls_all_see_the_ragged_fill():
    """Every block's commit adds frames to every rollout; the bench restores
    a ragged workload's fill before each block, so every attention call (warm
    up, timed, end to end) sees the fill whose work the line counts."""
    line, fills = _stub_run("ragged")
    w = bench.workloads()["ragged"]
    want = bench.prefill_frames(w, 0)
    assert len(set(want)) > 1          # the fill really is ragged
    assert fills and all(f == want for f in fills), fills[:3]
    assert line["config"]["keys_per_rollout"] == bench.keys_per_rollout(w, want)


@pytest.mark.parametrize("workload", ["480p", "gqa", "ragged", "multiview", "tiny"])
def test_gpu_arm_line_keeps_the_contract(workload):
    line = _stub_line(workload)
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "roofline", "gpu_launches", "clocks", "e2e"):
        assert key in line, key
    assert line["unit"] == "TFLOP/s" and line["higher_is_better"] is True
    assert line["scaling"] == "weak" and line["n_gpus"] == 1 and line["warmup"] >= 3
    assert line["config"]["workload"] == bench.workloads()[workload].name
    roof = line["roofline"]
    for key in ("bound", "achieved", "peak", "unit", "frac", "traffic"):
        assert key in roof, key
    w0 = bench.workloads()[workload]
    if w0.dtype == "bf16":
        assert roof["bound"] == "tensor" and roof["unit"] == "TFLOP/s"
        assert line["dtype"] == "bf16"
    else:
        assert roof["bound"] == "hbm" and roof["unit"] == "GB/s" and line["dtype"] == "f32"
    assert roof["frac"] == pytest.approx(roof["achieved"] / roof["peak"])
    esz = 2 if w0.dtype == "bf16" else 4
    e2e = line["e2e"]
    for key in ("value", "unit", "h2d_bytes_per_step", "d2h_bytes_per_step"):
        assert key in e2e, key
    w = w0.scaled(layers=min(w0.layers, 2))   # as bench_stub.py runs it
    # every call copies q, k, v in and out back: bytes from the tensors' sizes
    q = w.rollouts * w.queries * w.heads * w.head_dim * esz
    kv = w.rollouts * w.block_frames * w.frame_tokens * w.hkv * w.head_dim * esz
    calls = w.steps * w.layers
    assert e2e["h2d_bytes_per_step"] == calls * (q + 2 * kv)
    assert e2e["d2h_bytes_per_step"] == calls * q
    assert line["gpu_launches"] > 0
    # commit bytes: read k, v; write K, V and rotated K, with Hkv heads
    assert line["commit_roofline"]["algorithmic_bytes_per_launch"] == 5 * w.layers * kv
    assert line["commit_roofline"]["frac_4stream"] == pytest.approx(
        0.8 * line["commit_roofline"]["frac"])
    # the cache's storage and the K/V the method keeps
    assert line["config"]["cache_bytes"] == fd_cache_bytes(w)
    assert line["config"]["kv_bytes"] == 2 * w.layers * w.rollouts * w.slots * \
        w.frame_tokens * w.hkv * w.head_dim * esz
    if w0.ragged_window:
        # a ragged fill is restored before every timed block; the background
        # commit comparison is made on steady-state workloads only
        assert "finalize_overlap" not in line
    else:
        fo = line["finalize_overlap"]
        assert fo["layers"] == w.layers and fo["ms_per_step_side_stream_commits"] > 0
    if workload == "480p":
        oc = line["other_configs"]
        assert sorted(oc) == ["d64", "gqa", "large", "long", "multiview", "ragged", "tiny"]
        for name, e in oc.items():
            for key in ("ms_per_call", "tflops_per_call", "frac_of_burst_bf16", "clocks",
                        "commit_frac_of_hbm", "workload"):
                assert key in e, (name, key)
        assert oc["tiny"]["dtype"] == "f32" and "us_per_call" in oc["tiny"]
        ro = oc["long"]["rollout"]   # the 10,000-block rollout, timed whole
        assert ro["blocks"] == bench.workloads()["long"].blocks == 10000
        assert ro["device_bytes_constant"] is True and ro["ms_per_block"] > 0
    else:
        assert "other_configs" not in line


def fd_cache_bytes(w):
    from streaming_autoregressive_video_b200 import binding as fd
    return fd.fd_cache_bytes(fd.make_desc(w))


def test_reference_arm_line_matches_the_gpu_arm_config(capsys):
    w = Workload("contract-tiny", layers=2, rollouts=1, heads=2, head_dim=16, grid_h=3,
                 grid_w=4, action_tokens=1, block_frames=1, sink_frames=1,
                 window_frames=2, steps=1, blocks=1, dtype="bf16")
    bench.run_reference(types.SimpleNamespace(steps=1, warmup=0, gpus=1), w, 0)
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert line["impl"] == "reference"
    assert line["config"] == bench.workload_config(w, 1)
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["value"] == line["value"]
