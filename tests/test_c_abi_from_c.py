"""The boundary as a C caller sees it: a C99 program compiled with gcc against
include/fd.h, linked to libfd.so, makes the host-only calls (sizes, layout,
status strings, argument errors) and prints the results, which must equal
what the Python binding gets.  No GPU: every call here returns before any
CUDA work."""
import os
import shutil
import subprocess

import pytest

from streaming_autoregressive_video_b200 import binding as fd
from streaming_autoregressive_video_b200.workloads import GQA_480P, SINGLE_480P

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "streaming_autoregressive_video_b200")

PROGRAM = r"""
#include <stdio.h>
#include <string.h>
#include "fd.h"

static fd_cache_desc desc480(int32_t kv_heads) {
  fd_cache_desc d;
  memset(&d, 0, sizeof d);
  d.num_layers = 30; d.max_rollouts = 1; d.num_heads = 12; d.head_dim = 128;
  d.grid_h = 30; d.grid_w = 52; d.action_tokens = 0; d.block_frames = 3;
  d.sink_frames = 1; d.window_frames = 6; d.rope_theta = 1.0e4f; d.dtype = FD_BF16;
  d.num_kv_heads = kv_heads; d.num_views = 1; d.num_shards = 1; d.shard_index = 0;
  return d;
}

int main(void) {
  fd_cache_desc d = desc480(0);
  fd_cache_layout lay;
  printf("bytes %zu\n", fd_cache_bytes(&d));
  int st = (int)fd_cache_get_layout(&d, &lay);  /* before reading lay */
  printf("layout %d %zu %zu %zu %d %d %d\n", st, lay.krot, lay.layer_kv_bytes, lay.total,
         lay.rope_pairs_t, lay.rope_pairs_h, lay.rope_pairs_w);
  d = desc480(4);
  printf("gqa_bytes %zu\n", fd_cache_bytes(&d));
  d.block_frames = 7;  /* more than the window */
  printf("bad_bytes %zu\n", fd_cache_bytes(&d));
  printf("bad_layout %d\n", (int)fd_cache_get_layout(&d, &lay));
  printf("null_attention %d\n",
         (int)fd_block_attention(NULL, 0, 1, NULL, NULL, NULL, NULL, NULL, NULL));
  printf("status7 %s\n", fd_status_string(FD_ERR_UNSUPPORTED));
  return 0;
}
"""


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_c_program_sees_the_same_boundary(tmp_path):
    fd.load()                                      # builds libfd.so if needed
    src = tmp_path / "abi.c"
    exe = tmp_path / "abi"
    src.write_text(PROGRAM)
    cc = subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", "-pedantic",
                         "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe),
                         "-L", PKG, "-lfd", f"-Wl,-rpath,{PKG}"],
                        capture_output=True, text=True)
    assert cc.returncode == 0, cc.stderr
    run = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert run.returncode == 0, run.stderr
    got = dict(line.split(" ", 1) for line in run.stdout.strip().splitlines())

    lay = fd.fd_cache_get_layout(fd.make_desc(SINGLE_480P))
    assert int(got["bytes"]) == fd.fd_cache_bytes(fd.make_desc(SINGLE_480P)) == lay.total
    st, krot, layer_kv, total, pt, ph, pw = (int(x) for x in got["layout"].split())
    assert (st, krot, layer_kv, total) == (0, lay.krot, lay.layer_kv_bytes, lay.total)
    assert (pt, ph, pw) == (22, 21, 21)
    assert int(got["gqa_bytes"]) == fd.fd_cache_bytes(fd.make_desc(GQA_480P))
    assert int(got["bad_bytes"]) == 0 and int(got["bad_layout"]) == 2
    assert int(got["null_attention"]) == 1
    assert got["status7"] == fd.fd_status_string(7)
