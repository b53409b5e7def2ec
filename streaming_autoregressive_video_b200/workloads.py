"""Workload shapes of the streaming chunk-attention hot path.

Each workload is a cache geometry plus a rollout schedule.  The shapes follow
the serving scenarios on the pages:

* 832x480 video under 16x16 spatial VAE compression gives a 30x52 latent grid
  ("Cosmos3-H-Dreams" model card, Model Architecture / Input sections);
* each latent frame consumes 4 action vectors ("Cosmos3-H-Dreams", Model
  Architecture), carried here as 4 extra key/value tokens per frame;
* two or four denoising steps per block ("Cosmos3-H-Dreams" Model
  Architecture; AlpaDreams write-up, section VII);
* a bounded per-rollout cache of sink frames plus a rolling window
  ("NVIDIA FlashDreams Is the Open-Source Inference Engine Robotics World
  Models Needed", Bounded Memory for Infinite Rollouts).

Nothing here computes any part of the method.
"""
from __future__ import annotations

from dataclasses import dataclass, replace
from typing import Optional, Tuple


@dataclass(frozen=True)
class Workload:
    name: str
    layers: int
    rollouts: int
    heads: int
    head_dim: int
    grid_h: int
    grid_w: int
    action_tokens: int
    block_frames: int      # F
    sink_frames: int       # S
    window_frames: int     # W
    steps: int             # denoising steps per block
    blocks: int            # blocks in the rollout schedule
    dtype: str             # "bf16" or "f32"
    theta: float = 1.0e4
    value_scale: float = 1.0
    # ragged cache fill: window frames committed per rollout drawn uniformly
    # from [lo, hi] before the measured block (None = uniform fill)
    ragged_window: Optional[Tuple[int, int]] = None
    # key/value heads (grouped-query attention); 0 = heads
    kv_heads: int = 0
    # camera views per frame (multi-view models); tokens = views * Gh * Gw
    views: int = 1

    @property
    def hkv(self) -> int:             # key/value heads
        return self.kv_heads or self.heads

    @property
    def tokens(self) -> int:          # T: video tokens per latent frame
        return self.views * self.grid_h * self.grid_w

    @property
    def view_tokens(self) -> int:     # video tokens per view
        return self.grid_h * self.grid_w

    @property
    def frame_tokens(self) -> int:    # Tf: key/value tokens per frame
        return self.tokens + self.action_tokens

    @property
    def queries(self) -> int:         # Mq: query rows per rollout and head
        return self.block_frames * self.tokens

    @property
    def slots(self) -> int:           # S + W cache slots per rollout and layer
        return self.sink_frames + self.window_frames

    def scaled(self, **kw) -> "Workload":
        return replace(self, **kw)


# 1: tiny fp32 rollout, 20 blocks through the ring (latency bound)
TINY_F32 = Workload("tiny-f32-4x4-h2-d64-w3", layers=1, rollouts=1, heads=2,
                    head_dim=64, grid_h=4, grid_w=4, action_tokens=0,
                    block_frames=1, sink_frames=0, window_frames=3, steps=2,
                    blocks=20, dtype="f32")

# 2: one rollout at the 480x832 class shape, 1 sink + 6 window frames
SINGLE_480P = Workload("bf16-30x52-h12-d128-F3-S1-W6-L30", layers=30,
                       rollouts=1, heads=12, head_dim=128, grid_h=30,
                       grid_w=52, action_tokens=0, block_frames=3,
                       sink_frames=1, window_frames=6, steps=4, blocks=3,
                       dtype="bf16")

# 3: large-model shape, 40 heads, 12-frame window, 4 action tokens per frame
LARGE_ACTIONS = Workload("bf16-30x52+4a-h40-d128-F3-S1-W12-L40", layers=40,
                         rollouts=1, heads=40, head_dim=128, grid_h=30,
                         grid_w=52, action_tokens=4, block_frames=3,
                         sink_frames=1, window_frames=12, steps=4, blocks=5,
                         dtype="bf16", value_scale=0.5)

# 4: long rollout, one frame per block, 10,000 blocks through the ring
LONG_ROLLOUT = Workload("bf16-30x52-h12-d128-F1-S1-W8-10k", layers=1,
                        rollouts=1, heads=12, head_dim=128, grid_h=30,
                        grid_w=52, action_tokens=0, block_frames=1,
                        sink_frames=1, window_frames=8, steps=2, blocks=10000,
                        dtype="bf16")

# 5: 16 concurrent rollouts with ragged window fill
BATCHED_RAGGED = Workload("bf16-16x20-h24-d128-F3-W12-R16-ragged", layers=1,
                          rollouts=16, heads=24, head_dim=128, grid_h=16,
                          grid_w=20, action_tokens=0, block_frames=3,
                          sink_frames=0, window_frames=12, steps=2, blocks=1,
                          dtype="bf16", ragged_window=(3, 12))

# 6: four-camera frames at 704x1280 (44x80 latent grid per view under the same
#    16x spatial compression), 2 denoising steps (AlpaDreams write-up, section
#    VIII: four-view model, two-step diffusion, 704x1280); one latent frame per
#    block, 1 sink + 3 window frames; 16 heads of 128 (a 2B-parameter DiT,
#    hidden 2048).  14080 query tokens x 70400 keys per call.
MULTIVIEW_4 = Workload("bf16-4x44x80-h16-d128-F1-S1-W3", layers=28, rollouts=1,
                       heads=16, head_dim=128, grid_h=44, grid_w=80, action_tokens=0,
                       block_frames=1, sink_frames=1, window_frames=3, steps=2,
                       blocks=5, dtype="bf16", views=4)

# 7: the 480p shape with grouped-query attention (12 query heads, 4 key/value
#    heads): a cache-semantics variant, not a configuration of the pages
GQA_480P = SINGLE_480P.scaled(name="bf16-30x52-h12kv4-d128-F3-S1-W6-L30", kv_heads=4)

# 8: the 480p shape with head size 64 (the test matrix's second head size; 24
#    heads of 64 keep the 1536-wide model of the 12 x 128 workload)
D64_480P = SINGLE_480P.scaled(name="bf16-30x52-h24-d64-F3-S1-W6-L30", head_dim=64, heads=24)

ALL = [TINY_F32, SINGLE_480P, LARGE_ACTIONS, LONG_ROLLOUT, BATCHED_RAGGED, MULTIVIEW_4,
       GQA_480P, D64_480P]
