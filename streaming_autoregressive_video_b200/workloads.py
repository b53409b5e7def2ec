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

    @property
    def tokens(self) -> int:          # T: video tokens per latent frame
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

ALL = [TINY_F32, SINGLE_480P, LARGE_ACTIONS, LONG_ROLLOUT, BATCHED_RAGGED]
