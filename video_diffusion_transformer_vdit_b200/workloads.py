"""The Wan2.1-shaped attention workloads: shapes, masks and KV-cache histories (data only).

Token geometry: Wan2.1 at 832 x 480 gives a 30 x 52 latent patch grid (1,560 tokens per latent
frame); 5 s at 16 FPS is 81 pixel frames -> 21 latent frames (4x temporal compression,
1 + 4 * 20); Self-Forcing / Wave Forcing decode chunks of 3 latent frames (Wave Forcing / WaveRT
news item: the latent frame count must be divisible by 3); a 399-latent-frame rollout puts the
last chunk at global frame 396. Inputs are seeded N(0, 1) values (see the ``synth`` module); the
KV stream of a workload starts at ``kv_stream_first_frame``.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Tuple


@dataclass(frozen=True)
class Workload:
    id: int
    name: str
    grid_h: int
    grid_w: int
    heads: int
    head_dim: int
    bands: Tuple[int, int, int]
    mask_kind: int            # bit 0 block-causal, bit 1 radial, bit 2 dynamic threshold
    q_start: int              # global frame of the first query token
    q_frames: int
    capacity_frames: int      # KV ring capacity
    appends: Tuple[Tuple[int, int], ...]  # (start_frame, n_frames) KV appends, in order
    kv_stream_first_frame: int
    chunk_frames: int = 3
    w0: int = 52
    gamma_shift: int = 1
    lam: int = 8
    tau: float = 0.0          # dynamic threshold: logit margin below each row's maximum
    theta: float = 10000.0

    @property
    def frame_tokens(self) -> int:
        return self.grid_h * self.grid_w

    @property
    def q_tokens(self) -> int:
        return self.q_frames * self.frame_tokens

    @property
    def kv_tokens(self) -> int:
        return self.capacity_frames * self.frame_tokens

    @property
    def scale(self) -> float:
        return self.head_dim ** -0.5

    def window(self) -> Tuple[int, int]:
        """(first, last) global frame the cache holds after all appends."""
        first = last = None
        for s, n in self.appends:
            last = s + n - 1 if last is None else max(last, s + n - 1)
            first = s if first is None else first
            first = max(first, last - self.capacity_frames + 1)
        return first, last

    @property
    def kv_stream_frames(self) -> int:
        return max(s + n for s, n in self.appends) - self.kv_stream_first_frame


_WAN = dict(grid_h=30, grid_w=52, head_dim=128, bands=(44, 42, 42))

WORKLOADS = {
    1: Workload(1, "tiny 6x4x8 block-causal d64", grid_h=4, grid_w=8, heads=2, head_dim=64,
                bands=(24, 20, 20), mask_kind=1, q_start=0, q_frames=6, capacity_frames=6,
                appends=((0, 3), (3, 3)), kv_stream_first_frame=0),
    2: Workload(2, "wan2.1-1.3b bidirectional 21x30x52 h12 dense", heads=12, mask_kind=0,
                q_start=0, q_frames=21, capacity_frames=21, appends=((0, 21),),
                kv_stream_first_frame=0, **_WAN),
    3: Workload(3, "wan2.1-1.3b causal chunk q3@18 kv21 h12", heads=12, mask_kind=1,
                q_start=18, q_frames=3, capacity_frames=21,
                appends=tuple((s, 3) for s in range(0, 21, 3)), kv_stream_first_frame=0, **_WAN),
    4: Workload(4, "wan2.1-1.3b radial 21x30x52 h12 W0=52 g=1/2 l=8", heads=12, mask_kind=2,
                q_start=0, q_frames=21, capacity_frames=21, appends=((0, 21),),
                kv_stream_first_frame=0, **_WAN),
    5: Workload(5, "wan2.1-14b rollout chunk q3@396 kv21 h40 causal+radial", heads=40,
                mask_kind=3, q_start=396, q_frames=3, capacity_frames=21,
                appends=tuple((s, 3) for s in range(378, 399, 3)), kv_stream_first_frame=378,
                **_WAN),
    6: Workload(6, "wan2.1-1.3b radial + dynamic threshold tau=2 21x30x52 h12", heads=12,
                mask_kind=6, q_start=0, q_frames=21, capacity_frames=21, appends=((0, 21),),
                kv_stream_first_frame=0, tau=2.0, **_WAN),
}
