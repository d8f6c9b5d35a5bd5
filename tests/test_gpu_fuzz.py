"""Seeded random geometries and masks through the whole attention path (append, plan, forward)
against the oracle: grids from 1 x 1 to 9 x 40, 1-3 heads, head_dim 64 or 128, every mask kind
(with and without the dynamic threshold), ring windows with wrap-around and empty slots."""
import dataclasses

import numpy as np
import pytest

from video_diffusion_transformer_vdit_b200.workloads import Workload

import test_gpu_parity as P

pytestmark = pytest.mark.gpu


def _random_workload(seed):
    rng = np.random.default_rng(1000 + seed)
    gh, gw = int(rng.integers(1, 10)), int(rng.integers(1, 41))
    d = int(rng.choice([64, 128]))
    bands = (24, 20, 20) if d == 64 else (44, 42, 42)
    cap = int(rng.integers(1, 10))
    chunk = int(rng.integers(1, min(3, cap) + 1))
    n_chunks = int(rng.integers(1, 6))
    first_stream = int(rng.integers(0, 30))
    appends = tuple((first_stream + i * chunk, chunk) for i in range(n_chunks))
    last = appends[-1][0] + chunk - 1
    first = max(first_stream, last - cap + 1)
    q_frames = int(rng.integers(1, min(4, last - first + 1) + 1))
    q_start = int(rng.integers(first, last - q_frames + 2))  # query frames inside the window
    kind = int(rng.integers(0, 8))
    if kind & 4 and seed % 2:
        kind &= 3  # keep half of the cases static
    return Workload(200 + seed, f"fuzz{seed}", grid_h=gh, grid_w=gw, heads=int(rng.integers(1, 4)),
                    head_dim=d, bands=bands, mask_kind=kind, q_start=q_start, q_frames=q_frames,
                    capacity_frames=cap, appends=appends, kv_stream_first_frame=first_stream,
                    chunk_frames=chunk, w0=int(rng.integers(1, 30)), gamma_shift=int(rng.integers(0, 3)),
                    lam=int(rng.integers(0, 6)), tau=float(rng.choice([0.5, 1.5, 3.0])))


@pytest.mark.parametrize("seed", range(16))
def test_attention_random_geometry(seed):
    w = _random_workload(seed)
    if w.q_tokens * w.kv_tokens > 4_000_000:
        w = dataclasses.replace(w, grid_w=max(1, w.grid_w // 4))
    if w.mask_kind & 4:
        P._dynamic_check(w)
    else:
        P._full_check(w)
