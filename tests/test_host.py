"""Host logic of the Python binding that needs no GPU: the KV cache's window bookkeeping (which
global frames the ring holds after a sequence of appends) against the workloads' own window
rule and a brute-force replay of the ring, and the rejection of appends that would leave a gap
or rewrite a frame older than the window."""
import numpy as np
import pytest

import video_diffusion_transformer_vdit_b200 as vdit
from video_diffusion_transformer_vdit_b200.workloads import WORKLOADS, Workload


def _replay(cap, appends):
    """Brute force: the global frame each ring slot holds after the appends (-1: never written)."""
    slot = [-1] * cap
    for s, n in appends:
        for f in range(s, s + n):
            slot[f % cap] = f
    return slot


def _window(cap, appends):
    cache = vdit.KVCache(vdit.Geometry(2, 3, 1, 64, (24, 20, 20)), cap, device="cpu")
    for s, n in appends:
        cache._check_next(s)
        cache._note(s, n)
    return cache.first_frame, cache.last_frame


@pytest.mark.parametrize("wid", sorted(WORKLOADS))
def test_cache_window_of_the_workloads(wid):
    w = WORKLOADS[wid]
    assert _window(w.capacity_frames, w.appends) == w.window()


def test_cache_window_matches_a_replay_of_the_ring():
    rng = np.random.default_rng(21)
    for _ in range(200):
        cap = int(rng.integers(1, 12))
        start = int(rng.integers(0, 50))
        appends, f = [], start
        for _ in range(int(rng.integers(1, 8))):
            n = int(rng.integers(1, cap + 1))
            back = int(rng.integers(0, 2)) * int(rng.integers(0, n))  # sometimes re-append recent frames
            s = max(start, f - back)
            if appends:
                first, _ = _window(cap, appends)
                s = max(s, first)
            appends.append((s, n))
            f = max(f, s + n)
        first, last = _window(cap, appends)
        held = _replay(cap, appends)
        # the window is exactly the frames the ring holds, and they are contiguous
        assert sorted(x for x in held if x >= 0) == list(range(first, last + 1))
        w = Workload(0, "replay", 2, 3, 1, 64, (24, 20, 20), 0, first, 1, cap, tuple(appends), start)
        assert w.window() == (first, last)


def test_cache_rejects_gaps_and_frames_older_than_the_window():
    cache = vdit.KVCache(vdit.Geometry(2, 3, 1, 64, (24, 20, 20)), 4, device="cpu")
    cache._note(0, 3)
    cache._note(3, 3)                       # holds 2 .. 5
    assert (cache.first_frame, cache.last_frame) == (2, 5)
    with pytest.raises(ValueError, match="gap"):
        cache._check_next(7)
    with pytest.raises(ValueError, match="older"):
        cache._check_next(1)
    cache._check_next(6)                    # the next frame
    cache._check_next(2)                    # rewriting a held frame is allowed
