"""The workloads' shapes against the figures the pages print (tests/golden/wan_shapes.txt): the
latent patch grid of an 832 x 480 video, chunks of 3 latent frames, and the 399-latent-frame
long-video benchmark (1593 decoded frames) that puts the last chunk at global frame 396."""
import os

from video_diffusion_transformer_vdit_b200.workloads import WORKLOADS

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "wan_shapes.txt")


def _golden():
    out = {}
    for line in open(GOLDEN):
        line = line.split("#", 1)[0].split()
        if len(line) == 2:
            out[line[0]] = int(line[1])
    return out


def test_latent_grid_of_the_printed_resolution():
    g = _golden()
    for w in WORKLOADS.values():
        if w.grid_h * w.grid_w > 100:  # the Wan2.1-shaped workloads (not the tiny oracle case)
            assert (w.grid_h, w.grid_w) == (g["height"] // 16, g["width"] // 16) == (30, 52)


def test_long_video_benchmark_frames():
    g = _golden()
    n = g["long_video_latent_frames"]
    assert n % g["latent_frames_divisible_by"] == 0
    assert 1 + 4 * (n - 1) == g["long_video_decoded_frames"]
    roll = WORKLOADS[5]
    # the rollout chunk is the last chunk of the 399-frame benchmark: frames 396 .. 398
    assert roll.q_start + roll.q_frames == n and roll.q_frames == g["latent_frames_divisible_by"]
    assert max(s + k for s, k in roll.appends) == n


def test_chunks_are_three_latent_frames_and_clips_decode_from_whole_frames():
    g = _golden()
    c = g["latent_frames_divisible_by"]
    for w in WORKLOADS.values():
        if w.mask_kind & 1:
            assert w.chunk_frames == c
        # every clip or cache window of the Wan2.1-shaped workloads is a whole number of chunks
        if w.grid_h * w.grid_w > 100:
            assert w.capacity_frames % c == 0 and w.q_frames % c == 0
    # the 5 s clip at 16 FPS: 80 frames after the first, 81 decoded frames, 21 latent frames
    assert 1 + 4 * (WORKLOADS[2].q_frames - 1) == 1 + g["clip_seconds"] * g["fps"]
