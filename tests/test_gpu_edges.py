"""Edge cases of the GPU path against the oracle: degenerate grids and masks, positions at the
table limits, empty calls. Same tolerances as the parity tests (max-abs 2e-2, relative RMS 1e-2
for attention; the bf16 rounding bound for RoPE)."""
import numpy as np
import pytest
import torch

import oracle
import synth
import video_diffusion_transformer_vdit_b200 as vdit
from video_diffusion_transformer_vdit_b200.workloads import Workload

from _parity import assert_close, dev, f64, inputs, ogeom, rope_tolerance, run_oracle, run_product

pytestmark = pytest.mark.gpu

D64 = dict(head_dim=64, bands=(24, 20, 20))


def _full(w):
    q, k, v = inputs(w)
    o, lse, _, plan = run_product(w, q, k, v)
    ro, rl = run_oracle(w, q, k, v, np.arange(w.q_tokens), range(w.heads))
    assert_close(f64(o), ro)
    l = lse.cpu().numpy()
    fin = np.isfinite(rl)
    assert np.abs(l[fin] - rl[fin]).max() < 2e-2 and np.isneginf(l[~fin]).all()
    assert vdit.get_status() == vdit.OK
    return plan


EDGES = {
    # one patch per frame: 128-key tiles span 128 frames of the ring
    "grid_1x1_causal_radial": Workload(71, "1x1", grid_h=1, grid_w=1, heads=2, mask_kind=3,
                                       q_start=150, q_frames=20, capacity_frames=160,
                                       appends=((0, 100), (100, 70)), kv_stream_first_frame=0,
                                       w0=0, lam=5, **D64),
    # lambda = 1: every frame is a long-range frame, so the radial mask is dense
    "lambda_1": Workload(72, "lam1", grid_h=5, grid_w=7, heads=2, mask_kind=2, q_start=0,
                         q_frames=6, capacity_frames=6, appends=((0, 6),), kv_stream_first_frame=0,
                         w0=1, lam=1, **D64),
    # w0 = 0 and no long-range frames: each query keeps only its own patch in every frame
    "w0_0_diagonal": Workload(73, "w0", grid_h=6, grid_w=10, heads=2, mask_kind=2, q_start=0,
                              q_frames=5, capacity_frames=5, appends=((0, 5),),
                              kv_stream_first_frame=0, w0=0, lam=0, **D64),
    # chunks of one frame: frame-causal
    "chunk_1": Workload(74, "c1", grid_h=4, grid_w=9, heads=2, mask_kind=1, q_start=4, q_frames=3,
                        capacity_frames=7, appends=((0, 4), (4, 3)), kv_stream_first_frame=0,
                        chunk_frames=1, **D64),
    # positions at the end of the time table (frames 16379 .. 16383)
    "max_frame": Workload(75, "tmax", grid_h=3, grid_w=4, heads=2, mask_kind=1, q_start=16381,
                          q_frames=3, capacity_frames=5, appends=((16379, 2), (16381, 3)),
                          kv_stream_first_frame=16379, head_dim=128, bands=(44, 42, 42)),
    # a 2 x 1024 grid: w positions up to the end of the spatial table
    "wide_grid": Workload(76, "wide", grid_h=2, grid_w=1024, heads=1, mask_kind=2, q_start=0,
                          q_frames=2, capacity_frames=2, appends=((0, 2),),
                          kv_stream_first_frame=0, w0=300, lam=0, **D64),
}


@pytest.mark.parametrize("name", sorted(EDGES))
def test_attention_edge_cases(name):
    _full(EDGES[name])


def test_lambda_1_radial_plan_is_dense():
    w = EDGES["lambda_1"]
    plan = _full(w)
    assert plan.info["kept_pairs"] == w.q_tokens * w.kv_tokens


def test_rope_at_the_last_frame_and_grid_corner():
    g = vdit.Geometry(2, 1024, 2, 64, (24, 20, 20))
    n = 2 * 2048
    bits = synth.qkv_bf16(77, n, 2, 64, "q")
    y = vdit.rope3d_apply(dev(bits), g, 16382)
    torch.cuda.synchronize()
    pos = oracle.positions(n, 2, 1024, 16382)
    og = oracle.Geometry(2, 1024, 2, 64, 24, 20, 20, 10000.0)
    x64 = synth.bf16_bits_to_f64(bits)
    ref = oracle.rope3d(x64, pos, og)
    assert np.all(np.abs(f64(y) - ref) <= rope_tolerance(ref, x64))


def test_empty_calls_are_no_ops():
    g = vdit.Geometry(3, 4, 2, 64, (24, 20, 20))
    x = torch.empty(0, 2, 64, dtype=torch.bfloat16, device="cuda")
    y = vdit.rope3d_apply(x, g, 0)
    assert y.shape == (0, 2, 64)
    send = torch.empty(2, 3, 0, 1, 64, dtype=torch.bfloat16, device="cuda")
    full = tuple(torch.empty(0, 1, 64, dtype=torch.bfloat16, device="cuda") for _ in range(3))
    vdit.seq_pack(x, x, x, g, 0, 1, 2, send, full)
    out = torch.empty(0, 2, 64, dtype=torch.bfloat16, device="cuda")
    vdit.seq_unpack(torch.empty(2, 0, 1, 64, dtype=torch.bfloat16, device="cuda"), full[0], out, g, 1, 2)
    torch.cuda.synchronize()
    assert vdit.get_status() == vdit.OK


def test_frames_past_the_table_are_rejected():
    g = vdit.Geometry(3, 4, 2, 64, (24, 20, 20))
    x = torch.zeros(2 * 12, 2, 64, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(vdit.VditError):
        vdit.rope3d_apply(x, g, 16383)  # its second frame would be 16384
