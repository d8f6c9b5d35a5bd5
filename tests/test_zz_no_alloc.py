"""The attention entry point that allocates nothing (vdit_attn_forward_noalloc), called through
the C ABI and checked against vdit_attn_forward on the same inputs (bit-identical: the same
kernels run on the same plan) and against the fp64 oracle.

It exists for callers that cannot allocate device memory when they run attention (another
framework owns the GPU's memory through its own pool, or a latency-critical loop must not enter
the allocator): the partial results of the key pieces of its cut units go to a fixed device buffer
inside the library instead of the workspace the plan allocates. This file is collected last so that a run that
stops at the first failure has already run every other test; it also passes on its own in a
fresh process (it builds everything it needs, including the RoPE tables, before the call).
"""
import ctypes

import numpy as np
import pytest
import torch

import synth
import video_diffusion_transformer_vdit_b200 as vdit
from video_diffusion_transformer_vdit_b200.workloads import WORKLOADS, Workload

from _parity import MAX_ABS, REL_RMS, assert_close, dev, f64, geom, inputs, mask, run_oracle

pytestmark = pytest.mark.gpu


def _setup(w):
    q, k, v = inputs(w)
    g = geom(w)
    cache = vdit.KVCache(g, w.capacity_frames)  # vdit_kv_append builds the RoPE tables
    kd, vd = dev(k), dev(v)
    ft = w.frame_tokens
    for s, n in w.appends:
        off = (s - w.kv_stream_first_frame) * ft
        cache.append(kd[off:off + n * ft], vd[off:off + n * ft], s)
    plan = vdit.Plan(g, mask(w), w.q_start, w.q_frames, cache=cache)
    return dev(q), cache, plan


def _call(fn, plan, q, cache, w):
    o = torch.full_like(q, float("nan"))
    lse = torch.full((w.heads, w.q_tokens), float("nan"), device="cuda")
    rc = fn(plan._h, ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(cache.k.data_ptr()),
            ctypes.c_void_p(cache.v.data_ptr()), ctypes.c_void_p(o.data_ptr()),
            ctypes.c_void_p(lse.data_ptr()), ctypes.c_float(w.scale),
            ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    torch.cuda.synchronize()
    return rc, o, lse


def test_noalloc_forward_matches_forward_twice_in_a_row():
    # one head of the causal-chunk shape: 19 query blocks x 1 head leave most SMs idle, so the
    # schedule cuts every unit into key pieces and the scratch path is the one exercised
    base = WORKLOADS[3]
    w = Workload(**{**base.__dict__, "id": 95, "heads": 1})
    q, cache, plan = _setup(w)
    info = plan.info
    assert info["kv_splits"] > 1 and info["cut_units"] == 19
    assert 0 < info["workspace_bytes"] <= 32 << 20
    L = vdit.lib()
    rc, o_ref, lse_ref = _call(L.vdit_attn_forward, plan, q, cache, w)
    assert rc == vdit.OK
    # another query between the two calls leaves different partial results in the shared buffer,
    # so a call that read stale entries instead of its own would not match
    q_other = dev(synth.qkv_bf16(96, w.q_tokens, w.heads, w.head_dim, "q"))
    for i in range(2):
        rc, o, lse = _call(L.vdit_attn_forward_noalloc, plan, q, cache, w)
        assert rc == vdit.OK, L.vdit_last_error()
        # the same kernels on the same inputs and plan: bit-identical to vdit_attn_forward
        assert torch.equal(o, o_ref) and torch.equal(lse, lse_ref)
        if i == 0:
            rc, o_x, _ = _call(L.vdit_attn_forward_noalloc, plan, q_other, cache, w)
            assert rc == vdit.OK and not torch.equal(o_x, o_ref)
    assert vdit.get_status() == vdit.OK
    # and against the fp64 oracle on sampled rows (first tile, random rows, the ragged last tile)
    qb, kb, vb = inputs(w)
    rng = np.random.default_rng(95)
    rows = np.unique(np.r_[np.arange(0, 64), rng.integers(0, w.q_tokens, 96),
                           np.arange((w.q_tokens - 1) // 128 * 128, w.q_tokens)])
    ro, rl = run_oracle(w, qb, kb, vb, rows, [0])
    assert_close(f64(o[rows]), ro, max_abs=MAX_ABS, rel_rms=REL_RMS)
    assert np.max(np.abs(lse[0][rows].cpu().numpy() - rl[0])) < 2e-2


def test_noalloc_forward_runs_the_full_causal_chunk():
    # all 12 heads of the causal-chunk shape: the schedule cuts units into key pieces, and their
    # partial slots stay within the fixed buffer, so the call runs and matches vdit_attn_forward
    w = WORKLOADS[3]
    q, cache, plan = _setup(w)
    info = plan.info
    assert 0 < info["workspace_bytes"] <= 32 << 20
    L = vdit.lib()
    rc, o_ref, lse_ref = _call(L.vdit_attn_forward, plan, q, cache, w)
    assert rc == vdit.OK
    rc, o, lse = _call(L.vdit_attn_forward_noalloc, plan, q, cache, w)
    assert rc == vdit.OK, L.vdit_last_error()
    assert torch.equal(o, o_ref) and torch.equal(lse, lse_ref)
    assert vdit.get_status() == vdit.OK
