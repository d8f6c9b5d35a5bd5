"""Shared helpers of the GPU parity tests: seeded inputs, the product run through the C ABI,
the oracle run on the same bf16 values, and the tolerance checks."""
from __future__ import annotations

import math

import numpy as np
import torch

import oracle
import synth
import video_diffusion_transformer_vdit_b200 as vdit

# spec tolerances: bf16 in, fp32 accumulate
MAX_ABS = 2e-2
REL_RMS = 1e-2


def dev(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def geom(w):
    return vdit.Geometry(w.grid_h, w.grid_w, w.heads, w.head_dim, w.bands, w.theta)


def ogeom(w, heads=None):
    return oracle.Geometry(w.grid_h, w.grid_w, heads or w.heads, w.head_dim, *w.bands, w.theta)


def mask(w):
    return vdit.Mask(w.mask_kind, w.chunk_frames, w.w0, w.gamma_shift, w.lam, w.tau)


def omask(w):
    return oracle.Mask(block_causal=bool(w.mask_kind & 1), radial=bool(w.mask_kind & 2),
                       chunk_frames=w.chunk_frames, w0=w.w0, gamma_shift=w.gamma_shift, lam=w.lam)


def inputs(w, q_scale: float = 1.0):
    """uint16 bf16 bits: q [q_tokens, H, D], k and v streams [stream tokens, H, D]."""
    n_kv = w.kv_stream_frames * w.frame_tokens
    q = synth.qkv_bf16(w.id, w.q_tokens, w.heads, w.head_dim, "q", scale=q_scale)
    k = synth.qkv_bf16(w.id, n_kv, w.heads, w.head_dim, "k")
    v = synth.qkv_bf16(w.id, n_kv, w.heads, w.head_dim, "v")
    return q, k, v


def run_product(w, q, k, v, lse: bool = True):
    g = geom(w)
    cache = vdit.KVCache(g, w.capacity_frames)
    kd, vd = dev(k), dev(v)
    ft = w.frame_tokens
    for s, n in w.appends:
        off = (s - w.kv_stream_first_frame) * ft
        cache.append(kd[off:off + n * ft], vd[off:off + n * ft], s)
    plan = vdit.Plan(g, mask(w), w.q_start, w.q_frames, cache=cache)
    qd = dev(q)
    l = torch.full((w.heads, w.q_tokens), float("nan"), device="cuda") if lse else None
    o = vdit.attn_forward(plan, qd, cache, lse=l, scale=w.scale)
    torch.cuda.synchronize()
    return o, l, cache, plan


def run_oracle(w, q, k, v, rows, heads):
    """Oracle o [len(rows), len(heads), D] and lse [len(heads), len(rows)] for the given query
    rows and heads (the method is independent per head, so a head subset is exact)."""
    hs = list(heads)
    og = ogeom(w, len(hs))
    ft = w.frame_tokens
    kc = np.zeros((len(hs), w.kv_tokens, w.head_dim))
    vc = np.zeros_like(kc)
    k64 = synth.bf16_bits_to_f64(k[:, hs])
    v64 = synth.bf16_bits_to_f64(v[:, hs])
    for s, n in w.appends:
        off = (s - w.kv_stream_first_frame) * ft
        oracle.kv_append(kc, vc, w.capacity_frames, og, k64[off:off + n * ft], v64[off:off + n * ft], s, n)
    first, last = w.window()
    kpos, kvalid = oracle.cache_positions(w.capacity_frames, first, last, w.grid_h, w.grid_w)
    qpos_all = oracle.positions(w.q_tokens, w.grid_h, w.grid_w, w.q_start)
    qpos = tuple(p[rows] for p in qpos_all)
    qrot = oracle.rope3d(synth.bf16_bits_to_f64(q[rows][:, hs]), qpos, og)
    m = oracle.mask_rows(qpos, kpos, kvalid, omask(w))
    if w.mask_kind & 4:  # dynamic threshold over the candidates of the static bits
        o, lse, _ = oracle.attention_dynamic(qrot, kc.transpose(1, 0, 2), vc.transpose(1, 0, 2), m,
                                             w.scale, w.tau)
        return o, lse
    return oracle.attention(qrot, kc.transpose(1, 0, 2), vc.transpose(1, 0, 2), m, w.scale)


def assert_close(got: np.ndarray, ref: np.ndarray, max_abs=MAX_ABS, rel_rms=REL_RMS):
    err = got - ref
    ma = float(np.max(np.abs(err)))
    rr = float(math.sqrt(np.mean(err ** 2)) / max(1e-30, math.sqrt(np.mean(ref ** 2))))
    assert ma <= max_abs and rr <= rel_rms, f"max_abs {ma:.3e} (<= {max_abs}), rel_rms {rr:.3e} (<= {rel_rms})"
    return ma, rr


def rope_tolerance(ref: np.ndarray, x: np.ndarray) -> np.ndarray:
    """Per-element bound for fp32 rotation rounded to bf16: half an ulp of bf16 relative to the
    value (2^-8 |y|) plus the fp32 table and FMA error (a few 2^-24 of the pair magnitude)."""
    pair = np.abs(x[..., 0::2]) + np.abs(x[..., 1::2])
    pair = np.repeat(pair, 2, axis=-1)
    return 2.0 ** -8 * np.abs(ref) + 2.0 ** -20 * pair + 1e-30
