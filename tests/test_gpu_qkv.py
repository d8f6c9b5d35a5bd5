"""GPU parity of the fused QKV projection + RoPE + cache append (vdit_qkv_rope) against the fp64
oracle (qkv_project, then rope3d for Q and kv_append for K and V) on the same bf16 inputs.

Tolerance, per element of a rotated output y0 = a cos - b sin (likewise y1): the bf16 products
are exact in fp32, and summing d_model of them in fp32 errs by at most gamma * sum_k |x_k w_k|
with gamma = d_model * 2^-24 (Higham's first-order bound for recursive summation, u = 2^-24;
any summation order of the tensor core is covered, since every order's bound is at most that of
the longest chain). The test uses c = max(2^-12, d_model * 2^-24) times S_a + S_b with
S = |x| |w|^T: 2^-12 up to d_model 4096, 3.05e-4 at the Wan2.1-14B width 5120. The final rounding
to bf16 adds half an ulp, at most 2^-8 |y|."""
import numpy as np
import pytest
import torch

import oracle
import synth
import video_diffusion_transformer_vdit_b200 as vdit

from _parity import dev, f64

pytestmark = pytest.mark.gpu


def _inputs(seed, n_tok, d_model, hd):
    x = synth.normal_bf16(seed, n_tok * d_model).reshape(n_tok, d_model)
    w = synth.normal_bf16(seed + 1, 3 * hd * d_model, scale=d_model ** -0.5).reshape(3 * hd, d_model)
    return x, w


def _tolerance(x64, w64, heads, d, ref):
    s = np.abs(x64) @ np.abs(w64).T                      # [n, 3 hd]
    s = s.reshape(s.shape[0], 3, heads, d)
    pair = s[..., 0::2] + s[..., 1::2]
    pair = np.repeat(pair, 2, axis=-1)                   # S_a + S_b for both members of a pair
    c = max(2.0 ** -12, x64.shape[1] * 2.0 ** -24)       # fp32 summation of d_model products
    return 2.0 ** -8 * np.abs(ref) + c * pair + 1e-30


def _run_and_check(gh, gw, heads, d, bands, d_model, start, n_frames, cap, seed, rows=None):
    g = vdit.Geometry(gh, gw, heads, d, bands)
    og = oracle.Geometry(gh, gw, heads, d, *bands, 10000.0)
    ft = gh * gw
    n = n_frames * ft
    hd = heads * d
    xb, wb = _inputs(seed, n, d_model, hd)
    cache = vdit.KVCache(g, cap)
    q = vdit.qkv_rope(dev(xb), dev(wb), g, start, cache.k, cache.v, cap)
    torch.cuda.synchronize()
    assert vdit.get_status() == 0

    x64, w64 = synth.bf16_bits_to_f64(xb), synth.bf16_bits_to_f64(wb)
    sel = np.arange(n) if rows is None else rows
    qr, kr, vr = oracle.qkv_project(x64[sel], w64, heads, d)
    pos = oracle.positions(n, gh, gw, start)
    qrot = oracle.rope3d(qr, tuple(p[sel] for p in pos), og)
    tol = _tolerance(x64[sel], w64, heads, d, np.stack([qrot, qrot, vr], axis=1))
    got_q = f64(q)[sel]
    assert np.all(np.abs(got_q - qrot) <= tol[:, 0])

    # K', V in the ring: the oracle appends the same frames into an fp64 cache
    kc = np.zeros((heads, cap * ft, d))
    vc = np.zeros_like(kc)
    if rows is None:
        oracle.kv_append(kc, vc, cap, og, kr, vr, start, n_frames)
        gk, gv = f64(cache.k), f64(cache.v)
        k_tol = _tolerance(x64, w64, heads, d, np.stack([qrot, kc_rows(kc, start, n_frames, ft, cap), vr], axis=1))
        slots = ring_rows(start, n_frames, ft, cap)
        assert np.all(np.abs(gk[:, slots].transpose(1, 0, 2) - kc[:, slots].transpose(1, 0, 2)) <= k_tol[:, 1])
        assert np.all(np.abs(gv[:, slots].transpose(1, 0, 2) - vc[:, slots].transpose(1, 0, 2)) <= k_tol[:, 2])
        other = np.setdiff1d(np.arange(cap * ft), slots)
        assert not gk[:, other].any() and not gv[:, other].any()  # untouched slots stay zero
    else:
        # sampled rows: the K' / V cache rows of the same tokens
        kf = oracle.rope3d(kr, tuple(p[sel] for p in pos), og)
        slots = ring_rows(start, n_frames, ft, cap)[sel]
        gk, gv = f64(cache.k[:, slots]).transpose(1, 0, 2), f64(cache.v[:, slots]).transpose(1, 0, 2)
        t2 = _tolerance(x64[sel], w64, heads, d, np.stack([qrot, kf, vr], axis=1))
        assert np.all(np.abs(gk - kf) <= t2[:, 1])
        assert np.all(np.abs(gv - vr) <= t2[:, 2])


def ring_rows(start, n_frames, ft, cap):
    """Cache rows of the chunk's tokens, in token order."""
    return np.concatenate([((start + f) % cap) * ft + np.arange(ft) for f in range(n_frames)])


def kc_rows(kc, start, n_frames, ft, cap):
    """The chunk's K' rows of an oracle cache, [tokens, heads, d] in token order."""
    return kc[:, ring_rows(start, n_frames, ft, cap)].transpose(1, 0, 2)


def test_qkv_rope_small_ragged_with_ring_wrap():
    # 96 tokens (a ragged 128-row tile), 3 k steps, frames 8..10 into slots 3, 4, 0 (two launches)
    _run_and_check(gh=4, gw=8, heads=2, d=128, bands=(44, 42, 42), d_model=192, start=8,
                   n_frames=3, cap=5, seed=501)


def test_qkv_rope_head_dim_64_many_tiles():
    # head_dim 64 (bands 24/20/20), 4 heads: 256 columns per section; 7 frames of 5 x 9 tokens
    _run_and_check(gh=5, gw=9, heads=4, d=64, bands=(24, 20, 20), d_model=136, start=3,
                   n_frames=7, cap=9, seed=502)


def test_qkv_rope_wan13b_causal_chunk_sampled():
    # Wan2.1-1.3B-shaped chunk: 3 frames x 30 x 52 tokens at frame 18 of a 21-frame ring,
    # d_model 1536 -> 3 x 12 x 128; checked on sampled rows (first / last tiles and 300 random)
    rng = np.random.default_rng(5)
    n = 3 * 1560
    rows = np.unique(np.r_[np.arange(128), np.arange(n - 130, n), rng.integers(0, n, 300)])
    _run_and_check(gh=30, gw=52, heads=12, d=128, bands=(44, 42, 42), d_model=1536, start=18,
                   n_frames=3, cap=21, seed=503, rows=rows)


def test_qkv_rope_wan14b_rollout_chunk_sampled():
    # Wan2.1-14B-shaped rollout chunk: 3 frames x 30 x 52 tokens at global frame 396 of a
    # 21-frame ring (slots 18..20), d_model 5120 -> 3 x 40 x 128 (the shape the benchmark times);
    # sampled rows: first and last tiles and 200 random
    rng = np.random.default_rng(14)
    n = 3 * 1560
    rows = np.unique(np.r_[np.arange(128), np.arange(n - 130, n), rng.integers(0, n, 200)])
    _run_and_check(gh=30, gw=52, heads=40, d=128, bands=(44, 42, 42), d_model=5120, start=396,
                   n_frames=3, cap=21, seed=504, rows=rows)


def test_qkv_rope_rejects_bad_shapes():
    g = vdit.Geometry(4, 8, 1, 128, (44, 42, 42))  # heads * head_dim = 128: not a multiple of 256
    cache = vdit.KVCache(g, 3)
    x = torch.zeros(32, 64, dtype=torch.bfloat16, device="cuda")
    w = torch.zeros(3 * 128, 64, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(vdit.VditError):
        vdit.qkv_rope(x, w, g, 0, cache.k, cache.v, 3)
