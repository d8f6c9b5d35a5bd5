"""GPU parity: libvdit's CUDA kernels (through the C ABI) against the fp64 oracle on the same
seeded bf16 inputs. Bit-exact where the operation is a copy or an integer decision (V in the
cache, the tile schedule); within the bf16 rounding bound for RoPE; max-abs 2e-2 and relative RMS
1e-2 for attention (bf16 inputs, fp32 accumulation)."""
import numpy as np
import pytest
import torch

import oracle
import synth
import video_diffusion_transformer_vdit_b200 as vdit
from video_diffusion_transformer_vdit_b200.workloads import WORKLOADS, Workload

from _parity import (assert_close, dev, f64, geom, inputs, mask, ogeom, omask, rope_tolerance,
                     run_oracle, run_product)

pytestmark = pytest.mark.gpu


# ----------------------------------------------------------------------------- RoPE

@pytest.mark.parametrize("wid,start", [(1, 0), (1, 3), (2, 0), (5, 396)])
def test_rope3d_apply_parity(wid, start):
    w = WORKLOADS[wid]
    n = w.q_tokens if wid != 2 else 3 * w.frame_tokens + 77  # ragged token count
    bits = synth.qkv_bf16(w.id, n, w.heads, w.head_dim, "q")
    x = dev(bits)
    y = vdit.rope3d_apply(x, geom(w), start)
    torch.cuda.synchronize()
    rng = np.random.default_rng(wid)
    rows = np.unique(np.r_[rng.integers(0, n, 1500), np.arange(n - 40, n), np.arange(0, 40)])
    pos = oracle.positions(n, w.grid_h, w.grid_w, start)
    x64 = synth.bf16_bits_to_f64(bits[rows])
    ref = oracle.rope3d(x64, tuple(p[rows] for p in pos), ogeom(w))
    got = f64(y)[rows]
    assert np.all(np.abs(got - ref) <= rope_tolerance(ref, x64))


def test_rope3d_apply_in_place_matches_out_of_place():
    w = WORKLOADS[1]
    bits = synth.qkv_bf16(9, 5 * w.frame_tokens + 3, w.heads, w.head_dim, "k")
    a = vdit.rope3d_apply(dev(bits), geom(w), 7)
    x = dev(bits)
    vdit.rope3d_apply(x, geom(w), 7, out=x)
    torch.cuda.synchronize()
    assert torch.equal(a, x)


# ----------------------------------------------------------------------------- KV append

def test_kv_append_ring_parity_small():
    w = Workload(90, "ring", grid_h=3, grid_w=5, heads=3, head_dim=128, bands=(44, 42, 42),
                 mask_kind=0, q_start=12, q_frames=3, capacity_frames=7,
                 appends=tuple((s, 3) for s in range(0, 15, 3)), kv_stream_first_frame=0)
    _, k, v = inputs(w)
    _, _, cache, _ = run_product(w, synth.qkv_bf16(90, w.q_tokens, 3, 128, "q"), k, v, lse=False)
    og = ogeom(w)
    kc = np.zeros((3, w.kv_tokens, 128))
    vc = np.zeros_like(kc)
    ft = w.frame_tokens
    for s, n in w.appends:
        oracle.kv_append(kc, vc, 7, og, synth.bf16_bits_to_f64(k[s * ft:(s + n) * ft]),
                         synth.bf16_bits_to_f64(v[s * ft:(s + n) * ft]), s, n)
    assert np.array_equal(f64(cache.v), vc)  # V is a bit-exact copy
    kx = np.zeros_like(kc)
    for f in range(8, 15):  # unrotated source of each held frame, for the bound
        slot = f % 7
        kx[:, slot * ft:(slot + 1) * ft] = synth.bf16_bits_to_f64(k[f * ft:(f + 1) * ft]).transpose(1, 0, 2)
    got = f64(cache.k)
    assert np.all(np.abs(got - kc) <= rope_tolerance(kc, kx))
    assert (cache.first_frame, cache.last_frame) == (8, 14)


def test_kv_append_parity_long_rollout_sampled():
    w = WORKLOADS[5]
    q, k, v = inputs(w)
    _, _, cache, _ = run_product(w, q, k, v, lse=False)
    hs = [0, 17, 39]
    og = ogeom(w, len(hs))
    ft = w.frame_tokens
    kc = np.zeros((3, w.kv_tokens, 128))
    vc = np.zeros_like(kc)
    for s, n in w.appends:
        off = (s - 378) * ft
        oracle.kv_append(kc, vc, 21, og, synth.bf16_bits_to_f64(k[off:off + n * ft][:, hs]),
                         synth.bf16_bits_to_f64(v[off:off + n * ft][:, hs]), s, n)
    rng = np.random.default_rng(3)
    toks = np.unique(np.r_[rng.integers(0, w.kv_tokens, 3000), np.arange(w.kv_tokens - 60, w.kv_tokens)])
    gk = f64(cache.k[hs][:, toks])
    gv = f64(cache.v[hs][:, toks])
    assert np.array_equal(gv, vc[:, toks])
    # unrotated source values for the bound: slot s holds frame 378 + s here (378 = 18 * 21)
    src = synth.bf16_bits_to_f64(k[toks][:, hs]).transpose(1, 0, 2)
    assert np.all(np.abs(gk - kc[:, toks]) <= rope_tolerance(kc[:, toks], src))


# ----------------------------------------------------------------------------- attention

def _full_check(w, q_scale=1.0):
    q, k, v = inputs(w, q_scale)
    o, lse, _, _ = run_product(w, q, k, v)
    rows = np.arange(w.q_tokens)
    ro, rl = run_oracle(w, q, k, v, rows, range(w.heads))
    assert_close(f64(o), ro)
    assert np.max(np.abs(lse.cpu().numpy() - rl)) < 2e-2
    assert vdit.get_status() == vdit.OK


def test_attention_tiny_workload_full():
    _full_check(WORKLOADS[1])


def _medium(kind, q_start, q_frames, cap, appends, first_stream=0, d=128, wid=91, heads=2):
    return Workload(wid, "medium", grid_h=6, grid_w=10, heads=heads, head_dim=d,
                    bands=(44, 42, 42) if d == 128 else (24, 20, 20), mask_kind=kind,
                    q_start=q_start, q_frames=q_frames, capacity_frames=cap, appends=appends,
                    kv_stream_first_frame=first_stream, chunk_frames=3, w0=4, gamma_shift=1, lam=4)


MEDIUM = {
    # 9 frames x 60 tokens = 540 = 4 x 128 + 28: several tiles and a ragged tail
    "dense": _medium(0, 0, 9, 9, ((0, 9),)),
    "causal": _medium(1, 3, 6, 9, ((0, 3), (3, 3), (6, 3))),
    "radial_ring_wrap": _medium(2, 9, 3, 8, tuple((s, 3) for s in range(0, 12, 3)) + ((12, 1),)),
    "causal_radial": _medium(3, 6, 3, 9, tuple((s, 3) for s in range(0, 9, 3))),
    "partial_fill": _medium(1, 3, 3, 12, ((0, 3), (3, 3))),
    "d64_radial": _medium(2, 0, 7, 7, ((0, 7),), d=64, wid=92, heads=3),
    # 3-wide grid: a 128-key tile spans more than 32 row segments, so partial tiles take the
    # per-key predicate path instead of the per-segment intervals
    "narrow_grid_causal_radial": Workload(94, "narrow", grid_h=7, grid_w=3, heads=2, head_dim=128,
                                          bands=(44, 42, 42), mask_kind=3, q_start=9, q_frames=6,
                                          capacity_frames=16,
                                          appends=tuple((s, 3) for s in range(0, 15, 3)),
                                          kv_stream_first_frame=0, chunk_frames=3, w0=4,
                                          gamma_shift=1, lam=4),
}


@pytest.mark.parametrize("name", sorted(MEDIUM))
def test_attention_medium_full(name):
    _full_check(MEDIUM[name])


def _single_patch(kind, q_start, q_frames, cap, appends, tau=0.0):
    # 8 x 20 = 160 tokens per frame (tiles straddle frames), radius 4 >> dt: 0 from 3 frames
    # apart (lambda 0: no long-range frames), so the plan moves those frames' same-patch pairs
    # into single-patch entries at unaligned key rows
    return Workload(96, "single-patch", grid_h=8, grid_w=20, heads=2, head_dim=128,
                    bands=(44, 42, 42), mask_kind=kind, q_start=q_start, q_frames=q_frames,
                    capacity_frames=cap, appends=appends, kv_stream_first_frame=0, chunk_frames=3,
                    w0=4, gamma_shift=1, lam=0, tau=tau)


SINGLE_PATCH = {
    "radial": _single_patch(2, 0, 9, 9, ((0, 9),)),
    # a ring of 10 holding frames 2..11 (slots 2..9, 0, 1): the queries' single-patch key frames
    # 3..8 sit in consecutive slots
    "causal_radial_ring": _single_patch(3, 9, 3, 10, tuple((s, 3) for s in range(0, 12, 3))),
    "radial_odd_start": _single_patch(2, 2, 5, 8, ((0, 8),)),
}


@pytest.mark.parametrize("name", sorted(SINGLE_PATCH))
def test_attention_single_patch_entries_full(name):
    w = SINGLE_PATCH[name]
    first, last = w.window()
    plan = vdit.Plan(geom(w), mask(w), w.q_start, w.q_frames, capacity_frames=w.capacity_frames,
                     kv_first_frame=first, kv_last_frame=last, upload=False)
    assert plan.info["single_patch_entries"] > 0
    _full_check(w)


def test_attention_single_patch_entries_dynamic_threshold():
    import dataclasses
    w = dataclasses.replace(SINGLE_PATCH["radial"], mask_kind=6, tau=1.5)
    _dynamic_check(w)


@pytest.mark.parametrize("name", ["causal_radial", "dense"])
def test_attention_sharp_softmax(name):
    # Q scaled by 4: logits of standard deviation ~4 and a peaked softmax (|o| ~ 1), where the
    # relative-RMS bound is the binding one. The kernel multiplies bf16 operands, so the rotated
    # q and k carry a relative rounding of up to 2^-9 per element; on 128-term dot products with
    # |q_i k_i| * scale ~ 0.35 that moves a logit by ~0.015 typically (a few times that at the
    # tail), i.e. a softmax weight by a few percent, so single outputs near 1 can move by several
    # 1e-2. Observed on B200 for these inputs: max-abs 0.044 (causal_radial) and 0.026 (dense),
    # relative RMS 5.1e-3 and 4.9e-3, lse 0.022 and 0.025. Bounds: max-abs 0.09 and lse 0.05 (about
    # twice the larger observation), relative RMS 1e-2 unchanged.
    w = MEDIUM[name]
    q, k, v = inputs(w, 4.0)
    o, lse, _, _ = run_product(w, q, k, v)
    ro, rl = run_oracle(w, q, k, v, np.arange(w.q_tokens), range(w.heads))
    assert_close(f64(o), ro, max_abs=0.09, rel_rms=1e-2)
    assert np.max(np.abs(lse.cpu().numpy() - rl)) < 5e-2


@pytest.mark.parametrize("wid", [2, 3, 4, 5])
def test_attention_full_size_sampled(wid):
    w = WORKLOADS[wid]
    q, k, v = inputs(w)
    o, lse, _, plan = run_product(w, q, k, v)
    rng = np.random.default_rng(wid)
    last_tile = np.arange((w.q_tokens - 1) // 128 * 128, w.q_tokens)
    rows = np.unique(np.r_[np.arange(0, 64), rng.integers(0, w.q_tokens, 96), last_tile])
    hs = [0, w.heads // 2, w.heads - 1]
    # the sample includes rows of units that the CTA schedule cut into key pieces, where it cuts
    cta, merge = plan.schedule_for(torch.cuda.get_device_properties(0).multi_processor_count)
    assert plan.info["ctas"] == len(cta) and plan.info["cut_units"] == len(merge)
    cut = {(hd, r) for qb, hd, _, _ in merge.tolist() for r in range(qb * 256, min(qb * 256 + 256, w.q_tokens))}
    assert not cut or any((hd, int(r)) in cut for hd in hs for r in rows)
    ro, rl = run_oracle(w, q, k, v, rows, hs)
    assert_close(f64(o[rows][:, hs]), ro)
    assert np.max(np.abs(lse[hs][:, rows].cpu().numpy() - rl)) < 2e-2
    # every output row is finite and the kernel reported no timeout
    assert torch.isfinite(o).all()
    assert vdit.get_status() == vdit.OK


def test_attention_is_deterministic():
    w = MEDIUM["causal_radial"]
    q, k, v = inputs(w)
    o1, l1, cache, plan = run_product(w, q, k, v)
    o2 = vdit.attn_forward(plan, dev(q), cache, scale=w.scale)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2)


@pytest.mark.parametrize("q_start,q_frames", [(2, 2), (0, 1)])
def test_attention_rows_without_keys(q_start, q_frames):
    # block-causal, cache holds only frame 3 (chunk 1): query frames of chunk 0 see no key
    # (o = 0, lse = -inf); with q_start=0, q_frames=1 the plan lists no tile at all
    w = _medium(1, q_start, q_frames, 4, ((3, 1),), first_stream=3, wid=93)
    q, k, v = inputs(w)
    o, lse, _, plan = run_product(w, q, k, v)
    ro, rl = run_oracle(w, q, k, v, np.arange(w.q_tokens), range(w.heads))
    assert_close(f64(o), ro)
    gl = lse.cpu().numpy()
    assert np.array_equal(np.isinf(gl), np.isinf(rl))
    fin = np.isfinite(rl)
    assert np.max(np.abs(gl[fin] - rl[fin]), initial=0.0) < 2e-2
    if q_frames == 1:
        assert plan.info["tiles"] == 0 and not o.float().abs().sum().item()


# ----------------------------------------------------------------------------- dynamic threshold

def _rounding_slack(x, pair_mag):
    """Per element of the oracle's fp64 rotated values x: the amount (one bf16 spacing, or 0) by
    which the kernel's bf16 operand may differ from round_bf16(x). The kernel rotates in fp32 with
    fp32 (cos, sin) from fp64 tables, within 2^-22 (|x0| + |x1|) of the fp64 rotation, so it may
    round to the other neighbour only when x lies that close to a rounding midpoint (2^-21 taken)."""
    b = oracle.round_bf16(x)
    _, e = np.frexp(np.where(b == 0, 1.0, b))
    ulp = np.ldexp(1.0, e - 8)                   # bf16 spacing at b: 8 significant bits
    near = np.abs(np.abs(x - b) - ulp / 2) <= 2.0 ** -21 * pair_mag
    return np.where(near & (x != 0), ulp, 0.0)


def _pair_mag(x_unrot):
    m = np.abs(x_unrot[..., 0::2]) + np.abs(x_unrot[..., 1::2])
    return np.repeat(m, 2, axis=-1)


def _dynamic_check(w, rows=None, heads=None, q_scale=1.0):
    """Dynamic-threshold parity. The keep decision (logit within tau of the row maximum) is an
    integer decision taken from floating point, so the reference takes it in the kernel's
    precision: the oracle's dynamic_keep with logits="bf16" (bf16-rounded rotated q and K', fp64
    sums; the tensor core's fp32 sums of the same exact bf16 products differ by ~1e-6). The
    kernel's bf16 operands come from an fp32 rotation, so an element lying within the fp32 error
    of a bf16 rounding midpoint may round to the other neighbour: each candidate's logit carries
    a bound from those elements (_rounding_slack), and a candidate whose distance to its row's
    threshold is within its bound plus the row maximum's bound (plus 2e-5) may fall either way.
    A row with such candidates must match the reference under one of their keep / drop
    combinations. The values are the fp64 oracle's attention on the decided set."""
    import itertools
    q, k, v = inputs(w, q_scale)
    o, lse, _, _ = run_product(w, q, k, v)
    rows = np.arange(w.q_tokens) if rows is None else rows
    heads = list(range(w.heads)) if heads is None else heads
    og = ogeom(w, len(heads))
    ft = w.frame_tokens
    kc = np.zeros((len(heads), w.kv_tokens, w.head_dim))
    vc = np.zeros_like(kc)
    kx = np.zeros_like(kc)   # unrotated K in the ring layout, for the rotation error bound
    k64, v64 = synth.bf16_bits_to_f64(k[:, heads]), synth.bf16_bits_to_f64(v[:, heads])
    for s, n in w.appends:
        off = (s - w.kv_stream_first_frame) * ft
        oracle.kv_append(kc, vc, w.capacity_frames, og, k64[off:off + n * ft], v64[off:off + n * ft], s, n)
        for f in range(n):
            slot = (s + f) % w.capacity_frames
            kx[:, slot * ft:(slot + 1) * ft] = k64[off + f * ft:off + (f + 1) * ft].transpose(1, 0, 2)
    first, last = w.window()
    kpos, kvalid = oracle.cache_positions(w.capacity_frames, first, last, w.grid_h, w.grid_w)
    qpos = tuple(p[rows] for p in oracle.positions(w.q_tokens, w.grid_h, w.grid_w, w.q_start))
    q64 = synth.bf16_bits_to_f64(q[rows][:, heads])
    qrot = oracle.rope3d(q64, qpos, og)
    cand = oracle.mask_rows(qpos, kpos, kvalid, omask(w)).astype(bool)
    got = f64(o[rows][:, heads])
    n_amb_rows = 0
    keep_all, z_all, thr_all = oracle.dynamic_keep(qrot, kc.transpose(1, 0, 2), cand, w.scale,
                                                   w.tau, logits="bf16")
    dq = _rounding_slack(qrot, _pair_mag(q64))
    dk = _rounding_slack(kc, _pair_mag(kx))
    qb, kb = np.abs(oracle.round_bf16(qrot)), np.abs(oracle.round_bf16(kc))
    for hi in range(len(heads)):
        keep = keep_all[hi]
        z, thr = z_all[hi], thr_all[hi]
        band = w.scale * (dq[:, hi] @ kb[hi].T + qb[:, hi] @ dk[hi].T)     # [rows, keys]
        jmax = np.argmax(np.where(cand, z, -np.inf), axis=1)
        band_thr = band[np.arange(len(rows)), jmax][:, None]
        amb = cand & (np.abs(z - thr) <= band + band_thr + 2e-5)
        assert (amb.sum(axis=1) <= 4).all()
        ref, ref_lse = oracle.attention(qrot[:, hi:hi + 1], kc[hi][:, None], vc[hi][:, None],
                                        keep.astype(np.uint8), w.scale)
        err = np.abs(got[:, hi] - ref[:, 0]).max(axis=1)
        row_amb = amb.any(axis=1)
        n_amb_rows += int(row_amb.sum())
        assert (err[~row_amb] <= 2e-2).all(), float(err[~row_amb].max())
        for r in np.where(row_amb)[0]:
            js = np.where(amb[r])[0]
            best = np.inf
            for flips in itertools.product([False, True], repeat=len(js)):
                kr = keep[r].copy()
                kr[js[list(flips)]] ^= True
                alt, _ = oracle.attention(qrot[r:r + 1, hi:hi + 1], kc[hi][:, None], vc[hi][:, None],
                                          kr[None].astype(np.uint8), w.scale)
                best = min(best, float(np.abs(got[r, hi] - alt[0, 0]).max()))
            assert best <= 2e-2, (r, best)
        d = got[~row_amb, hi] - ref[~row_amb, 0]
        rr = np.sqrt((d ** 2).mean()) / max(1e-30, np.sqrt((ref[~row_amb, 0] ** 2).mean()))
        assert rr <= 1e-2, rr
        l_gpu = lse[heads[hi]][rows].cpu().numpy()
        ok_l = ~row_amb & np.isfinite(ref_lse[0])
        assert np.abs(l_gpu[ok_l] - ref_lse[0][ok_l]).max() < 2e-2
        assert np.isneginf(l_gpu[np.isneginf(ref_lse[0])]).all()
    assert n_amb_rows <= max(3, len(rows) * len(heads) // 20)
    assert vdit.get_status() == vdit.OK


DYNAMIC = {
    "dense_candidates": _medium(4, 0, 9, 9, ((0, 9),)),
    "causal_radial": _medium(7, 6, 3, 9, tuple((s, 3) for s in range(0, 9, 3))),
    "d64_radial": _medium(6, 0, 7, 7, ((0, 7),), d=64, wid=92, heads=3),
}


@pytest.mark.parametrize("name", sorted(DYNAMIC))
@pytest.mark.parametrize("tau", [0.5, 2.0])
def test_attention_dynamic_threshold_medium(name, tau):
    import dataclasses
    _dynamic_check(dataclasses.replace(DYNAMIC[name], tau=tau))


def test_attention_dynamic_threshold_full_size_sampled():
    w = WORKLOADS[6]
    rng = np.random.default_rng(6)
    rows = np.unique(np.r_[np.arange(0, 32), rng.integers(0, w.q_tokens, 64),
                           np.arange(w.q_tokens - 24, w.q_tokens)])
    _dynamic_check(w, rows=rows, heads=[0, w.heads - 1])
