"""Pins of the fp64 CPU oracle against what the pages and the mathematics fix.

Each test checks the oracle against something other than itself: a closed form, an
invariant, a library routine (torch fp64 SDPA, numpy reshape/any), brute force in pure
Python, or hand-worked cases stored under tests/golden/ with their source. The choice is
made so that a plausible slip (a sign, an index, a band offset, a comparison, the causal
direction, the time origin) fails at least one of them.
"""
import math
import os

import numpy as np
import pytest
import torch

import oracle
import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
G128 = oracle.Geometry(grid_h=30, grid_w=52, heads=2, head_dim=128, band_t=44, band_h=42, band_w=42)
G64 = oracle.Geometry(grid_h=4, grid_w=8, heads=2, head_dim=64, band_t=24, band_h=20, band_w=20)


def _rand(seed, shape):
    return synth.normal(seed, int(np.prod(shape))).reshape(shape)


# ----------------------------------------------------------------------------- positions

def test_positions_frame_major_then_h_then_w():
    # token order reading: frame-major, then patch row, then patch column; t is global
    t, h, w = oracle.positions(2 * 3 * 5, 3, 5, start_frame=18)
    exp = [(18 + f, y, x) for f in range(2) for y in range(3) for x in range(5)]
    assert list(zip(t.tolist(), h.tolist(), w.tolist())) == exp


def test_positions_global_time_index_example():
    # Causal-RoPE SP section 2.B: t_global = t_local + s. Token 1561 of a chunk starting at
    # frame 18 on a 30 x 52 grid is local frame 1, row 0, column 1 -> global frame 19.
    t, h, w = oracle.positions(1562, 30, 52, start_frame=18)
    assert (t[1561], h[1561], w[1561]) == (19, 0, 1)
    assert (t[1559], h[1559], w[1559]) == (18, 29, 51)


# ----------------------------------------------------------------------------- RoPE

def _pos(n, g, start):
    return oracle.positions(n, g.grid_h, g.grid_w, start)


@pytest.mark.parametrize("g", [G128, G64])
def test_rope_preserves_norm_of_every_pair(g):
    n = 3 * g.frame_tokens
    x = _rand(11, (n, g.heads, g.head_dim))
    y = oracle.rope3d(x, _pos(n, g, 396), g)
    px = np.hypot(x[..., 0::2], x[..., 1::2])
    py = np.hypot(y[..., 0::2], y[..., 1::2])
    assert np.max(np.abs(px - py) / px) < 1e-13
    nx = np.linalg.norm(x, axis=-1)
    ny = np.linalg.norm(y, axis=-1)
    assert np.max(np.abs(nx - ny) / nx) < 1e-14


def test_rope_identity_at_origin():
    x = _rand(12, (5, 2, 128))
    z = np.zeros(5, np.int32)
    y = oracle.rope3d(x, (z, z, z), G128)
    assert np.array_equal(x, y)


def test_rope_group_property():
    # rotating by p1 then by p2 equals rotating by p1 + p2
    g = G128
    x = _rand(13, (7, 2, 128))
    rng = np.random.default_rng(0)
    p1 = [rng.integers(0, 400, 7).astype(np.int32) for _ in range(3)]
    p2 = [rng.integers(0, 60, 7).astype(np.int32) for _ in range(3)]
    a = oracle.rope3d(oracle.rope3d(x, p1, g), p2, g)
    b = oracle.rope3d(x, [u + v for u, v in zip(p1, p2)], g)
    assert np.max(np.abs(a - b)) < 1e-11


@pytest.mark.parametrize("shift", [(18, 0, 0), (396, 0, 0), (0, 7, 0), (0, 0, 11), (396, 3, 5)])
def test_rope_scores_depend_only_on_relative_position(shift):
    # global time index invariant: q.k after rotation depends only on (dt, dh, dw), so moving
    # every token by the same (s_t, s_h, s_w) leaves every score unchanged
    g = G128
    rng = np.random.default_rng(1)
    n = 64
    q = _rand(14, (n, 2, 128))
    k = _rand(15, (n, 2, 128))
    pq = [rng.integers(0, 30, n).astype(np.int32) for _ in range(3)]
    pk = [rng.integers(0, 30, n).astype(np.int32) for _ in range(3)]
    s0 = np.einsum("nhd,mhd->hnm", oracle.rope3d(q, pq, g), oracle.rope3d(k, pk, g))
    pq2 = [p + s for p, s in zip(pq, shift)]
    pk2 = [p + s for p, s in zip(pk, shift)]
    s1 = np.einsum("nhd,mhd->hnm", oracle.rope3d(q, pq2, g), oracle.rope3d(k, pk2, g))
    assert np.max(np.abs(s0 - s1)) < 1e-10


def test_rope_chunk_with_start_frame_equals_slice_of_whole_clip():
    # Causal-RoPE SP 2.B: a chunk computes its own positions from its start frame alone and
    # gets exactly what the whole-sequence computation gives for those tokens
    g = G64
    ft = g.frame_tokens
    x = _rand(16, (21 * ft, 2, 64))
    whole = oracle.rope3d(x, _pos(21 * ft, g, 0), g)
    chunk = oracle.rope3d(x[18 * ft:], _pos(3 * ft, g, 18), g)
    assert np.array_equal(whole[18 * ft:], chunk)


@pytest.mark.parametrize("g", [G128, G64])
def test_rope_band_membership(g):
    # channels [0, bt) carry t, [bt, bt+bh) carry h, [bt+bh, D) carry w: moving one coordinate
    # changes exactly its own band and leaves the other channels bit-identical
    x = _rand(17, (1, 1, g.head_dim))
    bands = [(0, g.band_t), (g.band_t, g.band_t + g.band_h), (g.band_t + g.band_h, g.head_dim)]
    for axis in range(3):
        pos = [np.zeros(1, np.int32) for _ in range(3)]
        pos[axis][0] = 5
        y = oracle.rope3d(x, pos, g)
        lo, hi = bands[axis]
        outside = np.r_[0:lo, hi:g.head_dim]
        assert np.array_equal(y[0, 0, outside], x[0, 0, outside])
        assert np.all(np.abs(y[0, 0, lo:hi] - x[0, 0, lo:hi]) > 0)


@pytest.mark.parametrize("g", [G128, G64])
def test_rope_frequency_ladder_and_direction(g):
    # Standard rotary embedding per band: pair j turns counter-clockwise by pos * omega_j with
    # omega_0 = 1 rad per position and omega_{j+1} / omega_j = theta^(-2/width) (geometric
    # ladder down to theta^-(width-2)/width). Read off the angle of a unit vector on each pair.
    offs = [0, g.band_t, g.band_t + g.band_h]
    widths = [g.band_t, g.band_h, g.band_w]
    for axis in range(3):
        width, off = widths[axis], offs[axis]
        omegas = []
        for j in range(width // 2):
            x = np.zeros((1, 1, g.head_dim))
            x[0, 0, off + 2 * j] = 1.0
            pos = [np.zeros(1, np.int32) for _ in range(3)]
            pos[axis][0] = 1
            y = oracle.rope3d(x, pos, g)[0, 0]
            c, s = y[off + 2 * j], y[off + 2 * j + 1]
            assert abs(math.hypot(c, s) - 1) < 1e-15
            omegas.append(math.atan2(s, c))
        assert omegas[0] == pytest.approx(1.0, abs=1e-15)
        assert all(o > 0 for o in omegas)  # counter-clockwise
        ratios = np.array(omegas[1:]) / np.array(omegas[:-1])
        assert np.allclose(ratios, g.theta ** (-2.0 / width), rtol=1e-12, atol=0)


@pytest.mark.parametrize("g", [G128, G64])
def test_rope_each_band_equals_a_library_rotary_embedding(g):
    # External pin of the pairing and the ladder: each band of the 3-D RoPE is a 1-D rotary
    # embedding over adjacent channel pairs, which is the convention of the GPT-J rotary in
    # transformers (rotate_every_two, sinusoids with inverse frequencies 10000^(-2j/width)).
    # The library computes in fp32, so positions stay small enough for its angles to be exact
    # to ~1e-5; a rotate-half pairing, a reversed rotation or a shifted band fails by O(1).
    gptj = pytest.importorskip("transformers.models.gptj.modeling_gptj")
    assert g.theta == 10000.0
    n = 2 * g.frame_tokens
    x = _rand(29, (n, g.heads, g.head_dim))
    t, h, w = _pos(n, g, 37)
    y = oracle.rope3d(x, (t, h, w), g)
    bands = [(0, g.band_t, t), (g.band_t, g.band_t + g.band_h, h),
             (g.band_t + g.band_h, g.head_dim, w)]
    for lo, hi, p in bands:
        width = hi - lo
        table = gptj.create_sinusoidal_positions(int(p.max()) + 1, width)  # [pos, sin | cos]
        sincos = table[torch.from_numpy(p.astype(np.int64))]
        sin, cos = sincos[:, : width // 2], sincos[:, width // 2:]
        xb = torch.from_numpy(x[None, :, :, lo:hi].astype(np.float32))  # [1, n, heads, width]
        ref = gptj.apply_rotary_pos_emb(xb, sin[None], cos[None])[0].double().numpy()
        assert np.max(np.abs(y[:, :, lo:hi] - ref)) < 1e-4


# ----------------------------------------------------------------------------- mask

def _golden_mask_cases():
    rows = []
    with open(os.path.join(GOLDEN, "radial_mask_cases.txt")) as f:
        for line in f:
            line = line.split("#")[0].strip()
            if line:
                rows.append([int(v) for v in line.split()])
    return rows


def test_mask_hand_worked_cases():
    cases = _golden_mask_cases()
    assert len(cases) >= 20
    for bc, rad, tq, hq, wq, tk, hk, wk, keep in cases:
        m = oracle.Mask(block_causal=bool(bc), radial=bool(rad), chunk_frames=3, w0=52,
                        gamma_shift=1, lam=8)
        one = lambda a: np.array([a], np.int32)
        got = oracle.mask_rows((one(tq), one(hq), one(wq)), (one(tk), one(hk), one(wk)),
                               np.ones(1, np.uint8), m)[0, 0]
        assert got == keep, (bc, rad, tq, hq, wq, tk, hk, wk)


def _count_pairs_within(n, r):
    # ordered pairs (a, b) in [0, n)^2 with |a - b| <= r
    return n + 2 * sum(n - d for d in range(1, min(r, n - 1) + 1))


def _closed_form_radial_kept(q_frames, k_frames, grid_h, grid_w, w0, lam, causal_chunk=None):
    hw = grid_h * grid_w
    total = 0
    for fq in q_frames:
        for fk in k_frames:
            if causal_chunk and fk // causal_chunk > fq // causal_chunk:
                continue
            dt = abs(fq - fk)
            if lam and dt % lam == 0:
                total += hw * hw
            else:
                r = w0 >> dt if dt < 63 else 0
                total += _count_pairs_within(grid_h, r) * _count_pairs_within(grid_w, r)
    return total


def test_count_helper_brute_force():
    for n in (1, 4, 7):
        for r in range(0, 9):
            bf = sum(1 for a in range(n) for b in range(n) if abs(a - b) <= r)
            assert _count_pairs_within(n, r) == bf


def _kept(qframes0, nqf, kfirst, klast, cap, m, gh=30, gw=52):
    qpos = oracle.positions(nqf * gh * gw, gh, gw, qframes0)
    kpos, kvalid = oracle.cache_positions(cap, kfirst, klast, gh, gw)
    _, _, _, kept = oracle.tiles(qpos, kpos, kvalid, m)
    return kept


def test_radial_kept_count_closed_form_full_bidirectional_shape():
    # 21 frames x 30 x 52, W0 = 52, gamma = 1/2, lambda = 8, token-level mask
    m = oracle.Mask(radial=True, w0=52, gamma_shift=1, lam=8)
    kept = _kept(0, 21, 0, 20, 21, m)
    cf = _closed_form_radial_kept(range(21), range(21), 30, 52, 52, 8)
    assert kept == cf
    assert kept == 251_899_408


def test_causal_radial_kept_count_closed_form_long_rollout():
    # query chunk at global frames 396..398 against the rolling window 378..398
    m = oracle.Mask(block_causal=True, radial=True, chunk_frames=3, w0=52, gamma_shift=1, lam=8)
    kept = _kept(396, 3, 378, 398, 21, m)
    cf = _closed_form_radial_kept(range(396, 399), range(378, 399), 30, 52, 52, 8, causal_chunk=3)
    assert kept == cf
    assert kept == 35_059_624


def test_block_causal_newest_chunk_sees_everything():
    m = oracle.Mask(block_causal=True, chunk_frames=3)
    assert _kept(18, 3, 0, 20, 21, m) == 4680 * 32760


def test_block_causal_tiny_count_closed_form():
    # 6 frames x 4 x 8, chunks of 3: frames 0..2 see 3 frames, frames 3..5 see 6 frames
    m = oracle.Mask(block_causal=True, chunk_frames=3)
    qpos = oracle.positions(192, 4, 8, 0)
    kept = oracle.mask_rows(qpos, qpos, np.ones(192, np.uint8), m).sum()
    assert kept == 96 * 96 + 96 * 192
    assert kept / 192 ** 2 == 0.75


def test_single_chunk_block_causal_equals_bidirectional():
    g = G64
    n = 3 * g.frame_tokens
    for start in (0, 18, 396):
        pos = oracle.positions(n, g.grid_h, g.grid_w, start)
        mc = oracle.mask_rows(pos, pos, np.ones(n, np.uint8), oracle.Mask(block_causal=True))
        assert mc.all()
        q = oracle.rope3d(_rand(20, (n, 2, 64)), pos, g)
        k = oracle.rope3d(_rand(21, (n, 2, 64)), pos, g)
        v = _rand(22, (n, 2, 64))
        oc, lc = oracle.attention(q, k, v, mc, 0.125)
        od, ld = oracle.attention(q, k, v, np.ones((n, n), np.uint8), 0.125)
        assert np.array_equal(oc, od) and np.array_equal(lc, ld)


def test_infinite_radial_window_equals_dense():
    g = G64
    pos = oracle.positions(6 * g.frame_tokens, g.grid_h, g.grid_w, 0)
    ones = np.ones(len(pos[0]), np.uint8)
    for m in (oracle.Mask(radial=True, w0=1 << 40, lam=0),
              oracle.Mask(radial=True, w0=0, lam=1)):
        assert oracle.mask_rows(pos, pos, ones, m).all()


def test_empty_cache_slots_are_never_kept():
    kpos, kvalid = oracle.cache_positions(7, 0, 2, 2, 3)  # 3 of 7 frame slots filled
    assert kvalid.sum() == 3 * 6
    qpos = oracle.positions(6, 2, 3, 2)
    m = oracle.mask_rows(qpos, kpos, kvalid, oracle.Mask())
    assert m.sum() == 6 * 18 and not m[:, 18:].any()


# ----------------------------------------------------------------------------- attention

def test_attention_matches_torch_sdpa_fp64():
    g = G64
    n = 6 * g.frame_tokens
    pos = oracle.positions(n, g.grid_h, g.grid_w, 0)
    q = oracle.rope3d(_rand(30, (n, 2, 64)), pos, g)
    k = oracle.rope3d(_rand(31, (n, 2, 64)), pos, g)
    v = _rand(32, (n, 2, 64))
    for mk in (oracle.Mask(block_causal=True), oracle.Mask(radial=True, w0=4, lam=4),
               oracle.Mask()):
        m = oracle.mask_rows(pos, pos, np.ones(n, np.uint8), mk)
        o, lse = oracle.attention(q, k, v, m, 0.125)
        qt, kt, vt = (torch.from_numpy(a).permute(1, 0, 2) for a in (q, k, v))
        ref = torch.nn.functional.scaled_dot_product_attention(
            qt, kt, vt, attn_mask=torch.from_numpy(m.astype(bool)), scale=0.125)
        assert np.max(np.abs(ref.permute(1, 0, 2).numpy() - o)) < 1e-12
        s = torch.einsum("hnd,hmd->hnm", qt, kt) * 0.125
        s = s.masked_fill(~torch.from_numpy(m.astype(bool)), -math.inf)
        assert np.max(np.abs(torch.logsumexp(s, -1).numpy() - lse)) < 1e-12


def test_attention_brute_force_pure_python():
    rng = np.random.default_rng(5)
    nq, nk, heads, d = 5, 7, 2, 4
    q, k, v = rng.normal(size=(nq, heads, d)), rng.normal(size=(nk, heads, d)), rng.normal(size=(nk, heads, d))
    m = (rng.random((nq, nk)) < 0.6).astype(np.uint8)
    m[:, 0] = 1
    m[4, :] = 0  # a row with no kept key
    o, lse = oracle.attention(q, k, v, m, 0.7)
    for h in range(heads):
        for i in range(nq):
            js = [j for j in range(nk) if m[i, j]]
            if not js:
                assert all(o[i, h] == 0) and lse[h, i] == -math.inf
                continue
            sc = {j: 0.7 * sum(q[i, h, c] * k[j, h, c] for c in range(d)) for j in js}
            z = sum(math.exp(s) for s in sc.values())
            for c in range(d):
                ref = sum(math.exp(sc[j]) / z * v[j, h, c] for j in js)
                assert abs(ref - o[i, h, c]) < 1e-13
            assert abs(math.log(z) - lse[h, i]) < 1e-13


# ----------------------------------------------------------------------------- tiles

@pytest.mark.parametrize("tile", [16, 128])
def test_tiles_equal_reshape_any_of_explicit_mask(tile):
    g = oracle.Geometry(grid_h=5, grid_w=7, heads=1, head_dim=64, band_t=24, band_h=20, band_w=20)
    nq_frames, cap = 4, 11
    qpos = oracle.positions(nq_frames * 35, 5, 7, 6)
    kpos, kvalid = oracle.cache_positions(cap, 0, 9, 5, 7)  # slot 10 empty; ragged tails
    for mk in (oracle.Mask(block_causal=True), oracle.Mask(radial=True, w0=3, lam=4),
               oracle.Mask(block_causal=True, radial=True, w0=2, lam=3), oracle.Mask()):
        m = oracle.mask_rows(qpos, kpos, kvalid, mk)
        nq, nk = m.shape
        n_qt, n_kt = -(-nq // tile), -(-nk // tile)
        pad = np.zeros((n_qt * tile, n_kt * tile), np.uint8)
        pad[:nq, :nk] = m
        blocks = pad.reshape(n_qt, tile, n_kt, tile).transpose(0, 2, 1, 3)
        anyk = blocks.any(axis=(2, 3))
        inrange = np.zeros_like(pad)
        inrange[:nq, :nk] = 1
        complete = inrange.reshape(n_qt, tile, n_kt, tile).transpose(0, 2, 1, 3).all(axis=(2, 3))
        fullk = blocks.all(axis=(2, 3)) & complete
        row_ptr, col, full, kept = oracle.tiles(qpos, kpos, kvalid, mk, tile)
        assert kept == m.sum()
        exp_rows, exp_cols = np.nonzero(anyk)
        assert np.array_equal(col, exp_cols)
        assert np.array_equal(np.diff(row_ptr), np.bincount(exp_rows, minlength=n_qt))
        assert np.array_equal(full.astype(bool), fullk[exp_rows, exp_cols])


def test_dense_tile_list_closed_form():
    # 32,760 = 255 * 128 + 120: 256 x 256 tiles listed, the 255 x 255 complete ones full
    qpos = oracle.positions(32760, 30, 52, 0)
    kpos, kvalid = oracle.cache_positions(21, 0, 20, 30, 52)
    row_ptr, col, full, kept = oracle.tiles(qpos, kpos, kvalid, oracle.Mask())
    assert row_ptr[-1] == 256 * 256 and full.sum() == 255 * 255 and kept == 32760 ** 2


# ----------------------------------------------------------------------------- KV cache

def test_cache_positions_ring():
    (t, h, w), valid = oracle.cache_positions(7, 8, 14, 2, 3)
    ft = 6
    for slot in range(7):
        held = set(t[slot * ft:(slot + 1) * ft].tolist())
        assert held == {next(f for f in range(8, 15) if f % 7 == slot)}
    assert valid.all()
    assert h.tolist()[:6] == [0, 0, 0, 1, 1, 1] and w.tolist()[:6] == [0, 1, 2, 0, 1, 2]


def test_kv_append_ring_placement():
    g = oracle.Geometry(grid_h=2, grid_w=3, heads=2, head_dim=64, band_t=24, band_h=20, band_w=20)
    ft, cap = 6, 7
    k_all = _rand(40, (15 * ft, 2, 64))
    v_all = _rand(41, (15 * ft, 2, 64))
    kc = np.zeros((2, cap * ft, 64))
    vc = np.zeros((2, cap * ft, 64))
    for s in range(0, 15, 3):
        oracle.kv_append(kc, vc, cap, g, k_all[s * ft:(s + 3) * ft], v_all[s * ft:(s + 3) * ft], s, 3)
    krot = oracle.rope3d(k_all, oracle.positions(15 * ft, 2, 3, 0), g)
    for f in range(8, 15):  # the newest 7 frames survive, frame f in slot f mod 7
        slot = f % cap
        assert np.array_equal(vc[:, slot * ft:(slot + 1) * ft], v_all[f * ft:(f + 1) * ft].transpose(1, 0, 2))
        assert np.array_equal(kc[:, slot * ft:(slot + 1) * ft], krot[f * ft:(f + 1) * ft].transpose(1, 0, 2))


# ----------------------------------------------------------------------------- QKV projection

def test_qkv_project_hand_worked_example():
    # 2 tokens, d_model 2, one head of dimension 2; products worked out by hand
    x = np.array([[1.0, 2.0], [3.0, -1.0]])
    w = np.array([[1, 0], [0, 1], [2, 1], [1, -1], [0, 3], [1, 1]], dtype=np.float64)
    q, k, v = oracle.qkv_project(x, w, 1, 2)
    assert np.array_equal(q[:, 0], [[1, 2], [3, -1]])
    assert np.array_equal(k[:, 0], [[4, -1], [5, 4]])
    assert np.array_equal(v[:, 0], [[6, 3], [-3, 2]])


def test_qkv_project_identity_weights_split_heads():
    # W = [I; 2 I; -I] gives Q = x, K = 2 x, V = -x, cut into heads of head_dim channels
    rng = np.random.default_rng(3)
    heads, d = 3, 4
    x = rng.standard_normal((5, heads * d))
    eye = np.eye(heads * d)
    q, k, v = oracle.qkv_project(x, np.vstack([eye, 2 * eye, -eye]), heads, d)
    assert np.array_equal(q, x.reshape(5, heads, d))
    assert np.array_equal(k, 2 * x.reshape(5, heads, d))
    assert np.array_equal(v, -x.reshape(5, heads, d))


def test_qkv_project_is_linear_in_x():
    rng = np.random.default_rng(4)
    x1, x2 = rng.standard_normal((2, 7, 16))
    w = rng.standard_normal((3 * 8, 16))
    a = oracle.qkv_project(x1 + 3 * x2, w, 2, 4)
    b1, b2 = oracle.qkv_project(x1, w, 2, 4), oracle.qkv_project(x2, w, 2, 4)
    for i in range(3):
        assert np.allclose(a[i], b1[i] + 3 * b2[i], rtol=1e-12, atol=1e-12)


# ----------------------------------------------------------------------------- dynamic threshold

def test_dynamic_threshold_hand_worked_example():
    # one query, four candidate keys with logits 2.0, 1.0, -0.5, 1.9 (scale 1, d = 1): tau 0.5
    # keeps {0, 3}, tau 1.2 keeps {0, 1, 3}, and a masked-out key is never kept
    q = np.ones((1, 1, 1))
    k = np.array([2.0, 1.0, -0.5, 1.9, 5.0]).reshape(5, 1, 1)
    v = np.arange(5, dtype=np.float64).reshape(5, 1, 1)
    cand = np.array([[1, 1, 1, 1, 0]], np.uint8)
    _, _, keep = oracle.attention_dynamic(q, k, v, cand, 1.0, 0.5)
    assert keep[0, 0].tolist() == [True, False, False, True, False]
    o, lse, keep = oracle.attention_dynamic(q, k, v, cand, 1.0, 1.2)
    assert keep[0, 0].tolist() == [True, True, False, True, False]
    w = np.exp(np.array([2.0, 1.0, 1.9]))
    assert np.isclose(o[0, 0, 0], (w * np.array([0.0, 1.0, 3.0])).sum() / w.sum(), rtol=1e-14)
    assert np.isclose(lse[0, 0], np.log(w.sum()), rtol=1e-14)


def _rand_case(seed, nq=6, nk=40, heads=2, d=8):
    rng = np.random.default_rng(seed)
    q, k, v = rng.standard_normal((nq, heads, d)), rng.standard_normal((nk, heads, d)), rng.standard_normal((nk, heads, d))
    cand = (rng.random((nq, nk)) < 0.6).astype(np.uint8)
    cand[0] = 0  # a row without candidates
    return q, k, v, cand


def test_dynamic_threshold_large_tau_equals_the_candidate_mask():
    q, k, v, cand = _rand_case(1)
    o, lse, keep = oracle.attention_dynamic(q, k, v, cand, 0.35, 1e9)
    o2, lse2 = oracle.attention(q, k, v, cand, 0.35)
    assert (keep == cand.astype(bool)[None]).all()
    assert np.allclose(o, o2, atol=1e-13) and np.allclose(lse[:, 1:], lse2[:, 1:], atol=1e-13)
    assert (o[0] == 0).all() and np.isneginf(lse[:, 0]).all()


def test_dynamic_threshold_tiny_tau_keeps_only_the_argmax():
    q, k, v, cand = _rand_case(2)
    o, _, keep = oracle.attention_dynamic(q, k, v, cand, 0.35, 1e-12)
    for h in range(2):
        z = np.where(cand.astype(bool), 0.35 * q[:, h] @ k[:, h].T, -np.inf)
        for r in range(1, z.shape[0]):
            j = int(np.argmax(z[r]))
            assert keep[h, r].sum() == 1 and keep[h, r, j]
            assert np.allclose(o[r, h], v[j, h], atol=1e-13)


def test_dynamic_threshold_kept_sets_grow_with_tau():
    q, k, v, cand = _rand_case(3)
    prev = None
    for tau in (0.1, 0.5, 1.0, 2.0, 8.0):
        _, _, keep = oracle.attention_dynamic(q, k, v, cand, 0.35, tau)
        assert (keep <= cand.astype(bool)[None]).all()
        if prev is not None:
            assert (prev <= keep).all()
        prev = keep


# ----------------------------------------------------------------------------- bf16 decision rule

def test_round_bf16_hand_worked_values():
    # spacing 2^-7 on [1, 2): 1 + 2^-8 is a tie -> even (1.0); 1 + 3 * 2^-8 is a tie -> even
    # (1 + 2^-6); 0.7509765625 = 192.25 * 2^-8 -> 0.75; subnormal spacing 2^-133; overflow -> inf
    x = np.array([1 + 2 ** -8, 1 + 3 * 2 ** -8, 0.7509765625, -0.7490234375, 3 * 2 ** -135,
                  2.0 ** 128, 0.0, -1.5])
    want = np.array([1.0, 1 + 2 ** -6, 0.75, -0.75, 2.0 ** -133, np.inf, 0.0, -1.5])
    assert np.array_equal(oracle.round_bf16(x), want)


def test_round_bf16_equals_torch_float32_to_bfloat16():
    # for float32 inputs, round-to-nearest-even to 8 significant bits is torch's own conversion
    x = _rand(77, (20000,)).astype(np.float32) * np.float32(3.0)
    x[:5] = np.array([1 + 2 ** -8, 1 + 3 * 2 ** -8, 2 ** -130, -2 ** -127, 65504.0], np.float32)
    ref = torch.from_numpy(x).to(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(oracle.round_bf16(x.astype(np.float64)), ref)


def test_dynamic_keep_bf16_flips_a_decision_the_f64_rule_keeps():
    # one query q = (1, 0), scale 1, d = 2: logits are the keys' first channels. k0 = 1 - 2^-10
    # rounds up to 1.0 in bfloat16, k1 = 0.75 is exact. tau = 0.2495:
    #   f64:  z1 - z0 = 0.75 - 0.9990234375 = -0.2490234375 >= -0.2495  -> both kept
    #   bf16: z1 - z0 = 0.75 - 1.0 = -0.25 < -0.2495                    -> only k0 kept
    q = np.array([1.0, 0.0]).reshape(1, 1, 2)
    k = np.array([[1 - 2 ** -10, 0.0], [0.75, 0.0]]).reshape(2, 1, 2)
    v = np.array([[2.0, -1.0], [5.0, 3.0]]).reshape(2, 1, 2)
    cand = np.ones((1, 2), np.uint8)
    o64, l64, keep64 = oracle.attention_dynamic(q, k, v, cand, 1.0, 0.2495, logits="f64")
    ob, lb, keepb = oracle.attention_dynamic(q, k, v, cand, 1.0, 0.2495, logits="bf16")
    assert keep64[0, 0].tolist() == [True, True]
    assert keepb[0, 0].tolist() == [True, False]
    # bf16 rule: only key 0 is kept, so o = v0 and lse = its (unrounded) logit
    assert np.array_equal(ob[0, 0], [2.0, -1.0]) and lse_close(lb[0, 0], 1 - 2 ** -10)
    # f64 rule: softmax over the two unrounded logits, written out by hand
    e0, e1 = math.exp(1 - 2 ** -10), math.exp(0.75)
    assert np.allclose(o64[0, 0], [(2 * e0 + 5 * e1) / (e0 + e1), (-e0 + 3 * e1) / (e0 + e1)], rtol=1e-14)
    assert lse_close(l64[0, 0], math.log(e0 + e1))
    # the logits and threshold it returns are the rounded ones
    _, z, thr = oracle.dynamic_keep(q, k, cand, 1.0, 0.2495, logits="bf16")
    assert z[0, 0].tolist() == [1.0, 0.75] and thr[0, 0, 0] == 1.0 - 0.2495


def lse_close(a, b):
    return abs(a - b) <= 1e-14 * max(1.0, abs(b))


def test_dynamic_keep_rules_agree_on_bf16_exact_operands():
    # operands that are already bfloat16 values round to themselves: both rules are identical
    q, k, v, cand = _rand_case(4, nq=12, nk=64, d=16)
    q, k = oracle.round_bf16(q), oracle.round_bf16(k)
    for tau in (0.1, 0.7, 3.0):
        o1, l1, k1 = oracle.attention_dynamic(q, k, v, cand, 0.25, tau, logits="f64")
        o2, l2, k2 = oracle.attention_dynamic(q, k, v, cand, 0.25, tau, logits="bf16")
        assert np.array_equal(k1, k2) and np.array_equal(o1, o2) and np.array_equal(l1, l2)


def test_dynamic_keep_rules_differ_only_inside_the_rounding_band():
    # rounding q and k to bfloat16 moves each product q_i k_i by at most (2^-8 + 2^-16) |q_i k_i|
    # (relative error 2^-8 of each operand), so a logit moves by at most
    # eps = scale (2^-8 + 2^-16) sum_i |q_i k_i|; a decision can only flip for a candidate whose
    # f64 logit lies within eps_j + eps_max of the f64 threshold (the row maximum moves too)
    q, k, v, cand = _rand_case(5, nq=64, nk=400, d=32)
    scale, tau = 0.3, 2.0
    k64, z64, thr64 = oracle.dynamic_keep(q, k, cand, scale, tau, logits="f64")
    kb, _, _ = oracle.dynamic_keep(q, k, cand, scale, tau, logits="bf16")
    flips = 0
    for h in range(q.shape[1]):
        eps = scale * (2 ** -8 + 2 ** -16) * (np.abs(q[:, h]) @ np.abs(k[:, h]).T)
        eps_max = np.where(cand.astype(bool), eps, 0).max(axis=1, keepdims=True)
        band = np.abs(z64[h] - thr64[h]) <= eps + eps_max
        diff = k64[h] != kb[h]
        assert not (diff & ~band).any()
        flips += int(diff.sum())
    # the band is wide enough on these inputs that the two rules really do differ somewhere
    assert flips > 0


def test_dynamic_keep_bf16_limits_in_tau():
    q, k, v, cand = _rand_case(6)
    keep, _, _ = oracle.dynamic_keep(q, k, cand, 0.35, 1e9, logits="bf16")
    assert (keep == cand.astype(bool)[None]).all()
    keep, _, _ = oracle.dynamic_keep(q, k, cand, 0.35, 1e-12, logits="bf16")
    qb, kb = oracle.round_bf16(q), oracle.round_bf16(k)
    for h in range(2):
        z = np.where(cand.astype(bool), qb[:, h] @ kb[:, h].T, -np.inf)
        for r in range(1, z.shape[0]):
            assert keep[h, r].sum() == 1 and keep[h, r, int(np.argmax(z[r]))]
    assert not keep[:, 0].any()
