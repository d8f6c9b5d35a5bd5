"""Host-side checks of libvdit that need no GPU: the C ABI loads and exports every declared
symbol, the tile schedule is bit-identical to the oracle's explicit-mask tile list, and bad
arguments are rejected before any device work."""
import ctypes

import numpy as np
import pytest

import oracle
import video_diffusion_transformer_vdit_b200 as vdit
from video_diffusion_transformer_vdit_b200.workloads import WORKLOADS, Workload


def test_library_exports_every_declared_symbol():
    names = vdit.declared_symbols()
    assert len(names) >= 10
    L = vdit.lib()
    for n in names:
        assert hasattr(L, n), n
    # the ctypes prototypes cover the same set
    for n in names:
        assert getattr(L, n).argtypes is not None or n == "vdit_last_error", n


def _geom(w):
    return vdit.Geometry(w.grid_h, w.grid_w, w.heads, w.head_dim, w.bands, w.theta)


def _mask(w):
    return vdit.Mask(w.mask_kind, w.chunk_frames, w.w0, w.gamma_shift, w.lam, w.tau)


def _oracle_tiles(grid_h, grid_w, q_start, q_frames, cap, first, last, mask_kind, chunk, w0, g, lam):
    qpos = oracle.positions(q_frames * grid_h * grid_w, grid_h, grid_w, q_start)
    kpos, kvalid = oracle.cache_positions(cap, first, last, grid_h, grid_w)
    m = oracle.Mask(block_causal=bool(mask_kind & 1), radial=bool(mask_kind & 2),
                    chunk_frames=chunk, w0=w0, gamma_shift=g, lam=lam)
    return oracle.tiles(qpos, kpos, kvalid, m)


def _compare(plan, ref):
    rp, ci, fu = plan.export()
    orp, oci, ofu, kept = ref
    assert np.array_equal(rp.numpy(), orp)
    assert np.array_equal(ci.numpy(), oci)
    assert np.array_equal(fu.numpy(), ofu)
    assert plan.info["kept_pairs"] == kept
    assert plan.info["full_tiles"] == int(ofu.sum())


@pytest.mark.parametrize("wid", sorted(WORKLOADS))
def test_plan_bit_exact_vs_oracle_workloads(wid):
    w = WORKLOADS[wid]
    first, last = w.window()
    plan = vdit.Plan(_geom(w), _mask(w), w.q_start, w.q_frames, capacity_frames=w.capacity_frames,
                     kv_first_frame=first, kv_last_frame=last, upload=False)
    ref = _oracle_tiles(w.grid_h, w.grid_w, w.q_start, w.q_frames, w.capacity_frames, first, last,
                        w.mask_kind, w.chunk_frames, w.w0, w.gamma_shift, w.lam)
    _compare(plan, ref)


def test_plan_counts_of_the_wan_workloads():
    # non-empty / full tile counts and kept fractions of the four full-size workloads
    exp = {2: (65536, 65025), 3: (9472, 9180), 4: (30326, 7190), 5: (3998, 1134), 1: (4, 0)}
    for wid, (tiles, full) in exp.items():
        w = WORKLOADS[wid]
        first, last = w.window()
        info = vdit.Plan(_geom(w), _mask(w), w.q_start, w.q_frames,
                         capacity_frames=w.capacity_frames, kv_first_frame=first,
                         kv_last_frame=last, upload=False).info
        assert (info["tiles"], info["full_tiles"]) == (tiles, full), wid


def test_plan_bit_exact_vs_oracle_random_geometries():
    rng = np.random.default_rng(7)
    for _ in range(40):
        gh, gw = int(rng.integers(1, 9)), int(rng.integers(1, 40))
        cap = int(rng.integers(1, 12))
        last = int(rng.integers(0, 40))
        first = max(0, last - int(rng.integers(0, cap)))
        q_frames = int(rng.integers(1, 6))
        q_start = int(rng.integers(max(0, last - 8), last + 3))
        kind = int(rng.integers(0, 4))
        chunk = int(rng.integers(1, 5))
        w0 = int(rng.integers(0, 60))
        gs = int(rng.integers(0, 3))
        lam = int(rng.integers(0, 6))
        g = vdit.Geometry(gh, gw, 1, 64, (24, 20, 20))
        plan = vdit.Plan(g, vdit.Mask(kind, chunk, w0, gs, lam), q_start, q_frames,
                         capacity_frames=cap, kv_first_frame=first, kv_last_frame=last, upload=False)
        ref = _oracle_tiles(gh, gw, q_start, q_frames, cap, first, last, kind, chunk, w0, gs, lam)
        _compare(plan, ref)


def _check_masks(plan, grid_h, grid_w, q_start, q_frames, cap, first, last, kind, chunk, w0, g, lam,
                 q_tiles=None):
    """The plan's per-row keep masks of partial tiles equal the oracle's explicit mask, bit by
    bit (for the given q-tiles, all by default)."""
    rp, ci, fu = (t.numpy() for t in plan.export())
    idx, words = plan.export_masks()
    assert np.array_equal(idx >= 0, fu == 0)
    # identical blocks are stored once: every stored block is used by some entry and no two
    # stored blocks are equal (each entry is checked against the oracle below)
    used = np.unique(idx[idx >= 0])
    assert np.array_equal(used, np.arange(len(words)))
    if len(words):
        assert len(np.unique(words.reshape(len(words), -1), axis=0)) == len(words)
    n_q = q_frames * grid_h * grid_w
    qpos = oracle.positions(n_q, grid_h, grid_w, q_start)
    kpos, kvalid = oracle.cache_positions(cap, first, last, grid_h, grid_w)
    m = oracle.Mask(block_causal=bool(kind & 1), radial=bool(kind & 2), chunk_frames=chunk,
                    w0=w0, gamma_shift=g, lam=lam)
    n_k = len(kvalid)
    bits = np.arange(32, dtype=np.uint32)
    for qt in (range(len(rp) - 1) if q_tiles is None else q_tiles):
        q0, q1 = qt * 128, min(n_q, qt * 128 + 128)
        ref = oracle.mask_rows(tuple(p[q0:q1] for p in qpos), kpos, kvalid, m).astype(bool)
        for i in range(rp[qt], rp[qt + 1]):
            kt = ci[i]
            k0, k1 = kt * 128, min(n_k, kt * 128 + 128)
            want = np.zeros((128, 128), bool)
            want[:q1 - q0, :k1 - k0] = ref[:, k0:k1]
            if idx[i] < 0:
                assert want.all()
                continue
            got = ((words[idx[i]][:, :, None] >> bits) & 1).reshape(128, 128).astype(bool)
            assert np.array_equal(got, want), (qt, kt)


def _check_work(plan, grid_h, grid_w, q_start, q_frames, cap, first, last, kind, chunk, w0, g, lam,
                q_tiles=None):
    """The kernel's work list covers exactly the oracle's kept pairs, each once: per query tile,
    the entries' 128-key blocks (all ones for a full tile) placed at their key rows add up to the
    oracle's explicit mask rows, with no pair covered twice."""
    rp, kr, mi, words = plan.export_work()
    n_q = q_frames * grid_h * grid_w
    qpos = oracle.positions(n_q, grid_h, grid_w, q_start)
    kpos, kvalid = oracle.cache_positions(cap, first, last, grid_h, grid_w)
    m = oracle.Mask(block_causal=bool(kind & 1), radial=bool(kind & 2), chunk_frames=chunk,
                    w0=w0, gamma_shift=g, lam=lam)
    n_k = len(kvalid)
    bits = np.arange(32, dtype=np.uint32)
    for qt in (range(len(rp) - 1) if q_tiles is None else q_tiles):
        q0, q1 = qt * 128, min(n_q, qt * 128 + 128)
        ref = oracle.mask_rows(tuple(p[q0:q1] for p in qpos), kpos, kvalid, m).astype(bool)
        cover = np.zeros((q1 - q0, n_k + 128), np.int32)
        for e in range(rp[qt], rp[qt + 1]):
            k0 = int(kr[e])
            assert 0 <= k0 < n_k
            if mi[e] < 0:
                blk = np.ones((128, 128), bool)
            else:
                blk = ((words[mi[e]][:, :, None] >> bits) & 1).reshape(128, 128).astype(bool)
            cover[:, k0:k0 + 128] += blk[:q1 - q0]
        assert cover.max(initial=0) <= 1, qt          # no pair twice
        assert not cover[:, n_k:].any(), qt             # nothing past the last key
        assert np.array_equal(cover[:, :n_k].astype(bool), ref), qt


@pytest.mark.parametrize("wid", sorted(WORKLOADS))
def test_kernel_work_list_covers_the_mask_once_workloads(wid):
    w = WORKLOADS[wid]
    first, last = w.window()
    plan = vdit.Plan(_geom(w), _mask(w), w.q_start, w.q_frames, capacity_frames=w.capacity_frames,
                     kv_first_frame=first, kv_last_frame=last, upload=False)
    n_qt = plan.info["q_tiles"]
    sample = None if n_qt <= 8 else sorted({0, 1, n_qt // 3, n_qt // 2, (2 * n_qt) // 3, n_qt - 2, n_qt - 1})
    _check_work(plan, w.grid_h, w.grid_w, w.q_start, w.q_frames, w.capacity_frames, first, last,
                w.mask_kind, w.chunk_frames, w.w0, w.gamma_shift, w.lam, sample)
    info = plan.info
    if w.mask_kind & 2:
        # the radial workloads take their single-patch pairs off the aligned tiles
        assert info["single_patch_entries"] > 0 and info["work_entries"] < info["tiles"]
    else:
        assert info["single_patch_entries"] == 0 and info["work_entries"] == info["tiles"]


@pytest.mark.parametrize("kind,q_start,q_frames,cap,last", [(2, 0, 9, 9, 8), (3, 9, 3, 10, 11),
                                                            (2, 2, 5, 8, 7)])
def test_kernel_work_list_medium_single_patch_cases(kind, q_start, q_frames, cap, last):
    # the medium geometries the GPU parity tests run in full (8 x 20 patches, radius 4 >> dt)
    first = max(0, last - cap + 1)
    g = vdit.Geometry(8, 20, 2, 128, (44, 42, 42))
    plan = vdit.Plan(g, vdit.Mask(kind, 3, 4, 1, 0), q_start, q_frames, capacity_frames=cap,
                     kv_first_frame=first, kv_last_frame=last, upload=False)
    assert plan.info["single_patch_entries"] > 0
    _check_work(plan, 8, 20, q_start, q_frames, cap, first, last, kind, 3, 4, 1, 0)


def test_kernel_work_list_covers_the_mask_once_random_geometries():
    # frames of at least 128 tokens (where single-patch entries apply), rings that wrap, both
    # causal and not, radial radii that reach 0 within the window
    rng = np.random.default_rng(12)
    n_single = 0
    for _ in range(24):
        gh, gw = int(rng.integers(4, 14)), int(rng.integers(32, 60))
        cap = int(rng.integers(3, 14))
        last = int(rng.integers(0, 40))
        first = max(0, last - int(rng.integers(0, cap)))
        q_frames = int(rng.integers(1, 4))
        q_start = int(rng.integers(max(0, last - 6), last + 2))
        kind = int(rng.choice([2, 3]))
        chunk = int(rng.integers(1, 4))
        w0, gs, lam = int(rng.integers(0, 20)), int(rng.integers(1, 3)), int(rng.integers(0, 7))
        g = vdit.Geometry(gh, gw, 1, 64, (24, 20, 20))
        plan = vdit.Plan(g, vdit.Mask(kind, chunk, w0, gs, lam), q_start, q_frames,
                         capacity_frames=cap, kv_first_frame=first, kv_last_frame=last, upload=False)
        _check_work(plan, gh, gw, q_start, q_frames, cap, first, last, kind, chunk, w0, gs, lam)
        n_single += plan.info["single_patch_entries"]
    assert n_single > 0


@pytest.mark.parametrize("wid", sorted(WORKLOADS))
def test_plan_masks_bit_exact_vs_oracle_workloads(wid):
    w = WORKLOADS[wid]
    first, last = w.window()
    plan = vdit.Plan(_geom(w), _mask(w), w.q_start, w.q_frames, capacity_frames=w.capacity_frames,
                     kv_first_frame=first, kv_last_frame=last, upload=False)
    n_qt = plan.info["q_tiles"]
    # full-size workloads: the first, the last (ragged) and a spread of q-tiles in between
    sample = None if n_qt <= 8 else sorted({0, 1, n_qt // 3, n_qt // 2, (2 * n_qt) // 3, n_qt - 2, n_qt - 1})
    _check_masks(plan, w.grid_h, w.grid_w, w.q_start, w.q_frames, w.capacity_frames, first, last,
                 w.mask_kind, w.chunk_frames, w.w0, w.gamma_shift, w.lam, sample)


def test_plan_masks_bit_exact_vs_oracle_random_geometries():
    rng = np.random.default_rng(11)
    for _ in range(40):
        gh, gw = int(rng.integers(1, 9)), int(rng.integers(1, 40))
        cap = int(rng.integers(1, 12))
        last = int(rng.integers(0, 40))
        first = max(0, last - int(rng.integers(0, cap)))
        q_frames = int(rng.integers(1, 6))
        q_start = int(rng.integers(max(0, last - 8), last + 3))
        kind = int(rng.integers(0, 4))
        chunk = int(rng.integers(1, 5))
        w0 = int(rng.integers(0, 60))
        gs = int(rng.integers(0, 3))
        lam = int(rng.integers(0, 6))
        g = vdit.Geometry(gh, gw, 1, 64, (24, 20, 20))
        plan = vdit.Plan(g, vdit.Mask(kind, chunk, w0, gs, lam), q_start, q_frames,
                         capacity_frames=cap, kv_first_frame=first, kv_last_frame=last, upload=False)
        _check_masks(plan, gh, gw, q_start, q_frames, cap, first, last, kind, chunk, w0, gs, lam)


def test_plan_does_not_depend_on_the_host_thread_count(monkeypatch):
    """vdit_attn_plan computes query tiles on host threads and merges them in tile order: one,
    three and seven threads give the same tile lists, keep-mask blocks (numbering included) and
    work list."""
    def snapshot(w):
        first, last = w.window()
        plan = vdit.Plan(_geom(w), _mask(w), w.q_start, w.q_frames, capacity_frames=w.capacity_frames,
                         kv_first_frame=first, kv_last_frame=last, upload=False)
        return [np.ascontiguousarray(a) for a in (*plan.export(), *plan.export_masks(), *plan.export_work())]
    for wid in (4, 5):
        w = WORKLOADS[wid]
        got = []
        for n in ("1", "3", "7"):
            monkeypatch.setenv("VDIT_PLAN_THREADS", n)
            got.append(snapshot(w))
        for other in got[1:]:
            assert all(np.array_equal(a, b) for a, b in zip(got[0], other))


def _plan_of(w):
    first, last = w.window()
    return vdit.Plan(_geom(w), _mask(w), w.q_start, w.q_frames, capacity_frames=w.capacity_frames,
                     kv_first_frame=first, kv_last_frame=last, upload=False)


def _list_schedule_span(lengths, sms, fixed=12.0):
    """Makespan of CTAs of the given entry counts dispatched in order, each to the SM that frees
    first, a CTA costing its entries plus `fixed`."""
    import heapq
    free = [0.0] * sms
    for n in lengths:
        heapq.heapreplace(free, free[0] + n + fixed)
    return max(free)


def _check_schedule(plan, heads, sms, dynamic=False):
    """The CTA schedule (vdit_plan_export_schedule) runs every (q-block, head) unit's union list
    exactly once: whole (slot -1), or cut into consecutive pieces of at least 8 entries, each with
    its own partial slot, listed once in the merge table; head-major launch order; slots within
    the no-allocation buffer. Returns (cta, merge, unit lengths)."""
    whole, none = plan.schedule_for(1)  # one SM: nothing to balance, every unit whole
    assert len(none) == 0 and (whole[:, 2] == 0).all() and (whole[:, 4] == -1).all()
    length = {(int(r[0]), int(r[1])): int(r[3]) for r in whole}
    assert len(length) == len(whole) == plan.info["q_tiles"] // 2 * heads + (plan.info["q_tiles"] % 2) * heads
    cta, merge = plan.schedule_for(sms)
    assert (np.diff(cta[:, 1]) >= 0).all()                      # head-major
    pieces = {}
    for qb, hd, e0, n, slot in cta.tolist():
        pieces.setdefault((qb, hd), []).append((e0, n, slot))
    assert set(pieces) == set(length)
    slots = sorted(int(x) for x in cta[:, 4] if x >= 0)
    assert slots == list(range(len(slots)))                     # each slot used once
    assert len(slots) <= 32768 // (plan.g.head_dim + 1)
    cut = {(int(r[0]), int(r[1])): (int(r[2]), int(r[3])) for r in merge}
    assert len(cut) == len(merge)
    for u, ps in pieces.items():
        if len(ps) == 1 and u not in cut:
            assert ps[0] == (0, length[u], -1), u
            continue
        first, k = cut[u]
        assert k == len(ps) >= 2, u
        assert [p[2] for p in ps] == list(range(first, first + k)), u
        at = 0
        for e0, n, _ in ps:
            assert e0 == at and n >= 8, u
            at += n
        assert at == length[u], u
    if dynamic:
        assert len(merge) == 0
    return cta, merge, length


@pytest.mark.parametrize("wid", sorted(WORKLOADS))
def test_cta_schedule_covers_every_unit_once(wid):
    w = WORKLOADS[wid]
    plan = _plan_of(w)
    for sms in (148, 7, 1000):
        _check_schedule(plan, w.heads, sms, dynamic=bool(w.mask_kind & 4))


def test_cta_schedule_shortens_the_modelled_launch():
    """On a 148-SM B200 the cut schedule fills the last wave: the modelled makespan of the
    exported CTA table (list scheduling in launch order) is well below the whole-unit one on the
    dense, causal-chunk and 14B-rollout shapes (1 536, 228 and 760 units: 10.4, 1.5 and 5.1
    waves) and never above it; the dynamic threshold never cuts; one head of the causal chunk
    (19 units) is cut over the SMs."""
    for wid, gain in ((2, 0.04), (3, 0.10), (4, 0.0), (5, 0.05), (6, 0.0)):
        w = WORKLOADS[wid]
        plan = _plan_of(w)
        cta, merge, length = _check_schedule(plan, w.heads, 148, dynamic=bool(w.mask_kind & 4))
        whole, _ = plan.schedule_for(1)
        t_whole = _list_schedule_span(whole[:, 3], 148)
        t_cut = _list_schedule_span(cta[:, 3], 148)
        assert t_cut <= t_whole * (1 - gain), (wid, t_cut, t_whole)
        if w.mask_kind & 4:
            assert len(merge) == 0 and len(cta) == len(whole)
    # query blocks with empty lists (chunk 0 against a cache holding only frame 3) run whole
    for q_start, q_frames in ((0, 1), (2, 2)):
        empty = Workload(93, "no-keys", grid_h=6, grid_w=10, heads=2, head_dim=128, bands=(44, 42, 42),
                         mask_kind=1, q_start=q_start, q_frames=q_frames, capacity_frames=4,
                         appends=((3, 1),), kv_stream_first_frame=3, chunk_frames=3)
        for sms in (1, 2, 148):
            cta, merge, length = _check_schedule(_plan_of(empty), 2, sms)
            assert len(cta) == len(length) and len(merge) == 0
    one = Workload(**{**WORKLOADS[3].__dict__, "id": 95, "heads": 1})
    cta, merge, _ = _check_schedule(_plan_of(one), 1, 148)
    assert len(merge) == len(_plan_of(one).schedule_for(1)[0]) and len(cta) > 100
    with pytest.raises(vdit.VditError):
        _plan_of(one).schedule_for(0)


def test_plan_rejects_bad_arguments():
    L = vdit.lib()
    g = vdit.Geometry(30, 52, 12, 128, (44, 42, 42)).c()
    m = vdit.Mask.block_causal(3).c()
    h = ctypes.c_void_p()
    assert L.vdit_attn_plan(ctypes.byref(h), ctypes.byref(g), ctypes.byref(m), 0, 3, 21, 5, 2) == vdit.ERR_INVALID_ARG
    assert L.vdit_attn_plan(ctypes.byref(h), ctypes.byref(g), ctypes.byref(m), 0, 3, 2, 0, 5) == vdit.ERR_INVALID_ARG
    assert b"window" in L.vdit_last_error()
    bad = vdit.Geometry(30, 52, 12, 96, (32, 32, 32)).c()
    assert L.vdit_attn_plan(ctypes.byref(h), ctypes.byref(bad), ctypes.byref(m), 0, 3, 21, 0, 20) == vdit.ERR_UNSUPPORTED
    odd = vdit.Geometry(30, 52, 12, 128, (43, 43, 42)).c()
    assert L.vdit_attn_plan(ctypes.byref(h), ctypes.byref(odd), ctypes.byref(m), 0, 3, 21, 0, 20) == vdit.ERR_INVALID_ARG
    far = vdit.Mask.radial().c()
    assert L.vdit_attn_plan(ctypes.byref(h), ctypes.byref(g), ctypes.byref(far), 5000, 3, 21, 0, 20) == vdit.ERR_UNSUPPORTED


def test_calls_reject_null_and_misaligned_pointers_before_device_work():
    L = vdit.lib()
    g = vdit.Geometry(30, 52, 12, 128, (44, 42, 42)).c()
    assert L.vdit_rope3d_apply(ctypes.byref(g), None, None, 0, 10, None) == vdit.ERR_INVALID_ARG
    assert L.vdit_rope3d_apply(ctypes.byref(g), ctypes.c_void_p(8), ctypes.c_void_p(16), 0, 10, None) == vdit.ERR_MISALIGNED
    assert L.vdit_rope3d_apply(ctypes.byref(g), None, None, 0, 0, None) == vdit.OK  # empty is a no-op
    assert L.vdit_kv_append(ctypes.byref(g), ctypes.c_void_p(16), ctypes.c_void_p(32), 21,
                            ctypes.c_void_p(48), ctypes.c_void_p(64), 0, 22, None) == vdit.ERR_INVALID_ARG
    h = ctypes.c_void_p()
    m = vdit.Mask().c()
    assert L.vdit_attn_plan(ctypes.byref(h), ctypes.byref(g), ctypes.byref(m), 0, 21, 21, 0, 20) == vdit.OK
    assert L.vdit_attn_forward(h, ctypes.c_void_p(16), ctypes.c_void_p(16), ctypes.c_void_p(16),
                               ctypes.c_void_p(16), None, ctypes.c_float(0.1), None) == vdit.ERR_NOT_UPLOADED
    L.vdit_plan_destroy(h)
    # the peer-memory exchange: destination arrays checked entry by entry, ranks bounded
    ok = (ctypes.c_void_p * 2)(16, 32)
    null = (ctypes.c_void_p * 2)(16, 0)
    odd = (ctypes.c_void_p * 2)(16, 40)
    args = (ctypes.byref(g), ctypes.c_void_p(1 << 20), ctypes.c_void_p(2 << 20), ctypes.c_void_p(3 << 20))
    assert L.vdit_seq_pack_peers(*args, ok, ok, ok, 0, 2, 0, 0, 1, None) == vdit.OK  # empty: no-op
    assert L.vdit_seq_pack_peers(*args, null, ok, ok, 0, 2, 0, 5, 1, None) == vdit.ERR_INVALID_ARG
    assert L.vdit_seq_pack_peers(*args, ok, odd, ok, 0, 2, 0, 5, 1, None) == vdit.ERR_MISALIGNED
    assert L.vdit_seq_pack_peers(*args, ok, ok, ok, 0, 5, 0, 5, 1, None) == vdit.ERR_INVALID_ARG  # 5 !| 12
    assert L.vdit_seq_pack_peers(*args, ok, ok, ok, 2, 2, 0, 5, 1, None) == vdit.ERR_INVALID_ARG  # rank
    many = (ctypes.c_void_p * 24)(*[16] * 24)
    g24 = vdit.Geometry(30, 52, 24, 128, (44, 42, 42)).c()
    assert L.vdit_seq_pack_peers(ctypes.byref(g24), *args[1:], many, many, many, 0, 24, 0, 5, 1,
                                 None) == vdit.ERR_INVALID_ARG  # more ranks than VDIT_MAX_PEERS
    assert L.vdit_seq_push_peers(ctypes.byref(g), ctypes.c_void_p(16), null, 0, 2, 5, None) == vdit.ERR_INVALID_ARG
    assert L.vdit_seq_push_peers(ctypes.byref(g), ctypes.c_void_p(16), odd, 0, 2, 5, None) == vdit.ERR_MISALIGNED
    assert L.vdit_seq_push_peers(ctypes.byref(g), ctypes.c_void_p(16), ok, 0, 2, 0, None) == vdit.OK


def test_plan_and_masks_bit_exact_on_the_gpu_edge_workloads():
    # the degenerate grids and masks of the GPU edge tests: 1 x 1 grid, lambda 1, w0 0, chunks of
    # one frame, the last frames of the time table, a 2 x 1024 grid
    from test_gpu_edges import EDGES
    for name, w in EDGES.items():
        first, last = w.window()
        plan = vdit.Plan(_geom(w), _mask(w), w.q_start, w.q_frames, capacity_frames=w.capacity_frames,
                         kv_first_frame=first, kv_last_frame=last, upload=False)
        ref = _oracle_tiles(w.grid_h, w.grid_w, w.q_start, w.q_frames, w.capacity_frames, first, last,
                            w.mask_kind, w.chunk_frames, w.w0, w.gamma_shift, w.lam)
        _compare(plan, ref)
        _check_masks(plan, w.grid_h, w.grid_w, w.q_start, w.q_frames, w.capacity_frames, first, last,
                     w.mask_kind, w.chunk_frames, w.w0, w.gamma_shift, w.lam)
