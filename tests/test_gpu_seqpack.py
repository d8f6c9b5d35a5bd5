"""GPU parity of the sequence-parallel exchange kernels and of the attention step they serve
("Accelerating Video Generation Inference with Sequential-Parallel 3D Positional Encoding Using a
Global Time Index", sections 2.A-2.C): vdit_seq_pack (RoPE of Q and K at the shard's global
positions, Q, K and V into the all-to-all layout in one launch), vdit_seq_unpack (the return
layout), vdit_kv_write and vdit_attn_forward_rotated (the consumers of rotated data). The ranks of
a group are emulated on the one device: each rank's kernels run in turn and the test copies the
blocks an exchange would move; no kernel waits on another."""
import numpy as np
import pytest
import torch

import oracle
import synth
import video_diffusion_transformer_vdit_b200 as vdit
from video_diffusion_transformer_vdit_b200.workloads import WORKLOADS

from _parity import assert_close, dev, f64, geom, inputs, mask, rope_tolerance, run_oracle

pytestmark = pytest.mark.gpu

G13 = vdit.Geometry(30, 52, 12, 128, (44, 42, 42))


def _pack_all(q, k, v, g, start, ranks):
    """Every rank's pack of its token shard; returns per rank (send, (q_full, k_full, v_full))."""
    n = q.shape[0] // ranks
    hg = g.heads // ranks
    out = []
    for r in range(ranks):
        sl = slice(r * n, (r + 1) * n)
        send = torch.full((ranks, 3, n, hg, g.head_dim), float("nan"), dtype=torch.bfloat16, device="cuda") \
            if ranks > 1 else None
        full = tuple(torch.full((ranks * n, hg, g.head_dim), float("nan"), dtype=torch.bfloat16, device="cuda")
                     for _ in range(3))
        vdit.seq_pack(q[sl], k[sl], v[sl], g, start, r, ranks, send, full)
        out.append((send, full))
    return out


def _exchange_on_one_device(packs, n):
    """What the all-to-all moves: rank s's send block r lands in rank r's rows s * n .. ."""
    ranks = len(packs)
    for r in range(ranks):
        for s in range(ranks):
            if s != r:
                for x in range(3):
                    packs[r][1][x][s * n:(s + 1) * n].copy_(packs[s][0][r, x])


@pytest.mark.parametrize("ranks", [1, 2, 3, 4])
def test_seq_pack_matches_oracle(ranks):
    # a 3-frame chunk at global frame 396 (the long-rollout positions) split over the ranks; after
    # the emulated exchange each rank's head-sharded Q and K are the oracle's RoPE of the whole
    # chunk at global positions (within the RoPE bound), V is an exact copy
    n_all, start = 3 * 1560, 396
    qb, kb, vb = (synth.qkv_bf16(81, n_all, 12, 128, w) for w in ("q", "k", "v"))
    packs = _pack_all(dev(qb), dev(kb), dev(vb), G13, start, ranks)
    _exchange_on_one_device(packs, n_all // ranks)
    torch.cuda.synchronize()
    og = oracle.Geometry(30, 52, 12, 128, 44, 42, 42, 10000.0)
    pos = oracle.positions(n_all, 30, 52, start)
    rng = np.random.default_rng(ranks)
    rows = np.unique(np.r_[rng.integers(0, n_all, 400), np.arange(n_all - 40, n_all), np.arange(40)])
    hg = 12 // ranks
    for which, bits in ((0, qb), (1, kb), (2, vb)):
        x64 = synth.bf16_bits_to_f64(bits[rows])
        ref = oracle.rope3d(x64, tuple(p[rows] for p in pos), og) if which < 2 else x64
        for r in range(ranks):
            got = f64(packs[r][1][which])[rows]
            sl = slice(r * hg, (r + 1) * hg)
            if which < 2:
                assert np.all(np.abs(got - ref[:, sl]) <= rope_tolerance(ref[:, sl], x64[:, sl]))
            else:
                assert np.array_equal(got, ref[:, sl])


def test_seq_pack_rotation_equals_rope3d_apply_bits():
    # the pack's rotation is the same fp32 arithmetic as vdit_rope3d_apply: identical bits
    n = 2 * 1560 + 77
    qb, kb, vb = (synth.qkv_bf16(82, 2 * n, 12, 128, w) for w in ("q", "k", "v"))
    q, k, v = dev(qb), dev(kb), dev(vb)
    packs = _pack_all(q, k, v, G13, 18, 2)
    _exchange_on_one_device(packs, n)
    rq, rk = vdit.rope3d_apply(q, G13, 18), vdit.rope3d_apply(k, G13, 18)
    torch.cuda.synchronize()
    for r in range(2):
        sl = slice(6 * r, 6 * r + 6)
        assert torch.equal(packs[r][1][0], rq[:, sl].contiguous())
        assert torch.equal(packs[r][1][1], rk[:, sl].contiguous())
        assert torch.equal(packs[r][1][2], v[:, sl].contiguous())


@pytest.mark.parametrize("ranks", [1, 2, 3])
def test_seq_unpack_is_the_inverse_layout(ranks):
    n = 1000
    hg = 12 // ranks
    o_bits = [synth.qkv_bf16(90 + r, ranks * n, hg, 128, "v") for r in range(ranks)]
    o_full = [dev(b) for b in o_bits]  # rank r's attention output: all tokens, its heads
    for r in range(ranks):
        recv = None
        if ranks > 1:
            recv = torch.full((ranks, n, hg, 128), float("nan"), dtype=torch.bfloat16, device="cuda")
            for s in range(ranks):
                if s != r:
                    recv[s].copy_(o_full[s][r * n:(r + 1) * n])
        out = torch.empty(n, 12, 128, dtype=torch.bfloat16, device="cuda")
        vdit.seq_unpack(recv, o_full[r][r * n:(r + 1) * n], out, G13, r, ranks)
        torch.cuda.synchronize()
        ref = np.concatenate([synth.bf16_bits_to_f64(o_bits[s][r * n:(r + 1) * n]) for s in range(ranks)], axis=1)
        assert np.array_equal(f64(out), ref)


def test_kv_write_is_an_exact_ring_copy():
    g = vdit.Geometry(3, 5, 3, 128, (44, 42, 42))
    cache = vdit.KVCache(g, 4)
    kb = synth.qkv_bf16(94, 3 * 15, 3, 128, "k")
    vb = synth.qkv_bf16(94, 3 * 15, 3, 128, "v")
    cache.write(dev(kb), dev(vb), 2)  # frames 2, 3, 4 -> slots 2, 3, 0
    torch.cuda.synchronize()
    k64, v64 = synth.bf16_bits_to_f64(kb), synth.bf16_bits_to_f64(vb)
    for f, slot in ((2, 2), (3, 3), (4, 0)):
        src = slice((f - 2) * 15, (f - 1) * 15)
        assert np.array_equal(f64(cache.k[:, slot * 15:(slot + 1) * 15]), k64[src].transpose(1, 0, 2))
        assert np.array_equal(f64(cache.v[:, slot * 15:(slot + 1) * 15]), v64[src].transpose(1, 0, 2))
    assert not cache.k[:, 15:30].float().abs().sum().item()  # slot 1 untouched
    assert (cache.first_frame, cache.last_frame) == (2, 4)


@pytest.mark.parametrize("ranks", [1, 2, 3])
def test_sequence_parallel_causal_chunk_matches_oracle(ranks):
    # the Wan2.1-1.3B causal chunk (3 frames at global frame 18 against 21 cached frames, 12 heads)
    # through the sequence-parallel step on `ranks` emulated ranks: pack -> exchange -> ring write
    # of the rotated K', V -> plan -> attention of the rank's heads with rotated Q -> return
    # exchange -> unpack; the concatenated outputs are checked on sampled rows against the oracle
    w = WORKLOADS[3]
    qb, kb, vb = inputs(w)
    ft = w.frame_tokens
    n_all = w.q_tokens
    n = n_all // ranks
    hg = w.heads // ranks
    s_last = w.appends[-1][0]
    kd, vd = dev(kb), dev(vb)
    chunk = slice(s_last * ft, (s_last + 3) * ft)
    packs = _pack_all(dev(qb), kd[chunk], vd[chunk], geom(w), w.q_start, ranks)
    _exchange_on_one_device(packs, n)
    o_full = []
    for r in range(ranks):
        gr = vdit.Geometry(w.grid_h, w.grid_w, hg, w.head_dim, w.bands, w.theta)
        cache = vdit.KVCache(gr, w.capacity_frames)
        hs = slice(r * hg, (r + 1) * hg)
        for s, nf in w.appends[:-1]:  # this rank's heads of the history
            cache.append(kd[s * ft:(s + nf) * ft, hs].contiguous(), vd[s * ft:(s + nf) * ft, hs].contiguous(), s)
        q_full, k_full, v_full = packs[r][1]
        cache.write(k_full, v_full, s_last)
        plan = vdit.Plan(gr, mask(w), w.q_start, w.q_frames, cache=cache)
        o_full.append(vdit.attn_forward(plan, q_full, cache, scale=w.scale, q_rotated=True))
    outs = []
    for r in range(ranks):
        recv = None
        if ranks > 1:
            recv = torch.empty(ranks, n, hg, w.head_dim, dtype=torch.bfloat16, device="cuda")
            for s in range(ranks):
                if s != r:
                    recv[s].copy_(o_full[s][r * n:(r + 1) * n])
        out = torch.empty(n, w.heads, w.head_dim, dtype=torch.bfloat16, device="cuda")
        outs.append(vdit.seq_unpack(recv, o_full[r][r * n:(r + 1) * n], out, geom(w), r, ranks))
    o = torch.cat(outs, 0)
    torch.cuda.synchronize()
    assert vdit.get_status() == vdit.OK
    rng = np.random.default_rng(30 + ranks)
    rows = np.unique(np.r_[np.arange(64), rng.integers(0, n_all, 96), np.arange(n_all - 100, n_all)])
    hs = [0, 5, 6, 11]
    ro, _ = run_oracle(w, qb, kb, vb, rows, hs)
    assert_close(f64(o[rows][:, hs]), ro)


def test_seq_to_heads_single_rank_and_return():
    # one rank: seq_to_heads is the pack alone (identity layout, Q and K rotated as
    # vdit_rope3d_apply), heads_to_seq the unpack alone (identity)
    qb, kb, vb = (synth.qkv_bf16(83, 3 * 1560, 12, 128, w) for w in ("q", "k", "v"))
    q, k, v = dev(qb), dev(kb), dev(vb)
    qf, kf, vf = vdit.seq_to_heads(q, k, v, G13, 18)
    back = vdit.heads_to_seq(vf, G13)
    torch.cuda.synchronize()
    assert torch.equal(qf, vdit.rope3d_apply(q, G13, 18))
    assert torch.equal(kf, vdit.rope3d_apply(k, G13, 18))
    assert torch.equal(vf, v) and torch.equal(back, v)


def test_seq_pack_rejects_bad_arguments():
    x = torch.zeros(16, 12, 128, dtype=torch.bfloat16, device="cuda")
    full = tuple(torch.zeros(16 * 5, 2, 128, dtype=torch.bfloat16, device="cuda") for _ in range(3))
    send = torch.zeros(5, 3, 16, 2, 128, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(ValueError):  # 5 ranks do not divide 12 heads
        vdit.seq_pack(x, x, x, G13, 0, 0, 5, send, full)
    full = tuple(torch.zeros(32, 6, 128, dtype=torch.bfloat16, device="cuda") for _ in range(3))
    send = torch.zeros(2, 3, 16, 6, 128, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(vdit.VditError):  # rank outside [0, n_ranks)
        vdit.seq_pack(x, x, x, G13, 0, 2, 2, send, full)
    with pytest.raises(vdit.VditError):  # two outputs overlapping
        vdit.seq_pack(x, x, x, G13, 0, 0, 2, send,
                      (full[0], full[1], send.view(-1)[:32 * 6 * 128].view(32, 6, 128)))


@pytest.mark.parametrize("wid", [3, 5])
def test_rotated_forward_equals_forward_on_rotated_queries(wid):
    # vdit_attn_forward_rotated on RoPE(q) (vdit_rope3d_apply at the plan's query positions) runs
    # the same kernel as vdit_attn_forward on q with the rotation in the Q load: bit-identical
    w = WORKLOADS[wid]
    qb, kb, vb = inputs(w)
    g = geom(w)
    cache = vdit.KVCache(g, w.capacity_frames)
    kd, vd = dev(kb), dev(vb)
    ft = w.frame_tokens
    for s, n in w.appends:
        off = (s - w.kv_stream_first_frame) * ft
        cache.append(kd[off:off + n * ft], vd[off:off + n * ft], s)
    plan = vdit.Plan(g, mask(w), w.q_start, w.q_frames, cache=cache)
    q = dev(qb)
    la = torch.empty(w.heads, w.q_tokens, device="cuda")
    lb = torch.empty_like(la)
    a = vdit.attn_forward(plan, q, cache, lse=la, scale=w.scale)
    b = vdit.attn_forward(plan, vdit.rope3d_apply(q, g, w.q_start), cache, lse=lb, scale=w.scale,
                          q_rotated=True)
    torch.cuda.synchronize()
    assert torch.equal(a, b) and torch.equal(la, lb)
    assert vdit.get_status() == vdit.OK


# ---------------------------------------------------------------- peer-memory form of the exchange

G64 = vdit.Geometry(6, 10, 4, 64, (24, 20, 20))


@pytest.mark.parametrize("ranks,d", [(1, 128), (2, 128), (3, 128), (4, 128), (2, 64), (4, 64)])
def test_seq_pack_peers_equals_pack_and_exchange(ranks, d):
    # vdit_seq_pack_peers writes each rank's rows straight into every rank's head-sharded
    # buffers (here all on the one device, one rank after the other): the result equals, bit for
    # bit, the pack into send blocks plus the exchange, for Q, K (rotated) and V
    g = G13 if d == 128 else G64
    n_all, start = (3 * 1560 + 12 * 7, 396) if d == 128 else (7 * 60 + 4 * 3, 11)
    qb, kb, vb = (synth.qkv_bf16(83, n_all, g.heads, d, w) for w in ("q", "k", "v"))
    q, k, v = dev(qb), dev(kb), dev(vb)
    n = n_all // ranks
    packs = _pack_all(q, k, v, g, start, ranks)
    _exchange_on_one_device(packs, n)
    hg = g.heads // ranks
    full = [tuple(torch.full((ranks * n, hg, d), float("nan"), dtype=torch.bfloat16, device="cuda")
                  for _ in range(3)) for _ in range(ranks)]
    addrs = [[full[r][x].data_ptr() for r in range(ranks)] for x in range(3)]
    for r in range(ranks):
        sl = slice(r * n, (r + 1) * n)
        vdit.seq_pack_peers(q[sl], k[sl], v[sl], g, start, r, ranks, *addrs)
    torch.cuda.synchronize()
    for r in range(ranks):
        for x in range(3):
            assert torch.equal(full[r][x], packs[r][1][x])


@pytest.mark.parametrize("ranks", [1, 2, 3])
def test_seq_push_peers_is_the_inverse_layout(ranks):
    n = 1000
    hg = 12 // ranks
    o_bits = [synth.qkv_bf16(95 + r, ranks * n, hg, 128, "v") for r in range(ranks)]
    o_full = [dev(b) for b in o_bits]
    outs = [torch.full((n, 12, 128), float("nan"), dtype=torch.bfloat16, device="cuda") for _ in range(ranks)]
    for r in range(ranks):
        vdit.seq_push_peers(o_full[r], G13, r, ranks, [o.data_ptr() for o in outs])
    torch.cuda.synchronize()
    for s in range(ranks):
        ref = np.concatenate([synth.bf16_bits_to_f64(o_bits[r][s * n:(s + 1) * n]) for r in range(ranks)], axis=1)
        assert np.array_equal(f64(outs[s]), ref)
