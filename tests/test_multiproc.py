"""Multi-process host logic on gloo ranks (CPU): the bench's max-over-ranks step time and
whole-job throughput (its replicas share no data-path collective); the sequence-parallel
attention step (pack, one batched exchange of Q, K and V, ring write, attention of the rank's
heads, return exchange, unpack) with the oracle standing in for the device kernels; and Wave
Parallelism's K/V push."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world)
    try:
        ms = 10.0 + 5.0 * rank  # the slower rank sets the step time
        got = bench.max_over_ranks(ms, world)
        dist.barrier()
        out[rank] = (got, bench.aggregate_tflops(world, 6.594e12, got))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_weak_scaling_aggregate_gloo_two_ranks():
    world = 2
    port = _free_port()
    with mp.Manager() as man:
        out = man.dict()
        mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    assert res[0][0] == res[1][0] == 15.0
    # two replicas, each 6.594e12 FLOP per 15 ms step
    assert res[0][1] == pytest.approx(2 * 6.594e12 / 15e-3 / 1e12)


def test_single_rank_needs_no_process_group():
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    assert bench.max_over_ranks(3.5, 1) == 3.5
    assert bench.aggregate_tflops(1, 1e12, 1.0) == pytest.approx(1000.0)


# ----------------------------------------------------------------------------- sequence parallel

def _oracle_pack(q, k, v, g, start_frame, rank, n_ranks, send, full, rotate=True, stream=None):
    """CPU stand-in of vdit_seq_pack for the gloo test (test infrastructure: the oracle's RoPE of
    q and k at the shard's global positions, then the [ranks, 3, tokens, heads / ranks, D] send
    layout and the own block into the head-sharded buffers)."""
    import oracle
    n = q.shape[0]
    tok0 = rank * n
    og = oracle.Geometry(g.grid_h, g.grid_w, g.heads, g.head_dim, *g.bands, g.theta)
    pos = tuple(p[tok0:] for p in oracle.positions(tok0 + n, g.grid_h, g.grid_w, start_frame))
    xs = [t.double().numpy() for t in (q, k, v)]
    if rotate:
        xs[0], xs[1] = oracle.rope3d(xs[0], pos, og), oracle.rope3d(xs[1], pos, og)
    hg = g.heads // n_ranks
    for x in range(3):
        blocks = torch.from_numpy(xs[x].reshape(n, n_ranks, hg, g.head_dim).transpose(1, 0, 2, 3).copy())
        for r in range(n_ranks):
            if r == rank:
                full[x][rank * n:(rank + 1) * n] = blocks[r]
            else:
                send[r, x] = blocks[r]


def _oracle_unpack(recv, own, out, g, rank, n_ranks, stream=None):
    """CPU stand-in of vdit_seq_unpack (a copy)."""
    hg = g.heads // n_ranks
    for r in range(n_ranks):
        out[:, r * hg:(r + 1) * hg] = own if r == rank else recv[r]
    return out


SP_GRID = (3, 4)        # 12 tokens per latent frame
SP_HEADS, SP_D = 6, 64
# the chunk is frames 9..11 (36 tokens); the ring (10 frames) also holds frames 3..8


def _sp_inputs():
    import synth
    ft = SP_GRID[0] * SP_GRID[1]
    n_kv = 9 * ft  # frames 3..11
    k = synth.bf16_bits_to_f64(synth.qkv_bf16(31, n_kv, SP_HEADS, SP_D, "k"))
    v = synth.bf16_bits_to_f64(synth.qkv_bf16(31, n_kv, SP_HEADS, SP_D, "v"))
    q = synth.bf16_bits_to_f64(synth.qkv_bf16(31, 3 * ft, SP_HEADS, SP_D, "q"))
    return q, k, v


def _sp_reference():
    """Single-process oracle: the chunk's block-causal attention over frames 3..11, all heads."""
    import oracle
    q, k, v = _sp_inputs()
    gh, gw = SP_GRID
    ft = gh * gw
    og = oracle.Geometry(gh, gw, SP_HEADS, SP_D, 24, 20, 20, 10000.0)
    kc = np.zeros((SP_HEADS, 10 * ft, SP_D))
    vc = np.zeros_like(kc)
    for s in (3, 6, 9):
        off = (s - 3) * ft
        oracle.kv_append(kc, vc, 10, og, k[off:off + 3 * ft], v[off:off + 3 * ft], s, 3)
    kpos, kvalid = oracle.cache_positions(10, 3, 11, gh, gw)
    qpos = oracle.positions(3 * ft, gh, gw, 9)
    qrot = oracle.rope3d(q, qpos, og)
    m = oracle.mask_rows(qpos, kpos, kvalid, oracle.Mask(block_causal=True, chunk_frames=3))
    o, _ = oracle.attention(qrot, kc.transpose(1, 0, 2), vc.transpose(1, 0, 2), m, SP_D ** -0.5)
    return o


def _sp_worker(rank, world, port, out):
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    import oracle
    import video_diffusion_transformer_vdit_b200 as vdit
    # the pack / unpack kernels need a GPU; the exchange and the composition do not
    vdit.seq_pack = _oracle_pack
    vdit.seq_unpack = _oracle_unpack
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world)
    try:
        q, k, v = _sp_inputs()
        gh, gw = SP_GRID
        ft = gh * gw
        g = vdit.Geometry(gh, gw, SP_HEADS, SP_D, (24, 20, 20))
        n = 3 * ft // world
        sl = slice(rank * n, (rank + 1) * n)
        hg = SP_HEADS // world
        hs = slice(rank * hg, (rank + 1) * hg)
        t = lambda a: torch.from_numpy(np.ascontiguousarray(a))  # noqa: E731
        qf, kf, vf = vdit.seq_to_heads(t(q[sl]), t(k[6 * ft:][sl]), t(v[6 * ft:][sl]), g, 9)
        # this rank's cache holds its heads: the history (frames 3..8) appended by the oracle,
        # then the exchanged, already rotated chunk written into the ring as is
        og = oracle.Geometry(gh, gw, hg, SP_D, 24, 20, 20, 10000.0)
        kc = np.zeros((hg, 10 * ft, SP_D))
        vc = np.zeros_like(kc)
        for s in (3, 6):
            off = (s - 3) * ft
            oracle.kv_append(kc, vc, 10, og, k[off:off + 3 * ft][:, hs], v[off:off + 3 * ft][:, hs], s, 3)
        for f in range(3):  # kv_write: frame 9 + f -> slot (9 + f) mod 10
            slot = (9 + f) % 10
            kc[:, slot * ft:(slot + 1) * ft] = kf.numpy()[f * ft:(f + 1) * ft].transpose(1, 0, 2)
            vc[:, slot * ft:(slot + 1) * ft] = vf.numpy()[f * ft:(f + 1) * ft].transpose(1, 0, 2)
        kpos, kvalid = oracle.cache_positions(10, 3, 11, gh, gw)
        qpos = oracle.positions(3 * ft, gh, gw, 9)
        m = oracle.mask_rows(qpos, kpos, kvalid, oracle.Mask(block_causal=True, chunk_frames=3))
        o_full, _ = oracle.attention(qf.numpy(), kc.transpose(1, 0, 2), vc.transpose(1, 0, 2), m, SP_D ** -0.5)
        o = vdit.heads_to_seq(t(o_full), g)
        out[rank] = o.numpy().copy()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_sequence_parallel_attention_composition_gloo(world):
    # pack (RoPE at global positions) -> one batched exchange of Q, K, V -> ring write of the
    # rotated K', V -> attention of this rank's heads -> return exchange -> unpack, on `world`
    # gloo ranks; together the ranks' outputs equal the single-process attention of the chunk
    port = _free_port()
    with mp.Manager() as man:
        out = man.dict()
        mp.spawn(_sp_worker, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    got = np.concatenate([res[r] for r in range(world)], axis=0)
    ref = _sp_reference()
    assert got.shape == ref.shape
    assert np.abs(got - ref).max() < 1e-12


# ----------------------------------------------------------------------------- K/V push

def _oracle_append(k_cache, v_cache, g, capacity_frames, k, v, start_frame, stream=None):
    """CPU stand-in of vdit_kv_append for the gloo test (test infrastructure: the oracle's
    append, in float64, on CPU caches)."""
    import numpy as np
    import oracle
    og = oracle.Geometry(g.grid_h, g.grid_w, g.heads, g.head_dim, *g.bands, g.theta)
    kc, vc = k_cache.numpy(), v_cache.numpy()
    oracle.kv_append(kc, vc, capacity_frames, og, k.double().numpy(), v.double().numpy(),
                     start_frame, k.shape[0] // g.frame_tokens)


def _push_worker(rank, world, port, out):
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    import numpy as np
    import synth
    import video_diffusion_transformer_vdit_b200 as vdit
    vdit.kv_append = _oracle_append  # the append kernel needs a GPU; the push protocol does not
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world)
    try:
        g = vdit.Geometry(3, 4, 2, 64, (24, 20, 20))
        cache = vdit.KVCache(g, 5, device="cpu")
        cache.k, cache.v = cache.k.double(), cache.v.double()
        for start in (0, 3, 6):  # three chunks of 3 frames into a 5-frame ring (wraps)
            if rank == 0:
                k = torch.from_numpy(synth.bf16_bits_to_f64(synth.qkv_bf16(5, 36, 2, 64, "k", token_offset=12 * start)))
                v = torch.from_numpy(synth.bf16_bits_to_f64(synth.qkv_bf16(5, 36, 2, 64, "v", token_offset=12 * start)))
                cache.append(k, v, start)
                for wk in cache.push(k, v, 1):
                    wk.wait()
            else:
                cache.receive(start, 3, 0)
        out[rank] = (cache.k.double().numpy().copy(), cache.v.double().numpy().copy(),
                     cache.first_frame, cache.last_frame)
    finally:
        dist.destroy_process_group()


def test_kv_push_gloo_two_ranks():
    world = 2
    port = _free_port()
    with mp.Manager() as man:
        out = man.dict()
        mp.spawn(_push_worker, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    k0, v0, f0, l0 = res[0]
    k1, v1, f1, l1 = res[1]
    assert (f0, l0) == (f1, l1) == (4, 8)
    # the receiver appended exactly what the sender appended
    assert (k0 == k1).all() and (v0 == v1).all()
    assert abs(k0).max() > 0


# ----------------------------------------------------------------------------- head shards

def _shard_worker(rank, world, port, out):
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world)
    try:
        h0, h1 = bench.head_shard(12, world, rank)
        # per-rank FLOPs of a dense step on this rank's heads; step time: the slowest rank
        flops_rank = 4.0 * 128 * (h1 - h0) * 32760 * 32760
        got = bench.max_over_ranks(4.0 + rank, world)
        out[rank] = (h0, h1, got, bench.aggregate_tflops(world, flops_rank, got))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_head_shards_cover_the_heads_and_aggregate_strong_scaling(world):
    port = _free_port()
    with mp.Manager() as man:
        out = man.dict()
        mp.spawn(_shard_worker, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    spans = sorted((res[r][0], res[r][1]) for r in range(world))
    assert spans[0][0] == 0 and spans[-1][1] == 12
    assert all(a[1] == b[0] for a, b in zip(spans, spans[1:]))  # disjoint and contiguous
    slowest = 4.0 + world - 1
    assert all(res[r][2] == slowest for r in range(world))
    # the whole step (all 12 heads) over the slowest rank's time
    assert res[0][3] == pytest.approx(6.594e12 / (slowest * 1e-3) / 1e12, rel=1e-3)


def test_head_shard_rejects_an_uneven_split():
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    with pytest.raises(ValueError):
        bench.head_shard(12, 8, 0)
