"""The multi-GPU bench path runs one independent replica per rank (weak scaling); its only
collective is the max-over-ranks step time. This checks that reduction and the whole-job
throughput formula with two gloo ranks on CPU."""
import os
import socket

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


# ----------------------------------------------------------------------------- sequence -> heads

def _oracle_pack(x, send, g, start_frame, tok0, n_ranks, rotate=True, stream=None):
    """CPU stand-in of vdit_seq_pack for the gloo test (test infrastructure: the oracle's RoPE
    at the tokens' global positions, then the [ranks, tokens, heads / ranks, D] layout)."""
    import numpy as np
    import oracle
    n = x.shape[0]
    y = x.double().numpy()
    if rotate:
        pos = oracle.positions(tok0 + n, g.grid_h, g.grid_w, start_frame)
        og = oracle.Geometry(g.grid_h, g.grid_w, g.heads, g.head_dim, *g.bands, g.theta)
        y = oracle.rope3d(y, tuple(p[tok0:] for p in pos), og)
    hpr = g.heads // n_ranks
    send.copy_(torch.from_numpy(np.ascontiguousarray(
        y.reshape(n, n_ranks, hpr, g.head_dim).transpose(1, 0, 2, 3))).to(send.dtype))
    return send


def _seq_worker(rank, world, port, out):
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    import numpy as np
    import oracle
    import synth
    import video_diffusion_transformer_vdit_b200 as vdit
    vdit.seq_pack = _oracle_pack  # the pack kernel needs a GPU; the exchange logic does not
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world)
    try:
        g = vdit.Geometry(3, 5, 4, 64, (24, 20, 20))
        n_all = 2 * 15 + 6                       # a chunk of 36 tokens (2.4 frames of 3 x 5)
        full = synth.bf16_bits_to_f64(synth.qkv_bf16(7, n_all, 4, 64, "q"))
        n = n_all // world
        x = torch.from_numpy(full[rank * n:(rank + 1) * n]).float()
        got = vdit.seq_to_heads(x, g, 9, rotate=True)
        # the oracle's whole-chunk RoPE, this rank's heads
        og = oracle.Geometry(3, 5, 4, 64, 24, 20, 20, 10000.0)
        ref = oracle.rope3d(full, oracle.positions(n_all, 3, 5, 9), og)[:, rank * 2:(rank + 1) * 2]
        out[rank] = float(np.abs(got.double().numpy() - ref).max())
    finally:
        dist.destroy_process_group()


def test_seq_to_heads_exchange_gloo_two_ranks():
    world = 2
    port = _free_port()
    with mp.Manager() as man:
        out = man.dict()
        mp.spawn(_seq_worker, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    # float32 transport of float64 values: exact up to float32 rounding
    assert res[0] < 1e-5 and res[1] < 1e-5


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
