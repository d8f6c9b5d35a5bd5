"""The sequence-parallel exchange over peer memory (vdit.PeerExchange: "Accelerating Video
Generation Inference with Sequential-Parallel 3D Positional Encoding Using a Global Time Index",
section 2.C) with real CUDA IPC mappings: two gloo ranks share the one device, each allocates its
head-sharded buffers and output, the IPC handles are exchanged, and each rank's kernels write into
the other's buffers. The barrier between the ranks is a device synchronisation plus a host
barrier (gloo), so no kernel of one rank waits on the other's. Each rank's results must equal, bit
for bit, the single-process pack + exchange of the same inputs."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

pytestmark = pytest.mark.gpu

N_ALL, START = 2 * 1560 + 12 * 7, 396


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    sys.path.insert(0, os.path.join(root, "tests"))
    import synth
    import video_diffusion_transformer_vdit_b200 as vdit
    torch.cuda.set_device(0)
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world)
    try:
        g = vdit.Geometry(30, 52, 12, 128, (44, 42, 42))
        n = N_ALL // world

        def dev(bits):
            return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()

        q, k, v = (dev(synth.qkv_bf16(84, N_ALL, 12, 128, w))[rank * n:(rank + 1) * n] for w in ("q", "k", "v"))
        ex = vdit.PeerExchange(g, n)
        full = ex.seq_to_heads(q.contiguous(), k.contiguous(), v.contiguous(), START)
        got_full = [t.view(torch.int16).cpu().numpy().copy() for t in full]
        # the return exchange of a per-rank "attention output" (its heads, every token)
        o_full = dev(synth.qkv_bf16(85 + rank, world * n, 12 // world, 128, "v"))
        o = ex.heads_to_seq(o_full)
        torch.cuda.synchronize()
        assert vdit.get_status() == vdit.OK
        out[rank] = (got_full, o.view(torch.int16).cpu().numpy().copy())
        ex.close()  # collective: no rank unmaps while another may still write
        del ex
    finally:
        dist.destroy_process_group()


def test_peer_exchange_two_ranks_share_the_device():
    import synth
    import video_diffusion_transformer_vdit_b200 as vdit
    world = 2
    port = _free_port()
    with mp.Manager() as man:
        res = man.dict()
        mp.spawn(_worker, args=(world, port, res), nprocs=world, join=True)
        res = dict(res)
    g = vdit.Geometry(30, 52, 12, 128, (44, 42, 42))
    n = N_ALL // world
    hg = 12 // world
    q, k, v = (torch.from_numpy(synth.qkv_bf16(84, N_ALL, 12, 128, w).view(np.int16)).view(torch.bfloat16).cuda()
               for w in ("q", "k", "v"))
    # reference: the pack into send blocks plus the exchange, all ranks in this process
    packs = []
    for r in range(world):
        sl = slice(r * n, (r + 1) * n)
        send = torch.empty(world, 3, n, hg, 128, dtype=torch.bfloat16, device="cuda")
        full = tuple(torch.empty(world * n, hg, 128, dtype=torch.bfloat16, device="cuda") for _ in range(3))
        vdit.seq_pack(q[sl], k[sl], v[sl], g, START, r, world, send, full)
        packs.append((send, full))
    for r in range(world):
        for s in range(world):
            if s != r:
                for x in range(3):
                    packs[r][1][x][s * n:(s + 1) * n].copy_(packs[s][0][r, x])
    torch.cuda.synchronize()
    o_bits = [synth.qkv_bf16(85 + r, world * n, hg, 128, "v") for r in range(world)]
    for r in range(world):
        got_full, got_o = res[r]
        for x in range(3):
            assert np.array_equal(got_full[x], packs[r][1][x].view(torch.int16).cpu().numpy())
        ref_o = np.concatenate([o_bits[s].view(np.int16)[r * n:(r + 1) * n] for s in range(world)], axis=1)
        assert np.array_equal(got_o, ref_o)
