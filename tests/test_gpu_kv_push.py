"""Wave Parallelism's K/V forward push (Wave Forcing / WaveRT: each layer's K/V are sent one way
ahead so the transfer hides under attention) with the real append kernel: two gloo ranks share the
one device; rank 0 appends each chunk to its own ring cache and pushes the chunk's K and V (as
given to the append) to rank 1, which receives them through host memory (gloo has no device
point-to-point) and appends them with vdit_kv_append on the device. The receiver's cache must equal
the sender's bit for bit and the oracle's within the RoPE bound (V exactly). No kernel of one rank
waits on the other's; the overlap of the push with attention is not measured here."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

pytestmark = pytest.mark.gpu

GRID, HEADS, D, BANDS, CAP = (6, 10), 4, 128, (44, 42, 42), 7
STARTS = (0, 3, 6, 9)  # four 3-frame chunks into a 7-frame ring: the last one wraps


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _chunk(start, which):
    import synth
    ft = GRID[0] * GRID[1]
    return synth.qkv_bf16(41, 3 * ft, HEADS, D, which, token_offset=ft * start)


def _worker(rank, world, port, out):
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    import video_diffusion_transformer_vdit_b200 as vdit
    torch.cuda.set_device(0)
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world)
    try:
        g = vdit.Geometry(*GRID, HEADS, D, BANDS)
        cache = vdit.KVCache(g, CAP, device="cuda")

        def dev(bits):
            return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()

        for start in STARTS:
            if rank == 0:
                k, v = dev(_chunk(start, "k")), dev(_chunk(start, "v"))
                cache.append(k, v, start)
                for wk in cache.push(k, v, 1):
                    wk.wait()
            else:
                cache.receive(start, 3, 0)
        torch.cuda.synchronize()
        assert vdit.get_status() == vdit.OK
        out[rank] = (cache.k.view(torch.int16).cpu().numpy().copy(),
                     cache.v.view(torch.int16).cpu().numpy().copy(), cache.first_frame, cache.last_frame)
    finally:
        dist.destroy_process_group()


def test_kv_push_receiver_cache_equals_sender_and_oracle():
    import oracle
    import synth
    from _parity import rope_tolerance
    world = 2
    port = _free_port()
    with mp.Manager() as man:
        res = man.dict()
        mp.spawn(_worker, args=(world, port, res), nprocs=world, join=True)
        res = dict(res)
    k0, v0, f0, l0 = res[0]
    k1, v1, f1, l1 = res[1]
    assert (f0, l0) == (f1, l1) == (5, 11)
    assert np.array_equal(k0, k1) and np.array_equal(v0, v1)
    # the receiver's ring against the oracle's appends of the same chunks
    ft = GRID[0] * GRID[1]
    og = oracle.Geometry(*GRID, HEADS, D, *BANDS, 10000.0)
    kc = np.zeros((HEADS, CAP * ft, D))
    vc = np.zeros_like(kc)
    kx = np.zeros_like(kc)
    for s in STARTS:
        kb, vb = synth.bf16_bits_to_f64(_chunk(s, "k")), synth.bf16_bits_to_f64(_chunk(s, "v"))
        oracle.kv_append(kc, vc, CAP, og, kb, vb, s, 3)
        for f in range(3):  # unrotated source of each slot, for the bound
            slot = (s + f) % CAP
            kx[:, slot * ft:(slot + 1) * ft] = kb[f * ft:(f + 1) * ft].transpose(1, 0, 2)
    got_k = synth.bf16_bits_to_f64(k1.view(np.uint16))
    got_v = synth.bf16_bits_to_f64(v1.view(np.uint16))
    assert np.array_equal(got_v, vc)
    assert np.all(np.abs(got_k - kc) <= rope_tolerance(kc, kx))
