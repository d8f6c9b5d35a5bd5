"""Guard bands around every output buffer the kernels write (a bounds check while the CUDA
sanitizer is unavailable on the test machines): each output is the middle of a larger buffer whose
margins are filled with a bit pattern before the call and must hold it afterwards. The writes most
at risk: the ragged last query tile of attention (o, lse), the ring append across the end of the
ring, the fused QKV projection's tensor-memory stores (a chunk wrapping the ring: two launches), and
the sequence-parallel pack and unpack blocks."""
import numpy as np
import pytest
import torch

import synth
import video_diffusion_transformer_vdit_b200 as vdit
from video_diffusion_transformer_vdit_b200.workloads import Workload

from _parity import dev, geom, inputs, mask

pytestmark = pytest.mark.gpu

GUARD = 8192  # elements on each side (16 KiB of bf16, 32 KiB of fp32)


class Guarded:
    """A tensor of `shape` inside a 1-D buffer with GUARD pattern-filled elements on each side."""

    def __init__(self, shape, dtype=torch.bfloat16, fill=None):
        n = int(np.prod(shape))
        self.base = torch.empty(n + 2 * GUARD, dtype=dtype, device="cuda")
        ib = torch.int16 if dtype == torch.bfloat16 else torch.int32
        self.bits = self.base.view(ib)
        self.pattern = 0x5A5B if ib == torch.int16 else 0x5A5B5C5D
        self.bits.fill_(self.pattern)
        self.t = self.base[GUARD:GUARD + n].view(shape)
        if fill is not None:
            self.t.copy_(fill)

    def intact(self) -> bool:
        torch.cuda.synchronize()
        return bool((self.bits[:GUARD] == self.pattern).all() and (self.bits[-GUARD:] == self.pattern).all())


def _attention_case(w):
    q, k, v = inputs(w)
    g = geom(w)
    kc, vc = Guarded((w.heads, w.kv_tokens, w.head_dim)), Guarded((w.heads, w.kv_tokens, w.head_dim))
    kc.t.zero_()
    vc.t.zero_()
    cache = vdit.KVCache(g, w.capacity_frames)
    cache.k, cache.v = kc.t, vc.t
    kd, vd = dev(k), dev(v)
    ft = w.frame_tokens
    for s, n in w.appends:
        off = (s - w.kv_stream_first_frame) * ft
        cache.append(kd[off:off + n * ft], vd[off:off + n * ft], s)
    assert kc.intact() and vc.intact()
    plan = vdit.Plan(g, mask(w), w.q_start, w.q_frames, cache=cache)
    o = Guarded((w.q_tokens, w.heads, w.head_dim))
    lse = Guarded((w.heads, w.q_tokens), torch.float32)
    vdit.attn_forward(plan, dev(q), cache, out=o.t, lse=lse.t, scale=w.scale)
    assert o.intact() and lse.intact()
    assert torch.isfinite(o.t.float()).all()
    assert vdit.get_status() == vdit.OK
    return plan


@pytest.mark.parametrize("kind", [0, 3, 6])
def test_attention_outputs_guarded_ragged_last_tile(kind):
    # 9 frames x 6 x 10 = 540 queries = 4 x 128 + 28: a ragged last tile; ring of 8 frames with a
    # wrap (frames 4..12); dense, block-causal + radial, and radial with the dynamic threshold
    w = Workload(97, "guard", grid_h=6, grid_w=10, heads=3, head_dim=128, bands=(44, 42, 42),
                 mask_kind=kind, q_start=4, q_frames=9, capacity_frames=9,
                 appends=tuple((s, 3) for s in range(0, 12, 3)) + ((12, 1),), kv_stream_first_frame=0,
                 chunk_frames=3, w0=4, gamma_shift=1, lam=4, tau=2.0)
    _attention_case(w)


def test_attention_outputs_guarded_with_key_split():
    # one head of the Wan2.1-1.3B causal-chunk shape: the plan splits the keys, so the outputs are
    # written by the merge kernel (4,680 = 36 x 128 + 72 queries)
    w = Workload(98, "guard-split", grid_h=30, grid_w=52, heads=1, head_dim=128, bands=(44, 42, 42),
                 mask_kind=1, q_start=18, q_frames=3, capacity_frames=21,
                 appends=tuple((s, 3) for s in range(0, 21, 3)), kv_stream_first_frame=0)
    plan = _attention_case(w)
    assert plan.info["kv_splits"] > 1


def test_append_and_rope_guarded_across_the_ring_end():
    g = vdit.Geometry(5, 7, 3, 64, (24, 20, 20))
    ft = 35
    kc, vc = Guarded((3, 4 * ft, 64)), Guarded((3, 4 * ft, 64))
    kc.t.zero_()
    vc.t.zero_()
    k = dev(synth.qkv_bf16(61, 3 * ft, 3, 64, "k"))
    v = dev(synth.qkv_bf16(61, 3 * ft, 3, 64, "v"))
    vdit.kv_append(kc.t, vc.t, g, 4, k, v, 2)  # frames 2, 3, 4 -> slots 2, 3, 0
    vdit.kv_write(kc.t, vc.t, g, 4, k, v, 3)   # frames 3, 4, 5 -> slots 3, 0, 1
    assert kc.intact() and vc.intact()
    y = Guarded((3 * ft + 5, 3, 64))
    vdit.rope3d_apply(dev(synth.qkv_bf16(62, 3 * ft + 5, 3, 64, "q")), g, 9, out=y.t)
    assert y.intact()


def test_qkv_projection_guarded_two_launch_wrap():
    # 96 tokens (a ragged 128-row tile), frames 8..10 into slots 3, 4, 0 of a 5-frame ring
    g = vdit.Geometry(4, 8, 2, 128, (44, 42, 42))
    n, dm = 96, 192
    x = dev(synth.normal_bf16(511, n * dm).reshape(n, dm))
    wt = dev(synth.normal_bf16(512, 3 * 256 * dm, scale=dm ** -0.5).reshape(3 * 256, dm))
    kc, vc = Guarded((2, 5 * 32, 128)), Guarded((2, 5 * 32, 128))
    kc.t.zero_()
    vc.t.zero_()
    qo = Guarded((n, 2, 128))
    vdit.qkv_rope(x, wt, g, 8, kc.t, vc.t, 5, q_out=qo.t)
    assert kc.intact() and vc.intact() and qo.intact()
    assert vdit.get_status() == vdit.OK


@pytest.mark.parametrize("ranks", [2, 3])
def test_seq_pack_and_unpack_guarded(ranks):
    g = vdit.Geometry(30, 52, 12, 128, (44, 42, 42))
    n = 390
    hg = 12 // ranks
    q, k, v = (dev(synth.qkv_bf16(63, n, 12, 128, x)) for x in ("q", "k", "v"))
    send = Guarded((ranks, 3, n, hg, 128))
    full = [Guarded((ranks * n, hg, 128)) for _ in range(3)]
    vdit.seq_pack(q, k, v, g, 18, ranks - 1, ranks, send.t, tuple(f.t for f in full))
    assert send.intact() and all(f.intact() for f in full)
    out = Guarded((n, 12, 128))
    recv = Guarded((ranks, n, hg, 128), fill=torch.zeros(ranks, n, hg, 128, dtype=torch.bfloat16, device="cuda"))
    vdit.seq_unpack(recv.t, full[2].t[(ranks - 1) * n:ranks * n], out.t, g, ranks - 1, ranks)
    assert out.intact() and recv.intact()
