"""GPU parity of the sequence-to-head pack (vdit_seq_pack): the oracle's RoPE at the shard's global
positions, then the [ranks, tokens, heads / ranks, D] layout. Rotated values within the bf16
rounding bound of the RoPE tests; the unrotated pack (V) bit-exact."""
import numpy as np
import pytest
import torch

import oracle
import synth
import video_diffusion_transformer_vdit_b200 as vdit

from _parity import dev, f64, rope_tolerance

pytestmark = pytest.mark.gpu

G13 = vdit.Geometry(30, 52, 12, 128, (44, 42, 42))


def _reference(bits, g, start, tok0, ranks, rotate):
    n = bits.shape[0]
    y = synth.bf16_bits_to_f64(bits)
    if rotate:
        pos = oracle.positions(tok0 + n, g.grid_h, g.grid_w, start)
        og = oracle.Geometry(g.grid_h, g.grid_w, g.heads, g.head_dim, *g.bands, g.theta)
        y = oracle.rope3d(y, tuple(p[tok0:] for p in pos), og)
    hpr = g.heads // ranks
    return np.ascontiguousarray(y.reshape(n, ranks, hpr, g.head_dim).transpose(1, 0, 2, 3))


@pytest.mark.parametrize("ranks", [1, 2, 3, 4])
def test_seq_pack_rotated_matches_oracle(ranks):
    # a shard of 1 000 tokens (ragged against frames and warps) that starts 2 000 tokens into a
    # chunk at global frame 396 (the long-rollout positions)
    n, tok0, start = 1000, 2000, 396
    bits = synth.qkv_bf16(81, n, 12, 128, "q")
    send = torch.empty(ranks, n, 12 // ranks, 128, dtype=torch.bfloat16, device="cuda")
    vdit.seq_pack(dev(bits), send, G13, start, tok0, ranks, rotate=True)
    torch.cuda.synchronize()
    ref = _reference(bits, G13, start, tok0, ranks, True)
    x64 = synth.bf16_bits_to_f64(bits).reshape(n, ranks, 12 // ranks, 128).transpose(1, 0, 2, 3)
    assert np.all(np.abs(f64(send) - ref) <= rope_tolerance(ref, x64))


def test_seq_pack_unrotated_is_an_exact_permutation():
    n = 777
    bits = synth.qkv_bf16(82, n, 12, 128, "v")
    send = torch.empty(3, n, 4, 128, dtype=torch.bfloat16, device="cuda")
    vdit.seq_pack(dev(bits), send, G13, 0, 0, 3, rotate=False)
    torch.cuda.synchronize()
    ref = _reference(bits, G13, 0, 0, 3, False)
    assert np.array_equal(f64(send), ref)


def test_seq_to_heads_single_rank_equals_rope():
    # one rank: the exchange is the identity layout and the rotation is vdit_rope3d_apply's
    bits = synth.qkv_bf16(83, 3 * 1560, 12, 128, "q")
    x = dev(bits)
    a = vdit.seq_to_heads(x, G13, 18)
    b = vdit.rope3d_apply(x, G13, 18)
    torch.cuda.synchronize()
    assert torch.equal(a, b)


def test_seq_pack_rejects_heads_not_divisible():
    x = torch.zeros(16, 12, 128, dtype=torch.bfloat16, device="cuda")
    send = torch.zeros(5, 16, 2, 128, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(ValueError):
        vdit.seq_pack(x, send, G13, 0, 0, 5)
