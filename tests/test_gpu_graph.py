"""CUDA-graph capture of the launching calls. A decode loop that runs many small launches per
step (the appends of every DiT block's cache, the attention of a 3-frame chunk) can capture them
once and replay the graph, taking the host's launch gaps out. These tests check that a captured
and replayed call gives bit-identical results to the same call launched eagerly, and that a
replay reads the current contents of the captured buffers (what a loop that refills its input
buffers relies on). The eager calls themselves are held to the oracle by the parity tests."""
import pytest
import torch

import video_diffusion_transformer_vdit_b200 as vdit
from video_diffusion_transformer_vdit_b200.workloads import WORKLOADS

pytestmark = pytest.mark.gpu


def _randn(shape, gen):
    return torch.randn(shape, device="cuda", generator=gen).to(torch.bfloat16)


def test_graph_of_block_appends_equals_eager_appends():
    # four blocks' caches (2 heads, 30 x 52 grid, 7-frame ring), 3-frame chunks at frames 0 .. 11:
    # the appends at 6 and 9 wrap the ring
    g = vdit.Geometry(30, 52, 2, 128, (44, 42, 42), 10000.0)
    cap, blocks, ft = 7, 4, 30 * 52
    gen = torch.Generator(device="cuda").manual_seed(5)
    src = [(_randn((3 * ft, 2, 128), gen), _randn((3 * ft, 2, 128), gen)) for _ in range(blocks)]
    eager = [vdit.KVCache(g, cap) for _ in range(blocks)]
    graphed = [vdit.KVCache(g, cap) for _ in range(blocks)]
    for s in (0, 3, 6, 9):
        for b in range(blocks):
            eager[b].append(src[b][0], src[b][1], s)  # also the first, uncaptured call per device
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            for b in range(blocks):
                graphed[b].append(src[b][0], src[b][1], s)
        graph.replay()
        torch.cuda.synchronize()
        for b in range(blocks):
            assert torch.equal(graphed[b].k, eager[b].k) and torch.equal(graphed[b].v, eager[b].v)
        # refill the sources in place; the same graph, replayed, appends the new contents
        for b in range(blocks):
            for t in src[b]:
                t.copy_(_randn(t.shape, gen))
            eager[b].append(src[b][0], src[b][1], s)
        graph.replay()
        torch.cuda.synchronize()
        for b in range(blocks):
            assert torch.equal(graphed[b].k, eager[b].k) and torch.equal(graphed[b].v, eager[b].v)
        del graph
    assert vdit.get_status() == vdit.OK


def test_graph_of_an_attention_step_equals_eager_step():
    # one step of the Wan2.1-1.3B block-causal chunk (3 query frames at frame 18 against the
    # 21-frame cache, 12 heads): the chunk's append, then the attention forward with its merge of
    # the units the plan's schedule cuts into key pieces
    w = WORKLOADS[3]
    g = vdit.Geometry(w.grid_h, w.grid_w, w.heads, w.head_dim, w.bands, w.theta)
    m = vdit.Mask(w.mask_kind, w.chunk_frames, w.w0, w.gamma_shift, w.lam, w.tau)
    ft = w.frame_tokens
    gen = torch.Generator(device="cuda").manual_seed(7)
    eager, graphed = vdit.KVCache(g, w.capacity_frames), vdit.KVCache(g, w.capacity_frames)
    for s, n in w.appends:
        k, v = _randn((n * ft, w.heads, w.head_dim), gen), _randn((n * ft, w.heads, w.head_dim), gen)
        eager.append(k, v, s)
        graphed.append(k, v, s)
    plan = vdit.Plan(g, m, w.q_start, w.q_frames, cache=eager)
    shape = (w.q_frames * ft, w.heads, w.head_dim)
    q, k, v = _randn(shape, gen), _randn(shape, gen), _randn(shape, gen)
    o = torch.empty_like(q)
    lse = torch.empty((w.heads, shape[0]), dtype=torch.float32, device="cuda")
    vdit.attn_forward(plan, q, eager, out=o, lse=lse, scale=w.scale)  # plan upload, device set-up
    assert plan.info["cut_units"] > 0  # the step has the merge launch too
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        graphed.append(k, v, w.q_start)
        vdit.attn_forward(plan, q, graphed, out=o, lse=lse, scale=w.scale)
    for _ in range(2):
        eager.append(k, v, w.q_start)
        o_ref = torch.empty_like(q)
        lse_ref = torch.empty_like(lse)
        vdit.attn_forward(plan, q, eager, out=o_ref, lse=lse_ref, scale=w.scale)
        graph.replay()
        torch.cuda.synchronize()
        assert torch.equal(o, o_ref) and torch.equal(lse, lse_ref)
        assert torch.equal(graphed.k, eager.k) and torch.equal(graphed.v, eager.v)
        for t in (q, k, v):  # the next step's inputs, written into the captured buffers
            t.copy_(_randn(t.shape, gen))
    del graph
    assert vdit.get_status() == vdit.OK
