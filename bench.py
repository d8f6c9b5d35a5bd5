"""Benchmark of the attention hot path: one step = KV append (RoPE of K at global frames + ring
write) + attention forward (RoPE of Q fused, masked online softmax on tcgen05) over one seeded
synthetic batch, on every GPU of one node.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload ID] [--impl reference]

Prints one JSON line on rank 0. For N > 1 launch with torch.distributed.run: each rank runs
its own independent step (weak scaling, no data-path collective); the step time is the max over
ranks. ``--impl reference`` times the fp64 CPU oracle on the host cores instead (bounded sample
of the same workload per step). Default workload: the Wan2.1-1.3B-shaped bidirectional denoise
step (21 x 30 x 52 tokens, 12 heads, head_dim 128, dense).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

import synth  # noqa: E402
from video_diffusion_transformer_vdit_b200.workloads import WORKLOADS  # noqa: E402

METRIC = "attention TFLOP/s (unmasked) & % of B200 BF16 peak; RoPE/KV-append GB/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
MASK_NAMES = {0: "dense", 1: "block-causal", 2: "radial", 3: "block-causal+radial",
              4: "dense candidates + dynamic threshold", 5: "block-causal + dynamic threshold",
              6: "radial + dynamic threshold", 7: "block-causal+radial + dynamic threshold"}
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "attn_fwd_traffic.txt")
ATTN_SRC = os.path.join(ROOT, "video_diffusion_transformer_vdit_b200", "csrc", "attn_fwd.cu")


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def dist_env():
    return int(os.environ.get("RANK", 0)), int(os.environ.get("WORLD_SIZE", 1)), \
        int(os.environ.get("LOCAL_RANK", 0))


def max_over_ranks(x: float, world: int) -> float:
    """Max of a per-rank scalar over the process group (the one collective of the bench: the
    timing reduction). World size 1 needs no process group."""
    if world <= 1:
        return float(x)
    import torch.distributed as dist
    dev = torch.device("cuda", torch.cuda.current_device()) if dist.get_backend() == "nccl" \
        else torch.device("cpu")
    t = torch.tensor([float(x)], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_tflops(world: int, flops_per_rank: float, ms_per_step: float) -> float:
    """Whole-job throughput: every rank does flops_per_rank per step (replicas: weak scaling;
    equal head shards of one step: strong scaling), the step time is the slowest rank's."""
    return world * flops_per_rank / (ms_per_step * 1e-3) / 1e12


def head_shard(heads: int, world: int, rank: int):
    """Heads [h0, h1) of `rank` when `world` ranks split one step's heads evenly (heads are
    independent in attention, so each rank runs the same plan on its slice of Q and of the
    cache, with no exchange)."""
    if world < 1 or heads % world:
        raise ValueError(f"{heads} heads do not split evenly over {world} ranks")
    hg = heads // world
    return rank * hg, (rank + 1) * hg


def config_of(w, extra=None):
    c = {"workload": w.name, "frames_x_grid": f"{w.q_frames}x{w.grid_h}x{w.grid_w}",
         "q_tokens": w.q_tokens, "kv_tokens": w.kv_tokens, "heads": w.heads,
         "head_dim": w.head_dim, "mask": MASK_NAMES[w.mask_kind], "q_start_frame": w.q_start,
         "batch": 1}
    if w.mask_kind & 4:
        c["tau"] = w.tau
        c["dynamic"] = ("two passes over the candidate tiles (row logit maxima, then attention "
                        "over candidates within tau of them); FLOPs count 4*d per candidate pair")
    if extra:
        c.update(extra)
    return c


# ------------------------------------------------------------------------------ oracle arm

class OracleArm:
    """The fp64 CPU oracle as a benchmark arm. Setup (not timed): the seeded inputs and the
    fp64 KV cache filled by the oracle's own appends. A timed sample: RoPE of a random set of
    query rows, their explicit mask rows, and two-pass masked attention of those rows for all
    heads against every key slot. Throughput counts 4*d FLOP per kept pair of the sample."""

    def __init__(self, w):
        import oracle
        self.oracle, self.w = oracle, w
        self.og = oracle.Geometry(w.grid_h, w.grid_w, w.heads, w.head_dim, *w.bands, w.theta)
        self.om = oracle.Mask(block_causal=bool(w.mask_kind & 1), radial=bool(w.mask_kind & 2),
                              chunk_frames=w.chunk_frames, w0=w.w0, gamma_shift=w.gamma_shift,
                              lam=w.lam)
        ft = w.frame_tokens
        n_kv = w.kv_stream_frames * ft
        k = synth.bf16_bits_to_f64(synth.qkv_bf16(w.id, n_kv, w.heads, w.head_dim, "k"))
        v = synth.bf16_bits_to_f64(synth.qkv_bf16(w.id, n_kv, w.heads, w.head_dim, "v"))
        kc = np.zeros((w.heads, w.kv_tokens, w.head_dim))
        vc = np.zeros_like(kc)
        for s, n in w.appends:
            off = (s - w.kv_stream_first_frame) * ft
            oracle.kv_append(kc, vc, w.capacity_frames, self.og, k[off:off + n * ft],
                             v[off:off + n * ft], s, n)
        self.kt = np.ascontiguousarray(kc.transpose(1, 0, 2))
        self.vt = np.ascontiguousarray(vc.transpose(1, 0, 2))
        first, last = w.window()
        self.kpos, self.kvalid = oracle.cache_positions(w.capacity_frames, first, last,
                                                        w.grid_h, w.grid_w)
        self.qpos = oracle.positions(w.q_tokens, w.grid_h, w.grid_w, w.q_start)
        self.qbits = synth.qkv_bf16(w.id, w.q_tokens, w.heads, w.head_dim, "q")
        self.rng = np.random.default_rng(0)
        self.rows_per_s = None

    def _run(self, n_rows):
        o, w = self.oracle, self.w
        rows = np.sort(self.rng.choice(w.q_tokens, n_rows, replace=False))
        t0 = time.perf_counter()
        qp = tuple(p[rows] for p in self.qpos)
        q = o.rope3d(synth.bf16_bits_to_f64(self.qbits[rows]), qp, self.og)
        m = o.mask_rows(qp, self.kpos, self.kvalid, self.om)
        if w.mask_kind & 4:
            o.attention_dynamic(q, self.kt, self.vt, m, w.scale, w.tau)
        else:
            o.attention(q, self.kt, self.vt, m, w.scale)
        dt = time.perf_counter() - t0
        return dt, 4.0 * w.head_dim * w.heads * int(m.sum()), n_rows

    def sample(self, budget_s):
        """One timed sample of about budget_s seconds: (TFLOP/s, seconds, rows)."""
        if self.rows_per_s is None:
            dt, _, n = self._run(8)
            self.rows_per_s = n / max(dt, 1e-4)
        n_rows = int(min(self.w.q_tokens, max(1, self.rows_per_s * budget_s)))
        dt, flops, n = self._run(n_rows)
        self.rows_per_s = n / max(dt, 1e-4)
        return flops / dt / 1e12, dt, n

    def describe(self, n_rows):
        w = self.w
        return (f"oracle (fp64 C, OpenMP): RoPE + explicit mask + two-pass attention of {n_rows} "
                f"random query rows x {w.heads} heads against all {w.kv_tokens} key slots (cache "
                f"built by the oracle's appends before timing); TFLOP/s counts 4*d per kept pair")


def run_reference(args, w):
    rank, world, _ = dist_env()
    if rank != 0:
        return
    arm = OracleArm(w)
    budget = max(0.1, 90.0 / max(1, args.steps + args.warmup))
    times, vals, rows = [], [], 0
    for i in range(args.warmup + args.steps):
        val, dt, n = arm.sample(budget)
        if i >= args.warmup:
            times.append(dt)
            vals.append(val)
            rows = n
    value = statistics.mean(vals)
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * statistics.mean(times), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic N(0,1), seeded SplitMix64 + Box-Muller, bf16-rounded",
            "config": config_of(w, {"parallelism": "host cores (OpenMP)"}),
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": arm.oracle.threads(),
                             "kind": "oracle", "sample": arm.describe(rows)},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------------------ GPU arm

class ClockSampler:
    """nvidia-smi clock / throttle-reason samples while the timed region runs."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.proc = None
        self.dev = device_index
        self.out = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.dev), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, ValueError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=10)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, mx, reasons, power = [], [], set(), []
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 8:
                continue
            try:
                sm.append(float(f[0]))
                mx.append(float(f[1]))
                power.append(float(f[2]))
            except ValueError:
                continue
            for n, val in zip(names, f[4:8]):
                if val.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None,
                "power_w_max": max(power) if power else None,
                "samples": len(sm), "reasons": sorted(reasons)}


def traffic_per_launch(w):
    """DRAM bytes per attention launch from the committed ncu summary, if it was taken on this
    workload from the current kernel source (else None)."""
    if not os.path.exists(TRAFFIC_FILE):
        return None, None
    kv = {}
    with open(TRAFFIC_FILE) as f:
        for line in f:
            if ":" in line:
                a, b = line.split(":", 1)
                kv[a.strip()] = b.strip()
    with open(ATTN_SRC, "rb") as f:
        sha = hashlib.sha256(f.read()).hexdigest()
    if kv.get("source_sha256") != sha or kv.get("workload_id") != str(w.id):
        return None, "kernel changed since the ncu capture" if kv.get("source_sha256") != sha else None
    try:
        return float(kv["dram_bytes_per_launch"]), kv.get("note")
    except (KeyError, ValueError):
        return None, None


def _nvtx(name):
    """NVTX range around a timed region (visible to Nsight tools; a no-op otherwise)."""
    import contextlib
    try:
        return torch.cuda.nvtx.range(name)
    except Exception:  # pragma: no cover - NVTX unavailable
        return contextlib.nullcontext()


def _time_back_to_back(fn, n, stream):
    """Mean device time (ms) of fn() over n back-to-back calls on `stream` (CUDA events)."""
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for i in range(n):
        fn(i)
    b.record(stream)
    torch.cuda.synchronize()
    return a.elapsed_time(b) / n


def _time_graph(fn, n_calls, stream, reps=5):
    """Mean device time (ms) per call of fn(i), i < n_calls, captured once into one CUDA graph
    and replayed `reps` times back to back (CUDA events on `stream`): the calls run with no host
    launch gap between them."""
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        for i in range(n_calls):
            fn(i)
    graph.replay()  # warm-up replay
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        a.record(stream)
        for _ in range(reps):
            graph.replay()
        b.record(stream)
    torch.cuda.synchronize()
    ms = a.elapsed_time(b) / (reps * n_calls)
    del graph
    return ms


def time_append(vdit, g, capacity_frames, n_frames, start_frame, dev, stream, n=20, graph_calls=30):
    """vdit_kv_append of one n_frames chunk, timed back to back over distinct (source, cache)
    sets whose total exceeds L2, so no launch finds its input in L2 and each pays for the
    write-back its predecessor left there; then the same appends, graph_calls of them (one per
    DiT block of Wan2.1-1.3B), captured in one CUDA graph, which takes the host's launch gaps
    out of small appends. Returns (ms, algorithmic bytes: read K, V + write K', V, torch copy ms,
    graph ms)."""
    ft = g.grid_h * g.grid_w
    shape = (n_frames * ft, g.heads, g.head_dim)
    per_set = 4 * int(np.prod(shape)) * 2
    n_sets = max(2, min(8, -(-400_000_000 // per_set)))
    gen = torch.Generator(device=dev).manual_seed(11)
    sets = []
    for _ in range(n_sets):
        k = torch.randn(shape, device=dev, generator=gen).to(torch.bfloat16)
        v = torch.randn(shape, device=dev, generator=gen).to(torch.bfloat16)
        cs = (g.heads, capacity_frames * ft, g.head_dim)
        sets.append((k, v, torch.zeros(cs, dtype=torch.bfloat16, device=dev),
                     torch.zeros(cs, dtype=torch.bfloat16, device=dev)))

    def one(i):
        k, v, kc, vc = sets[i % n_sets]
        vdit.kv_append(kc, vc, g, capacity_frames, k, v, start_frame)

    for i in range(n_sets):
        one(i)
    with _nvtx(f"kv_append {n_frames} frames x {g.heads} heads"):
        ms = _time_back_to_back(one, n, stream)
    # context: torch's device-to-device copy of the same bytes (K and V into the first frames of
    # the caches' storage), same sets, same launch pattern: what a plain copy of this size reaches
    def copy(i):
        k, v, kc, vc = sets[i % n_sets]
        kc.view(-1)[:k.numel()].copy_(k.view(-1))
        vc.view(-1)[:v.numel()].copy_(v.view(-1))

    for i in range(n_sets):
        copy(i)
    copy_ms = _time_back_to_back(copy, n, stream)
    with _nvtx(f"kv_append graph of {graph_calls}, {n_frames} frames x {g.heads} heads"):
        graph_ms = _time_graph(one, graph_calls, stream)
    return ms, per_set, copy_ms, graph_ms


def time_workload(vdit, w, dev, stream, burst_peak, n=10):
    """Attention forward (plus the split merge, when the plan splits) of workload w on seeded
    device-generated N(0, 1) bf16 inputs: its KV history appended first, then n timed launches
    after 3 warm-up launches. Inputs exceed L2 (cache K and V, Q, O)."""
    g = vdit.Geometry(w.grid_h, w.grid_w, w.heads, w.head_dim, w.bands, w.theta)
    m = vdit.Mask(w.mask_kind, w.chunk_frames, w.w0, w.gamma_shift, w.lam, w.tau)
    ft = w.frame_tokens
    gen = torch.Generator(device=dev).manual_seed(1000 + w.id)
    cache = vdit.KVCache(g, w.capacity_frames, device=dev)
    for s, nf in w.appends:
        shape = (nf * ft, w.heads, w.head_dim)
        k = torch.randn(shape, device=dev, generator=gen).to(torch.bfloat16)
        v = torch.randn(shape, device=dev, generator=gen).to(torch.bfloat16)
        cache.append(k, v, s)
        del k, v
    q = torch.randn((w.q_tokens, w.heads, w.head_dim), device=dev, generator=gen).to(torch.bfloat16)
    o = torch.empty_like(q)
    t0 = time.perf_counter()
    plan = vdit.Plan(g, m, w.q_start, w.q_frames, cache=cache)
    t_plan = time.perf_counter() - t0
    for _ in range(3):
        vdit.attn_forward(plan, q, cache, out=o, scale=w.scale)
    with _nvtx(f"attention workload {w.id}"):
        ms = _time_back_to_back(lambda i: vdit.attn_forward(plan, q, cache, out=o, scale=w.scale), n, stream)
    info = plan.info
    flops = plan.flops()
    tf = flops / (ms * 1e-3) / 1e12
    status = vdit.get_status()
    return {"workload": w.name, "mask": MASK_NAMES[w.mask_kind],
            "q_tokens": w.q_tokens, "kv_tokens": w.kv_tokens, "heads": w.heads,
            "attn_fwd_ms": ms, "tflops": tf, "frac_of_burst_peak": tf / burst_peak,
            "kept_fraction": info["kept_pairs"] / (w.q_tokens * w.kv_tokens),
            "tiles": info["tiles"], "full_tiles": info["full_tiles"],
            "ctas": info["ctas"], "cut_units": info["cut_units"],
            "kv_splits": info["kv_splits"],
            "launches": 1 + (1 if info["cut_units"] > 0 else 0),
            "plan_host_ms": 1e3 * t_plan, "status": status,
            "how": "%d back-to-back launches after 3 warm-up, CUDA events; ms includes the "
                   "merge kernel of the cut units' key pieces when cut_units > 0; TFLOP/s counts "
                   "4*d per kept pair" % n}


def run_gpu(args, w):
    import video_diffusion_transformer_vdit_b200 as vdit

    rank, world, local = dist_env()
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    else:
        torch.cuda.set_device(0)
    dev = torch.device("cuda", torch.cuda.current_device())
    full_heads = w.heads
    if args.shard == "heads":
        import dataclasses
        h0, h1 = head_shard(w.heads, world, rank)
        w = dataclasses.replace(w, heads=h1 - h0)
    g = vdit.Geometry(w.grid_h, w.grid_w, w.heads, w.head_dim, w.bands, w.theta)
    m = vdit.Mask(w.mask_kind, w.chunk_frames, w.w0, w.gamma_shift, w.lam, w.tau)
    ft = w.frame_tokens

    def bf16(bits):
        return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16)

    n_kv = w.kv_stream_frames * ft
    q_h = bf16(synth.qkv_bf16(w.id, w.q_tokens, full_heads, w.head_dim, "q"))
    k_h = bf16(synth.qkv_bf16(w.id, n_kv, full_heads, w.head_dim, "k"))
    v_h = bf16(synth.qkv_bf16(w.id, n_kv, full_heads, w.head_dim, "v"))
    if args.shard == "heads":  # this rank's heads of the same step
        q_h, k_h, v_h = (t[:, h0:h1].contiguous() for t in (q_h, k_h, v_h))
    q, k, v = q_h.to(dev), k_h.to(dev), v_h.to(dev)
    cache = vdit.KVCache(g, w.capacity_frames, device=dev)
    # history before the timed append (the earlier chunks of a causal rollout)
    s_last, n_last = w.appends[-1]
    for s, n in w.appends[:-1]:
        off = (s - w.kv_stream_first_frame) * ft
        cache.append(k[off:off + n * ft], v[off:off + n * ft], s)
    off_last = (s_last - w.kv_stream_first_frame) * ft
    k_step, v_step = k[off_last:off_last + n_last * ft], v[off_last:off_last + n_last * ft]
    cache.append(k_step, v_step, s_last)
    t_plan = time.perf_counter()
    plan = vdit.Plan(g, m, w.q_start, w.q_frames, cache=cache)
    t_plan = time.perf_counter() - t_plan
    o = torch.empty_like(q)
    flops = plan.flops()
    stream = torch.cuda.current_stream()
    append_bytes = 4 * k_step.numel() * 2  # read K, V; write K', V (bf16)

    def step(evs=None):
        if evs:
            evs[0].record(stream)
        vdit.kv_append(cache.k, cache.v, g, w.capacity_frames, k_step, v_step, s_last)
        if evs:
            evs[1].record(stream)
        vdit.attn_forward(plan, q, cache, out=o, scale=w.scale)
        if evs:
            evs[2].record(stream)

    def barrier():
        if world > 1:
            import torch.distributed as dist
            dist.barrier()
        torch.cuda.synchronize()

    for _ in range(args.warmup):
        step()
    barrier()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    clocks = ClockSampler(torch.cuda.current_device()) if rank == 0 else None
    if clocks:
        clocks.start()
        time.sleep(0.3)
    barrier()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with _nvtx("timed steps"):
        t0.record(stream)
        for i in range(args.steps):
            step(evs[i])
        t1.record(stream)
        barrier()
    clk = clocks.stop() if clocks else None
    ms = max_over_ranks(t0.elapsed_time(t1), world)
    ms_step = ms / args.steps
    attn_ms = statistics.mean(evs[i][1].elapsed_time(evs[i][2]) for i in range(args.steps))
    app_ms = statistics.mean(evs[i][0].elapsed_time(evs[i][1]) for i in range(args.steps))

    status = vdit.get_status()

    # standalone RoPE (the C-ABI call on Q, out of place) for its GB/s: back to back over four
    # distinct (input, output) pairs, 800 MB in all, so no launch finds its input in L2 and each
    # pays the write-back of the output the launch before it left in L2
    xs = [q] + [torch.empty_like(q).copy_(q) for _ in range(3)]
    ys = [torch.empty_like(q) for _ in range(4)]
    for i in range(4):
        vdit.rope3d_apply(xs[i], g, w.q_start, out=ys[i])
    torch.cuda.synchronize()
    r0, r1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    n_rope = 20
    with _nvtx("rope3d_apply"):
        r0.record(stream)
        for i in range(n_rope):
            vdit.rope3d_apply(xs[i % 4], g, w.q_start, out=ys[i % 4])
        r1.record(stream)
    torch.cuda.synchronize()
    rope_ms = r0.elapsed_time(r1) / n_rope
    del xs, ys
    rope_bytes = 2 * q.numel() * 2

    # sequence-to-head pack (vdit_seq_pack) as rank 0 of two sequence-parallel ranks: RoPE of Q and K
    # at the global positions, Q, K and V of half the tokens into the all-to-all layout (the block
    # of the other rank) and the own head-sharded buffers, in one launch; back to back over two
    # distinct input / output sets (1.2 GB in all)
    pack = None
    if g.heads % 2 == 0:
        n_half = q.shape[0] // 2
        hg = g.heads // 2
        sets = []
        for _ in range(2):
            ins = [q[:n_half].clone() for _ in range(3)]
            send = torch.empty(2, 3, n_half, hg, g.head_dim, dtype=q.dtype, device=q.device)
            full = tuple(torch.empty(2 * n_half, hg, g.head_dim, dtype=q.dtype, device=q.device)
                         for _ in range(3))
            sets.append((ins, send, full))

        def one_pack(i):
            ins, send, full = sets[i % 2]
            vdit.seq_pack(ins[0], ins[1], ins[2], g, w.q_start, 0, 2, send, full)

        for i in range(2):
            one_pack(i)
        with _nvtx("seq_pack"):
            pack_ms = _time_back_to_back(one_pack, 20, stream)
        pack_bytes = 3 * 2 * n_half * g.heads * g.head_dim * 2
        pack = {"ms": pack_ms, "bytes": pack_bytes, "gbs": pack_bytes / (pack_ms * 1e-3) / 1e9,
                "frac_hbm": pack_bytes / (pack_ms * 1e-3) / 1e9 / peaks()[0]["hbm_gbs"]}
        # the peer-memory form (vdit_seq_pack_peers) with both ranks' destination buffers on this
        # device: the same reads and writes, the writes as the kernel's own stores into the
        # head-sharded buffers of every rank (over NVLink when they are another GPU's)
        peer_sets = []
        for ins, _, full in sets:
            other = tuple(torch.empty_like(t) for t in full)
            peer_sets.append((ins, [[full[x].data_ptr(), other[x].data_ptr()] for x in range(3)], other))

        def one_peer_pack(i):
            ins, addrs, _ = peer_sets[i % 2]
            vdit.seq_pack_peers(ins[0], ins[1], ins[2], g, w.q_start, 0, 2, *addrs)

        for i in range(2):
            one_peer_pack(i)
        with _nvtx("seq_pack_peers"):
            peer_ms = _time_back_to_back(one_peer_pack, 20, stream)
        pack["peers"] = {"ms": peer_ms, "gbs": pack_bytes / (peer_ms * 1e-3) / 1e9,
                         "frac_hbm": pack_bytes / (peer_ms * 1e-3) / 1e9 / peaks()[0]["hbm_gbs"],
                         "how": "vdit_seq_pack_peers as rank 0 of 2, both ranks' buffers on this "
                                "device; same bytes"}
        del sets, peer_sets

    # fused QKV projection + RoPE + cache append (vdit_qkv_rope) of the step's newest frames,
    # d_model = heads * head_dim (as in Wan2.1), random bf16 weights, its own cache
    qkv = None
    dm = g.heads * g.head_dim
    if dm % 256 == 0:
        n_tok = w.appends[-1][1] * ft
        gen = torch.Generator(device="cuda").manual_seed(7)
        xq = torch.randn(n_tok, dm, device="cuda", generator=gen).to(torch.bfloat16)
        wq = (torch.randn(3 * dm, dm, device="cuda", generator=gen) * dm ** -0.5).to(torch.bfloat16)
        qc = vdit.KVCache(g, w.capacity_frames)
        qo = torch.empty(n_tok, g.heads, g.head_dim, dtype=torch.bfloat16, device="cuda")
        for _ in range(3):
            vdit.qkv_rope(xq, wq, g, s_last, qc.k, qc.v, w.capacity_frames, q_out=qo)
        torch.cuda.synchronize()
        # X and W (115 MB at the 1.3B clip) fit in L2: every timed launch follows a 256 MB write
        # that evicts them, and is timed alone with its own events (median of 10)
        flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
        n_qkv = 10
        evq = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(n_qkv)]
        with _nvtx("qkv_rope"):
            for i in range(n_qkv):
                flush.fill_(i & 0xFF)
                evq[i][0].record(stream)
                vdit.qkv_rope(xq, wq, g, s_last, qc.k, qc.v, w.capacity_frames, q_out=qo)
                evq[i][1].record(stream)
        torch.cuda.synchronize()
        qkv_ms = statistics.median(a.elapsed_time(b) for a, b in evq)
        del flush
        qkv = {"ms": qkv_ms, "tflops": 2.0 * n_tok * dm * 3 * dm / (qkv_ms * 1e-3) / 1e12,
               "shape": f"[{n_tok}, {dm}] x [{3 * dm}, {dm}]^T"}
        del xq, wq, qc, qo

    # KV append on its own, over distinct buffers (no deferred write-back into the next
    # kernel): the clip-sized append of this workload and the 3-frame chunks of the Wan2.1-1.3B
    # (12 heads) and Wan2.1-14B (40 heads) decode
    appends = {}
    pk0 = peaks()[0]
    for name, heads, nf, start in (("clip", g.heads, n_last, s_last),
                                   ("chunk_1.3b_h12", 12, 3, 18), ("chunk_14b_h40", 40, 3, 396)):
        ga = vdit.Geometry(g.grid_h, g.grid_w, heads, g.head_dim, g.bands, g.theta)
        a_ms, a_bytes, c_ms, g_ms = time_append(vdit, ga, w.capacity_frames if name == "clip" else 21,
                                                nf, start, dev, stream)
        gbs = a_bytes / (a_ms * 1e-3) / 1e9
        appends[name] = {"frames": nf, "heads": heads, "ms": a_ms, "bytes": a_bytes, "gbs": gbs,
                         "frac_hbm": gbs / pk0["hbm_gbs"],
                         "graph_ms": g_ms, "graph_gbs": a_bytes / (g_ms * 1e-3) / 1e9,
                         "graph_frac_hbm": a_bytes / (g_ms * 1e-3) / 1e9 / pk0["hbm_gbs"],
                         "torch_copy_same_bytes_gbs": a_bytes / (c_ms * 1e-3) / 1e9}
    torch.cuda.synchronize()

    # the other attention configurations, timed in the same run (not part of the step)
    per_workload = {}
    if not args.no_per_workload:
        for wid in (2, 3, 4, 5, 6):
            if wid == w.id:
                continue
            per_workload[str(wid)] = time_workload(vdit, WORKLOADS[wid], dev, stream,
                                                   pk0["bf16_tflops"])
            torch.cuda.empty_cache()

    # End to end through the public API: every step copies its Q, K, V from pinned host memory
    # and its O back to pinned host memory. Inputs and outputs are double-buffered and the copies
    # run on their own streams, so step i's copies overlap step i-1's kernels (a stream of denoise
    # steps); the KV cache is only touched by the compute stream, in step order.
    k_src, v_src = k_h[off_last:off_last + n_last * ft], v_h[off_last:off_last + n_last * ft]
    q_p, k_p, v_p = q_h.pin_memory(), k_src.pin_memory(), v_src.pin_memory()
    o_p = [torch.empty(o.shape, dtype=o.dtype).pin_memory() for _ in range(2)]
    q_d = [torch.empty_like(q) for _ in range(2)]
    k_d = [torch.empty_like(k_step) for _ in range(2)]
    v_d = [torch.empty_like(v_step) for _ in range(2)]
    o_d = [torch.empty_like(o) for _ in range(2)]
    s_h2d, s_d2h = torch.cuda.Stream(), torch.cuda.Stream()
    ev = lambda: torch.cuda.Event()  # noqa: E731
    h2d_done, comp_done, d2h_done = [ev(), ev()], [ev(), ev()], [ev(), ev()]
    for e in comp_done + d2h_done:
        e.record(stream)

    def e2e_step(i):
        b = i % 2
        with torch.cuda.stream(s_h2d):
            s_h2d.wait_event(comp_done[b])  # buffer b's inputs are free once step i-2 ran
            q_d[b].copy_(q_p, non_blocking=True)
            k_d[b].copy_(k_p, non_blocking=True)
            v_d[b].copy_(v_p, non_blocking=True)
            h2d_done[b].record(s_h2d)
        stream.wait_event(h2d_done[b])
        stream.wait_event(d2h_done[b])  # o_d[b] was read back by step i-2's copy
        vdit.kv_append(cache.k, cache.v, g, w.capacity_frames, k_d[b], v_d[b], s_last, stream=stream)
        vdit.attn_forward(plan, q_d[b], cache, out=o_d[b], scale=w.scale, stream=stream)
        comp_done[b].record(stream)
        with torch.cuda.stream(s_d2h):
            s_d2h.wait_event(comp_done[b])
            o_p[b].copy_(o_d[b], non_blocking=True)
            d2h_done[b].record(s_d2h)

    n_e2e = max(3, min(args.steps, 20))
    for i in range(3):
        e2e_step(i)
    torch.cuda.synchronize()
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s_h2d)
    for i in range(n_e2e):
        e2e_step(i)
    s_d2h.wait_event(comp_done[(n_e2e - 1) % 2])
    e1.record(s_d2h)
    torch.cuda.synchronize()
    barrier()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / n_e2e, world)
    h2d = (q_p.numel() + k_p.numel() + v_p.numel()) * 2
    d2h = o_p[0].numel() * 2

    if rank == 0:
        pk, src = peaks()
        # the attention kernel is timed in a short region: the burst peak applies unless the
        # region ran for a second or more, or the SM clock sat well below its maximum
        # (power-capped), where the sustained peak (measured under the cap) does
        timed_s = ms * 1e-3
        clk_ok = bool(clk and clk.get("sm_mhz") and clk.get("sm_max_mhz")
                      and clk["sm_mhz"] >= 0.95 * clk["sm_max_mhz"])
        burst = timed_s < 1.0 and (clk_ok or not clk or not clk.get("sm_mhz"))
        peak = pk["bf16_tflops"] if burst else pk.get("bf16_tflops_sustained", pk["bf16_tflops"])
        peak_kind = ("bf16 dense, burst (%s): timed region %.2f s at full clock" % (src, timed_s)
                     if burst else "bf16 dense, sustained (%s): timed region %.2f s" % (src, timed_s))
        achieved = flops / (attn_ms * 1e-3) / 1e12
        traffic, tnote = traffic_per_launch(w)
        cpu = None
        if world == 1 and not args.no_cpu_baseline:
            arm = OracleArm(w)
            val, dt, n = arm.sample(args.cpu_budget)
            cpu = {"value": val, "unit": "TFLOP/s", "cores": arm.oracle.threads(), "kind": "oracle",
                   "sample": arm.describe(n), "seconds": dt}
        info = plan.info
        line = {
            "metric": METRIC,
            "value": aggregate_tflops(world, flops, ms_step),
            "unit": "TFLOP/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": ms_step,
            "higher_is_better": True,
            "scaling": "strong" if args.shard == "heads" else "weak", "vs_baseline": None,
            "dtype": "bf16",
            "data": "synthetic N(0,1), seeded SplitMix64 + Box-Muller, bf16-rounded",
            "config": config_of(w, {
                "parallelism": (f"{world} head shards of {w.heads} of {full_heads} heads (no collective)"
                                if args.shard == "heads" else
                                f"{world} independent replicas (no collective)"),
                "l2": "inputs larger than L2: %.0f MB touched per step (Q, K/V chunk, caches, O)"
                      % ((q.numel() * 2 * 2 + append_bytes + cache.k.numel() * 4) / 1e6),
                "step": "kv_append(newest chunk) + attn_forward (RoPE of Q fused); plan built "
                        "once per geometry outside the timed region (%.1f ms host)" % (1e3 * t_plan),
                "tiles": info["tiles"], "full_tiles": info["full_tiles"],
                "ctas": info["ctas"], "cut_units": info["cut_units"],
                "kept_fraction": info["kept_pairs"] / (w.q_tokens * w.kv_tokens)}),
            "roofline": {"bound": "tensor", "kernel": "attn_fwd",
                         "timed": "one vdit_attn_forward call: attn_fwd_kernel, plus split_combine_kernel "
                                  "when the CTA schedule cuts units into key pieces (%d cut units here)"
                                  % plan.info["cut_units"],
                         "achieved": achieved,
                         "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak,
                         "peak_kind": peak_kind,
                         "frac_of_burst_peak": achieved / pk["bf16_tflops"],
                         "frac_of_sustained_peak": achieved / pk.get("bf16_tflops_sustained",
                                                                     pk["bf16_tflops"]),
                         "traffic": traffic, "traffic_note": tnote,
                         "algorithmic": "4*head_dim FLOP per kept (query, key, head): %.4g per launch" % flops},
            "cpu_baseline": cpu,
            "e2e": {"value": aggregate_tflops(world, flops, e2e_ms), "unit": "TFLOP/s",
                    "ms_per_step": e2e_ms, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "how": "public API; per step H2D of Q, K, V from pinned memory and D2H of O, "
                           "double-buffered on copy streams overlapping the previous step"},
            "attended": {
                "pairs_per_s": world * g.heads * info["kept_pairs"] / (attn_ms * 1e-3),
                "query_tokens_per_s": (1 if args.shard == "heads" else world) * w.q_tokens / (ms_step * 1e-3),
                "how": "pairs_per_s: kept (query, key, head) triples per second of attn_fwd; "
                       "query_tokens_per_s: query tokens through the whole step (append + "
                       "attention, all heads) per second; both summed over the ranks (head "
                       "shards share their query tokens)"},
            # per step: the append, the attention kernel and, when units are cut, the merge
            "gpu_launches": args.steps * (2 + (1 if info["cut_units"] > 0 else 0)),
            "clocks": clk,
            "kernels": {
                "attn_fwd_ms": attn_ms, "attn_fwd_tflops": achieved,
                "kv_append_ms": appends["clip"]["ms"], "kv_append_gbs": appends["clip"]["gbs"],
                "kv_append_frac_hbm": appends["clip"]["frac_hbm"],
                "kv_append": dict(appends, how="vdit_kv_append alone, 20 launches back to back "
                                  "over distinct source and cache buffers (> 400 MB in all); "
                                  "graph_*: 30 of the same appends (one per DiT block) captured "
                                  "in one CUDA graph, 5 replays; "
                                  "bytes = read K, V + write K', V; torch_copy_same_bytes_gbs: "
                                  "torch's device copy of K and V (two launches) over the same "
                                  "buffers, for context"),
                "kv_append_in_step_ms": app_ms,
                "kv_append_in_step_gbs": append_bytes / (app_ms * 1e-3) / 1e9,
                "rope3d_apply_ms": rope_ms, "rope3d_apply_gbs": rope_bytes / (rope_ms * 1e-3) / 1e9,
                "rope3d_apply_frac_hbm": rope_bytes / (rope_ms * 1e-3) / 1e9 / pk["hbm_gbs"],
                "hbm_peak_gbs": pk["hbm_gbs"],
                "seq_pack": None if pack is None else dict(
                    pack, how="vdit_seq_pack of Q, K, V of one of 2 sequence-parallel ranks (RoPE "
                              "of Q and K + all-to-all layout, one launch), read + write bytes, "
                              "not part of the step"),
                "qkv_rope": None if qkv is None else dict(
                    qkv, frac_of_sustained_peak=qkv["tflops"] / peak,
                    frac_of_burst_peak=qkv["tflops"] / pk["bf16_tflops"],
                    how="vdit_qkv_rope: X W^T on tcgen05, RoPE of Q and K, K' and V into the "
                        "ring cache; median of 10 launches, each after a 256 MB write that "
                        "evicts X and W from L2; not part of the step")},
            "per_workload": per_workload,
            "status": status,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", type=int, default=2, choices=sorted(WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-budget", type=float, default=10.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--shard", default="replicas", choices=["replicas", "heads"],
                    help="N > 1: independent replicas of the step (weak scaling, default) or one "
                         "step's heads split evenly over the ranks (strong scaling)")
    ap.add_argument("--no-per-workload", action="store_true",
                    help="skip timing the other attention configurations")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    world = dist_env()[1]
    if args.gpus != world:
        ap.error(f"--gpus {args.gpus} but {world} rank(s): launch one process per GPU "
                 f"(python -m torch.distributed.run --nproc-per-node {args.gpus} bench.py ...)")
    w = WORKLOADS[args.workload]
    if args.impl == "reference":
        run_reference(args, w)
    else:
        run_gpu(args, w)


if __name__ == "__main__":
    main()
