"""Python binding of libvdit: B200 (sm_100a) spatio-temporal attention for video DiTs.

Argument marshalling only: every step runs in libvdit's CUDA kernels through its C ABI
(include/vdit.h). PyTorch supplies device memory and the current CUDA stream. There is no CPU
fallback: without the built library every call raises.

    import video_diffusion_transformer_vdit_b200 as vdit
    g = vdit.Geometry(grid_h=30, grid_w=52, heads=12, head_dim=128, bands=(44, 42, 42))
    cache = vdit.KVCache(g, capacity_frames=21, device="cuda")
    cache.append(k_chunk, v_chunk, start_frame=18)          # RoPE(K) at global frames + ring write
    plan = vdit.Plan(g, vdit.Mask.block_causal(3), q_start_frame=18, q_frames=3, cache=cache)
    o = vdit.attn_forward(plan, q_chunk, cache)              # RoPE(Q) fused into the Q load
"""
from __future__ import annotations

import ctypes
import math
import os
import re
from dataclasses import dataclass
from typing import Optional, Tuple

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
# the in-tree build; there is no fallback: a missing library is an error
LIB_PATH = os.path.join(_PKG, "libvdit.so")
HEADER_PATH = os.path.join(os.path.dirname(_PKG), "include", "vdit.h")

OK = 0
ERR_INVALID_ARG = -1
ERR_UNSUPPORTED = -2
ERR_MISALIGNED = -3
ERR_CUDA = -4
ERR_TIMEOUT = -5
ERR_NOT_UPLOADED = -6

MASK_DENSE = 0
MASK_BLOCK_CAUSAL = 1
MASK_RADIAL = 2
MASK_DYNAMIC = 4
TILE = 128


class VditError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"libvdit error {code}: {msg}")
        self.code = code


class _Geom(ctypes.Structure):
    _fields_ = [("grid_h", ctypes.c_int), ("grid_w", ctypes.c_int), ("heads", ctypes.c_int),
                ("head_dim", ctypes.c_int), ("band_t", ctypes.c_int), ("band_h", ctypes.c_int),
                ("band_w", ctypes.c_int), ("theta", ctypes.c_double)]


class _Mask(ctypes.Structure):
    _fields_ = [("kind", ctypes.c_int), ("chunk_frames", ctypes.c_int), ("w0", ctypes.c_longlong),
                ("gamma_shift", ctypes.c_int), ("lambda_", ctypes.c_int), ("tau", ctypes.c_double)]


class _PlanInfo(ctypes.Structure):
    _fields_ = [("q_tokens", ctypes.c_int), ("kv_tokens", ctypes.c_int), ("q_tiles", ctypes.c_int),
                ("kv_tiles", ctypes.c_int), ("tiles", ctypes.c_int), ("full_tiles", ctypes.c_int),
                ("kept_pairs", ctypes.c_longlong), ("uploaded", ctypes.c_int),
                ("kv_splits", ctypes.c_int), ("workspace_bytes", ctypes.c_longlong),
                ("mask_bytes", ctypes.c_longlong), ("work_entries", ctypes.c_int),
                ("single_patch_entries", ctypes.c_int), ("work_mask_bytes", ctypes.c_longlong),
                ("ctas", ctypes.c_int), ("cut_units", ctypes.c_int)]


_lib = None


def lib() -> ctypes.CDLL:
    """The loaded libvdit.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is not built: run "
                               "`python -m video_diffusion_transformer_vdit_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        P, I, LL, F = ctypes.c_void_p, ctypes.c_int, ctypes.c_longlong, ctypes.c_float
        gp, mp = ctypes.POINTER(_Geom), ctypes.POINTER(_Mask)
        L.vdit_rope3d_apply.argtypes = [gp, P, P, I, LL, P]
        L.vdit_kv_append.argtypes = [gp, P, P, I, P, P, I, I, P]
        L.vdit_attn_plan.argtypes = [ctypes.POINTER(P), gp, mp, I, I, I, I, I]
        L.vdit_plan_upload.argtypes = [P, P]
        L.vdit_plan_info.argtypes = [P, ctypes.POINTER(_PlanInfo)]
        L.vdit_plan_export.argtypes = [P, P, P, P]
        L.vdit_plan_export_masks.argtypes = [P, P, P]
        L.vdit_plan_export_work.argtypes = [P, P, P, P, P]
        L.vdit_plan_export_schedule.argtypes = [P, I, ctypes.POINTER(I), ctypes.POINTER(I), P, P]
        L.vdit_qkv_rope.argtypes = [P, P, P, I, I, I, P, P, P, I, P]
        L.vdit_seq_pack.argtypes = [gp, P, P, P, P, P, P, P, I, I, I, LL, I, P]
        L.vdit_seq_unpack.argtypes = [gp, P, P, P, I, I, LL, P]
        L.vdit_seq_pack_peers.argtypes = [gp, P, P, P, P, P, P, I, I, I, LL, I, P]
        L.vdit_seq_push_peers.argtypes = [gp, P, P, I, I, LL, P]
        L.vdit_kv_write.argtypes = [gp, P, P, I, P, P, I, I, P]
        L.vdit_attn_forward_rotated.argtypes = [P, P, P, P, P, P, F, P]
        L.vdit_plan_destroy.argtypes = [P]
        L.vdit_plan_destroy.restype = None
        L.vdit_attn_forward.argtypes = [P, P, P, P, P, P, F, P]
        L.vdit_attn_forward_noalloc.argtypes = [P, P, P, P, P, P, F, P]
        L.vdit_get_status.argtypes = [ctypes.POINTER(I)]
        L.vdit_debug_skip_loads.argtypes = [I]
        L.vdit_debug_skip_loads.restype = None
        L.vdit_last_error.restype = ctypes.c_char_p
        _lib = L
    return _lib


def declared_symbols() -> list:
    """Names of the functions include/vdit.h declares (for export checks)."""
    with open(HEADER_PATH) as f:
        text = f.read()
    return re.findall(r"VDIT_API\s+[\w\s\*]+?\b(vdit_\w+)\s*\(", text)


def _check(rc: int) -> None:
    if rc != OK:
        raise VditError(rc, lib().vdit_last_error().decode())


def _stream(stream=None) -> ctypes.c_void_p:
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _dev_ptr(t: torch.Tensor, name: str) -> ctypes.c_void_p:
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


@dataclass(frozen=True)
class Geometry:
    """grid_h x grid_w patches per latent frame, heads x head_dim, RoPE bands (t, h, w)."""
    grid_h: int
    grid_w: int
    heads: int
    head_dim: int
    bands: Tuple[int, int, int]
    theta: float = 10000.0

    @property
    def frame_tokens(self) -> int:
        return self.grid_h * self.grid_w

    def c(self) -> _Geom:
        return _Geom(self.grid_h, self.grid_w, self.heads, self.head_dim, *self.bands,
                     float(self.theta))


@dataclass(frozen=True)
class Mask:
    """Mask kind bits (MASK_BLOCK_CAUSAL | MASK_RADIAL | MASK_DYNAMIC) and parameters."""
    kind: int = MASK_DENSE
    chunk_frames: int = 3
    w0: int = 52
    gamma_shift: int = 1
    lam: int = 8
    tau: float = 0.0

    @staticmethod
    def dense() -> "Mask":
        return Mask(MASK_DENSE)

    @staticmethod
    def block_causal(chunk_frames: int = 3) -> "Mask":
        return Mask(MASK_BLOCK_CAUSAL, chunk_frames=chunk_frames)

    @staticmethod
    def radial(w0: int = 52, gamma_shift: int = 1, lam: int = 8, chunk_frames: Optional[int] = None) -> "Mask":
        kind = MASK_RADIAL | (MASK_BLOCK_CAUSAL if chunk_frames else 0)
        return Mask(kind, chunk_frames=chunk_frames or 3, w0=w0, gamma_shift=gamma_shift, lam=lam)

    def c(self) -> _Mask:
        return _Mask(self.kind, self.chunk_frames, self.w0, self.gamma_shift, self.lam, float(self.tau))


def rope3d_apply(x: torch.Tensor, g: Geometry, start_frame: int,
                 out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """3-D RoPE of x [n_tokens, heads, head_dim] (bf16, CUDA) whose first token is at global
    frame start_frame. out=x rotates in place."""
    if x.dtype != torch.bfloat16 or x.dim() != 3 or x.shape[1:] != (g.heads, g.head_dim):
        raise ValueError("x must be bf16 [n_tokens, heads, head_dim]")
    y = torch.empty_like(x) if out is None else out
    gc = g.c()
    _check(lib().vdit_rope3d_apply(ctypes.byref(gc), _dev_ptr(x, "x"), _dev_ptr(y, "out"),
                                   int(start_frame), x.shape[0], _stream(stream)))
    return y


def kv_append(k_cache: torch.Tensor, v_cache: torch.Tensor, g: Geometry, capacity_frames: int,
              k: torch.Tensor, v: torch.Tensor, start_frame: int, stream=None) -> None:
    """Rotate K at its global frames and write K', V into ring slots f mod capacity_frames."""
    ft = g.frame_tokens
    if k.shape != v.shape or k.shape[0] % ft or k.shape[1:] != (g.heads, g.head_dim):
        raise ValueError("k, v must be [n_frames * frame_tokens, heads, head_dim]")
    for t in (k, v, k_cache, v_cache):
        if t.dtype != torch.bfloat16:
            raise ValueError("tensors must be bf16")
    gc = g.c()
    _check(lib().vdit_kv_append(ctypes.byref(gc), _dev_ptr(k_cache, "k_cache"),
                                _dev_ptr(v_cache, "v_cache"), int(capacity_frames),
                                _dev_ptr(k, "k"), _dev_ptr(v, "v"), int(start_frame),
                                k.shape[0] // ft, _stream(stream)))


def qkv_rope(x: torch.Tensor, w: torch.Tensor, g: Geometry, start_frame: int,
             k_cache: torch.Tensor, v_cache: torch.Tensor, capacity_frames: int,
             q_out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """Fused [Q | K | V] = x w^T, RoPE of Q and K at global frames from start_frame, K' and V into
    ring slots f mod capacity_frames. x: bf16 [n_frames * frame_tokens, d_model]; w: bf16
    [3 * heads * head_dim, d_model]. Returns the rotated Q [tokens, heads, head_dim]."""
    ft = g.frame_tokens
    if x.dtype != torch.bfloat16 or x.dim() != 2 or x.shape[0] % ft:
        raise ValueError("x must be bf16 [n_frames * frame_tokens, d_model]")
    hd = g.heads * g.head_dim
    if w.dtype != torch.bfloat16 or tuple(w.shape) != (3 * hd, x.shape[1]):
        raise ValueError("w must be bf16 [3 * heads * head_dim, d_model]")
    q = torch.empty(x.shape[0], g.heads, g.head_dim, dtype=torch.bfloat16, device=x.device) \
        if q_out is None else q_out
    gc = g.c()
    _check(lib().vdit_qkv_rope(ctypes.byref(gc), _dev_ptr(x, "x"), _dev_ptr(w, "w"), x.shape[1],
                               int(start_frame), x.shape[0] // ft, _dev_ptr(q, "q_out"),
                               _dev_ptr(k_cache, "k_cache"), _dev_ptr(v_cache, "v_cache"),
                               int(capacity_frames), _stream(stream)))
    return q


def kv_write(k_cache: torch.Tensor, v_cache: torch.Tensor, g: Geometry, capacity_frames: int,
             k_rotated: torch.Tensor, v: torch.Tensor, start_frame: int, stream=None) -> None:
    """Write already rotated K' and V into ring slots f mod capacity_frames (vdit_kv_write)."""
    ft = g.frame_tokens
    if k_rotated.shape != v.shape or k_rotated.shape[0] % ft or k_rotated.shape[1:] != (g.heads, g.head_dim):
        raise ValueError("k, v must be [n_frames * frame_tokens, heads, head_dim]")
    for t in (k_rotated, v, k_cache, v_cache):
        if t.dtype != torch.bfloat16:
            raise ValueError("tensors must be bf16")
    gc = g.c()
    _check(lib().vdit_kv_write(ctypes.byref(gc), _dev_ptr(k_cache, "k_cache"),
                               _dev_ptr(v_cache, "v_cache"), int(capacity_frames),
                               _dev_ptr(k_rotated, "k"), _dev_ptr(v, "v"), int(start_frame),
                               k_rotated.shape[0] // ft, _stream(stream)))


def seq_pack(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, g: Geometry, start_frame: int,
             rank: int, n_ranks: int, send: Optional[torch.Tensor], full, rotate: bool = True,
             stream=None) -> None:
    """vdit_seq_pack: this rank's q, k, v [n, heads, head_dim] (chunk-local tokens rank * n ..)
    -> send [n_ranks, 3, n, heads / n_ranks, head_dim] (blocks for the other ranks) and the own
    block into full = (q_full, k_full, v_full), each [n_ranks * n, heads / n_ranks, head_dim];
    Q and K rotated at their global positions when rotate."""
    n = q.shape[0]
    for name, t in (("q", q), ("k", k), ("v", v)):
        if t.dtype != torch.bfloat16 or t.dim() != 3 or tuple(t.shape) != (n, g.heads, g.head_dim):
            raise ValueError(f"{name} must be bf16 [n_tokens, heads, head_dim]")
    if n_ranks < 1 or g.heads % n_ranks:
        raise ValueError("n_ranks must divide heads")
    hg = g.heads // n_ranks
    for t in full:
        if t.dtype != torch.bfloat16 or tuple(t.shape) != (n_ranks * n, hg, g.head_dim):
            raise ValueError("full buffers must be bf16 [n_ranks * n_tokens, heads / n_ranks, head_dim]")
    if n_ranks > 1 and (send is None or tuple(send.shape) != (n_ranks, 3, n, hg, g.head_dim)):
        raise ValueError("send must be [n_ranks, 3, n_tokens, heads / n_ranks, head_dim]")
    gc = g.c()
    sp = _dev_ptr(send, "send") if send is not None else ctypes.c_void_p(0)
    _check(lib().vdit_seq_pack(ctypes.byref(gc), _dev_ptr(q, "q"), _dev_ptr(k, "k"), _dev_ptr(v, "v"),
                               sp, _dev_ptr(full[0], "q_full"), _dev_ptr(full[1], "k_full"),
                               _dev_ptr(full[2], "v_full"), int(rank), int(n_ranks), int(start_frame),
                               n, int(bool(rotate)), _stream(stream)))


def seq_unpack(recv: Optional[torch.Tensor], own: torch.Tensor, out: torch.Tensor, g: Geometry,
               rank: int, n_ranks: int, stream=None) -> torch.Tensor:
    """vdit_seq_unpack: out [n, heads, head_dim] from recv [n_ranks, n, heads / n_ranks,
    head_dim] (block r from rank r) and own [n, heads / n_ranks, head_dim] (block rank)."""
    n = out.shape[0]
    hg = g.heads // n_ranks
    if out.dtype != torch.bfloat16 or tuple(out.shape) != (n, g.heads, g.head_dim):
        raise ValueError("out must be bf16 [n_tokens, heads, head_dim]")
    if tuple(own.shape) != (n, hg, g.head_dim):
        raise ValueError("own must be [n_tokens, heads / n_ranks, head_dim]")
    if n_ranks > 1 and (recv is None or tuple(recv.shape) != (n_ranks, n, hg, g.head_dim)):
        raise ValueError("recv must be [n_ranks, n_tokens, heads / n_ranks, head_dim]")
    gc = g.c()
    rp = _dev_ptr(recv, "recv") if recv is not None else ctypes.c_void_p(0)
    _check(lib().vdit_seq_unpack(ctypes.byref(gc), rp, _dev_ptr(own, "own"), _dev_ptr(out, "out"),
                                 int(rank), int(n_ranks), n, _stream(stream)))
    return out


def _group_info(group):
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return 1, 0
    return dist.get_world_size(group), dist.get_rank(group)


def exchange(sends: dict, recvs: dict, group=None) -> None:
    """One batched point-to-point exchange: sends[r] (a list of tensors) go to group rank r, and
    recvs[r] (a list of tensors, the same sizes in the same order as rank r's sends here) are
    filled from group rank r, all posted together (batch_isend_irecv; one grouped NCCL launch on
    GPUs). Backends without device-tensor point-to-point (gloo) stage device tensors through host
    memory."""
    import torch.distributed as dist
    peers = sorted(set(sends) | set(recvs))
    if not peers:
        return
    staged = dist.get_backend(group) != "nccl"

    def host(t):
        return t.detach().cpu() if (staged and t.is_cuda) else t

    def glob(r):
        return r if group is None else dist.get_global_rank(group, r)

    ops, back = [], []
    for r in peers:
        for t in sends.get(r, ()):
            ops.append(dist.P2POp(dist.isend, host(t).contiguous(), glob(r), group))
        for t in recvs.get(r, ()):
            buf = torch.empty(t.shape, dtype=t.dtype) if (staged and t.is_cuda) else t
            ops.append(dist.P2POp(dist.irecv, buf, glob(r), group))
            if buf is not t:
                back.append((t, buf))
    for req in dist.batch_isend_irecv(ops):
        req.wait()
    for t, buf in back:
        t.copy_(buf)


def seq_to_heads(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, g: Geometry, start_frame: int,
                 group=None, rotate: bool = True, stream=None):
    """Sequence-parallel to head-parallel exchange of one chunk ("Accelerating Video Generation
    Inference with Sequential-Parallel 3D Positional Encoding Using a Global Time Index", sections
    2.A-2.C): rank r of the group holds tokens [r n, (r + 1) n) of q, k, v [n, heads, head_dim];
    returns (q_full, k_full, v_full), each [world * n, heads / world, head_dim]: all tokens of
    this rank's heads, Q and K rotated at their global positions when rotate. One pack launch
    (vdit_seq_pack) and one batched exchange of Q, K and V together."""
    world, rank = _group_info(group)
    n = q.shape[0]
    hg = g.heads // world
    full = tuple(torch.empty(world * n, hg, g.head_dim, dtype=q.dtype, device=q.device) for _ in range(3))
    send = torch.empty(world, 3, n, hg, g.head_dim, dtype=q.dtype, device=q.device) if world > 1 else None
    seq_pack(q, k, v, g, start_frame, rank, world, send, full, rotate, stream)
    if world > 1:
        exchange({r: [send[r, x] for x in range(3)] for r in range(world) if r != rank},
                 {r: [full[x][r * n:(r + 1) * n] for x in range(3)] for r in range(world) if r != rank},
                 group)
    return full


def heads_to_seq(o_full: torch.Tensor, g: Geometry, group=None, out: Optional[torch.Tensor] = None,
                 stream=None) -> torch.Tensor:
    """Return exchange after attention: o_full [world * n, heads / world, head_dim] (this rank's
    heads, all tokens) -> out [n, heads, head_dim] (this rank's tokens, all heads): one batched
    exchange and one unpack launch (vdit_seq_unpack)."""
    world, rank = _group_info(group)
    n = o_full.shape[0] // world
    hg = g.heads // world
    if out is None:
        out = torch.empty(n, g.heads, g.head_dim, dtype=o_full.dtype, device=o_full.device)
    recv = None
    if world > 1:
        recv = torch.empty(world, n, hg, g.head_dim, dtype=o_full.dtype, device=o_full.device)
        exchange({r: [o_full[r * n:(r + 1) * n]] for r in range(world) if r != rank},
                 {r: [recv[r]] for r in range(world) if r != rank}, group)
    return seq_unpack(recv, o_full[rank * n:(rank + 1) * n], out, g, rank, world, stream)


def _addr_array(addrs, n_ranks: int, name: str):
    addrs = [int(a) for a in addrs]
    if len(addrs) != n_ranks or any(a == 0 for a in addrs):
        raise ValueError(f"{name} must hold n_ranks device addresses")
    return (ctypes.c_void_p * n_ranks)(*addrs)


def seq_pack_peers(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, g: Geometry, start_frame: int,
                   rank: int, n_ranks: int, q_dst, k_dst, v_dst, rotate: bool = True, stream=None) -> None:
    """vdit_seq_pack_peers: this rank's q, k, v [n, heads, head_dim] (chunk-local tokens rank * n
    ..) written straight into every rank's head-sharded buffers; q_dst, k_dst, v_dst: n_ranks
    device addresses valid in this process (rank r's q_full / k_full / v_full [n_ranks * n,
    heads / n_ranks, head_dim]), Q and K rotated at their global positions when rotate."""
    n = q.shape[0]
    for name, t in (("q", q), ("k", k), ("v", v)):
        if t.dtype != torch.bfloat16 or t.dim() != 3 or tuple(t.shape) != (n, g.heads, g.head_dim):
            raise ValueError(f"{name} must be bf16 [n_tokens, heads, head_dim]")
    gc = g.c()
    _check(lib().vdit_seq_pack_peers(ctypes.byref(gc), _dev_ptr(q, "q"), _dev_ptr(k, "k"), _dev_ptr(v, "v"),
                                     _addr_array(q_dst, n_ranks, "q_dst"), _addr_array(k_dst, n_ranks, "k_dst"),
                                     _addr_array(v_dst, n_ranks, "v_dst"), int(rank), int(n_ranks),
                                     int(start_frame), n, int(bool(rotate)), _stream(stream)))


def seq_push_peers(o_full: torch.Tensor, g: Geometry, rank: int, n_ranks: int, out_dst, stream=None) -> None:
    """vdit_seq_push_peers: o_full [n_ranks * n, heads / n_ranks, head_dim] (this rank's heads,
    every rank's tokens) into every rank's out [n, heads, head_dim] at this rank's head columns;
    out_dst: n_ranks device addresses valid in this process."""
    hg = g.heads // n_ranks if n_ranks >= 1 else 0
    if (o_full.dtype != torch.bfloat16 or o_full.dim() != 3 or n_ranks < 1 or g.heads % n_ranks
            or o_full.shape[0] % n_ranks or tuple(o_full.shape[1:]) != (hg, g.head_dim)):
        raise ValueError("o_full must be bf16 [n_ranks * n_tokens, heads / n_ranks, head_dim]")
    gc = g.c()
    _check(lib().vdit_seq_push_peers(ctypes.byref(gc), _dev_ptr(o_full, "o_full"),
                                     _addr_array(out_dst, n_ranks, "out_dst"), int(rank), int(n_ranks),
                                     o_full.shape[0] // n_ranks, _stream(stream)))


class PeerExchange:
    """The sequence-parallel exchange over peer memory ("Accelerating Video Generation Inference
    with Sequential-Parallel 3D Positional Encoding Using a Global Time Index", section 2.C: the
    RoPE and the all-to-all of Q, K and V in one operation). Each rank allocates its head-sharded
    buffers q_full, k_full, v_full [world * n, heads / world, head_dim] and its output out [n,
    heads, head_dim] once; their CUDA IPC handles (torch's CUDA storage sharing) are exchanged with
    all_gather_object, so every rank holds the device addresses of every rank's buffers, and
    vdit_seq_pack_peers / vdit_seq_push_peers do the transfer with their own stores (over NVLink
    between GPUs). A barrier between the ranks precedes each kernel (no rank may still read the
    buffers it is about to overwrite) and follows it (every rank's rows have landed): a
    one-element all-reduce on the current stream with NCCL; with other backends (ranks sharing a
    GPU, tests) a device synchronisation and a host barrier. Calls run on the current stream.
    Every rank's buffers are mapped by the others, so the ranks keep their exchanges alive
    together and release them together: close() (a barrier, then the mappings are dropped) on
    every rank before any rank frees its exchange."""

    def __init__(self, g: Geometry, n_tokens: int, group=None, device=None):
        import torch.distributed as dist
        self.g, self.n, self.group = g, int(n_tokens), group
        self.world, self.rank = _group_info(group)
        if g.heads % self.world:
            raise ValueError("the group size must divide heads")
        dev = torch.device(device) if device is not None else torch.device("cuda", torch.cuda.current_device())
        hg = g.heads // self.world
        self.full = tuple(torch.empty(self.world * self.n, hg, g.head_dim, dtype=torch.bfloat16, device=dev)
                          for _ in range(3))
        self.out = torch.empty(self.n, g.heads, g.head_dim, dtype=torch.bfloat16, device=dev)
        bufs = (*self.full, self.out)
        self._mapped = []  # peer storages kept open for the lifetime of this object
        if self.world == 1:
            self.addrs = [[t.data_ptr()] for t in bufs]
            self._nccl = False
            return
        self._nccl = dist.get_backend(group) == "nccl"
        mine = []
        for t in bufs:
            st = t.untyped_storage()
            mine.append((st._share_cuda_(), t.data_ptr() - st.data_ptr()))
        everyone = [None] * self.world
        dist.all_gather_object(everyone, mine, group=group)
        self.addrs = [[0] * self.world for _ in bufs]
        for r in range(self.world):
            for i, (handle, offset) in enumerate(everyone[r]):
                if r == self.rank:
                    self.addrs[i][r] = bufs[i].data_ptr()
                    continue
                st = torch.UntypedStorage._new_shared_cuda(*handle)
                self._mapped.append(st)
                self.addrs[i][r] = st.data_ptr() + offset
        self._flag = torch.zeros(1, device=dev)

    def _barrier(self):
        if self.world == 1:
            return
        import torch.distributed as dist
        if self._nccl:
            dist.all_reduce(self._flag, group=self.group)
        else:
            torch.cuda.synchronize()
            dist.barrier(group=self.group)

    def close(self) -> None:
        """Collective: waits until no rank can still write into this rank's buffers, then drops
        the mappings of the other ranks' buffers."""
        self._barrier()
        self._mapped.clear()
        self.addrs = None

    def seq_to_heads(self, q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, start_frame: int,
                     rotate: bool = True):
        """This rank's q, k, v [n, heads, head_dim] (tokens rank * n ..) -> (q_full, k_full,
        v_full), each [world * n, heads / world, head_dim] (every token of this rank's heads)."""
        self._barrier()
        seq_pack_peers(q, k, v, self.g, start_frame, self.rank, self.world, *self.addrs[:3], rotate=rotate)
        self._barrier()
        return self.full

    def heads_to_seq(self, o_full: torch.Tensor) -> torch.Tensor:
        """o_full [world * n, heads / world, head_dim] -> out [n, heads, head_dim] (this rank's
        tokens, every head)."""
        self._barrier()
        seq_push_peers(o_full, self.g, self.rank, self.world, self.addrs[3])
        self._barrier()
        return self.out


class KVCache:
    """Ring KV cache [heads, capacity_frames * frame_tokens, head_dim] (bf16, zero-filled) plus
    the bookkeeping of which global frames it holds."""

    def __init__(self, g: Geometry, capacity_frames: int, device="cuda"):
        self.g = g
        self.capacity_frames = capacity_frames
        shape = (g.heads, capacity_frames * g.frame_tokens, g.head_dim)
        self.k = torch.zeros(shape, dtype=torch.bfloat16, device=device)
        self.v = torch.zeros(shape, dtype=torch.bfloat16, device=device)
        self.first_frame: Optional[int] = None
        self.last_frame: Optional[int] = None

    def _check_next(self, start_frame: int) -> None:
        if self.last_frame is not None:
            if start_frame > self.last_frame + 1:
                raise ValueError("append would leave a gap of frames")
            if start_frame < self.first_frame:
                raise ValueError("frame older than the cache window")

    def _note(self, start_frame: int, n: int) -> None:
        last = start_frame + n - 1
        self.last_frame = last if self.last_frame is None else max(self.last_frame, last)
        first = start_frame if self.first_frame is None else self.first_frame
        self.first_frame = max(first, self.last_frame - self.capacity_frames + 1)

    def append(self, k: torch.Tensor, v: torch.Tensor, start_frame: int, stream=None) -> None:
        """Rotate K at its global frames and write K', V into the ring (vdit_kv_append)."""
        self._check_next(start_frame)
        kv_append(self.k, self.v, self.g, self.capacity_frames, k, v, start_frame, stream)
        self._note(start_frame, k.shape[0] // self.g.frame_tokens)

    def write(self, k_rotated: torch.Tensor, v: torch.Tensor, start_frame: int, stream=None) -> None:
        """Write an already rotated chunk (K' and V) into the ring (vdit_kv_write)."""
        self._check_next(start_frame)
        kv_write(self.k, self.v, self.g, self.capacity_frames, k_rotated, v, start_frame, stream)
        self._note(start_frame, k_rotated.shape[0] // self.g.frame_tokens)

    def push(self, k: torch.Tensor, v: torch.Tensor, dst: int, group=None) -> list:
        """Wave Parallelism's K/V forward push (Wave Forcing / WaveRT): send a chunk's K and V as
        given to append (before RoPE: one contiguous message each; the receiver's append rotates
        K at the same global frames in the same pass that places it in its ring, so sending K'
        would save no work) one way to rank dst, which appends them to its own cache with
        receive(). The sends are asynchronous (isend; NCCL on GPUs), so they overlap the attention
        that follows; returns the work handles to wait on before k, v are reused. Backends
        without device-tensor point-to-point (gloo) stage through host memory."""
        import torch.distributed as dist
        glob = dst if group is None else dist.get_global_rank(group, dst)
        staged = dist.get_backend(group) != "nccl"
        bufs = [t.detach().cpu() if (staged and t.is_cuda) else t.contiguous() for t in (k, v)]
        return [dist.isend(b, glob, group=group) for b in bufs]

    def receive(self, start_frame: int, n_frames: int, src: int, group=None, stream=None) -> None:
        """Receive a chunk pushed by rank src and append it here (RoPE at its global frames, ring
        write), as the sender appended it to its own cache."""
        import torch.distributed as dist
        glob = src if group is None else dist.get_global_rank(group, src)
        staged = dist.get_backend(group) != "nccl"
        shape = (n_frames * self.g.frame_tokens, self.g.heads, self.g.head_dim)
        dev = torch.device("cpu") if staged else self.k.device
        k = torch.empty(shape, dtype=self.k.dtype, device=dev)
        v = torch.empty_like(k)
        dist.recv(k, glob, group=group)
        dist.recv(v, glob, group=group)
        if staged and self.k.is_cuda:
            k, v = k.to(self.k.device), v.to(self.k.device)
        self.append(k, v, start_frame, stream)

    def project_append(self, x: torch.Tensor, w: torch.Tensor, start_frame: int,
                       q_out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
        """Fused QKV projection of the chunk x (vdit_qkv_rope): K', V into the ring; returns the
        rotated Q."""
        self._check_next(start_frame)
        q = qkv_rope(x, w, self.g, start_frame, self.k, self.v, self.capacity_frames, q_out, stream)
        self._note(start_frame, x.shape[0] // self.g.frame_tokens)
        return q


class Plan:
    """Tile schedule of the mask for q_frames query frames from q_start_frame against the frames
    a ring cache holds (host-built, exact); uploaded to the current device on construction unless
    upload=False."""

    def __init__(self, g: Geometry, mask: Mask, q_start_frame: int, q_frames: int,
                 cache: Optional[KVCache] = None, capacity_frames: Optional[int] = None,
                 kv_first_frame: Optional[int] = None, kv_last_frame: Optional[int] = None,
                 upload: bool = True, stream=None):
        if cache is not None:
            capacity_frames, kv_first_frame, kv_last_frame = (
                cache.capacity_frames, cache.first_frame, cache.last_frame)
        self.g, self.mask = g, mask
        self.q_start_frame, self.q_frames = q_start_frame, q_frames
        self._h = ctypes.c_void_p()
        gc, mc = g.c(), mask.c()
        _check(lib().vdit_attn_plan(ctypes.byref(self._h), ctypes.byref(gc), ctypes.byref(mc),
                                    int(q_start_frame), int(q_frames), int(capacity_frames),
                                    int(kv_first_frame), int(kv_last_frame)))
        if upload:
            self.upload(stream)

    def upload(self, stream=None) -> None:
        _check(lib().vdit_plan_upload(self._h, _stream(stream)))

    @property
    def info(self) -> dict:
        i = _PlanInfo()
        _check(lib().vdit_plan_info(self._h, ctypes.byref(i)))
        return {f: getattr(i, f) for f, _ in _PlanInfo._fields_}

    def export(self):
        """(row_ptr, col_idx, full) as CPU int32 / int32 / uint8 tensors."""
        inf = self.info
        rp = torch.zeros(inf["q_tiles"] + 1, dtype=torch.int32)
        ci = torch.zeros(max(1, inf["tiles"]), dtype=torch.int32)
        fu = torch.zeros(max(1, inf["tiles"]), dtype=torch.uint8)
        _check(lib().vdit_plan_export(self._h, ctypes.c_void_p(rp.data_ptr()),
                                      ctypes.c_void_p(ci.data_ptr()), ctypes.c_void_p(fu.data_ptr())))
        n = inf["tiles"]
        return rp, ci[:n], fu[:n]

    def export_masks(self):
        """(mask_index [tiles] int32, words [blocks, 128, 4] uint32 as int64 numpy): the per-row
        keep masks of the partial tiles (mask_index -1 for a full tile)."""
        import numpy as np
        inf = self.info
        idx = np.zeros(max(1, inf["tiles"]), np.int32)
        words = np.zeros(max(4, inf["mask_bytes"] // 4), np.uint32)
        _check(lib().vdit_plan_export_masks(self._h, ctypes.c_void_p(idx.ctypes.data),
                                            ctypes.c_void_p(words.ctypes.data)))
        return idx[:inf["tiles"]], words[:inf["mask_bytes"] // 4].reshape(-1, 128, 4)

    def export_work(self):
        """The kernel's work list: (row_ptr [q_tiles + 1], key_row [entries], mask_index
        [entries], words [blocks, 128, 4]) as numpy arrays (vdit_plan_export_work)."""
        import numpy as np
        inf = self.info
        rp = np.zeros(inf["q_tiles"] + 1, np.int32)
        kr = np.zeros(max(1, inf["work_entries"]), np.int32)
        mi = np.zeros(max(1, inf["work_entries"]), np.int32)
        words = np.zeros(max(4, inf["work_mask_bytes"] // 4), np.uint32)
        _check(lib().vdit_plan_export_work(self._h, ctypes.c_void_p(rp.ctypes.data),
                                           ctypes.c_void_p(kr.ctypes.data),
                                           ctypes.c_void_p(mi.ctypes.data),
                                           ctypes.c_void_p(words.ctypes.data)))
        n = inf["work_entries"]
        return rp, kr[:n], mi[:n], words[:inf["work_mask_bytes"] // 4].reshape(-1, 128, 4)

    def schedule_for(self, sm_count: int):
        """The CTA schedule vdit_plan_upload would fix on a device with sm_count SMs
        (vdit_plan_export_schedule): (cta [ctas, 5]: q-block, head, first entry, entries, slot or
        -1; merge [cut units, 4]: q-block, head, first slot, pieces) as numpy int32 arrays."""
        import numpy as np
        n_cta, n_cut = ctypes.c_int(), ctypes.c_int()
        _check(lib().vdit_plan_export_schedule(self._h, int(sm_count), ctypes.byref(n_cta),
                                               ctypes.byref(n_cut), None, None))
        cta = np.zeros((max(1, n_cta.value), 5), np.int32)
        merge = np.zeros((max(1, n_cut.value), 4), np.int32)
        _check(lib().vdit_plan_export_schedule(self._h, int(sm_count), ctypes.byref(n_cta),
                                               ctypes.byref(n_cut), ctypes.c_void_p(cta.ctypes.data),
                                               ctypes.c_void_p(merge.ctypes.data)))
        return cta[:n_cta.value], merge[:n_cut.value]

    def flops(self) -> float:
        """Unmasked-entry FLOPs of one forward: 4 * head_dim per kept (query, key, head)."""
        return 4.0 * self.g.head_dim * self.g.heads * self.info["kept_pairs"]

    def __del__(self):
        h = getattr(self, "_h", None)
        if h is not None and h.value and _lib is not None:
            _lib.vdit_plan_destroy(h)
            self._h = ctypes.c_void_p()


def attn_forward(plan: Plan, q: torch.Tensor, cache: Optional[KVCache] = None,
                 k_cache: Optional[torch.Tensor] = None, v_cache: Optional[torch.Tensor] = None,
                 out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
                 scale: Optional[float] = None, stream=None, q_rotated: bool = False) -> torch.Tensor:
    """o = masked softmax(RoPE(q) . K'^T * scale) V over the plan; q is unrotated (RoPE fused into
    the Q load, vdit_attn_forward) unless q_rotated (vdit_attn_forward_rotated)."""
    if cache is not None:
        k_cache, v_cache = cache.k, cache.v
    g = plan.g
    if q.dtype != torch.bfloat16 or q.dim() != 3 or q.shape[1:] != (g.heads, g.head_dim):
        raise ValueError("q must be bf16 [q_tokens, heads, head_dim]")
    if q.shape[0] != plan.info["q_tokens"]:
        raise ValueError("q has a different token count than the plan")
    o = torch.empty_like(q) if out is None else out
    if scale is None:
        scale = 1.0 / math.sqrt(g.head_dim)
    lse_ptr = ctypes.c_void_p(0)
    if lse is not None:
        if lse.dtype != torch.float32 or lse.shape != (g.heads, q.shape[0]) or not lse.is_contiguous():
            raise ValueError("lse must be fp32 [heads, q_tokens]")
        lse_ptr = ctypes.c_void_p(lse.data_ptr())
    fn = lib().vdit_attn_forward_rotated if q_rotated else lib().vdit_attn_forward
    _check(fn(plan._h, _dev_ptr(q, "q"), _dev_ptr(k_cache, "k_cache"), _dev_ptr(v_cache, "v_cache"),
              _dev_ptr(o, "out"), lse_ptr, float(scale), _stream(stream)))
    return o


def get_status() -> int:
    """Reads and clears the device status word (OK or ERR_TIMEOUT); synchronises the device."""
    s = ctypes.c_int(0)
    _check(lib().vdit_get_status(ctypes.byref(s)))
    return s.value
