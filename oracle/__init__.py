"""Python marshalling for the fp64 CPU oracle in ``vdit_oracle.c``.

TEST INFRASTRUCTURE: only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline /
reference leg of ``bench.py`` import this package. It shares no code with the product
(``video_diffusion_transformer_vdit_b200``) and never imports it.

Every function converts numpy arrays to contiguous C buffers and calls the C oracle; the
arithmetic lives in ``vdit_oracle.c`` (see its header for the pages each step follows), except
``qkv_project`` and the logits of ``dynamic_keep``, whose one step is numpy's float64 matrix
product.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "vdit_oracle.c")
_LIB = os.path.join(_HERE, "libvdit_oracle.so")
_lib = None

_i32p = np.ctypeslib.ndpointer(dtype=np.int32, flags="C_CONTIGUOUS")
_u8p = np.ctypeslib.ndpointer(dtype=np.uint8, flags="C_CONTIGUOUS")
_f64p = np.ctypeslib.ndpointer(dtype=np.float64, flags="C_CONTIGUOUS")
_L = ctypes.c_long
_I = ctypes.c_int
_LL = ctypes.c_longlong
_D = ctypes.c_double


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (plain -O2, no fast-math, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fno-fast-math", "-ffp-contract=off", "-fopenmp",
                               "-fPIC", "-shared", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_LIB)
        L.vo_positions.argtypes = [_L, _I, _I, _I, _i32p, _i32p, _i32p]
        L.vo_rope3d.argtypes = [_f64p, _f64p, _L, _I, _I, _i32p, _i32p, _i32p, _I, _I, _I, _D]
        L.vo_mask_rows.argtypes = [_u8p, _L, _i32p, _i32p, _i32p, _L, _i32p, _i32p, _i32p, _u8p,
                                   _I, _I, _I, _LL, _I, _I]
        L.vo_attention.argtypes = [_f64p, _f64p, _f64p, _u8p, _L, _L, _I, _I, _D, _f64p, _f64p]
        L.vo_tiles.argtypes = [_L, _i32p, _i32p, _i32p, _L, _i32p, _i32p, _i32p, _u8p,
                               _I, _I, _I, _LL, _I, _I, _I, _i32p, _i32p, _u8p]
        L.vo_tiles.restype = _LL
        L.vo_cache_positions.argtypes = [_I, _I, _I, _I, _I, _i32p, _i32p, _i32p, _u8p]
        L.vo_kv_append.argtypes = [_f64p, _f64p, _I, _I, _I, _I, _I, _I, _I, _I, _D,
                                   _f64p, _f64p, _I, _I]
        L.vo_threads.restype = _I
        L.vo_round_bf16.argtypes = [_f64p, _L]
        _lib = L
    return _lib


def threads() -> int:
    """OpenMP threads the oracle's parallel loops use."""
    return int(lib().vo_threads())


@dataclass(frozen=True)
class Geometry:
    """Latent grid and head layout: grid_h x grid_w patches per frame, RoPE bands t/h/w."""
    grid_h: int
    grid_w: int
    heads: int
    head_dim: int
    band_t: int
    band_h: int
    band_w: int
    theta: float = 10000.0

    @property
    def frame_tokens(self) -> int:
        return self.grid_h * self.grid_w


@dataclass(frozen=True)
class Mask:
    """Mask predicate: block-causal over chunks of ``chunk_frames`` global frames and/or the
    radial window (Chebyshev distance <= w0 * 2^(-gamma_shift * |dt|), full width when |dt| is
    a multiple of ``lam``). Both off = dense."""
    block_causal: bool = False
    radial: bool = False
    chunk_frames: int = 3
    w0: int = 52
    gamma_shift: int = 1
    lam: int = 8

    def args(self):
        return (int(self.block_causal), int(self.radial), int(self.chunk_frames),
                int(self.w0), int(self.gamma_shift), int(self.lam))


def _c(a, dt):
    return np.ascontiguousarray(a, dtype=dt)


def positions(n_tokens: int, grid_h: int, grid_w: int, start_frame: int):
    t = np.empty(n_tokens, np.int32)
    h = np.empty(n_tokens, np.int32)
    w = np.empty(n_tokens, np.int32)
    lib().vo_positions(n_tokens, grid_h, grid_w, start_frame, t, h, w)
    return t, h, w


def rope3d(x: np.ndarray, pos, g: Geometry) -> np.ndarray:
    """RoPE of x [n, heads, D] (float64) at positions pos = (t, h, w)."""
    x = _c(x, np.float64)
    n, heads, d = x.shape
    y = np.empty_like(x)
    t, h, w = (_c(p, np.int32) for p in pos)
    lib().vo_rope3d(x, y, n, heads, d, t, h, w, g.band_t, g.band_h, g.band_w, g.theta)
    return y


def qkv_project(x: np.ndarray, w: np.ndarray, heads: int, head_dim: int):
    """The QKV projections ("Accelerating Video Generation Inference with Sequential-Parallel 3D
    Positional Encoding Using a Global Time Index", section 2.C, names them as the producer of the
    rotated Q and K): [Q | K | V] = x w^T in float64, x [n, d_model], w [3 * heads * head_dim,
    d_model] (rows of W_q, W_k, W_v), split into three [n, heads, head_dim] arrays. Its one step
    is numpy's matrix product (a library primitive); RoPE and the cache write are the separate
    oracle functions rope3d and kv_append."""
    x = np.asarray(x, np.float64)
    w = np.asarray(w, np.float64)
    hd = heads * head_dim
    if w.shape != (3 * hd, x.shape[1]):
        raise ValueError("w must be [3 * heads * head_dim, d_model]")
    y = x @ w.T
    return tuple(y[:, i * hd:(i + 1) * hd].reshape(-1, heads, head_dim) for i in range(3))


def mask_rows(qpos, kpos, kvalid, m: Mask) -> np.ndarray:
    tq, hq, wq = (_c(p, np.int32) for p in qpos)
    tk, hk, wk = (_c(p, np.int32) for p in kpos)
    nq, nk = len(tq), len(tk)
    out = np.empty((nq, nk), np.uint8)
    lib().vo_mask_rows(out, nq, tq, hq, wq, nk, tk, hk, wk, _c(kvalid, np.uint8), *m.args())
    return out


def attention(q, k, v, mask, scale: float):
    """(o [nq, heads, D], lse [heads, nq]) of masked softmax attention in float64."""
    q = _c(q, np.float64)
    k = _c(k, np.float64)
    v = _c(v, np.float64)
    nq, heads, d = q.shape
    nk = k.shape[0]
    o = np.empty((nq, heads, d), np.float64)
    lse = np.empty((heads, nq), np.float64)
    lib().vo_attention(q, k, v, _c(mask, np.uint8), nq, nk, heads, d, float(scale), o, lse)
    return o, lse


def round_bf16(x) -> np.ndarray:
    """x rounded to the nearest bfloat16 value (ties to even), returned as float64."""
    y = np.array(x, dtype=np.float64, order="C", copy=True)
    lib().vo_round_bf16(y.reshape(-1), y.size)
    return y


def dynamic_keep(q, k, cand, scale: float, tau: float, logits: str = "f64"):
    """Keep decision of the dynamic-threshold mode of "DynamicRad: Content-Adaptive Sparse
    Attention for Long Video Diffusion", section 2: the pre-softmax logits are the importance
    proxies and an adaptive threshold filters the structured candidate set. Reading taken: per
    head and query row, with z = scale * q . k over the row's candidates (cand [nq, nk], from
    mask_rows) and z_max their maximum, a candidate is kept iff z >= z_max - tau.

    logits selects the precision of the decision. "f64": q and k as given. "bf16": q and k are
    first rounded to bfloat16 (round_bf16), the operand precision of the tensor-core kernel, and
    the products are summed in float64: a threshold is a decision taken from floating point, and
    both sides take it in the same precision. The logits are numpy float64 matrix products (a
    library primitive). Returns (keep [heads, nq, nk] bool, z [heads, nq, nk] with -inf outside
    the candidates, thr [heads, nq, 1] = z_max - tau)."""
    if logits not in ("f64", "bf16"):
        raise ValueError("logits must be 'f64' or 'bf16'")
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    if logits == "bf16":
        q, k = round_bf16(q), round_bf16(k)
    cand = np.asarray(cand).astype(bool)
    nq, heads, _ = q.shape
    keep = np.zeros((heads,) + cand.shape, bool)
    z_all = np.full((heads,) + cand.shape, -np.inf)
    thr = np.full((heads, nq, 1), -np.inf)
    for h in range(heads):
        z = scale * (q[:, h] @ k[:, h].T)
        zc = np.where(cand, z, -np.inf)
        zmax = zc.max(axis=1, keepdims=True) if cand.shape[1] else np.full((nq, 1), -np.inf)
        keep[h] = cand & (z >= zmax - tau)
        z_all[h] = zc
        thr[h] = zmax - tau
    return keep, z_all, thr


def attention_dynamic(q, k, v, cand, scale: float, tau: float, logits: str = "f64"):
    """Attention in the dynamic-threshold mode (dynamic_keep's decision, in the precision
    `logits` selects), then masked softmax attention over the kept keys with the float64 q, k and
    v (the C oracle's attention). Returns (o [nq, heads, D], lse [heads, nq], keep [heads, nq, nk])."""
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    nq, heads, d = q.shape
    keep, _, _ = dynamic_keep(q, k, cand, scale, tau, logits)
    o = np.empty((nq, heads, d))
    lse = np.empty((heads, nq))
    for h in range(heads):
        oh, lh = attention(q[:, h:h + 1], k[:, h:h + 1], v[:, h:h + 1], keep[h].astype(np.uint8), scale)
        o[:, h] = oh[:, 0]
        lse[h] = lh[0]
    return o, lse, keep


def tiles(qpos, kpos, kvalid, m: Mask, tile: int = 128):
    """(row_ptr, col_idx, full, kept_pairs) of the explicit mask's tile list."""
    tq, hq, wq = (_c(p, np.int32) for p in qpos)
    tk, hk, wk = (_c(p, np.int32) for p in kpos)
    nq, nk = len(tq), len(tk)
    n_qt, n_kt = -(-nq // tile), -(-nk // tile)
    row_ptr = np.zeros(n_qt + 1, np.int32)
    col = np.zeros(max(1, n_qt * n_kt), np.int32)
    full = np.zeros(max(1, n_qt * n_kt), np.uint8)
    kept = lib().vo_tiles(nq, tq, hq, wq, nk, tk, hk, wk, _c(kvalid, np.uint8), *m.args(),
                          tile, row_ptr, col, full)
    n = int(row_ptr[-1])
    return row_ptr, col[:n].copy(), full[:n].copy(), int(kept)


def cache_positions(capacity_frames: int, first_frame: int, last_frame: int,
                    grid_h: int, grid_w: int):
    n = capacity_frames * grid_h * grid_w
    t = np.empty(n, np.int32)
    h = np.empty(n, np.int32)
    w = np.empty(n, np.int32)
    valid = np.empty(n, np.uint8)
    lib().vo_cache_positions(capacity_frames, first_frame, last_frame, grid_h, grid_w,
                             t, h, w, valid)
    return (t, h, w), valid


def kv_append(k_cache: np.ndarray, v_cache: np.ndarray, capacity_frames: int, g: Geometry,
              k: np.ndarray, v: np.ndarray, start_frame: int, n_frames: int) -> None:
    """In-place append into float64 caches [heads, capacity_frames * frame_tokens, D]."""
    assert k_cache.flags.c_contiguous and v_cache.flags.c_contiguous
    assert k_cache.dtype == np.float64 and v_cache.dtype == np.float64
    lib().vo_kv_append(k_cache, v_cache, capacity_frames, g.grid_h, g.grid_w, g.heads,
                       g.head_dim, g.band_t, g.band_h, g.band_w, g.theta,
                       _c(k, np.float64), _c(v, np.float64), start_frame, n_frames)
