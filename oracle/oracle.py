"""numpy front end of the C oracle (``csa_oracle.c``).

TEST INFRASTRUCTURE ONLY.  Every function here marshals numpy arrays into the
C oracle and back; the arithmetic lives in ``csa_oracle.c``.  The composite
helpers (``csa_prefill``, ``hca_prefill``, ``csa_decode``) chain the oracle's
steps in the order the pages describe: compress -> (norm, RoPE) -> indexer ->
top-k -> attention over selected entries plus the sliding window.
"""
from __future__ import annotations

import ctypes
import math
import os
import subprocess
import threading

import numpy as np

__all__ = [
    "build", "lib", "n_visible", "pool", "rmsnorm", "rope", "mxfp4_quantize", "mxfp4_dequantize",
    "index_scores", "topk", "attention", "hca_select", "csa_prefill", "hca_prefill", "csa_decode",
    "window_rows", "prep_queries", "entries_rows", "grouped_out_proj", "F64", "F32", "BF16",
]

F64, F32, BF16 = 0, 1, 2
_HERE = os.path.dirname(os.path.abspath(__file__))
_SO = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile csa_oracle.c into liboracle.so (gcc -O2, OpenMP, no fast-math)."""
    src = os.path.join(_HERE, "csa_oracle.c")
    hdr = os.path.join(_HERE, "csa_oracle.h")
    fresh = os.path.exists(_SO) and os.path.getmtime(_SO) >= max(os.path.getmtime(src), os.path.getmtime(hdr))
    if force or not fresh:
        tmp = _SO + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared", "-Wall",
                               "-ffp-contract=off", "-o", tmp, src, "-lm"])
        os.replace(tmp, _SO)
    return _SO


def lib():
    global _lib
    with _lock:
        if _lib is None:
            build()
            L = ctypes.CDLL(_SO)
            P, I, I64, D = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_double
            L.orc_n_visible.argtypes = [I64, I, I64]
            L.orc_n_visible.restype = I64
            L.orc_pool.argtypes = [I, I, I, I, I, P, P, P, P]
            L.orc_pool.restype = I
            L.orc_rmsnorm.argtypes = [I64, I, D, P]
            L.orc_rope.argtypes = [I64, I, I, D, P, P]
            L.orc_mxfp4_quantize.argtypes = [I64, I, P, P, P]
            L.orc_mxfp4_dequantize.argtypes = [I64, I, P, P, P]
            L.orc_index_scores.argtypes = [I, I, I, P, P, P, P, P, I, P, P, P, P]
            L.orc_index_scores.restype = I64
            L.orc_topk.argtypes = [I, I, P, P, I, P, P, P]
            L.orc_attention.argtypes = [I, I, I, D, I, P, P, P, I, I, P, I, P, P, I, I, I, P, P, P, P]
            L.orc_grouped_out_proj.argtypes = [I, I, I, I, I, I, I, P, P, P, P, P]
            _lib = L
    return _lib


def _p(a: np.ndarray | None):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _dt(a: np.ndarray) -> int:
    if a.dtype == np.float64:
        return F64
    if a.dtype == np.float32:
        return F32
    if a.dtype == np.uint16:
        return BF16
    raise TypeError(f"oracle inputs must be float64, float32 or bf16 bits (uint16), got {a.dtype}")


def _c(a, dtype=None):
    return np.ascontiguousarray(a if dtype is None else np.asarray(a, dtype=dtype))


def n_visible(t: int, m: int, n_entries: int) -> int:
    return int(lib().orc_n_visible(int(t), int(m), int(n_entries)))


def pool(kv: np.ndarray, z: np.ndarray, bias: np.ndarray, m: int, overlap: bool) -> np.ndarray:
    """Softmax pooling of one sequence: kv, z [T, C] -> [T//m, C] float64."""
    kv, z = _c(kv), _c(z)
    assert kv.dtype == z.dtype and kv.shape == z.shape and kv.ndim == 2
    T, C = kv.shape
    bias = _c(bias, np.float32)
    assert bias.shape == ((2 if overlap else 1) * m, C)
    out = np.zeros((T // m, C), dtype=np.float64)
    lib().orc_pool(T, C, m, int(bool(overlap)), _dt(kv), _p(kv), _p(z), _p(bias), _p(out))
    return out


def rmsnorm(x: np.ndarray, eps: float) -> np.ndarray:
    y = _c(x, np.float64).copy()
    C = y.shape[-1]
    lib().orc_rmsnorm(y.size // C, C, float(eps), _p(y))
    return y


def rope(x: np.ndarray, pos: np.ndarray, rope_dims: int, theta: float) -> np.ndarray:
    """Partial RoPE on rows of x [..., C]; pos broadcast over the leading dims of x."""
    y = _c(x, np.float64).copy()
    C = y.shape[-1]
    rows = y.size // C
    p = np.broadcast_to(np.asarray(pos, dtype=np.int64).reshape(pos.shape + (1,) * (y.ndim - 1 - np.ndim(pos))),
                        y.shape[:-1])
    p = _c(p.reshape(rows), np.int64)
    lib().orc_rope(rows, C, int(rope_dims), float(theta), _p(p), _p(y))
    return y


def mxfp4_quantize(x: np.ndarray):
    """float32 [..., cols] -> (packed uint8 [..., cols/2], scales uint8 [..., cols/32])."""
    x = _c(x, np.float32)
    cols = x.shape[-1]
    assert cols % 32 == 0
    rows = x.size // cols
    packed = np.zeros(x.shape[:-1] + (cols // 2,), dtype=np.uint8)
    scales = np.zeros(x.shape[:-1] + (cols // 32,), dtype=np.uint8)
    lib().orc_mxfp4_quantize(rows, cols, _p(x), _p(packed), _p(scales))
    return packed, scales


def mxfp4_dequantize(packed: np.ndarray, scales: np.ndarray) -> np.ndarray:
    packed, scales = _c(packed, np.uint8), _c(scales, np.uint8)
    cols = packed.shape[-1] * 2
    rows = packed.size // (cols // 2)
    out = np.zeros(packed.shape[:-1] + (cols,), dtype=np.float64)
    lib().orc_mxfp4_dequantize(rows, cols, _p(packed), _p(scales), _p(out))
    return out


def index_scores(q_packed, q_scales, w, q_seq, n_vis, k_packed, k_scales, want64: bool = False):
    """Indexer scores.  q_* [nq,Hi,Di/2|Di/32], w [nq,Hi], k_* [B,E_max,Di/2|Di/32].

    Returns (s32 [nq,E_max] float32 with -inf where not visible, s64 or None, n_inexact)."""
    q_packed, q_scales = _c(q_packed, np.uint8), _c(q_scales, np.uint8)
    k_packed, k_scales = _c(k_packed, np.uint8), _c(k_scales, np.uint8)
    w = _c(w, np.float32)
    nq, Hi, half = q_packed.shape
    Di = half * 2
    B, E_max, _ = k_packed.shape
    q_seq, n_vis = _c(q_seq, np.int32), _c(n_vis, np.int32)
    s32 = np.full((nq, E_max), -np.inf, dtype=np.float32)
    s64 = np.full((nq, E_max), -np.inf, dtype=np.float64) if want64 else None
    bad = lib().orc_index_scores(nq, Hi, Di, _p(q_packed), _p(q_scales), _p(w), _p(q_seq), _p(n_vis), E_max,
                                 _p(k_packed), _p(k_scales), _p(s32), _p(s64))
    return s32, s64, int(bad)


def topk(scores: np.ndarray, n_vis: np.ndarray, k: int):
    """-> (idx [nq,k] int32 ascending / -1 padded, cnt [nq], kth [nq,2] float32)."""
    scores = _c(scores, np.float32)
    nq, E_stride = scores.shape
    n_vis = _c(n_vis, np.int32)
    idx = np.zeros((nq, k), dtype=np.int32)
    cnt = np.zeros((nq,), dtype=np.int32)
    kth = np.zeros((nq, 2), dtype=np.float32)
    lib().orc_topk(nq, E_stride, _p(scores), _p(n_vis), int(k), _p(idx), _p(cnt), _p(kth))
    return idx, cnt, kth


def attention(q, q_pos, q_seq, entries, idx, cnt, window, wbase, W: int, scale: float | None = None):
    """Joint-softmax MQA over selected entries plus window rows.

    q [nq,H,D]; entries [B,E_max,D]; idx [nq,k]; window [B,Tw,D]; arrays may be
    float64, float32 or bf16 bits.  Returns (out [nq,H,D] float64, lse [nq,H])."""
    q, entries, window = _c(q), _c(entries), _c(window)
    nq, H, D = q.shape
    B, E_max, _ = entries.shape
    Tw = window.shape[1]
    idx, cnt = _c(idx, np.int32), _c(cnt, np.int32)
    k = idx.shape[1]
    q_pos, q_seq, wbase = _c(q_pos, np.int64), _c(q_seq, np.int32), _c(wbase, np.int64)
    scale = 1.0 / math.sqrt(D) if scale is None else float(scale)
    out = np.zeros((nq, H, D), dtype=np.float64)
    lse = np.zeros((nq, H), dtype=np.float64)
    lib().orc_attention(nq, H, D, scale, _dt(q), _p(q), _p(q_pos), _p(q_seq), E_max, _dt(entries), _p(entries),
                        k, _p(idx), _p(cnt), int(W), Tw, _dt(window), _p(window), _p(wbase), _p(out), _p(lse))
    return out, lse


def hca_select(q_pos: np.ndarray, q_seq: np.ndarray, n_entries: np.ndarray, mprime: int):
    """HCA selects every visible entry: idx = 0..n_vis-1 (as an index list for ``attention``)."""
    nv = np.array([n_visible(t, mprime, n_entries[s]) for t, s in zip(q_pos, q_seq)], dtype=np.int32)
    kmax = max(1, int(nv.max()) if nv.size else 1)
    idx = np.full((len(nv), kmax), -1, dtype=np.int32)
    for i, v in enumerate(nv):
        idx[i, :v] = np.arange(v, dtype=np.int32)
    return idx, nv


def window_rows(kv: np.ndarray, norm: bool, eps: float, rope_dims: int, theta: float) -> np.ndarray:
    """Raw-token window rows of one sequence: RoPE_u(RMSNorm(kv[u])) (norm optional), float64 [T, C]."""
    x = _c(kv)
    if x.dtype == np.uint16:
        x = (x.astype(np.uint32) << 16).view(np.float32)
    x = x.astype(np.float64)
    if norm:
        x = rmsnorm(x, eps)
    return rope(x, np.arange(x.shape[0], dtype=np.int64), rope_dims, theta)


def prep_queries(q: np.ndarray, pos: np.ndarray, norm: bool, eps: float, rope_dims: int, theta: float):
    """Queries [T, H, D] -> RoPE_t(RMSNorm per head), float64."""
    x = _c(q)
    if x.dtype == np.uint16:
        x = (x.astype(np.uint32) << 16).view(np.float32)
    x = x.astype(np.float64)
    if norm:
        x = rmsnorm(x, eps)
    return rope(x, np.asarray(pos, dtype=np.int64), rope_dims, theta)


def entries_rows(kv, z, bias, m, overlap, norm, eps, rope_dims, theta):
    """Compressed entries of one sequence: RoPE at m(j+1)-1 of RMSNorm (optional) of the pooled rows."""
    e = pool(kv, z, bias, m, overlap)
    if norm:
        e = rmsnorm(e, eps)
    pos = (np.arange(e.shape[0], dtype=np.int64) + 1) * m - 1
    return rope(e, pos, rope_dims, theta)


def csa_prefill(wl, inp: dict, b: int = 0, rows: np.ndarray | None = None):
    """Whole CSA prefill layer for sequence b of a prefill workload.

    Returns a dict with the intermediates (entries, window, q, indexer keys,
    scores, top-k) and the attention output for the query rows ``rows``
    (default: all tokens)."""
    T = inp["kv"].shape[1]
    rows = np.arange(T) if rows is None else np.asarray(rows)
    ent = entries_rows(inp["kv"][b], inp["z"][b], inp["bias"], wl.m, wl.overlap, wl.norm, wl.eps, wl.rope_dims,
                   wl.theta)
    win = window_rows(inp["kv"][b], wl.norm, wl.eps, wl.rope_dims, wl.theta)
    qf = prep_queries(inp["q"][b][rows], rows, wl.norm, wl.eps, wl.rope_dims, wl.theta)
    # indexer keys: pooled raw indexer keys (no norm, no RoPE), then MXFP4
    ki = pool(inp["ki"][b], inp["zi"][b], inp["bias_i"], wl.m, wl.overlap)
    k_packed, k_scales = mxfp4_quantize(ki.astype(np.float32))
    qi = inp["qi"][b][rows]
    if qi.dtype == np.uint16:
        qi = (qi.astype(np.uint32) << 16).view(np.float32)
    q_packed, q_scales = mxfp4_quantize(qi.astype(np.float32))
    E = ent.shape[0]
    n_vis = np.array([n_visible(t, wl.m, E) for t in rows], dtype=np.int32)
    q_seq = np.zeros(len(rows), dtype=np.int32)
    s32, _, bad = index_scores(q_packed, q_scales, inp["w"][b][rows], q_seq, n_vis, k_packed[None], k_scales[None])
    idx, cnt, kth = topk(s32, n_vis, wl.k)
    out, lse = attention(qf, rows, q_seq, ent[None], idx, cnt, win[None], np.zeros(1, np.int64), wl.W)
    return dict(entries=ent, window=win, q=qf, ki=ki, k_packed=k_packed, k_scales=k_scales, q_packed=q_packed,
                q_scales=q_scales, n_vis=n_vis, scores=s32, idx=idx, cnt=cnt, kth=kth, out=out, lse=lse,
                inexact=bad, rows=rows)


def hca_prefill(wl, inp: dict, b: int = 0, rows: np.ndarray | None = None):
    """Whole HCA prefill layer (pool with m', dense attention over all visible entries + window)."""
    T = inp["kv"].shape[1]
    rows = np.arange(T) if rows is None else np.asarray(rows)
    ent = entries_rows(inp["kv"][b], inp["z"][b], inp["bias"], wl.m, False, wl.norm, wl.eps, wl.rope_dims, wl.theta)
    win = window_rows(inp["kv"][b], wl.norm, wl.eps, wl.rope_dims, wl.theta)
    qf = prep_queries(inp["q"][b][rows], rows, wl.norm, wl.eps, wl.rope_dims, wl.theta)
    q_seq = np.zeros(len(rows), dtype=np.int32)
    idx, cnt = hca_select(rows, q_seq, np.array([ent.shape[0]]), wl.m)
    out, lse = attention(qf, rows, q_seq, ent[None], idx, cnt, win[None], np.zeros(1, np.int64), wl.W)
    return dict(entries=ent, window=win, q=qf, idx=idx, cnt=cnt, out=out, lse=lse, rows=rows)


def csa_decode(wl, entries, k_packed, k_scales, q, qi_packed, qi_scales, w, window, pos, seqs=None):
    """CSA decode for sequences ``seqs``: indexer over all visible entries, top-k, attention.

    entries [B,E,D] bf16 bits; k_* [B,E,..]; q [B,H,D]; qi_* [B,Hi,..]; w [B,Hi];
    window [B,W,D] holding tokens pos-W+1..pos; pos [B]."""
    B, E, D = entries.shape
    seqs = np.arange(B) if seqs is None else np.asarray(seqs)
    n_vis = np.array([n_visible(pos[s], wl.m, E) for s in seqs], dtype=np.int32)
    s32, _, bad = index_scores(qi_packed[seqs], qi_scales[seqs], w[seqs], seqs.astype(np.int32), n_vis,
                               k_packed, k_scales)
    idx, cnt, kth = topk(s32, n_vis, wl.k)
    Tw = window.shape[1]
    wbase = np.asarray(pos, dtype=np.int64) - Tw + 1
    out, lse = attention(q[seqs], np.asarray(pos)[seqs], seqs.astype(np.int32), entries, idx, cnt, window,
                         wbase, wl.W)
    return dict(scores=s32, n_vis=n_vis, idx=idx, cnt=cnt, kth=kth, out=out, lse=lse, inexact=bad)


def grouped_out_proj(o, A, Bm, G: int):
    """Grouped output projection: o [T, H, D] (or [T, H*D]); A [G, R, (H/G)*D]; Bm [d_model, G*R];
    all of one element type (float64, float32 or bf16 bits).  Returns (z [T, G*R], y [T, d_model])
    in float64."""
    o, A, Bm = _c(o), _c(A), _c(Bm)
    assert o.dtype == A.dtype == Bm.dtype
    T = o.shape[0]
    HD = int(np.prod(o.shape[1:]))
    Gc, R, Kg = A.shape
    assert Gc == G and Kg * G == HD
    d_model, GR = Bm.shape
    assert GR == G * R
    # heads and head dim only enter through their product and the group split
    H, D = (o.shape[1], o.shape[2]) if o.ndim == 3 else (G, Kg)
    assert H % G == 0 and (H // G) * D == Kg
    z = np.zeros((T, G * R), dtype=np.float64)
    y = np.zeros((T, d_model), dtype=np.float64)
    lib().orc_grouped_out_proj(T, H, D, G, R, d_model, _dt(o), _p(o), _p(A), _p(Bm), _p(z), _p(y))
    return z, y
