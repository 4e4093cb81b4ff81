"""ctypes binding of libcsa.so (include/csa.h) for torch tensors.

Argument marshalling only: every function checks device, dtype, shape and
contiguity, passes raw device pointers and the current CUDA stream to the C ABI
function of the same name, and raises ``CsaError`` on a non-OK status.  There is
no CPU fallback: if the library is missing or fails to load, every call raises.
Scratch workspaces are torch allocations unless the caller passes one.
"""
from __future__ import annotations

import ctypes
import math
import os
import threading

import torch

__all__ = ["CsaError", "lib", "csa_compress", "csa_compress_step", "csa_norm_rope", "csa_quantize_mxfp4", "csa_index_topk",
           "csa_index_score", "csa_index_score_q", "csa_topk_select",
           "csa_index_topk_workspace", "csa_index_topk_launches", "csa_sparse_attn", "csa_sparse_attn_workspace", "hca_attn",
           "csa_sparse_attn_ex", "hca_attn_ex", "csa_index_topk_grouped",
           "hca_attn_workspace", "csa_grouped_out_proj", "csa_get_device_error", "csa_set_batch_invariant", "csa_set_index_fusion", "LIB_PATH", "DEVERR_NONE", "DEVERR_TIMEOUT",
           "DEVERR_INDEX"]

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libcsa.so")
DEVERR_NONE, DEVERR_TIMEOUT, DEVERR_INDEX = 0, 1, 2
_F32, _BF16 = 0, 1
_lock = threading.Lock()
_lib = None


class CsaError(RuntimeError):
    def __init__(self, fn: str, status: int, msg: str):
        super().__init__(f"{fn}: status {status} ({msg})")
        self.status = status


class _QPrep(ctypes.Structure):
    _fields_ = [("norm", ctypes.c_int), ("eps", ctypes.c_float), ("rope_dims", ctypes.c_int),
                ("rope_theta", ctypes.c_float)]


def _q_prep(prep: dict | None):
    """csa_q_prep from dict(norm=..., eps=..., rope_dims=..., theta=...), or NULL."""
    if prep is None:
        return None
    return ctypes.byref(_QPrep(int(bool(prep.get("norm", True))), float(prep.get("eps", 1e-6)),
                               int(prep.get("rope_dims", 0)), float(prep.get("theta", 10000.0))))


class _PoolCfg(ctypes.Structure):
    _fields_ = [("m", ctypes.c_int), ("overlap", ctypes.c_int), ("C", ctypes.c_int), ("norm", ctypes.c_int),
                ("eps", ctypes.c_float), ("rope_dims", ctypes.c_int), ("rope_theta", ctypes.c_float),
                ("in_dtype", ctypes.c_int)]


def lib() -> ctypes.CDLL:
    """Load libcsa.so (built in-tree by ``__graft_entry__.build()``); raise if it is absent."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise RuntimeError(f"{LIB_PATH} is missing: build it with `python -m compressed_sparse_long_02_b200.build`")
            L = ctypes.CDLL(LIB_PATH)
            P, I, I64, F, SZ = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_float, ctypes.c_size_t
            L.csa_compress.argtypes = [ctypes.POINTER(_PoolCfg), I, I, P, P, P, P, I, P, P, P, P]
            L.csa_compress_step.argtypes = [ctypes.POINTER(_PoolCfg), I, P, P, P, P, P, I, P, P, P]
            L.csa_norm_rope.argtypes = [P, I, I64, I, I, P, I64, I, F, I, F, P, P]
            L.csa_quantize_mxfp4.argtypes = [P, I, I64, I, P, P, P]
            L.csa_index_topk.argtypes = [I, I, I, I, I, P, P, P, P, P, I, I, P, P, P, P, P, P, P, SZ, P]
            L.csa_index_score.argtypes = [I, I, I, I, P, P, P, P, P, I, I, P, P, P, P, I, P]
            L.csa_index_score_q.argtypes = [I, I, I, I, P, I, P, P, P, I, I, P, P, P, P, I, P]
            L.csa_topk_select.argtypes = [I, I, I, P, I, P, P, I, I, P, P, P, P]
            L.csa_index_topk_grouped.argtypes = [I] + L.csa_index_topk.argtypes
            L.csa_index_topk_launches.argtypes = [I, I, I, I, I]
            L.csa_index_topk_launches.restype = I
            L.csa_index_topk_workspace.argtypes = [I, I, I]
            L.csa_index_topk_workspace.restype = SZ
            L.csa_sparse_attn.argtypes = [I, I, I, I, I, F, P, P, P, I, I, P, P, P, I, P, P, P, P, P, SZ, P]
            L.csa_sparse_attn_workspace.argtypes = [I, I, I, I, I]
            L.csa_sparse_attn_workspace.restype = SZ
            L.hca_attn.argtypes = [I, I, I, I, I, F, P, P, P, I, I, P, P, I, P, P, P, P, P, SZ, P]
            L.csa_sparse_attn_ex.argtypes = [ctypes.POINTER(_QPrep)] + L.csa_sparse_attn.argtypes
            L.hca_attn_ex.argtypes = [ctypes.POINTER(_QPrep)] + L.hca_attn.argtypes
            L.hca_attn_workspace.argtypes = [I, I, I, I, I]
            L.hca_attn_workspace.restype = SZ
            L.csa_grouped_out_proj.argtypes = [I, I, I, I, I, I, P, P, P, P, P, P]
            L.csa_get_device_error.argtypes = [ctypes.POINTER(ctypes.c_int32), P]
            L.csa_set_index_fusion.argtypes = [I]
            L.csa_set_index_fusion.restype = I
            L.csa_set_batch_invariant.argtypes = [I]
            L.csa_set_batch_invariant.restype = I
            L.csa_status_string.argtypes = [I]
            L.csa_status_string.restype = ctypes.c_char_p
            L.csa_last_cuda_error.argtypes = []
            L.csa_last_cuda_error.restype = ctypes.c_char_p
            for fn in ("csa_compress", "csa_compress_step", "csa_norm_rope", "csa_quantize_mxfp4", "csa_index_topk", "csa_index_score",
                       "csa_index_score_q",
                       "csa_topk_select", "csa_sparse_attn",
                       "hca_attn", "csa_sparse_attn_ex", "hca_attn_ex", "csa_grouped_out_proj", "csa_index_topk_grouped",
                       "csa_get_device_error"):
                getattr(L, fn).restype = I
            _lib = L
    return _lib


def _check(fn: str, status: int):
    if status != 0:
        msg = lib().csa_status_string(status).decode()
        if status == 5:  # CSA_ERR_CUDA
            msg += " (" + lib().csa_last_cuda_error().decode() + ")"
        raise CsaError(fn, status, msg)


def _ptr(t: torch.Tensor | None):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("tensor must live on a CUDA device")
    if not t.is_contiguous():
        raise ValueError("tensor must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _stream(t: torch.Tensor):
    return ctypes.c_void_p(torch.cuda.current_stream(t.device).cuda_stream)


def _dt(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return _BF16
    if t.dtype == torch.float32:
        return _F32
    raise TypeError(f"unsupported dtype {t.dtype} (float32 or bfloat16)")


def _need(t: torch.Tensor, dtype, shape=None, name="tensor"):
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")


def csa_compress(kv: torch.Tensor, logits: torch.Tensor, slot_bias: torch.Tensor, *, m: int, overlap: bool,
                 norm: bool, eps: float = 1e-6, rope_dims: int = 0, theta: float = 10000.0,
                 want_entries: bool = True, E_max: int | None = None, want_fp4: bool = False,
                 want_window: bool = False):
    """Pool kv/logits [B, T, C] into entries.  Returns dict(entries, fp4, fp4_scale, window)."""
    if kv.dim() == 2:
        kv, logits = kv[None], logits[None]
    B, T, C = kv.shape
    E = T // m
    E_max = E if E_max is None else E_max
    _need(slot_bias, torch.float32, ((2 if overlap else 1) * m, C), "slot_bias")
    dev = kv.device
    out = {"entries": None, "fp4": None, "fp4_scale": None, "window": None}
    if want_entries:
        out["entries"] = torch.empty((B, E_max, C), dtype=torch.bfloat16, device=dev)
    if want_fp4:
        out["fp4"] = torch.empty((B, E_max, C // 2), dtype=torch.uint8, device=dev)
        out["fp4_scale"] = torch.empty((B, E_max, C // 32), dtype=torch.uint8, device=dev)
    if want_window:
        out["window"] = torch.empty((B, T, C), dtype=torch.bfloat16, device=dev)
    cfg = _PoolCfg(m, int(bool(overlap)), C, int(bool(norm)), eps, rope_dims, theta, _dt(kv))
    st = lib().csa_compress(ctypes.byref(cfg), B, T, _ptr(kv.contiguous()), _ptr(logits.contiguous()),
                            _ptr(slot_bias), _ptr(out["entries"]), E_max, _ptr(out["fp4"]), _ptr(out["fp4_scale"]),
                            _ptr(out["window"]), _stream(kv))
    _check("csa_compress", st)
    return out


def csa_compress_step(kv: torch.Tensor, logits: torch.Tensor, slot_bias: torch.Tensor, pos: torch.Tensor, *, m: int,
                      overlap: bool, norm: bool, eps: float = 1e-6, rope_dims: int = 0, theta: float = 10000.0,
                      entries: torch.Tensor | None = None, fp4: torch.Tensor | None = None,
                      fp4_scale: torch.Tensor | None = None):
    """Decode-time compressor: kv/logits [B, (1+overlap)*m, C] hold each sequence's last raw
    tokens (row s = token pos - S + 1 + s); writes the entry that token pos completes into
    entries [B, E_max, C] (bf16) and / or fp4 [B, E_max, C/2] + fp4_scale [B, E_max, C/32]."""
    B, S, C = kv.shape
    assert S == (2 if overlap else 1) * m, "kv must hold the last (1 + overlap) * m tokens"
    _need(slot_bias, torch.float32, (S, C), "slot_bias")
    _need(pos, torch.int32, (B,), "pos")
    ref = entries if entries is not None else fp4
    assert ref is not None, "nothing to write"
    E_max = ref.shape[1]
    cfg = _PoolCfg(m, int(bool(overlap)), C, int(bool(norm)), eps, rope_dims, theta, _dt(kv))
    st = lib().csa_compress_step(ctypes.byref(cfg), B, _ptr(pos), _ptr(kv.contiguous()), _ptr(logits.contiguous()),
                                 _ptr(slot_bias), _ptr(entries), E_max, _ptr(fp4), _ptr(fp4_scale), _stream(kv))
    _check("csa_compress_step", st)


def csa_norm_rope(x: torch.Tensor, pos: torch.Tensor | None, *, norm: bool, eps: float = 1e-6, rope_dims: int = 0,
                  theta: float = 10000.0, pos_mod: int = 1, out: torch.Tensor | None = None):
    """RMSNorm + partial RoPE of x [rows, heads, C] (or [rows, C]); pos int32 [rows] or None."""
    xs = x if x.dim() == 3 else x[:, None, :]
    rows, heads, C = xs.shape
    if out is None:
        out = torch.empty(x.shape, dtype=torch.bfloat16, device=x.device)
    if pos is not None:
        _need(pos, torch.int32, (rows,), "pos")
    st = lib().csa_norm_rope(_ptr(xs.contiguous()), _dt(x), rows, heads, C, _ptr(pos), pos_mod, int(bool(norm)),
                             eps, rope_dims, theta, _ptr(out), _stream(x))
    _check("csa_norm_rope", st)
    return out


def csa_quantize_mxfp4(x: torch.Tensor, packed: torch.Tensor | None = None, scales: torch.Tensor | None = None):
    """x [..., cols] float32/bf16 -> (packed uint8 [..., cols/2], scales uint8 [..., cols/32])."""
    cols = x.shape[-1]
    rows = x.numel() // cols if cols else 0
    if packed is None:
        packed = torch.empty(x.shape[:-1] + (cols // 2,), dtype=torch.uint8, device=x.device)
    if scales is None:
        scales = torch.empty(x.shape[:-1] + (cols // 32,), dtype=torch.uint8, device=x.device)
    st = lib().csa_quantize_mxfp4(_ptr(x.contiguous()), _dt(x), rows, cols, _ptr(packed), _ptr(scales), _stream(x))
    _check("csa_quantize_mxfp4", st)
    return packed, scales


def csa_index_topk_launches(Nq: int, Hi: int, Di: int, E_max: int, k: int) -> int:
    """Kernels csa_index_topk launches for these sizes: 1 (fused decode kernel) or 2."""
    return int(lib().csa_index_topk_launches(Nq, Hi, Di, E_max, k))


def csa_index_topk_workspace(Nq: int, E_max: int, k: int) -> int:
    return int(lib().csa_index_topk_workspace(Nq, E_max, k))


def csa_index_topk(q_fp4, q_scale, w, q_pos, q_seq, k_fp4, k_scale, n_entries, *, k: int, m: int,
                   want_scores: bool = False, workspace: torch.Tensor | None = None, idx=None, cnt=None,
                   q_group: int = 1):
    """Lightning-indexer scores + top-k.  Returns (idx [Nq,k] int32, cnt [Nq] int32, scores or None).
    q_group = 2: rows 2g and 2g+1 name one sequence and share its key reads
    (csa_index_topk_grouped)."""
    Nq, Hi, half = q_fp4.shape
    Di = half * 2
    B, E_max, _ = k_fp4.shape
    dev = q_fp4.device
    for t, nm in ((q_fp4, "q_fp4"), (q_scale, "q_scale"), (k_fp4, "k_fp4"), (k_scale, "k_scale")):
        _need(t, torch.uint8, None, nm)
    _need(w, torch.float32, (Nq, Hi), "w")
    for t, nm in ((q_pos, "q_pos"), (q_seq, "q_seq"), (n_entries, "n_entries")):
        _need(t, torch.int32, None, nm)
    if idx is None:
        idx = torch.empty((Nq, k), dtype=torch.int32, device=dev)
    if cnt is None:
        cnt = torch.empty((Nq,), dtype=torch.int32, device=dev)
    scores = torch.full((Nq, E_max), float("-inf"), dtype=torch.float32, device=dev) if want_scores else None
    need = csa_index_topk_workspace(Nq, E_max, k)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    st = lib().csa_index_topk_grouped(q_group, Nq, Hi, Di, k, m, _ptr(q_fp4), _ptr(q_scale), _ptr(w), _ptr(q_pos),
                                      _ptr(q_seq), B, E_max, _ptr(k_fp4), _ptr(k_scale), _ptr(n_entries), _ptr(idx),
                                      _ptr(cnt), _ptr(scores), _ptr(workspace), workspace.numel(), _stream(q_fp4))
    _check("csa_index_topk", st)
    return idx, cnt, scores


def csa_index_topk_grouped(q_group: int, *args, **kw):
    """csa_index_topk with rows in groups of q_group sharing a sequence (see csa_index_topk)."""
    return csa_index_topk(*args, q_group=q_group, **kw)


def csa_index_score(q_fp4, q_scale, w, q_pos, q_seq, k_fp4, k_scale, n_entries, *, m: int,
                    scores: torch.Tensor | None = None):
    """Indexer scores only: scores float32 [Nq, E_stride] (E_stride >= E_max), filled for j < n_vis."""
    Nq, Hi, half = q_fp4.shape
    B, E_max, _ = k_fp4.shape
    if scores is None:
        scores = torch.full((Nq, E_max), float("-inf"), dtype=torch.float32, device=q_fp4.device)
    _need(scores, torch.float32, None, "scores")
    st = lib().csa_index_score(Nq, Hi, half * 2, m, _ptr(q_fp4), _ptr(q_scale), _ptr(w), _ptr(q_pos), _ptr(q_seq), B,
                               E_max, _ptr(k_fp4), _ptr(k_scale), _ptr(n_entries), _ptr(scores), scores.shape[1],
                               _stream(q_fp4))
    _check("csa_index_score", st)
    return scores


def csa_index_score_q(q, w, q_pos, q_seq, k_fp4, k_scale, n_entries, *, m: int,
                      scores: torch.Tensor | None = None):
    """csa_index_score with unencoded queries q [Nq, Hi, Di] float32/bf16 (encoded to MXFP4
    inside the indexer).  Returns scores float32 [Nq, E_stride]."""
    Nq, Hi, Di = q.shape
    B, E_max, _ = k_fp4.shape
    if scores is None:
        scores = torch.full((Nq, E_max), float("-inf"), dtype=torch.float32, device=q.device)
    _need(scores, torch.float32, None, "scores")
    q = q.contiguous()
    st = lib().csa_index_score_q(Nq, Hi, Di, m, _ptr(q), _dt(q), _ptr(w), _ptr(q_pos), _ptr(q_seq), B, E_max,
                                 _ptr(k_fp4), _ptr(k_scale), _ptr(n_entries), _ptr(scores), scores.shape[1],
                                 _stream(q))
    _check("csa_index_score_q", st)
    return scores


def csa_topk_select(scores, q_pos, q_seq, n_entries, *, k: int, m: int, E_max: int, idx=None, cnt=None):
    """Top-k of score rows (see csa_index_topk).  Returns (idx, cnt)."""
    Nq, E_stride = scores.shape
    B = n_entries.shape[0]
    if idx is None:
        idx = torch.empty((Nq, k), dtype=torch.int32, device=scores.device)
    if cnt is None:
        cnt = torch.empty((Nq,), dtype=torch.int32, device=scores.device)
    st = lib().csa_topk_select(Nq, k, m, _ptr(scores), E_stride, _ptr(q_pos), _ptr(q_seq), B, E_max, _ptr(n_entries),
                               _ptr(idx), _ptr(cnt), _stream(scores))
    _check("csa_topk_select", st)
    return idx, cnt


def csa_sparse_attn_workspace(Nq: int, H: int, D: int, k: int, W: int) -> int:
    return int(lib().csa_sparse_attn_workspace(Nq, H, D, k, W))


def hca_attn_workspace(Nq: int, H: int, D: int, E_max: int, W: int) -> int:
    return int(lib().hca_attn_workspace(Nq, H, D, E_max, W))


def csa_sparse_attn(q, q_pos, q_seq, entries, idx, cnt, window, window_base, *, W: int, scale: float | None = None,
                    out=None, want_lse: bool = False, workspace: torch.Tensor | None = None, prep: dict | None = None):
    """MQA over selected entries + window.  q [Nq,H,D] bf16; entries [B,E_max,D]; window [B,Tw,D].
    prep = dict(norm, eps, rope_dims, theta): q is raw and the kernel applies csa_norm_rope's
    transform as it loads it (csa_sparse_attn_ex)."""
    Nq, H, D = q.shape
    B, E_max, _ = entries.shape
    Tw = window.shape[1]
    k = idx.shape[1]
    _need(q, torch.bfloat16, None, "q")
    _need(entries, torch.bfloat16, None, "entries")
    _need(window, torch.bfloat16, None, "window")
    scale = 1.0 / math.sqrt(D) if scale is None else scale
    out = torch.empty_like(q) if out is None else out
    lse = torch.empty((Nq, H), dtype=torch.float32, device=q.device) if want_lse else None
    need = csa_sparse_attn_workspace(Nq, H, D, k, W)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    st = lib().csa_sparse_attn_ex(_q_prep(prep), Nq, H, D, k, W, scale, _ptr(q), _ptr(q_pos), _ptr(q_seq), B, E_max,
                                  _ptr(entries), _ptr(idx), _ptr(cnt), Tw, _ptr(window), _ptr(window_base), _ptr(out),
                                  _ptr(lse), _ptr(workspace), workspace.numel(), _stream(q))
    _check("csa_sparse_attn", st)
    return out, lse


def hca_attn(q, q_pos, q_seq, entries, n_entries, window, window_base, *, mprime: int, W: int,
             scale: float | None = None, out=None, want_lse: bool = False, workspace: torch.Tensor | None = None,
             prep: dict | None = None):
    """Dense MQA over every visible HCA entry + window (prep: as csa_sparse_attn)."""
    Nq, H, D = q.shape
    B, E_max, _ = entries.shape
    Tw = window.shape[1]
    _need(q, torch.bfloat16, None, "q")
    scale = 1.0 / math.sqrt(D) if scale is None else scale
    out = torch.empty_like(q) if out is None else out
    lse = torch.empty((Nq, H), dtype=torch.float32, device=q.device) if want_lse else None
    need = hca_attn_workspace(Nq, H, D, E_max, W)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    st = lib().hca_attn_ex(_q_prep(prep), Nq, H, D, mprime, W, scale, _ptr(q), _ptr(q_pos), _ptr(q_seq), B, E_max,
                           _ptr(entries), _ptr(n_entries), Tw, _ptr(window), _ptr(window_base), _ptr(out), _ptr(lse),
                           _ptr(workspace), workspace.numel(), _stream(q))
    _check("hca_attn", st)
    return out, lse


def csa_sparse_attn_ex(prep: dict | None, *args, **kw):
    """csa_sparse_attn with the query prepared in the kernel (prep: see csa_sparse_attn)."""
    return csa_sparse_attn(*args, prep=prep, **kw)


def hca_attn_ex(prep: dict | None, *args, **kw):
    """hca_attn with the query prepared in the kernel (prep: see csa_sparse_attn)."""
    return hca_attn(*args, prep=prep, **kw)


def csa_grouped_out_proj(o, A, Bm, *, z=None, y=None):
    """Grouped output projection: o [T, H, D] bf16; A [G, R, (H/G) D] bf16; Bm [d_model, G R] bf16.
    Returns (z [T, G R], y [T, d_model]) bf16."""
    T, H, D = o.shape
    G, R, Kg = A.shape
    d_model = Bm.shape[0]
    for t, nm in ((o, "o"), (A, "A"), (Bm, "Bm")):
        _need(t, torch.bfloat16, None, nm)
    if Kg * G != H * D or tuple(Bm.shape) != (d_model, G * R):
        raise ValueError("inconsistent projection shapes")
    z = torch.empty((T, G * R), dtype=torch.bfloat16, device=o.device) if z is None else z
    y = torch.empty((T, d_model), dtype=torch.bfloat16, device=o.device) if y is None else y
    st = lib().csa_grouped_out_proj(T, H, D, G, R, d_model, _ptr(o), _ptr(A), _ptr(Bm), _ptr(z), _ptr(y), _stream(o))
    _check("csa_grouped_out_proj", st)
    return z, y


def csa_set_index_fusion(on: bool) -> None:
    """Process-wide: csa_index_topk uses the fused decode kernel where it fits (off by default)."""
    _check("csa_set_index_fusion", lib().csa_set_index_fusion(int(bool(on))))


def csa_set_batch_invariant(on: bool) -> None:
    """Process-wide: attention splits each query's keys by a rule independent of the batch."""
    _check("csa_set_batch_invariant", lib().csa_set_batch_invariant(int(bool(on))))


def csa_get_device_error(device=None) -> int:
    """Synchronise the current stream and return (and clear) the device error word."""
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    code = ctypes.c_int32(0)
    st = lib().csa_get_device_error(ctypes.byref(code), ctypes.c_void_p(torch.cuda.current_stream(dev).cuda_stream))
    _check("csa_get_device_error", st)
    return int(code.value)
