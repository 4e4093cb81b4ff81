"""The CSA / HCA layer as a sequence of C-ABI calls (binding only; no arithmetic here).

CSA prefill ("DeepSeek-V4: Million-Token Context", CSA stage; "Follow the white
rabbit", CSA / window / indexer paragraphs):
    csa_compress(kv)            -> entries (norm + RoPE) and raw window rows
    csa_compress(indexer keys)  -> MXFP4 indexer key cache
    csa_quantize_mxfp4(q_I)     -> MXFP4 indexer queries
    csa_index_topk              -> top-k entry indices per query
    csa_sparse_attn_ex          -> output (the queries' RMSNorm + RoPE applied as the
                                   kernel loads them, bitwise csa_norm_rope's)
CSA decode: csa_quantize_mxfp4(q_I) -> csa_index_topk -> csa_sparse_attn over a resident
cache.  HCA prefill: csa_compress(m'=128) -> hca_attn_ex.
"""
from __future__ import annotations

import torch

from . import binding as B

__all__ = ["csa_prefill", "csa_decode", "hca_prefill", "q_prep"]


def _i32(x, dev):
    return torch.as_tensor(x, dtype=torch.int32, device=dev)


def q_prep(wl) -> dict:
    """The queries' RMSNorm + partial RoPE, applied by the attention kernel as it loads them."""
    return dict(norm=wl.norm, eps=wl.eps, rope_dims=wl.rope_dims, theta=wl.theta)


def csa_prefill(wl, t: dict, rows: torch.Tensor | None = None) -> dict:
    """t: device tensors kv, z [1,T,C]; bias; q [1,T,H,C]; qi [1,T,Hi,Di]; ki, zi [1,T,Di]; bias_i; w [1,T,Hi]."""
    dev = t["kv"].device
    T = t["kv"].shape[1]
    pool = B.csa_compress(t["kv"], t["z"], t["bias"], m=wl.m, overlap=wl.overlap, norm=wl.norm, eps=wl.eps,
                          rope_dims=wl.rope_dims, theta=wl.theta, want_window=True)
    E = T // wl.m
    E_pad = max(8, (E + 7) // 8 * 8)
    keys = B.csa_compress(t["ki"], t["zi"], t["bias_i"], m=wl.m, overlap=wl.overlap, norm=False,
                          want_entries=False, want_fp4=True, E_max=E_pad)
    pos = torch.arange(T, dtype=torch.int32, device=dev) if rows is None else rows.to(torch.int32)
    Nq = pos.numel()
    qi = t["qi"][0] if rows is None else t["qi"][0][rows]
    q_fp4, q_sc = B.csa_quantize_mxfp4(qi)
    q = (t["q"][0] if rows is None else t["q"][0][rows]).contiguous()  # raw: prepared inside the attention
    w = (t["w"][0] if rows is None else t["w"][0][rows]).contiguous()
    seq = torch.zeros(Nq, dtype=torch.int32, device=dev)
    n_ent = _i32([E], dev)
    idx, cnt, _ = B.csa_index_topk(q_fp4, q_sc, w, pos, seq, keys["fp4"], keys["fp4_scale"], n_ent, k=wl.k,
                                   m=wl.m)
    out, lse = B.csa_sparse_attn(q, pos, seq, pool["entries"], idx, cnt, pool["window"], _i32([0], dev), W=wl.W,
                                 want_lse=True, prep=q_prep(wl))
    return dict(out=out, lse=lse, idx=idx, cnt=cnt, entries=pool["entries"], window=pool["window"],
                k_fp4=keys["fp4"], k_scale=keys["fp4_scale"], q=q, q_fp4=q_fp4, q_scale=q_sc, w=w, n_ent=n_ent)


def csa_decode(wl, cache: dict, step: dict, ws: dict | None = None, out: torch.Tensor | None = None) -> dict:
    """One decode step over a resident cache.

    cache: entries [B,E,D] bf16, k_fp4 [B,E,Di/2], k_scale [B,E,Di/32], window [B,W,D] bf16,
           window_base int32 [B], n_entries int32 [B]
    step:  q [B,H,D] bf16 (normalised, rotated), qi [B,Hi,Di] float32, w [B,Hi], pos int32 [B]
    ws:    optional preallocated buffers (q_fp4, q_scale, index_ws (csa_index_topk's workspace),
           idx, cnt, seq, attn_ws).
    csa_quantize_mxfp4(qi) -> csa_index_topk (fused scores + selection when the shape suits it)
    -> csa_sparse_attn."""
    Bn = step["q"].shape[0]
    dev = step["q"].device
    ws = ws or {}
    seq = ws.get("seq")
    if seq is None:
        seq = torch.arange(Bn, dtype=torch.int32, device=dev)
    q_fp4, q_sc = B.csa_quantize_mxfp4(step["qi"], ws.get("q_fp4"), ws.get("q_scale"))
    idx, cnt, _ = B.csa_index_topk(q_fp4, q_sc, step["w"], step["pos"], seq, cache["k_fp4"], cache["k_scale"],
                                   cache["n_entries"], k=wl.k, m=wl.m, workspace=ws.get("index_ws"),
                                   idx=ws.get("idx"), cnt=ws.get("cnt"))
    o, lse = B.csa_sparse_attn(step["q"], step["pos"], seq, cache["entries"], idx, cnt, cache["window"],
                               cache["window_base"], W=wl.W, out=out, workspace=ws.get("attn_ws"))
    return dict(out=o, idx=idx, cnt=cnt)


def hca_prefill(wl, t: dict, rows: torch.Tensor | None = None) -> dict:
    dev = t["kv"].device
    T = t["kv"].shape[1]
    pool = B.csa_compress(t["kv"], t["z"], t["bias"], m=wl.m, overlap=False, norm=wl.norm, eps=wl.eps,
                          rope_dims=wl.rope_dims, theta=wl.theta, want_window=True)
    E = T // wl.m
    pos = torch.arange(T, dtype=torch.int32, device=dev) if rows is None else rows.to(torch.int32)
    q = (t["q"][0] if rows is None else t["q"][0][rows]).contiguous()  # raw: prepared inside the attention
    seq = torch.zeros(pos.numel(), dtype=torch.int32, device=dev)
    out, lse = B.hca_attn(q, pos, seq, pool["entries"], _i32([E], dev), pool["window"], _i32([0], dev),
                          mprime=wl.m, W=wl.W, want_lse=True, prep=q_prep(wl))
    return dict(out=out, lse=lse, entries=pool["entries"], window=pool["window"], q=q)
