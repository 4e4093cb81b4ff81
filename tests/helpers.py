"""Shared comparison helpers for the parity tests (no layer arithmetic here)."""
from __future__ import annotations

import numpy as np

# tolerances of the bf16 paths against the float64 oracle
REL_L2 = 1e-2
MAX_ABS = 3e-2
TOPK_REL_GAP = 1e-6


def bf16_bits_to_f64(a: np.ndarray) -> np.ndarray:
    return (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def to_dev_bf16(bits: np.ndarray, dev):
    import torch
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(dev)


def to_dev(a: np.ndarray, dev):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a)).to(dev)


def t2np(t) -> np.ndarray:
    import torch
    if t.dtype == torch.bfloat16:
        return t.float().cpu().numpy().astype(np.float64)
    return t.cpu().numpy()


def rel_l2(x: np.ndarray, ref: np.ndarray) -> float:
    return float(np.linalg.norm((x - ref).ravel()) / max(np.linalg.norm(ref.ravel()), 1e-30))


def assert_close_attn(out: np.ndarray, ref: np.ndarray, what: str = ""):
    r = rel_l2(out, ref)
    m = float(np.max(np.abs(out - ref))) if out.size else 0.0
    assert np.all(np.isfinite(out)), f"{what}: non-finite output"
    assert r <= REL_L2 and m <= MAX_ABS, f"{what}: relL2 {r:.3e} (<= {REL_L2}), max-abs {m:.3e} (<= {MAX_ABS})"
    return r, m


def assert_bf16_rounding(out: np.ndarray, ref: np.ndarray, what: str = "", atol: float = 1e-5):
    """bf16 output of a float32 computation vs the float64 oracle: within 2^-8 relative (one
    bf16 rounding of 2^-9 plus float32 arithmetic) or atol."""
    err = np.abs(out - ref)
    bad = err > (2.0 ** -8) * np.abs(ref) + atol
    assert not bad.any(), f"{what}: {int(bad.sum())} elements off, worst {float(err.max()):.3e}"


def check_topk(idx_gpu: np.ndarray, cnt_gpu: np.ndarray, idx_ref: np.ndarray, cnt_ref: np.ndarray,
               kth: np.ndarray, scores_ref: np.ndarray, n_vis: np.ndarray, k: int):
    """Index sets must be equal, except rows whose k-th and (k+1)-th oracle scores differ by
    less than 1e-6 relative; those must still keep every score clearly above the k-th and
    nothing clearly below it.  Returns the number of exempt rows."""
    assert np.array_equal(cnt_gpu, cnt_ref), "counts differ"
    exempt = 0
    for n in range(idx_ref.shape[0]):
        c = int(cnt_ref[n])
        g = idx_gpu[n, :c]
        assert np.all(np.diff(g) > 0), f"row {n}: indices not strictly ascending"
        assert np.all(idx_gpu[n, c:] == -1), f"row {n}: padding is not -1"
        if np.array_equal(g, idx_ref[n, :c]):
            continue
        sk, sk1 = float(kth[n, 0]), float(kth[n, 1])
        if not (n_vis[n] > k and (sk - sk1) < TOPK_REL_GAP * abs(sk)):
            raise AssertionError(f"row {n}: index set differs and the row is not exempt (s_k={sk}, s_k+1={sk1})")
        exempt += 1
        s = scores_ref[n, :n_vis[n]]
        must = np.nonzero(s > sk * (1 + TOPK_REL_GAP))[0]
        assert set(must.tolist()) <= set(g.tolist()), f"row {n}: exempt row misses a clear winner"
        assert np.all(s[g] >= sk * (1 - TOPK_REL_GAP)), f"row {n}: exempt row keeps a clear loser"
    return exempt


E2M1_BOUNDS = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0])


def fp4_mismatch_justified(x_ref: np.ndarray, packed_gpu: np.ndarray, scales_gpu: np.ndarray,
                           packed_ref: np.ndarray, scales_ref: np.ndarray, rel: float = 1e-5) -> int:
    """MXFP4 bytes of a float32 computation vs the oracle's float64 value: codes may differ only
    where the oracle value sits within `rel` of a rounding or scale boundary.  Returns #justified."""
    rows, cols = x_ref.shape
    blocks = x_ref.reshape(rows, cols // 32, 32)
    amax = np.abs(blocks).max(axis=2)
    E = scales_ref.astype(np.int64) - 127
    scale_edge = (np.abs(amax / (6.0 * np.exp2(E)) - 1) < rel) | (np.abs(amax / (6.0 * np.exp2(E - 1)) - 1) < rel)
    sc_bad = scales_gpu != scales_ref
    assert not (sc_bad & ~scale_edge).any(), "scale byte differs away from a scale boundary"
    cg = np.stack([packed_gpu & 15, packed_gpu >> 4], -1).reshape(rows, cols)
    cr = np.stack([packed_ref & 15, packed_ref >> 4], -1).reshape(rows, cols)
    y = np.abs(x_ref) / np.exp2(np.repeat(E, 32, axis=1))
    near = np.min(np.abs(y[..., None] - E2M1_BOUNDS) / E2M1_BOUNDS, axis=-1) < rel
    blk_edge = np.repeat(scale_edge, 32, axis=1)
    code_bad = cg != cr
    assert not (code_bad & ~near & ~blk_edge).any(), "E2M1 code differs away from a rounding boundary"
    return int(code_bad.sum() + sc_bad.sum())


def check_csa_prefill_rows(wl, host: dict, r: dict, rows: np.ndarray, check_entries: bool = True) -> dict:
    """Per-row parity of one CSA prefill layer run against the oracle.

    host: host arrays of one sequence's inputs (kv, z, bias, ki, zi, bias_i: full length;
    q, qi, w: only the query rows `rows`, in that order).  r: the layer's device outputs
    for every token as a query (entries, k_fp4, k_scale, q_fp4, q_scale, idx, cnt, out).

    Every sampled row must pass, none is allowed to miss:
    * the GPU pools indexer keys in float32 and the oracle in float64, so a key's MXFP4
      code may differ only where the float64 value sits on a rounding or scale boundary
      (`fp4_mismatch_justified`);
    * the query bytes are a pure function of the input bits: equal;
    * the oracle's scores and top-k over the GPU's key bytes: the GPU's index set equals
      the oracle's on every row, up to the 1e-6 tie exemption (`check_topk`);
    * the oracle's attention over that index set: within the attention tolerance.
    Returns counts (justified FP4 differences, exempt rows)."""
    import oracle
    E = wl.T // wl.m
    seq = np.zeros(len(rows), np.int32)
    ki_ref = oracle.pool(host["ki"], host["zi"], host["bias_i"], wl.m, wl.overlap)
    kp_ref, ks_ref = oracle.mxfp4_quantize(ki_ref.astype(np.float32))
    kp_gpu = t2np(r["k_fp4"])[0, :E]
    ks_gpu = t2np(r["k_scale"])[0, :E]
    n_fp4 = fp4_mismatch_justified(ki_ref, kp_gpu, ks_gpu, kp_ref, ks_ref)
    qi = host["qi"]
    qi = bf16_bits_to_f64(qi).astype(np.float32) if qi.dtype == np.uint16 else qi.astype(np.float32)
    qp, qs = oracle.mxfp4_quantize(qi)
    sel = np.asarray(rows)
    assert np.array_equal(t2np(r["q_fp4"])[sel], qp) and np.array_equal(t2np(r["q_scale"])[sel], qs), \
        "indexer query bytes differ"
    n_vis = np.array([oracle.n_visible(t, wl.m, E) for t in rows], np.int32)
    s32, _, _ = oracle.index_scores(qp, qs, host["w"], seq, n_vis, kp_gpu[None], ks_gpu[None])
    idx_ref, cnt_ref, kth = oracle.topk(s32, n_vis, wl.k)
    idx_gpu, cnt_gpu = t2np(r["idx"])[sel], t2np(r["cnt"])[sel]
    exempt = check_topk(idx_gpu, cnt_gpu, idx_ref, cnt_ref, kth, s32, n_vis, wl.k)
    ent = oracle.entries_rows(host["kv"], host["z"], host["bias"], wl.m, wl.overlap, wl.norm, wl.eps, wl.rope_dims,
                              wl.theta)
    if check_entries:
        assert_bf16_rounding(t2np(r["entries"])[0, :E], ent, "entries")
    win = oracle.window_rows(host["kv"], wl.norm, wl.eps, wl.rope_dims, wl.theta)
    qf = oracle.prep_queries(host["q"], rows, wl.norm, wl.eps, wl.rope_dims, wl.theta)
    out_ref, _ = oracle.attention(qf, rows, seq, ent[None], idx_gpu, cnt_gpu, win[None], np.zeros(1, np.int64), wl.W)
    assert_close_attn(t2np(r["out"])[sel], out_ref, f"CSA prefill T={wl.T}")
    return {"fp4_justified": n_fp4, "exempt_rows": exempt}
