"""GPU parity of each C-ABI call against the CPU oracle, on the same seeded inputs.

Stage inputs come from the seeded generator or from the oracle's own earlier
stages (never from the CUDA path).  Bars: MXFP4 bytes, scores and index sets
bit-exact (index sets up to the 1e-6 tie exemption); bf16 activations within one
bf16 rounding of the float64 oracle; attention outputs within relative L2 1e-2 and
max-abs 3e-2.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from compressed_sparse_long_02_b200 import synth
from tests.helpers import (assert_bf16_rounding, assert_close_attn, bf16_bits_to_f64, check_topk,
                           fp4_mismatch_justified, t2np, to_dev, to_dev_bf16)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def B(cuda):
    from compressed_sparse_long_02_b200 import binding
    binding.lib()
    return binding


def _err_clear(B):
    assert B.csa_get_device_error() == 0


# ------------------------------------------------------------------ MXFP4 encoding
def test_quantize_golden_vectors(B, cuda):
    import json, os
    cases = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "mxfp4_vectors.json")))["cases"]
    x = np.array([c["x"] for c in cases], np.float32)
    pk, sc = B.csa_quantize_mxfp4(to_dev(x, cuda))
    rp, rs = oracle.mxfp4_quantize(x)
    assert np.array_equal(t2np(pk), rp) and np.array_equal(t2np(sc), rs)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_quantize_bitexact_random(B, cuda, dtype):
    rng = np.random.default_rng(5)
    x = rng.standard_normal((1000, 128)) * np.exp(rng.uniform(-30, 30, (1000, 1)))
    x[3] = 0.0
    x[4, :5] = -0.0
    x[7] = 6.0 * 2.0 ** -130  # subnormal block
    x[9, 0] = 3.0e38
    if dtype == "f32":
        xs = x.astype(np.float32)
        xd = to_dev(xs, cuda)
        ref_in = xs
    else:
        bits = synth.to_dtype_np(x, "bf16")
        xd = to_dev_bf16(bits, cuda)
        ref_in = bf16_bits_to_f64(bits).astype(np.float32)
    pk, sc = B.csa_quantize_mxfp4(xd)
    rp, rs = oracle.mxfp4_quantize(ref_in)
    assert np.array_equal(t2np(sc), rs)
    assert np.array_equal(t2np(pk), rp)


# ------------------------------------------------------------------ compressor
def _pool_ref(wl, inp, b=0, which="kv"):
    if which == "kv":
        return oracle.entries_rows(inp["kv"][b], inp["z"][b], inp["bias"], wl.m, wl.overlap, wl.norm, wl.eps,
                               wl.rope_dims, wl.theta)
    return oracle.pool(inp["ki"][b], inp["zi"][b], inp["bias_i"], wl.m, wl.overlap)


def _dev_act(a, wl, dev):
    return to_dev_bf16(a, dev) if wl.dtype == "bf16" else to_dev(a, dev)


@pytest.mark.parametrize("name,T", [("tiny", 512), ("tiny", 37), ("csa_prefill_8k", 1024), ("hca_prefill_64k", 2048 + 77)])
def test_compress_entries_window_fp4(B, cuda, name, T):
    wl = synth.WORKLOADS[name]
    inp = synth.prefill_inputs(wl, T=T)
    kv, z = _dev_act(inp["kv"], wl, cuda), _dev_act(inp["z"], wl, cuda)
    r = B.csa_compress(kv, z, to_dev(inp["bias"], cuda), m=wl.m, overlap=wl.overlap, norm=wl.norm, eps=wl.eps,
                       rope_dims=wl.rope_dims, theta=wl.theta, want_window=True)
    E = T // wl.m
    ent = t2np(r["entries"])[0]
    assert ent.shape[0] == E
    if E:
        assert_bf16_rounding(ent, _pool_ref(wl, inp), f"{name} entries")
    win_ref = oracle.window_rows(inp["kv"][0], wl.norm, wl.eps, wl.rope_dims, wl.theta)
    assert_bf16_rounding(t2np(r["window"])[0], win_ref, f"{name} window rows")
    if wl.kind == "csa_prefill" and E:
        E_pad = (E + 7) // 8 * 8
        rk = B.csa_compress(_dev_act(inp["ki"], wl, cuda), _dev_act(inp["zi"], wl, cuda), to_dev(inp["bias_i"], cuda),
                            m=wl.m, overlap=wl.overlap, norm=False, want_entries=False, want_fp4=True, E_max=E_pad)
        kref = _pool_ref(wl, inp, which="ki")
        rp, rs = oracle.mxfp4_quantize(kref.astype(np.float32))
        gp, gs = t2np(rk["fp4"])[0, :E], t2np(rk["fp4_scale"])[0, :E]
        n_diff = fp4_mismatch_justified(kref, gp, gs, rp, rs)
        assert n_diff <= max(2, E * wl.Di // 10000)
    _err_clear(B)


def test_norm_rope_queries(B, cuda):
    wl = synth.WORKLOADS["csa_prefill_8k"]
    inp = synth.prefill_inputs(wl, T=300)
    rows = np.array([0, 1, 2, 3, 127, 128, 299])
    q = to_dev_bf16(inp["q"][0][rows], cuda)
    pos = to_dev(rows.astype(np.int32) * 217, cuda)   # spread positions up to ~65k
    out = B.csa_norm_rope(q, pos, norm=True, eps=wl.eps, rope_dims=wl.rope_dims, theta=wl.theta)
    ref = oracle.prep_queries(inp["q"][0][rows], rows * 217, True, wl.eps, wl.rope_dims, wl.theta)
    assert_bf16_rounding(t2np(out), ref, "queries")


# ------------------------------------------------------------------ indexer + top-k
def _index_case(wl, T, rows, dev, B):
    inp = synth.prefill_inputs(wl, T=T)
    ki = oracle.pool(inp["ki"][0], inp["zi"][0], inp["bias_i"], wl.m, wl.overlap)
    E = ki.shape[0]
    E_pad = max(8, (E + 7) // 8 * 8)
    kp, ks = oracle.mxfp4_quantize(ki.astype(np.float32))
    kp_pad = np.zeros((1, E_pad, wl.Di // 2), np.uint8)
    ks_pad = np.zeros((1, E_pad, wl.Di // 32), np.uint8)
    kp_pad[0, :E], ks_pad[0, :E] = kp, ks
    qi = inp["qi"][0][rows]
    qi = bf16_bits_to_f64(qi).astype(np.float32) if qi.dtype == np.uint16 else qi
    qp, qs = oracle.mxfp4_quantize(qi)
    w = inp["w"][0][rows]
    n_vis = np.array([oracle.n_visible(t, wl.m, E) for t in rows], np.int32)
    s32, s64, bad = oracle.index_scores(qp, qs, w, np.zeros(len(rows), np.int32), n_vis, kp_pad[:, :E], ks_pad[:, :E])
    assert bad == 0
    idx_r, cnt_r, kth = oracle.topk(s32, n_vis, wl.k)
    idx, cnt, sc = B.csa_index_topk(to_dev(qp, dev), to_dev(qs, dev), to_dev(w, dev), to_dev(rows.astype(np.int32), dev),
                                    to_dev(np.zeros(len(rows), np.int32), dev), to_dev(kp_pad, dev), to_dev(ks_pad, dev),
                                    to_dev(np.array([E], np.int32), dev), k=wl.k, m=wl.m, want_scores=True)
    return dict(idx=t2np(idx), cnt=t2np(cnt), sc=t2np(sc)[:, :E], s32=s32, idx_r=idx_r, cnt_r=cnt_r, kth=kth,
                n_vis=n_vis, E=E)


@pytest.mark.parametrize("name,T,nrows", [("tiny", 512, None), ("csa_prefill_8k", 2048, 160),
                                         ("csa_prefill_8k", 2048, None), ("csa_prefill_8k", 8192, 400)])
def test_index_topk_exact(B, cuda, name, T, nrows):
    """Scores bit-exact and index sets exact; 2048 and ~400 rows reach the persistent
    many-query indexer (at least two queries per SM), 160 rows the per-query one."""
    wl = synth.WORKLOADS[name]
    rng = np.random.default_rng(9)
    if nrows is None:
        rows = np.arange(T)
    else:
        special = [0, 3, 4, 7, 127, 128, wl.m * wl.k - 1, wl.m * wl.k, T - 1]
        rows = np.unique(np.concatenate([[r for r in special if r < T], rng.choice(T, nrows, replace=False)]))
    r = _index_case(wl, T, rows, cuda, B)
    vis = np.arange(r["E"])[None, :] < r["n_vis"][:, None]
    np.testing.assert_array_equal(r["sc"][vis], r["s32"][vis])  # scores bit-exact
    check_topk(r["idx"], r["cnt"], r["idx_r"], r["cnt_r"], r["kth"], r["s32"], r["n_vis"], wl.k)
    _err_clear(B)


def test_index_topk_decode_multi_sequence(B, cuda):
    """4 sequences with ragged entry counts, one query each at the end of its context."""
    wl = synth.WORKLOADS["csa_decode_128k"]
    d = synth.decode_inputs(wl, B=4, E=4096)
    kp, ks = oracle.mxfp4_quantize(d["ki"])
    qp, qs = oracle.mxfp4_quantize(d["qi"])
    n_ent = np.array([4096, 1000, 4095, 1025], np.int32)
    pos = n_ent.astype(np.int64) * wl.m - 1
    pos[2] -= 2                                  # unfinished group: one entry fewer is visible
    n_vis = np.array([oracle.n_visible(pos[b], wl.m, n_ent[b]) for b in range(4)], np.int32)
    seqs = np.arange(4, dtype=np.int32)
    s32, _, bad = oracle.index_scores(qp, qs, d["w"], seqs, n_vis, kp, ks)
    idx_r, cnt_r, kth = oracle.topk(s32, n_vis, wl.k)
    idx, cnt, sc = B.csa_index_topk(to_dev(qp, cuda), to_dev(qs, cuda), to_dev(d["w"], cuda),
                                    to_dev(pos.astype(np.int32), cuda), to_dev(seqs, cuda), to_dev(kp, cuda),
                                    to_dev(ks, cuda), to_dev(n_ent, cuda), k=wl.k, m=wl.m, want_scores=True)
    sc = t2np(sc)
    for b in range(4):
        np.testing.assert_array_equal(sc[b, :n_vis[b]], s32[b, :n_vis[b]])
    check_topk(t2np(idx), t2np(cnt), idx_r, cnt_r, kth, s32, n_vis, wl.k)
    _err_clear(B)


def test_index_score_many_queries_multi_sequence(B, cuda):
    """400 queries over 3 sequences with ragged entry counts (the persistent indexer, whose
    blocks of eight queries then span several sequences): scores bit-exact on every visible
    entry, the rest of each row untouched; rows whose sequence id is out of range, one
    whole block of them included, are left alone and flag CSA_DEVERR_INDEX."""
    rng = np.random.default_rng(77)
    Bs, E_max, Hi, Di, m = 3, 1024, 64, 128, 4
    n_ent = np.array([1024, 777, 1000], np.int32)
    kp, ks = oracle.mxfp4_quantize(rng.standard_normal((Bs, E_max, Di)).astype(np.float32))
    Nq = 400
    seq = rng.integers(0, Bs, Nq).astype(np.int32)
    seq[[5, 200, 399]] = [-1, 3, -1]
    seq[16:24] = -1                              # a whole block of eight queries without a sequence
    pos = (rng.integers(0, 4 * E_max + 40, Nq)).astype(np.int32)
    pos[:4] = [0, 3, 4 * 777 - 1, 4 * 1024 + 39]
    qp, qs = oracle.mxfp4_quantize(rng.standard_normal((Nq, Hi, Di)).astype(np.float32))
    w = rng.random((Nq, Hi)).astype(np.float32)
    ok = (seq >= 0) & (seq < Bs)
    n_vis = np.array([oracle.n_visible(int(pos[i]), m, int(n_ent[seq[i]])) if ok[i] else 0 for i in range(Nq)],
                     np.int32)
    s32, _, bad = oracle.index_scores(qp[ok], qs[ok], w[ok], seq[ok], n_vis[ok], kp, ks)
    assert bad == 0
    sentinel = np.float32(-7.25)
    scores = to_dev(np.full((Nq, E_max + 4), sentinel, np.float32), cuda)
    B.csa_index_score(to_dev(qp, cuda), to_dev(qs, cuda), to_dev(w, cuda), to_dev(pos, cuda), to_dev(seq, cuda),
                      to_dev(kp, cuda), to_dev(ks, cuda), to_dev(n_ent, cuda), m=m, scores=scores)
    sc = t2np(scores)
    ref = np.full_like(sc, sentinel)
    vis = np.arange(E_max)[None, :] < n_vis[ok][:, None]
    ref[np.where(ok)[0], :E_max] = np.where(vis, s32, sentinel)
    np.testing.assert_array_equal(sc, ref)
    assert B.csa_get_device_error() == B.DEVERR_INDEX  # read and cleared


@pytest.mark.parametrize("Hi,Di,dtype", [(64, 128, "f32"), (64, 128, "bf16"), (4, 64, "f32"), (20, 128, "bf16")])
def test_index_score_q_encodes_inside(B, cuda, Hi, Di, dtype):
    """Unencoded queries: the indexer's own MXFP4 encoding gives the oracle's scores bit for bit."""
    rng = np.random.default_rng(31 + Hi + Di)
    Bq, E = 3, 2048
    ki = rng.standard_normal((Bq, E, Di)).astype(np.float32)
    kp, ks = oracle.mxfp4_quantize(ki)
    qi = (rng.standard_normal((Bq, Hi, Di)) * rng.choice([1e-3, 1.0, 40.0], (Bq, Hi, 1))).astype(np.float32)
    if dtype == "bf16":
        bits = synth.to_dtype_np(qi, "bf16")
        q_dev = to_dev_bf16(bits, cuda)
        qi = bf16_bits_to_f64(bits).astype(np.float32)
    else:
        q_dev = to_dev(qi, cuda)
    qp, qs = oracle.mxfp4_quantize(qi)
    w = rng.uniform(0, 1, (Bq, Hi)).astype(np.float32)
    n_ent = np.array([E, 1500, 777], np.int32)
    pos = (n_ent.astype(np.int64) * 4 - 1).astype(np.int32)
    seqs = np.arange(Bq, dtype=np.int32)
    n_vis = np.array([oracle.n_visible(pos[b], 4, n_ent[b]) for b in range(Bq)], np.int32)
    s32, _, bad = oracle.index_scores(qp, qs, w, seqs, n_vis, kp, ks)
    assert bad == 0
    sc = t2np(B.csa_index_score_q(q_dev, to_dev(w, cuda), to_dev(pos, cuda), to_dev(seqs, cuda), to_dev(kp, cuda),
                                  to_dev(ks, cuda), to_dev(n_ent, cuda), m=4))
    for b in range(Bq):
        np.testing.assert_array_equal(sc[b, :n_vis[b]], s32[b, :n_vis[b]])
    _err_clear(B)


def test_topk_ties_lowest_index(B, cuda):
    """All keys identical: every score ties, the k lowest indices must win."""
    Hi, Di, E, k = 8, 128, 1024, 100
    x = np.ones((1, E, Di), np.float32)
    kp, ks = oracle.mxfp4_quantize(x)
    q = np.ones((1, Hi, Di), np.float32)
    qp, qs = oracle.mxfp4_quantize(q)
    w = np.full((1, Hi), 0.5, np.float32)
    idx, cnt, _ = B.csa_index_topk(to_dev(qp, cuda), to_dev(qs, cuda), to_dev(w, cuda),
                                   to_dev(np.array([4 * E - 1], np.int32), cuda), to_dev(np.zeros(1, np.int32), cuda),
                                   to_dev(kp, cuda), to_dev(ks, cuda), to_dev(np.array([E], np.int32), cuda), k=k, m=4)
    assert t2np(idx)[0].tolist() == list(range(k)) and int(t2np(cnt)[0]) == k


# ------------------------------------------------------------------ attention
def _attn_inputs(seed, Nq, E, Tw, k, W, dense=False):
    rng = np.random.default_rng(seed)
    D, H = 512, 64
    ent = synth.to_dtype_np(rng.standard_normal((1, E, D)), "bf16")
    win = synth.to_dtype_np(rng.standard_normal((1, Tw, D)), "bf16")
    q = synth.to_dtype_np(rng.standard_normal((Nq, H, D)) * 0.3, "bf16")
    return ent, win, q


@pytest.mark.parametrize("Nq,E,k,W,Tw", [(40, 600, 512, 128, 2400), (8, 5000, 1024, 128, 8000), (200, 300, 64, 128, 1300)])
def test_sparse_attn_matches_oracle(B, cuda, Nq, E, k, W, Tw):
    rng = np.random.default_rng(Nq + E)
    ent, win, q = _attn_inputs(Nq, Nq, E, Tw, k, W)
    pos = np.sort(rng.choice(np.arange(Tw), Nq, replace=False)).astype(np.int64)
    pos[0] = 0
    pos[-1] = Tw - 1
    n_vis = np.minimum((pos + 1) // 4, E).astype(np.int32)
    idx = np.full((Nq, k), -1, np.int32)
    cnt = np.zeros(Nq, np.int32)
    for i in range(Nq):       # a random ascending subset of the visible entries
        c = min(k, int(n_vis[i]))
        idx[i, :c] = np.sort(rng.choice(n_vis[i], c, replace=False)) if c else []
        cnt[i] = c
    seq = np.zeros(Nq, np.int32)
    ref, lse_ref = oracle.attention(q, pos, seq, ent, idx, cnt, win, np.zeros(1, np.int64), W)
    out, lse = B.csa_sparse_attn(to_dev_bf16(q, cuda), to_dev(pos.astype(np.int32), cuda), to_dev(seq, cuda),
                                 to_dev_bf16(ent, cuda), to_dev(idx, cuda), to_dev(cnt, cuda), to_dev_bf16(win, cuda),
                                 to_dev(np.zeros(1, np.int32), cuda), W=W, want_lse=True)
    assert_close_attn(t2np(out), ref, "sparse attention")
    np.testing.assert_allclose(t2np(lse), lse_ref, atol=2e-2)
    _err_clear(B)


def test_hca_attn_matches_oracle(B, cuda):
    rng = np.random.default_rng(4)
    T, m, W = 4096 + 300, 128, 128
    E = T // m
    ent, win, q = _attn_inputs(4, 64, E, T, 0, W)
    pos = np.unique(np.concatenate([[0, 126, 127, 128, 255, T - 1], rng.choice(T, 58, replace=False)])).astype(np.int64)
    q = q[:len(pos)]
    seq = np.zeros(len(pos), np.int32)
    idx, cnt = oracle.hca_select(pos, seq, np.array([E]), m)
    ref, lse_ref = oracle.attention(q, pos, seq, ent, idx, cnt, win, np.zeros(1, np.int64), W)
    out, lse = B.hca_attn(to_dev_bf16(q, cuda), to_dev(pos.astype(np.int32), cuda), to_dev(seq, cuda),
                          to_dev_bf16(ent, cuda), to_dev(np.array([E], np.int32), cuda), to_dev_bf16(win, cuda),
                          to_dev(np.zeros(1, np.int32), cuda), mprime=m, W=W, want_lse=True)
    assert_close_attn(t2np(out), ref, "hca attention")
    np.testing.assert_allclose(t2np(lse), lse_ref, atol=2e-2)
    _err_clear(B)


@pytest.mark.parametrize("dense", [False, True])
def test_attn_tile_aligned_boxes_match_oracle(B, cuda, dense):
    """One CTA per query (>= 148 queries): the key list is tile-aligned where that adds no
    tile, and full tiles of contiguous rows (dense entries, window rows) load as TMA boxes.
    Two sequences with their own entry counts and window bases, so that the box row
    coordinates carry the sequence offsets; queries with full, ragged and padded tiles."""
    rng = np.random.default_rng(31 + dense)
    D, H, m, W, E_max, Tw, k = 512, 64, 4, 128, 300, 1200, 256
    ent = synth.to_dtype_np(rng.standard_normal((2, E_max, D)), "bf16")
    win = synth.to_dtype_np(rng.standard_normal((2, Tw, D)), "bf16")
    wbase = np.array([0, 5000], np.int64)
    ne = np.array([300, 260], np.int32)
    p0 = np.concatenate([[0, 126, 127, 128, 511, 512, 515, 1023, 1024, 1199], rng.choice(Tw, 90, replace=False)])
    p1 = np.concatenate([[5000, 5126, 5127, 6199], 5000 + rng.choice(Tw, 96, replace=False)])
    pos = np.concatenate([np.unique(p0), np.unique(p1)]).astype(np.int64)
    seq = np.concatenate([np.zeros(len(np.unique(p0)), np.int32), np.ones(len(np.unique(p1)), np.int32)])
    Nq = len(pos)
    assert Nq >= 148
    q = synth.to_dtype_np(rng.standard_normal((Nq, H, D)) * 0.3, "bf16")
    if dense:
        idx, cnt = oracle.hca_select(pos, seq, ne, m)
    else:
        n_vis = np.minimum((pos + 1) // m, ne[seq]).astype(np.int32)
        idx = np.full((Nq, k), -1, np.int32)
        cnt = np.zeros(Nq, np.int32)
        for i in range(Nq):
            c = min(k, int(n_vis[i]))
            idx[i, :c] = np.sort(rng.choice(n_vis[i], c, replace=False)) if c else []
            cnt[i] = c
    ref, lse_ref = oracle.attention(q, pos, seq, ent, idx, cnt, win, wbase, W)
    args = (to_dev_bf16(q, cuda), to_dev(pos.astype(np.int32), cuda), to_dev(seq, cuda), to_dev_bf16(ent, cuda))
    wb = to_dev(wbase.astype(np.int32), cuda)
    if dense:
        out, lse = B.hca_attn(*args, to_dev(ne, cuda), to_dev_bf16(win, cuda), wb, mprime=m, W=W, want_lse=True)
    else:
        out, lse = B.csa_sparse_attn(*args, to_dev(idx, cuda), to_dev(cnt, cuda), to_dev_bf16(win, cuda), wb, W=W,
                                     want_lse=True)
    assert_close_attn(t2np(out), ref, "tile-aligned attention")
    np.testing.assert_allclose(t2np(lse), lse_ref, atol=2e-2)
    _err_clear(B)


@pytest.mark.parametrize("dense", [False, True])
@pytest.mark.parametrize("Nq", [6, 160])
def test_attn_query_prep_in_kernel(B, cuda, dense, Nq):
    """csa_sparse_attn_ex / hca_attn_ex on raw queries against the oracle from the raw
    queries, and against csa_norm_rope followed by the plain call (the same transform,
    with the norm folded into the logit scale: equal up to rounding).  Few queries (split
    key lists, two-pass pipeline) and many (one CTA per query, tile boundaries); positions
    up to 2^20 exercise the angle reduction."""
    rng = np.random.default_rng(41 + Nq + dense)
    D, H, m, W, E_max, k = 512, 64, 4, 128, 400, 256
    Tw = 1 << 20
    base = Tw - 3000
    pos = np.sort(rng.choice(np.arange(base, Tw), Nq, replace=False)).astype(np.int64)
    pos[-1] = Tw - 1
    seq = np.zeros(Nq, np.int32)
    ent = synth.to_dtype_np(rng.standard_normal((1, E_max, D)), "bf16")
    win = synth.to_dtype_np(rng.standard_normal((1, 3000, D)), "bf16")
    wbase = np.array([base], np.int32)
    qraw = synth.to_dtype_np(rng.standard_normal((Nq, H, D)) * 2.0, "bf16")
    idx = np.stack([np.sort(rng.choice(E_max, k, replace=False)) for _ in range(Nq)]).astype(np.int32)
    cnt = np.full(Nq, k, np.int32)
    q_d, pos_d, seq_d = to_dev_bf16(qraw, cuda), to_dev(pos.astype(np.int32), cuda), to_dev(seq, cuda)
    ent_d, win_d, wb_d = to_dev_bf16(ent, cuda), to_dev_bf16(win, cuda), to_dev(wbase, cuda)
    prep = dict(norm=True, eps=1e-6, rope_dims=64, theta=10000.0)
    qn = B.csa_norm_rope(q_d, pos_d, norm=True, eps=1e-6, rope_dims=64, theta=10000.0)
    if dense:
        ne = to_dev(np.array([E_max], np.int32), cuda)
        a, la = B.hca_attn(qn, pos_d, seq_d, ent_d, ne, win_d, wb_d, mprime=m, W=W, want_lse=True)
        b, lb = B.hca_attn_ex(prep, q_d, pos_d, seq_d, ent_d, ne, win_d, wb_d, mprime=m, W=W, want_lse=True)
    else:
        idx_d, cnt_d = to_dev(idx, cuda), to_dev(cnt, cuda)
        a, la = B.csa_sparse_attn(qn, pos_d, seq_d, ent_d, idx_d, cnt_d, win_d, wb_d, W=W, want_lse=True)
        b, lb = B.csa_sparse_attn_ex(prep, q_d, pos_d, seq_d, ent_d, idx_d, cnt_d, win_d, wb_d, W=W, want_lse=True)
    torch.cuda.synchronize()
    assert_close_attn(t2np(b), t2np(a), "in-kernel query prep vs csa_norm_rope + attention")
    np.testing.assert_allclose(t2np(lb), t2np(la), atol=1e-2)
    # and against the oracle from the raw queries
    qf = oracle.prep_queries(qraw, pos, True, 1e-6, 64, 10000.0)
    if dense:
        idx, cnt = oracle.hca_select(pos, seq, np.array([E_max]), m)
    ref, _ = oracle.attention(qf, pos, seq, ent, idx, cnt, win, wbase.astype(np.int64), W)
    assert_close_attn(t2np(b), ref, "attention with in-kernel query prep")
    _err_clear(B)


def test_attn_query_prep_rejects_unsupported_rope(B, cuda):
    q = torch.zeros((1, 64, 512), dtype=torch.bfloat16, device=cuda)
    i1 = torch.zeros(1, dtype=torch.int32, device=cuda)
    ent = torch.zeros((1, 8, 512), dtype=torch.bfloat16, device=cuda)
    idx = torch.zeros((1, 4), dtype=torch.int32, device=cuda)
    for rd in (66, 3, -2):
        with pytest.raises(B.CsaError):
            B.csa_sparse_attn_ex(dict(norm=True, eps=1e-6, rope_dims=rd, theta=1e4), q, i1, i1, ent, idx, i1, ent, i1,
                                 W=4)


def test_attn_bad_index_flagged_and_skipped(B, cuda):
    rng = np.random.default_rng(12)
    Nq, E, k, W, Tw = 4, 256, 32, 16, 1024
    ent, win, q = _attn_inputs(12, Nq, E, Tw, k, W)
    pos = np.array([700, 800, 900, 1000], np.int64)
    idx = np.stack([np.sort(rng.choice(E, k, replace=False)) for _ in range(Nq)]).astype(np.int32)
    cnt = np.full(Nq, k, np.int32)
    bad = idx.copy()
    bad[1, 5] = E + 1000       # outside the cache: must be skipped and flagged
    seq = np.zeros(Nq, np.int32)
    out, _ = B.csa_sparse_attn(to_dev_bf16(q, cuda), to_dev(pos.astype(np.int32), cuda), to_dev(seq, cuda),
                               to_dev_bf16(ent, cuda), to_dev(bad, cuda), to_dev(cnt, cuda), to_dev_bf16(win, cuda),
                               to_dev(np.zeros(1, np.int32), cuda), W=W)
    assert B.csa_get_device_error() == B.DEVERR_INDEX
    keep = np.delete(idx[1], 5)
    idx2 = np.full((Nq, k), -1, np.int32)
    idx2[:, :] = idx
    idx2[1, :k - 1] = keep
    idx2[1, k - 1] = -1
    cnt2 = cnt.copy()
    cnt2[1] = k - 1
    ref, _ = oracle.attention(q, pos, seq, ent, idx2, cnt2, win, np.zeros(1, np.int64), W)
    assert_close_attn(t2np(out), ref, "attention with a skipped index")
