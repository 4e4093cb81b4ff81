"""Pins of the CPU oracle to facts outside itself (closed forms, invariants,
brute force, hand-worked vectors, numbers the pages print).

Each test is chosen so that a plausible slip in the oracle (a wrong slot-to-token
map, a zero-padded instead of excluded slot, a transposed RoPE pair, an
off-by-one in entry visibility, a wrong tie rule, a dropped window row) fails.
"""
import json
import math
import os

import numpy as np
import pytest

import oracle
from compressed_sparse_long_02_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
rng0 = np.random.default_rng(1234)


# ------------------------------------------------------------------ pooling (compressor)
def _rand(shape, rng=rng0):
    return rng.standard_normal(shape)


@pytest.mark.parametrize("m,overlap", [(4, True), (128, False), (4, False), (2, True)])
def test_pool_uniform_logits_is_mean(m, overlap):
    """Equal logits and zero bias: softmax weights are uniform, so each entry is the
    plain mean of the tokens it pools (8 for a CSA entry, 4 for the first CSA entry,
    m' for HCA)."""
    T, C = 6 * m + 3, 16
    kv = _rand((T, C))
    z = np.full((T, C), 0.37)
    bias = np.zeros(((2 if overlap else 1) * m, C), np.float32)
    e = oracle.pool(kv, z, bias, m, overlap)
    assert e.shape == (T // m, C)
    for j in range(T // m):
        lo = m * (j - 1) if (overlap and j > 0) else m * j
        ref = kv[lo:m * (j + 1)].mean(axis=0)
        np.testing.assert_allclose(e[j], ref, rtol=0, atol=1e-13)


def test_pool_bias_slot_selects_token():
    """A large bias on slot s makes that slot's token dominate: slot s < m maps to
    token m(j-1)+s (previous group), slot s >= m to token mj+s-m (own group)."""
    m, T, C = 4, 40, 8
    kv = _rand((T, C))
    z = np.zeros((T, C))
    for s in range(2 * m):
        bias = np.zeros((2 * m, C), np.float32)
        bias[s] = 80.0
        e = oracle.pool(kv, z, bias, m, True)
        for j in range(1, T // m):
            np.testing.assert_allclose(e[j], kv[m * (j - 1) + s], atol=1e-12)
        if s >= m:  # first entry has no previous group: its own slot still wins
            np.testing.assert_allclose(e[0], kv[s - m], atol=1e-12)


def test_pool_first_entry_excludes_missing_slots():
    """Entry 0 has no previous group: those slots are left out of the softmax, not
    zero-padded (a zero row with zero logit would pull the mean toward 0)."""
    m, C = 4, 8
    kv = np.ones((8, C)) * 5.0
    z = np.zeros((8, C))
    e = oracle.pool(kv, z, np.zeros((8, C), np.float32), m, True)
    np.testing.assert_allclose(e, 5.0, atol=1e-13)


def test_pool_weights_sum_to_one_and_convex():
    """Softmax weights sum to one per channel: pooling a constant c gives c exactly
    (to rounding), and every entry lies within the per-channel range of its slots."""
    m, T, C = 4, 64, 12
    z = _rand((T, C)) * 3
    bias = (_rand((2 * m, C)) * 0.3).astype(np.float32)
    e1 = oracle.pool(np.full((T, C), 2.5), z, bias, m, True)
    assert np.max(np.abs(e1 - 2.5)) < 1e-12
    kv = _rand((T, C))
    e = oracle.pool(kv, z, bias, m, True)
    for j in range(T // m):
        lo = max(0, m * (j - 1))
        blk = kv[lo:m * (j + 1)]
        assert np.all(e[j] >= blk.min(axis=0) - 1e-12) and np.all(e[j] <= blk.max(axis=0) + 1e-12)


def test_pool_locality():
    """Changing token 4j+3 changes only entries j and j+1 with overlap, only entry j without."""
    m, T, C, j = 4, 48, 8, 5
    kv = _rand((T, C))
    z = _rand((T, C))
    bias = np.zeros((2 * m, C), np.float32)
    for overlap, touched in [(True, {j, j + 1}), (False, {j})]:
        b = bias if overlap else bias[:m]
        e0 = oracle.pool(kv, z, b, m, overlap)
        kv2 = kv.copy()
        kv2[4 * j + 3] += 1.0
        e1 = oracle.pool(kv2, z, b, m, overlap)
        changed = {i for i in range(T // m) if not np.array_equal(e0[i], e1[i])}
        assert changed == touched


def test_pool_two_slot_closed_form():
    """m=1 with overlap: entry j pools tokens j-1 and j with weights
    sigmoid(a_1 - a_0) -- written out for two slots."""
    T, C = 10, 3
    kv = _rand((T, C))
    z = _rand((T, C))
    bias = np.array([[0.2, -0.1, 0.0], [0.0, 0.3, -0.4]], np.float32)
    e = oracle.pool(kv, z, bias, 1, True)
    for j in range(1, T):
        a0 = z[j - 1] + bias[0].astype(np.float64)
        a1 = z[j] + bias[1].astype(np.float64)
        w1 = 1.0 / (1.0 + np.exp(a0 - a1))
        np.testing.assert_allclose(e[j], (1 - w1) * kv[j - 1] + w1 * kv[j], atol=1e-13)
    np.testing.assert_allclose(e[0], kv[0], atol=1e-15)


# ------------------------------------------------------------------ visibility and counts
def test_page_entry_counts_and_constants():
    facts = json.load(open(os.path.join(GOLDEN, "page_facts.json")))["facts"]
    for f in facts:
        if "context_tokens" in f:
            n = oracle.n_visible(f["context_tokens"] - 1, f["m"], 1 << 40)
            assert n == f["context_tokens"] // f["m"]
            assert abs(n - f["approx"]) <= f["rel_tol"] * f["approx"], f["what"]
    wl = synth.WORKLOADS
    assert wl["csa_decode_1m"].k == 1024 and wl["csa_decode_128k"].k == 1024
    assert all(w.W == 128 for n, w in wl.items() if n != "tiny")
    assert wl["csa_decode_1m"].E == 262144 and wl["csa_decode_128k"].E == 32768
    assert wl["hca_prefill_64k"].E == 512 and wl["csa_prefill_8k"].E == 2048


def test_visibility_unfinished_group():
    """A group becomes an entry only when complete: the query at 4j+2 does not see
    entry j, the query at 4j+3 does (its last token is the query itself)."""
    for j in range(0, 20):
        assert oracle.n_visible(4 * j + 2, 4, 10 ** 6) == j
        assert oracle.n_visible(4 * j + 3, 4, 10 ** 6) == j + 1
        assert oracle.n_visible(128 * j + 126, 128, 10 ** 6) == j
        assert oracle.n_visible(128 * j + 127, 128, 10 ** 6) == j + 1
    assert oracle.n_visible(10 ** 6, 4, 77) == 77


# ------------------------------------------------------------------ RMSNorm and RoPE
def test_rmsnorm_unit_mean_square():
    x = _rand((50, 64)) * 3
    y = oracle.rmsnorm(x, 1e-6)
    ms = (x ** 2).mean(axis=1)
    np.testing.assert_allclose((y ** 2).mean(axis=1), ms / (ms + 1e-6), rtol=1e-12)
    np.testing.assert_allclose(y / x, (1 / np.sqrt(ms + 1e-6))[:, None] * np.ones_like(x), rtol=1e-12)


def test_rope_closed_form_angles():
    """Pair i of the rotated slice turns by pos * theta^(-2i/d_r): pair 0 by pos
    radians, pair 1 of a 4-dim slice by pos/100 at theta=1e4; channels before the
    slice are untouched; the pair layout is (2i, 2i+1)."""
    C, dr = 12, 4
    x = np.zeros((1, C))
    x[0, 8] = 1.0   # pair 0 of the slice: (8, 9)
    x[0, 10] = 1.0  # pair 1: (10, 11)
    x[0, 0] = 7.0
    y = oracle.rope(x, np.array([3]), dr, 10000.0)
    np.testing.assert_allclose(y[0, 8:10], [math.cos(3.0), math.sin(3.0)], atol=1e-15)
    np.testing.assert_allclose(y[0, 10:12], [math.cos(0.03), math.sin(0.03)], atol=1e-15)
    assert y[0, 0] == 7.0 and np.all(y[0, 1:8] == 0)


def test_rope_norm_and_relative_position():
    C, dr = 64, 32
    q = _rand((1, C))
    k = _rand((1, C))
    for p, pp, delta in [(5, 2, 11), (1000, 17, 4096), (0, 0, 123)]:
        rq = oracle.rope(q, np.array([p]), dr, 10000.0)
        rk = oracle.rope(k, np.array([pp]), dr, 10000.0)
        rq2 = oracle.rope(q, np.array([p + delta]), dr, 10000.0)
        rk2 = oracle.rope(k, np.array([pp + delta]), dr, 10000.0)
        assert abs(np.dot(rq[0], rk[0]) - np.dot(rq2[0], rk2[0])) < 1e-10
        assert abs(np.linalg.norm(rq) - np.linalg.norm(q)) < 1e-12
    assert np.array_equal(oracle.rope(q, np.array([99]), 0, 10000.0), q)


# ------------------------------------------------------------------ MXFP4
def _codes(packed):
    lo = packed & 0xF
    hi = packed >> 4
    return np.stack([lo, hi], axis=-1).reshape(packed.shape[:-1] + (-1,))


def test_mxfp4_hand_worked_vectors():
    cases = json.load(open(os.path.join(GOLDEN, "mxfp4_vectors.json")))["cases"]
    for c in cases:
        x = np.array(c["x"], dtype=np.float32)[None]
        pk, sc = oracle.mxfp4_quantize(x)
        assert int(sc[0, 0]) == c["scale_byte"], c["name"]
        assert _codes(pk)[0].tolist() == c["codes"], c["name"]


def test_mxfp4_roundtrip_idempotent_and_bound():
    x = (rng0.standard_normal((64, 128)) * np.exp(rng0.uniform(-8, 8, (64, 1)))).astype(np.float32)
    pk, sc = oracle.mxfp4_quantize(x)
    deq = oracle.mxfp4_dequantize(pk, sc)
    pk2, sc2 = oracle.mxfp4_quantize(deq.astype(np.float32))
    # values are a fixed point; bytes need not be (a block whose amax rounds down to
    # 3*2^E re-encodes as 6*2^(E-1): same value, smaller exponent)
    np.testing.assert_array_equal(oracle.mxfp4_dequantize(pk2, sc2), deq)
    amax_code = np.abs(deq.reshape(64, 4, 32)).max(axis=2) / np.exp2(sc.astype(np.int64) - 127)
    same = (amax_code > 3) | (amax_code == 0)
    assert np.array_equal(sc[same], sc2[same])
    # scale rule: amax <= 6*2^E and amax > 6*2^(E-1) (E minimal)
    E = sc.astype(np.int64) - 127
    amax = np.abs(x.reshape(64, 4, 32)).max(axis=2)
    assert np.all(amax <= 6 * np.exp2(E)) and np.all(amax > 6 * np.exp2(E - 1))
    # error bound: half the local grid step (<= 1 at the top, 0.25 below 2) times 2^E
    err = np.abs(x.astype(np.float64) - deq).reshape(64, 4, 32)
    a = np.abs(x.astype(np.float64)).reshape(64, 4, 32) / np.exp2(E)[..., None]
    half_step = np.where(a > 4, 1.0, np.where(a > 2, 0.5, 0.25))
    assert np.all(err <= half_step * np.exp2(E)[..., None] + 1e-30)


def test_mxfp4_grid_values_roundtrip_exact():
    grid = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6], np.float64)
    for E in (-20, -3, 0, 5):
        vals = np.resize(np.concatenate([grid, -grid[1:]]), 32) * 2.0 ** E
        x = vals.astype(np.float32)[None]
        pk, sc = oracle.mxfp4_quantize(x)
        assert sc[0, 0] == E + 127
        np.testing.assert_array_equal(oracle.mxfp4_dequantize(pk, sc)[0], vals)


# ------------------------------------------------------------------ indexer scores
def _fp4_rows(vals_by_row):
    x = np.array(vals_by_row, np.float32)
    return oracle.mxfp4_quantize(x)


def test_index_score_closed_form():
    """q head 0 = all 1, head 1 = all -1, head 2 = first half 2; key = all 1 (Di=64).
    Dots: 64, -64, 64; ReLU drops head 1; score = 0.5*64 + 0.25*0 + 2*64 = 160."""
    Di, Hi = 64, 3
    q = np.zeros((1, Hi, Di), np.float32)
    q[0, 0] = 1.0
    q[0, 1] = -1.0
    q[0, 2, :32] = 2.0
    k = np.ones((1, 2, Di), np.float32)
    k[0, 1, :] = -0.5
    qp, qs = oracle.mxfp4_quantize(q)
    kp, ks = oracle.mxfp4_quantize(k)
    w = np.array([[0.5, 0.25, 2.0]], np.float32)
    s32, s64, bad = oracle.index_scores(qp, qs, w, np.array([0]), np.array([2]), kp, ks, want64=True)
    assert bad == 0
    assert s32[0, 0] == 160.0 and s64[0, 0] == 160.0
    # key 2 = -0.5: dots -32, 32, -32 -> only head 1 survives: 0.25*32 = 8
    assert s32[0, 1] == 8.0


def test_index_score_fp32_chain_within_bound_of_fp64():
    wl = synth.WORKLOADS["tiny"]
    inp = synth.prefill_inputs(wl)
    r = oracle.csa_prefill(wl, inp, rows=np.arange(100, 512, 37))
    s32, s64, bad = oracle.index_scores(r["q_packed"], r["q_scales"], inp["w"][0][r["rows"]],
                                        np.zeros(len(r["rows"]), np.int32), r["n_vis"],
                                        r["k_packed"][None], r["k_scales"][None], want64=True)
    assert bad == 0
    vis = np.isfinite(s64)
    rel = np.abs(s32[vis] - s64[vis]) / np.maximum(np.abs(s64[vis]), 1e-30)
    assert rel.max() <= wl.Hi * 2.0 ** -23
    assert np.all(s32[vis] >= 0)


# ------------------------------------------------------------------ top-k
def _brute_topk(s, nv, k):
    cand = [(-float(s[j]), j) for j in range(nv)]
    cand.sort()
    return sorted(j for _, j in cand[:k])


def test_topk_brute_force_and_ties():
    r = np.random.default_rng(7)
    nq, E, k = 40, 60, 9
    s = r.integers(0, 6, (nq, E)).astype(np.float32)   # many exact ties
    s[::3] = r.standard_normal((len(s[::3]), E)).astype(np.float32)
    s[5] = 0.0                                          # all-zero row: lowest indices
    nv = r.integers(0, E + 1, nq).astype(np.int32)
    nv[5] = E
    idx, cnt, kth = oracle.topk(s, nv, k)
    for n in range(nq):
        ref = _brute_topk(s[n], nv[n], k)
        assert cnt[n] == len(ref)
        assert idx[n, :cnt[n]].tolist() == ref
        assert np.all(idx[n, cnt[n]:] == -1)
    assert idx[5].tolist() == list(range(k))


def test_topk_all_visible_when_few_and_scale_invariance():
    r = np.random.default_rng(8)
    s = r.random((5, 30)).astype(np.float32)
    idx, cnt, _ = oracle.topk(s, np.array([0, 3, 7, 8, 30], np.int32), 8)
    assert cnt.tolist() == [0, 3, 7, 8, 8]
    assert idx[2, :7].tolist() == list(range(7)) and idx[2, 7] == -1
    idx2, _, _ = oracle.topk(s * 4.0, np.array([0, 3, 7, 8, 30], np.int32), 8)
    assert np.array_equal(idx, idx2)


# ------------------------------------------------------------------ attention
def _dense_masked_attention(q, keys, scale):
    """Textbook softmax attention of each head against a key list (K = V)."""
    logits = np.einsum("hd,rd->hr", q, keys) * scale
    logits -= logits.max(axis=1, keepdims=True)
    p = np.exp(logits)
    p /= p.sum(axis=1, keepdims=True)
    return p @ keys


def test_attention_full_selection_matches_dense_masked():
    """With k covering every visible entry, the layer equals plain attention over the
    concatenated [visible entries | window rows] key list (written out densely here)."""
    r = np.random.default_rng(11)
    E, D, H, W, Tw = 20, 16, 3, 5, 40
    ent = r.standard_normal((1, E, D))
    win = r.standard_normal((1, Tw, D))
    ts = np.array([0, 3, 4, 17, 39])
    nv = np.array([oracle.n_visible(t, 2, E) for t in ts], np.int32)
    idx = np.full((len(ts), E), -1, np.int32)
    for i, v in enumerate(nv):
        idx[i, :v] = np.arange(v)
    q = r.standard_normal((len(ts), H, D))
    out, lse = oracle.attention(q, ts, np.zeros(len(ts), np.int32), ent, idx, nv, win, np.zeros(1, np.int64), W)
    for i, t in enumerate(ts):
        keys = np.concatenate([ent[0, :nv[i]], win[0, max(0, t - W + 1):t + 1]])
        ref = _dense_masked_attention(q[i], keys, 1 / math.sqrt(D))
        np.testing.assert_allclose(out[i], ref, atol=1e-12)


def test_attention_duplicate_key_kept_and_single_key():
    D = 4
    k1 = np.array([1.0, 0.0, 0.0, 0.0])
    k2 = np.array([0.0, 1.0, 0.0, 0.0])
    ent = np.stack([k1, k2])[None]
    win = k1[None, None, :]            # window row at position 0 equals entry 0
    q = np.array([[[2.0, 1.0, 0.0, 0.0]]])
    out, lse = oracle.attention(q, np.array([0]), np.array([0]), ent, np.array([[0, 1]]), np.array([2]),
                                win, np.zeros(1, np.int64), 1, scale=1.0)
    e1, e2 = math.exp(2.0), math.exp(1.0)
    ref = (2 * e1 * k1 + e2 * k2) / (2 * e1 + e2)
    np.testing.assert_allclose(out[0, 0], ref, atol=1e-14)
    assert abs(lse[0, 0] - math.log(2 * e1 + e2)) < 1e-14
    out1, lse1 = oracle.attention(q, np.array([0]), np.array([0]), ent, np.array([[1, -1]]), np.array([1]),
                                  win, np.zeros(1, np.int64), 0, scale=1.0)
    np.testing.assert_allclose(out1[0, 0], k2, atol=0)
    assert lse1[0, 0] == 1.0


def test_hca_reduces_to_causal_attention():
    """HCA with m'=1, no window, zero bias and no RoPE/norm: each entry is its own
    token, visible iff j <= t, so the layer is textbook causal attention
    (torch scaled_dot_product_attention, float64, is_causal=True)."""
    import torch
    r = np.random.default_rng(3)
    T, D, H = 33, 8, 2
    kv = r.standard_normal((T, D))
    e = oracle.pool(kv, r.standard_normal((T, D)), np.zeros((1, D), np.float32), 1, False)
    np.testing.assert_array_equal(e, kv)
    q = r.standard_normal((T, H, D))
    ts = np.arange(T)
    idx, cnt = oracle.hca_select(ts, np.zeros(T, np.int32), np.array([T]), 1)
    out, _ = oracle.attention(q, ts, np.zeros(T, np.int32), e[None], idx, cnt, np.zeros((1, 1, D)),
                              np.zeros(1, np.int64), 0)
    qt = torch.from_numpy(q).permute(1, 0, 2)[None]
    kt = torch.from_numpy(kv)[None, None].expand(1, H, T, D)
    ref = torch.nn.functional.scaled_dot_product_attention(qt, kt, kt, is_causal=True)[0].permute(1, 0, 2)
    np.testing.assert_allclose(out, ref.numpy(), atol=1e-12)


def test_layer_causality():
    """Perturbing any token after t leaves the layer output at t bit-identical
    (entries of unfinished groups, future window rows and future indexer keys are
    all out of reach)."""
    wl = synth.WORKLOADS["tiny"].replace(T=64, k=4, W=8)
    inp = synth.prefill_inputs(wl, T=64)
    rows = np.array([0, 3, 4, 7, 13, 30])
    r0 = oracle.csa_prefill(wl, inp, rows=rows)
    for cut in (14, 31):
        inp2 = {k: v.copy() for k, v in inp.items()}
        for key in ("kv", "z", "ki", "zi"):
            inp2[key][:, cut:] = inp2[key][:, cut:][::-1] if inp2[key].dtype != np.uint16 else 0
        r1 = oracle.csa_prefill(wl, inp2, rows=rows)
        for i, t in enumerate(rows):
            if t < cut:
                assert np.array_equal(r0["out"][i], r1["out"][i]), (cut, t)


def test_tiny_workload_sanity():
    wl = synth.WORKLOADS["tiny"]
    inp = synth.prefill_inputs(wl)
    r = oracle.csa_prefill(wl, inp)
    assert r["entries"].shape == (128, 128)
    assert r["inexact"] == 0
    # the query at position t sees floor((t+1)/4) entries and min(k, that) are selected
    t = np.arange(512)
    np.testing.assert_array_equal(r["cnt"], np.minimum((t + 1) // 4, wl.k))
    assert np.all(np.isfinite(r["out"]))


# ------------------------------------------------------------------ grouped output projection
def _gop_case(seed, T=5, H=8, D=6, G=4, R=5, dm=7):
    rng = np.random.default_rng(seed)
    o = rng.standard_normal((T, H, D))
    A = rng.standard_normal((G, R, (H // G) * D))
    Bm = rng.standard_normal((dm, G * R))
    return o, A, Bm


def test_grouped_out_proj_identity_is_concatenation():
    """Identity group matrices (R = heads per group x D) and an identity dense matrix:
    the projection returns the head outputs concatenated, exactly."""
    T, H, D, G = 4, 8, 3, 2
    o = np.random.default_rng(1).standard_normal((T, H, D))
    Kg = (H // G) * D
    A = np.stack([np.eye(Kg)] * G)
    z, y = oracle.grouped_out_proj(o, A, np.eye(G * Kg), G)
    assert np.array_equal(z, o.reshape(T, H * D)) and np.array_equal(y, o.reshape(T, H * D))


def test_grouped_out_proj_one_group_is_two_matrix_products():
    """G = 1 is the textbook chain of two dense projections, y = (o A^T) B^T (a library
    matmul here); R differs from the group width, so a transposed operand cannot pass."""
    o, A, Bm = _gop_case(2, G=1)
    z, y = oracle.grouped_out_proj(o, A, Bm, 1)
    z_ref = o.reshape(o.shape[0], -1) @ A[0].T
    np.testing.assert_allclose(z, z_ref, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(y, z_ref @ Bm.T, rtol=1e-12, atol=1e-12)


def test_grouped_out_proj_equals_block_diagonal_single_group():
    """G groups equal one group whose matrix is block diagonal (group g's matrix on the
    block of its heads): the grouping only removes the zero blocks."""
    o, A, Bm = _gop_case(3)
    G, R, Kg = A.shape
    Abd = np.zeros((1, G * R, G * Kg))
    for g in range(G):
        Abd[0, g * R:(g + 1) * R, g * Kg:(g + 1) * Kg] = A[g]
    z, y = oracle.grouped_out_proj(o, A, Bm, G)
    z1, y1 = oracle.grouped_out_proj(o, Abd, Bm, 1)
    np.testing.assert_allclose(z, z1, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(y, y1, rtol=1e-12, atol=1e-12)


def test_grouped_out_proj_group_locality_and_linearity():
    """Changing the heads of group g changes only that group's R intermediate values; the
    projection is linear in the head outputs."""
    o, A, Bm = _gop_case(4)
    G, R, _ = A.shape
    H = o.shape[1]
    z, y = oracle.grouped_out_proj(o, A, Bm, G)
    for g in range(G):
        o2 = o.copy()
        o2[:, g * (H // G):(g + 1) * (H // G)] += 1.0
        z2, _ = oracle.grouped_out_proj(o2, A, Bm, G)
        changed = np.any(z2 != z, axis=0)
        assert changed[g * R:(g + 1) * R].all() and not np.delete(changed, np.s_[g * R:(g + 1) * R]).any()
    z3, y3 = oracle.grouped_out_proj(2.5 * o, A, Bm, G)
    np.testing.assert_allclose(y3, 2.5 * y, rtol=1e-12, atol=1e-12)
