"""End-to-end GPU parity of the whole layer (all C-ABI calls chained) against the
oracle, at the workloads' full sizes in the launch configuration the benchmark uses,
checked on sampled query rows that include the edge positions.

Inputs come from the seeded generators (drawn on the GPU with torch for the large
workloads and copied to the host for the oracle).  The GPU path computes its own
compressed indexer keys in float32, the oracle in float64, so an FP4 code may flip
where a pooled value sits on a rounding boundary: such flips must be justified by that
boundary, and the oracle then scores the GPU's key bytes, so that index sets must match
on every sampled row (up to the 1e-6 tie exemption) and outputs meet the attention
tolerance on all of them.
"""
import numpy as np
import pytest
import torch

import oracle
from compressed_sparse_long_02_b200 import synth
from tests.helpers import assert_close_attn, check_csa_prefill_rows, check_topk, t2np, to_dev, to_dev_bf16

pytestmark = pytest.mark.gpu


def _host(t: torch.Tensor) -> np.ndarray:
    if t.dtype == torch.bfloat16:
        return t.cpu().view(torch.int16).numpy().view(np.uint16)
    return t.cpu().numpy()


def _rows(T, wl, n, seed):
    rng = np.random.default_rng(seed)
    special = [0, 1, 3, 4, 7, 127, 128, wl.m * max(wl.k, 1) - 1, wl.m * max(wl.k, 1), wl.m - 1, wl.m, T - 1]
    return np.unique(np.concatenate([[r for r in special if 0 <= r < T], rng.choice(T, n, replace=False)]))


@pytest.fixture(scope="module")
def L(cuda):
    from compressed_sparse_long_02_b200 import binding, layer
    binding.lib()
    return layer


@pytest.mark.parametrize("T", [2048 + 5, 8192])
def test_csa_prefill_layer(L, cuda, T):
    """Every sampled row must match: index sets exact (up to the 1e-6 tie exemption) when the
    oracle scores the GPU's key bytes, those bytes within the FP4 boundary rule of the
    oracle's own, and outputs within the attention tolerance."""
    wl = synth.WORKLOADS["csa_prefill_8k"].replace(T=T)
    t = synth.prefill_inputs_torch(wl, cuda)
    rows = _rows(T, wl, 96, T)
    r = L.csa_prefill(wl, t)            # every row, as the benchmark runs it
    torch.cuda.synchronize()
    host = {k: (_host(v) if k in ("bias", "bias_i") else _host(v)[0]) for k, v in t.items()
            if k not in ("q", "qi", "w")}
    sel = torch.as_tensor(rows, device=cuda)
    host["q"] = _host(t["q"][0][sel].contiguous())
    host["qi"] = _host(t["qi"][0][sel].contiguous())
    host["w"] = _host(t["w"][0][sel].contiguous())
    check_csa_prefill_rows(wl, host, r, rows)
    assert L.B.csa_get_device_error() == 0


def test_hca_prefill_layer_full_size(L, cuda):
    wl = synth.WORKLOADS["hca_prefill_64k"]
    t = synth.prefill_inputs_torch(wl, cuda)
    T = wl.T
    rows = _rows(T, wl, 64, 4)
    rows = np.unique(np.concatenate([rows, [127, 128, 255, 256, 128 * 511 - 1, 128 * 511, 128 * 512 - 1]]))
    r = L.hca_prefill(wl, t)
    torch.cuda.synchronize()
    kv, z, bias = _host(t["kv"]), _host(t["z"]), _host(t["bias"])
    q = _host(t["q"][0, rows].contiguous())
    ent = oracle.entries_rows(kv[0], z[0], bias, wl.m, False, wl.norm, wl.eps, wl.rope_dims, wl.theta)
    win = oracle.window_rows(kv[0], wl.norm, wl.eps, wl.rope_dims, wl.theta)
    qf = oracle.prep_queries(q, rows, wl.norm, wl.eps, wl.rope_dims, wl.theta)
    seq = np.zeros(len(rows), np.int32)
    idx, cnt = oracle.hca_select(rows, seq, np.array([ent.shape[0]]), wl.m)
    ref, _ = oracle.attention(qf, rows, seq, ent[None], idx, cnt, win[None], np.zeros(1, np.int64), wl.W)
    assert_close_attn(t2np(r["out"][rows]), ref, "HCA prefill 64k")
    assert L.B.csa_get_device_error() == 0


def test_csa_decode_layer_full_size(L, cuda):
    """csa_decode_128k at full size: 32 sequences of 32768 entries; 4 sequences checked."""
    from compressed_sparse_long_02_b200 import binding as B
    wl = synth.WORKLOADS["csa_decode_128k"]
    d = synth.decode_inputs_torch(wl, cuda, replica=0)
    sample = np.array([0, 9, 22, 31])
    ki_host = d["ki"].cpu().numpy()
    kp, ks = oracle.mxfp4_quantize(ki_host)          # the cache bytes come from the oracle's encoder
    cache = {"entries": d["entries"], "k_fp4": to_dev(kp, cuda), "k_scale": to_dev(ks, cuda), "window": d["window"],
             "window_base": (d["pos"] - wl.W + 1).to(torch.int32),
             "n_entries": torch.full((wl.B,), wl.E, dtype=torch.int32, device=cuda)}
    step = {"q": d["q"], "qi": d["qi"], "w": d["w"], "pos": d["pos"]}
    r = L.csa_decode(wl, cache, step)
    torch.cuda.synchronize()
    ent = _host(d["entries"][sample].contiguous())
    qp, qs = oracle.mxfp4_quantize(d["qi"][sample].cpu().numpy())
    pos = d["pos"].cpu().numpy()[sample].astype(np.int64)
    ref = oracle.csa_decode(wl, ent, kp[sample], ks[sample], _host(d["q"][sample].contiguous()), qp, qs,
                            d["w"][sample].cpu().numpy(), _host(d["window"][sample].contiguous()), pos)
    check_topk(t2np(r["idx"])[sample], t2np(r["cnt"])[sample], ref["idx"], ref["cnt"], ref["kth"], ref["scores"],
               ref["n_vis"], wl.k)
    assert_close_attn(t2np(r["out"])[sample], ref["out"], "CSA decode 128k")
    assert B.csa_get_device_error() == 0


def test_csa_decode_1m_sampled(L, cuda):
    """csa_decode_1m: 4 sequences of 262144 entries, 1% boosted indexer keys; 2 sequences checked."""
    wl = synth.WORKLOADS["csa_decode_1m"]
    d = synth.decode_inputs_torch(wl, cuda, replica=0)
    sample = np.array([0, 3])
    kp_d, ks_d = L.B.csa_quantize_mxfp4(d["ki"])      # GPU cache for the run ...
    ki_s = d["ki"][sample].cpu().numpy()
    kp, ks = oracle.mxfp4_quantize(ki_s)             # ... must equal the oracle's bytes (bit-exact encoder)
    assert np.array_equal(t2np(kp_d[sample]), kp) and np.array_equal(t2np(ks_d[sample]), ks)
    cache = {"entries": d["entries"], "k_fp4": kp_d, "k_scale": ks_d, "window": d["window"],
             "window_base": (d["pos"] - wl.W + 1).to(torch.int32),
             "n_entries": torch.full((wl.B,), wl.E, dtype=torch.int32, device=cuda)}
    step = {"q": d["q"], "qi": d["qi"], "w": d["w"], "pos": d["pos"]}
    r = L.csa_decode(wl, cache, step)
    torch.cuda.synchronize()
    ent = _host(d["entries"][sample].contiguous())
    qp, qs = oracle.mxfp4_quantize(d["qi"][sample].cpu().numpy())
    pos = d["pos"].cpu().numpy()[sample].astype(np.int64)
    ref = oracle.csa_decode(wl, ent, kp, ks, _host(d["q"][sample].contiguous()), qp, qs, d["w"][sample].cpu().numpy(),
                            _host(d["window"][sample].contiguous()), pos)
    check_topk(t2np(r["idx"])[sample], t2np(r["cnt"])[sample], ref["idx"], ref["cnt"], ref["kth"], ref["scores"],
               ref["n_vis"], wl.k)
    assert_close_attn(t2np(r["out"])[sample], ref["out"], "CSA decode 1M")


def test_decode_edge_cases(L, cuda):
    """Short contexts: t = 0 (window only), unfinished first group, k larger than the visible set."""
    from compressed_sparse_long_02_b200 import binding as B
    wl = synth.WORKLOADS["csa_decode_128k"].replace(k=16, W=8)
    E = 64
    d = synth.decode_inputs(wl, B=5, E=E)
    kp, ks = oracle.mxfp4_quantize(d["ki"])
    qp, qs = oracle.mxfp4_quantize(d["qi"])
    pos = np.array([0, 2, 3, 37, 4 * E - 1], np.int64)
    n_ent = np.array([E, E, E, 9, E], np.int32)
    wbase = np.maximum(pos - wl.W + 1, 0)
    # window buffer rows hold tokens wbase..wbase+W-1 (a prefix of the buffer is used near t=0)
    cache = {"entries": to_dev_bf16(d["entries"], cuda), "k_fp4": to_dev(kp, cuda), "k_scale": to_dev(ks, cuda),
             "window": to_dev_bf16(d["window"], cuda), "window_base": to_dev(wbase.astype(np.int32), cuda),
             "n_entries": to_dev(n_ent, cuda)}
    step = {"q": to_dev_bf16(d["q"], cuda), "qi": to_dev(d["qi"], cuda), "w": to_dev(d["w"], cuda),
            "pos": to_dev(pos.astype(np.int32), cuda)}
    r = L.csa_decode(wl, cache, step)
    torch.cuda.synchronize()
    seqs = np.arange(5, dtype=np.int32)
    n_vis = np.array([oracle.n_visible(pos[b], wl.m, n_ent[b]) for b in range(5)], np.int32)
    s32, _, _ = oracle.index_scores(qp, qs, d["w"], seqs, n_vis, kp, ks)
    idx, cnt, kth = oracle.topk(s32, n_vis, wl.k)
    ref, _ = oracle.attention(d["q"], pos, seqs, d["entries"], idx, cnt, d["window"], wbase, wl.W)
    check_topk(t2np(r["idx"]), t2np(r["cnt"]), idx, cnt, kth, s32, n_vis, wl.k)
    assert t2np(r["cnt"]).tolist() == [0, 0, 1, 9, 16]
    assert_close_attn(t2np(r["out"]), ref, "decode edge cases")
    assert B.csa_get_device_error() == 0


def test_empty_batches(L, cuda):
    from compressed_sparse_long_02_b200 import binding as B
    z8 = torch.empty((0, 64, 64), dtype=torch.uint8, device=cuda)
    p, s = B.csa_quantize_mxfp4(torch.empty((0, 128), dtype=torch.float32, device=cuda))
    assert p.shape == (0, 64) and s.shape == (0, 4)
    q = torch.empty((0, 64, 512), dtype=torch.bfloat16, device=cuda)
    e = torch.zeros((1, 8, 512), dtype=torch.bfloat16, device=cuda)
    i0 = torch.empty((0,), dtype=torch.int32, device=cuda)
    out, _ = B.csa_sparse_attn(q, i0, i0, e, torch.empty((0, 4), dtype=torch.int32, device=cuda), i0, e,
                               torch.zeros(1, dtype=torch.int32, device=cuda), W=4)
    assert out.shape == (0, 64, 512)
    assert B.csa_get_device_error() == 0
