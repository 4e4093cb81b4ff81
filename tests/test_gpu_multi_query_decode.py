"""Multi-query decode: two new tokens of each sequence scored together by the lightning
indexer (csa_index_topk_grouped, q_group = 2), every key tile read once per pair.

Bars: scores, indices and counts bitwise equal to csa_index_topk on the same rows (the
per-pair head chain is the same fixed order), scores bit-exact against the oracle on
every visible entry and index sets exact (check_topk); a pair whose rows name different
sequences flags CSA_DEVERR_INDEX and its second row scores -inf.
"""
import numpy as np
import pytest

import oracle
from compressed_sparse_long_02_b200 import synth
from tests.helpers import check_topk, t2np, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def B(cuda):
    from compressed_sparse_long_02_b200 import binding
    binding.lib()
    return binding


def _inputs(seed, n_ent, E_max, nq, Hi=64, Di=128):
    rng = np.random.default_rng(seed)
    Bs = len(n_ent)
    kp, ks = oracle.mxfp4_quantize(rng.standard_normal((Bs, E_max, Di)).astype(np.float32))
    qp, qs = oracle.mxfp4_quantize(rng.standard_normal((nq, Hi, Di)).astype(np.float32))
    w = rng.random((nq, Hi)).astype(np.float32)
    return kp, ks, qp, qs, w


def _run(B, cuda, q_group, qp, qs, w, pos, seq, kp, ks, n_ent, k, m=4):
    return B.csa_index_topk(to_dev(qp, cuda), to_dev(qs, cuda), to_dev(w, cuda), to_dev(pos.astype(np.int32), cuda),
                            to_dev(seq.astype(np.int32), cuda), to_dev(kp, cuda), to_dev(ks, cuda),
                            to_dev(n_ent.astype(np.int32), cuda), k=k, m=m, want_scores=True, q_group=q_group)


@pytest.mark.parametrize("odd", [False, True])
def test_grouped_indexer_bitwise_and_oracle(B, cuda, odd):
    """Six sequences with ragged entry counts, two queries each at consecutive positions
    (the second sees one entry more); with `odd` the last group has a single row."""
    m, k, E_max = 4, 512, 4096
    n_ent = np.array([4096, 1000, 4095, 1025, 2048, 96], np.int32)
    seq = np.repeat(np.arange(len(n_ent)), 2).astype(np.int32)
    pos = np.stack([n_ent * m - 2, n_ent * m - 1], 1).reshape(-1).astype(np.int64)
    if odd:
        seq, pos = seq[:-1], pos[:-1]
    nq = len(seq)
    kp, ks, qp, qs, w = _inputs(5 + odd, n_ent, E_max, nq)
    g_idx, g_cnt, g_sc = _run(B, cuda, 2, qp, qs, w, pos, seq, kp, ks, n_ent, k)
    assert B.csa_get_device_error() == 0
    u_idx, u_cnt, u_sc = _run(B, cuda, 1, qp, qs, w, pos, seq, kp, ks, n_ent, k)
    assert B.csa_get_device_error() == 0
    n_vis = np.array([oracle.n_visible(int(pos[i]), m, int(n_ent[seq[i]])) for i in range(nq)], np.int32)
    assert n_vis[0] + 1 == n_vis[1]
    g_sc, u_sc = t2np(g_sc), t2np(u_sc)
    for i in range(nq):  # the workspace rows past n_vis are not part of the result
        assert np.array_equal(g_sc[i, :n_vis[i]].view(np.uint32), u_sc[i, :n_vis[i]].view(np.uint32)), f"row {i}"
    assert np.array_equal(t2np(g_idx), t2np(u_idx)) and np.array_equal(t2np(g_cnt), t2np(u_cnt))
    s32, _, bad = oracle.index_scores(qp, qs, w, seq, n_vis, kp, ks)
    assert bad == 0
    for i in range(nq):
        np.testing.assert_array_equal(g_sc[i, :n_vis[i]], s32[i, :n_vis[i]])
    idx_r, cnt_r, kth = oracle.topk(s32, n_vis, k)
    check_topk(t2np(g_idx), t2np(g_cnt), idx_r, cnt_r, kth, s32, n_vis, k)


def test_grouped_indexer_128k_decode_shape(B, cuda):
    """16 sequences x 2 new tokens at the 128K decode shape (32768 entries, k = 1024):
    bitwise the ungrouped call on every row, two rows against the oracle."""
    wl = synth.WORKLOADS["csa_decode_128k"]
    Bs, E = 16, wl.E
    n_ent = np.full(Bs, E, np.int32)
    n_ent[3] = E - 5
    seq = np.repeat(np.arange(Bs), 2).astype(np.int32)
    pos = np.stack([n_ent * wl.m - 2, n_ent * wl.m + 1], 1).reshape(-1).astype(np.int64)
    kp, ks, qp, qs, w = _inputs(11, n_ent, E, 2 * Bs)
    g = _run(B, cuda, 2, qp, qs, w, pos, seq, kp, ks, n_ent, wl.k, wl.m)
    u = _run(B, cuda, 1, qp, qs, w, pos, seq, kp, ks, n_ent, wl.k, wl.m)
    assert B.csa_get_device_error() == 0
    assert np.array_equal(t2np(g[0]), t2np(u[0])) and np.array_equal(t2np(g[1]), t2np(u[1]))
    rows = np.array([6, 7])
    n_vis = np.array([oracle.n_visible(int(pos[i]), wl.m, int(n_ent[seq[i]])) for i in rows], np.int32)
    s32, _, bad = oracle.index_scores(qp[rows], qs[rows], w[rows], seq[rows], n_vis, kp, ks)
    assert bad == 0
    sc = t2np(g[2])[rows]
    for j in range(len(rows)):
        np.testing.assert_array_equal(sc[j, :n_vis[j]], s32[j, :n_vis[j]])
    idx_r, cnt_r, kth = oracle.topk(s32, n_vis, wl.k)
    check_topk(t2np(g[0])[rows], t2np(g[1])[rows], idx_r, cnt_r, kth, s32, n_vis, wl.k)


def test_grouped_pair_of_two_sequences_is_flagged(B, cuda):
    """Rows 2 and 3 name different sequences: the error word says so, row 2 is scored as
    usual and row 3 scores -inf on every entry visible to it; the other pairs are exact."""
    m, k, E_max = 4, 64, 1024
    n_ent = np.array([1024, 900, 1000], np.int32)
    seq = np.array([0, 0, 1, 2, 2, 2], np.int32)
    pos = np.array([4000, 4001, 3599, 3999, 3000, 3001], np.int64)
    kp, ks, qp, qs, w = _inputs(21, n_ent, E_max, len(seq))
    g_idx, g_cnt, g_sc = _run(B, cuda, 2, qp, qs, w, pos, seq, kp, ks, n_ent, k)
    assert B.csa_get_device_error() == B.DEVERR_INDEX
    u_idx, u_cnt, u_sc = _run(B, cuda, 1, qp, qs, w, pos, seq, kp, ks, n_ent, k)
    assert B.csa_get_device_error() == 0
    n_vis = np.array([oracle.n_visible(int(pos[i]), m, int(n_ent[seq[i]])) for i in range(len(seq))], np.int32)
    g_sc, u_sc = t2np(g_sc), t2np(u_sc)
    for i in (0, 1, 2, 4, 5):
        assert np.array_equal(g_sc[i, :n_vis[i]], u_sc[i, :n_vis[i]]), f"row {i}"
        assert np.array_equal(t2np(g_idx)[i], t2np(u_idx)[i])
    assert np.all(np.isneginf(g_sc[3, :n_vis[3]]))
    assert int(t2np(g_cnt)[3]) == min(k, int(n_vis[3]))


def test_grouped_indexer_rejects_unsupported(B, cuda):
    m, k, E_max = 4, 16, 64
    n_ent = np.array([64], np.int32)
    kp, ks, qp, qs, w = _inputs(3, n_ent, E_max, 2, Hi=32)
    seq, pos = np.zeros(2, np.int32), np.array([100, 101])
    with pytest.raises(B.CsaError) as e:
        _run(B, cuda, 2, qp, qs, w, pos, seq, kp, ks, n_ent, k)
    assert e.value.status == 3
    kp, ks, qp, qs, w = _inputs(3, n_ent, E_max, 2)
    with pytest.raises(B.CsaError) as e:
        _run(B, cuda, 3, qp, qs, w, pos, seq, kp, ks, n_ent, k)
    assert e.value.status == 3
