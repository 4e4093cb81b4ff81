"""The fused decode indexer + top-k (csa_index_topk with csa_set_index_fusion on, when the
clusters of CTAs per query, two CTAs per SM, are at least as many CTAs as SMs and their
slices hold the row: Hi = 64, Di = 128, pre-encoded queries).  Scores stay in shared memory and the cluster selects the top-k, so its
indices, counts and optional score output must equal the two-kernel path's
(csa_index_score then csa_topk_select) bit for bit, and the oracle's selection on the
same key bytes up to the 1e-6 tie exemption.

Shapes (148 SMs): 32 queries x 32768 entries (clusters of 8, 16 entries per thread: the
128K decode), 37 x 16000 (8, 8), 20 x 6000 (8, 8), 60 x 12000 (4, 16); positions vary so
that some queries see at most k entries (taken whole, no scoring), the rest more.
"""
import numpy as np
import pytest
import torch

import oracle
from tests.helpers import check_topk, t2np

pytestmark = pytest.mark.gpu


@pytest.fixture
def B(cuda):
    from compressed_sparse_long_02_b200 import binding
    binding.lib()
    binding.csa_set_index_fusion(True)
    yield binding
    binding.csa_set_index_fusion(False)


def test_fusion_switch_selects_the_kernel_count(B):
    assert B.csa_index_topk_launches(32, 64, 128, 32768, 1024) == 1
    assert B.csa_index_topk_launches(4, 64, 128, 262144, 1024) == 2   # a row too long for the clusters
    B.csa_set_index_fusion(False)
    assert B.csa_index_topk_launches(32, 64, 128, 32768, 1024) == 2
    B.csa_set_index_fusion(True)


def _case(dev, Nq, E, seed, n_seq=None, k=1024):
    g = torch.Generator(device=dev)
    g.manual_seed(seed)
    n_seq = n_seq or Nq
    from compressed_sparse_long_02_b200 import binding as Bd
    keys = torch.randn((n_seq, E, 128), generator=g, device=dev)
    keys[:, ::53] += 1.5
    kp, ks = Bd.csa_quantize_mxfp4(keys)
    qi = torch.randn((Nq, 64, 128), generator=g, device=dev)
    qp, qs = Bd.csa_quantize_mxfp4(qi)
    w = torch.rand((Nq, 64), generator=g, device=dev)
    seq = (torch.arange(Nq, device=dev) % n_seq).to(torch.int32)
    rng = np.random.default_rng(seed)
    # positions: most queries see many entries, a few at most k (taken whole)
    pos = rng.integers(4 * (k + 1), 4 * E, size=Nq)
    pos[:: max(1, Nq // 5)] = rng.integers(0, 4 * k, size=len(pos[:: max(1, Nq // 5)]))
    pos = torch.as_tensor(pos.astype(np.int32), device=dev)
    n_ent = torch.full((n_seq,), E, dtype=torch.int32, device=dev)
    return dict(kp=kp, ks=ks, qp=qp, qs=qs, w=w, seq=seq, pos=pos, n_ent=n_ent, k=k)


@pytest.mark.parametrize("Nq,E,n_seq", [(32, 32768, 32), (37, 16000, 5), (20, 6000, 20), (60, 12000, 7)])
def test_fused_equals_two_kernel_path(B, cuda, Nq, E, n_seq):
    c = _case(cuda, Nq, E, seed=Nq + E, n_seq=n_seq)
    idx_f, cnt_f, sc_f = B.csa_index_topk(c["qp"], c["qs"], c["w"], c["pos"], c["seq"], c["kp"], c["ks"], c["n_ent"],
                                          k=c["k"], m=4, want_scores=True)
    scores = B.csa_index_score(c["qp"], c["qs"], c["w"], c["pos"], c["seq"], c["kp"], c["ks"], c["n_ent"], m=4)
    idx_2, cnt_2 = B.csa_topk_select(scores, c["pos"], c["seq"], c["n_ent"], k=c["k"], m=4, E_max=E)
    torch.cuda.synchronize()
    assert torch.equal(cnt_f, cnt_2), "counts differ from the two-kernel path"
    assert torch.equal(idx_f, idx_2), "indices differ from the two-kernel path"
    # scores are written for the visible entries of queries that needed a selection
    nvis = torch.clamp((c["pos"] + 1) // 4, max=E)
    for n in range(Nq):
        v = int(nvis[n])
        if v > c["k"]:
            assert torch.equal(sc_f[n, :v], scores[n, :v]), f"query {n}: fused score output differs"
    assert B.csa_get_device_error() == 0


def test_fused_matches_oracle_on_sampled_rows(B, cuda):
    Nq, E = 32, 32768
    c = _case(cuda, Nq, E, seed=7)
    idx, cnt, _ = B.csa_index_topk(c["qp"], c["qs"], c["w"], c["pos"], c["seq"], c["kp"], c["ks"], c["n_ent"],
                                   k=c["k"], m=4)
    torch.cuda.synchronize()
    rows = np.array([0, 1, 13, 31])
    seqs = t2np(c["seq"])[rows]
    kp = t2np(c["kp"])[seqs]
    ks = t2np(c["ks"])[seqs]
    pos = t2np(c["pos"])[rows]
    n_vis = np.array([oracle.n_visible(int(t), 4, E) for t in pos], np.int32)
    s32, _, _ = oracle.index_scores(t2np(c["qp"])[rows], t2np(c["qs"])[rows], t2np(c["w"])[rows],
                                    np.arange(len(rows), dtype=np.int32), n_vis, kp, ks)
    idx_r, cnt_r, kth = oracle.topk(s32, n_vis, c["k"])
    check_topk(t2np(idx)[rows], t2np(cnt)[rows], idx_r, cnt_r, kth, s32, n_vis, c["k"])
    assert B.csa_get_device_error() == 0
