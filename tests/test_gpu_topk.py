"""GPU parity of the top-k selection (`csa_topk_select`) against the oracle's top-k.

The same float32 score rows go to both sides, so index sets must be identical (no tie
exemption: ties resolve to the lowest index on both sides).  Cases span every kernel
variant -- rows held in the registers of a thread-block cluster of 2, 4, 8 or 16 CTAs
(few rows: 8, 16 or 32 entries per thread), of one CTA (many rows: 16 / 32 entries per
thread, rows up to 2048, 8192 and 32768 entries), and rows staged in shared memory
(longer rows, read from global memory beyond its capacity) -- with ragged visible
counts, rows at or below k, exact ties across warp and CTA boundaries, -0/+0, negative
scores, an outlier that crowds the threshold bin (the digit-pass path), and a score
stride wider than E_max.
"""
import numpy as np
import pytest

import oracle
from tests.helpers import t2np, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def B(cuda):
    from compressed_sparse_long_02_b200 import binding
    binding.lib()
    return binding


def _rows(kind: str, Nq: int, E: int, rng) -> np.ndarray:
    if kind == "normal":
        return rng.standard_normal((Nq, E)).astype(np.float32)
    if kind == "positive":        # sums of ReLU terms: positive, concentrated
        return (rng.gamma(20.0, 1.0, (Nq, E))).astype(np.float32)
    if kind == "levels":          # a few distinct values: huge tie groups at the threshold
        return rng.integers(0, 7, (Nq, E)).astype(np.float32)
    if kind == "equal":           # every score identical
        return np.full((Nq, E), 1.5, np.float32)
    if kind == "signed_zero":     # only -0, +0 and a handful of positives
        s = np.where(rng.random((Nq, E)) < 0.5, np.float32(-0.0), np.float32(0.0)).astype(np.float32)
        s[:, ::97] = 1.0
        return s
    if kind == "outlier":         # one huge score squeezes the rest into the lowest bins
        s = rng.standard_normal((Nq, E)).astype(np.float32)
        s[:, E // 3] = 1e30
        return s
    raise ValueError(kind)


def _run(B, cuda, scores: np.ndarray, n_vis: np.ndarray, k: int, E_max: int, m: int = 4):
    Nq = scores.shape[0]
    pos = (n_vis.astype(np.int64) * m - 1).astype(np.int32)     # visible count = n_vis exactly
    seq = np.arange(Nq, dtype=np.int32)
    n_ent = np.full(Nq, E_max, np.int32)
    idx, cnt = B.csa_topk_select(to_dev(scores, cuda), to_dev(pos, cuda), to_dev(seq, cuda), to_dev(n_ent, cuda),
                                 k=k, m=m, E_max=E_max)
    idx_r, cnt_r, _ = oracle.topk(scores, n_vis, k)
    np.testing.assert_array_equal(t2np(cnt), cnt_r)
    np.testing.assert_array_equal(t2np(idx), idx_r)
    assert B.csa_get_device_error() == 0


@pytest.mark.parametrize("E,k", [(2000, 512), (8000, 1024), (9000, 1024), (40000, 1024)])
@pytest.mark.parametrize("kind", ["normal", "positive", "levels", "outlier"])
def test_topk_row_lengths(B, cuda, E, k, kind):
    rng = np.random.default_rng(100 + E)
    Nq = 40
    s = _rows(kind, Nq, E, rng)
    n_vis = rng.integers(0, E + 1, Nq).astype(np.int32)
    n_vis[:6] = [E, k, k + 1, 0, 1, E - 1]
    _run(B, cuda, s, n_vis, k, E)


@pytest.mark.parametrize("E,k", [(2000, 256), (8000, 1024), (30000, 1024)])
@pytest.mark.parametrize("kind", ["normal", "levels", "outlier"])
def test_topk_many_rows(B, cuda, E, k, kind):
    """160 rows: more rows than a wave of clusters, so one CTA per row holds it."""
    rng = np.random.default_rng(300 + E)
    Nq = 160
    s = _rows(kind, Nq, E, rng)
    n_vis = rng.integers(0, E + 1, Nq).astype(np.int32)
    n_vis[:5] = [E, k, k + 1, 0, E - 1]
    _run(B, cuda, s, n_vis, k, E)


@pytest.mark.parametrize("Nq,E", [(4, 262144), (8, 100000), (16, 65536)])
def test_topk_cluster_of_eight(B, cuda, Nq, E):
    """Few long rows: eight CTAs per row, up to 32 entries per thread (the 1M-token decode shape)."""
    rng = np.random.default_rng(400 + Nq)
    k = 1024
    s = _rows("normal", Nq, E, rng)
    s[0, E // 8 - 700:E // 8 + 700] = 6.5     # a tie group across the first CTA boundary
    n_vis = np.full(Nq, E, np.int32)
    n_vis[-1] = E - 12345
    _run(B, cuda, s, n_vis, k, E)


@pytest.mark.parametrize("Nq,E", [(4, 262144), (9, 150000)])
@pytest.mark.parametrize("kind", ["normal", "levels", "outlier", "equal"])
def test_topk_cluster_of_sixteen(B, cuda, Nq, E, kind):
    """Rows beyond 131072 entries with at most 9 rows: a non-portable cluster of 16 CTAs per
    row, 16 entries per thread, where 16-CTA clusters can be resident (else 8 CTAs of 32);
    a tie group across the first CTA boundary, ragged visible counts."""
    rng = np.random.default_rng(500 + Nq + len(kind))
    k = 1024
    s = _rows(kind, Nq, E, rng)
    if kind == "normal":
        s[0, E // 16 - 900:E // 16 + 900] = 6.5
    n_vis = np.full(Nq, E, np.int32)
    n_vis[-1] = E - 54321
    n_vis[1] = k + 1
    _run(B, cuda, s, n_vis, k, E)


@pytest.mark.parametrize("kind", ["normal", "equal", "signed_zero", "outlier", "levels"])
def test_topk_decode_shape(B, cuda, kind):
    """32 rows of 32768 scores, k = 1024: the 128K-context decode selection."""
    rng = np.random.default_rng(7)
    E, k = 32768, 1024
    s = _rows(kind, 32, E, rng)
    n_vis = np.full(32, E, np.int32)
    n_vis[1:5] = [E - 1, k + 3, 8191, 20001]
    _run(B, cuda, s, n_vis, k, E)


def test_topk_slices_beyond_shared_memory(B, cuda):
    """2 rows of 500,000 scores: longer than shared memory holds, read from global memory."""
    rng = np.random.default_rng(11)
    E, k = 500_000, 1024
    s = _rows("normal", 2, E, rng)
    s[1, 123_456:123_456 + 3000] = 9.0          # a tie group straddling the threshold
    _run(B, cuda, s, np.array([E, E - 17], np.int32), k, E)


def test_topk_wide_stride(B, cuda):
    """Score rows wider than E_max: only the first n_vis of each row are read."""
    rng = np.random.default_rng(12)
    E_max, stride, k = 16384, 16400, 512
    s = rng.standard_normal((8, stride)).astype(np.float32)
    s[:, E_max:] = 1e9                           # beyond E_max: must never be selected
    n_vis = np.array([E_max, 600, 512, 513, 9000, 16383, 1, 12345], np.int32)
    Nq = s.shape[0]
    pos = (n_vis.astype(np.int64) * 4 - 1).astype(np.int32)
    idx, cnt = B.csa_topk_select(to_dev(s, cuda), to_dev(pos, cuda), to_dev(np.arange(Nq, dtype=np.int32), cuda),
                                 to_dev(np.full(Nq, E_max, np.int32), cuda), k=k, m=4, E_max=E_max)
    idx_r, cnt_r, _ = oracle.topk(np.ascontiguousarray(s[:, :E_max]), n_vis, k)
    np.testing.assert_array_equal(t2np(cnt), cnt_r)
    np.testing.assert_array_equal(t2np(idx), idx_r)


def test_topk_bad_sequence_rows_empty(B, cuda):
    """A row whose sequence id is out of range selects nothing (count 0, all -1)."""
    E, k = 10000, 64
    s = np.random.default_rng(13).standard_normal((4, E)).astype(np.float32)
    pos = np.full(4, 4 * E - 1, np.int32)
    seq = np.array([0, -1, 7, 1], np.int32)      # B = 2: rows 1 and 2 are invalid
    idx, cnt = B.csa_topk_select(to_dev(s, cuda), to_dev(pos, cuda), to_dev(seq, cuda),
                                 to_dev(np.full(2, E, np.int32), cuda), k=k, m=4, E_max=E)
    cnt, idx = t2np(cnt), t2np(idx)
    assert cnt.tolist() == [k, 0, 0, k]
    assert np.all(idx[1:3] == -1)
    idx_r, _, _ = oracle.topk(s[[0, 3]], np.array([E, E], np.int32), k)
    np.testing.assert_array_equal(idx[[0, 3]], idx_r)
