"""The C-ABI library builds, loads without a GPU and exports every declared entry point;
host-side validation answers with status codes before any device work."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "csa.h")


@pytest.fixture(scope="module")
def L():
    from compressed_sparse_long_02_b200 import build as bld
    bld.build()
    from compressed_sparse_long_02_b200 import binding
    return binding.lib()


def declared_functions():
    text = open(HEADER).read()
    return re.findall(r"^CSA_API\s+[\w\s\*]+?\b(\w+)\(", text, flags=re.M)


def test_header_declares_the_boundary():
    names = set(declared_functions())
    for fn in ("csa_compress", "csa_index_topk", "csa_sparse_attn", "hca_attn", "csa_quantize_mxfp4",
               "csa_norm_rope", "csa_get_device_error", "csa_status_string"):
        assert fn in names


def test_library_exports_every_declared_symbol(L):
    for fn in declared_functions():
        assert hasattr(L, fn), f"{fn} declared in csa.h but not exported"


def test_status_strings(L):
    L.csa_status_string.restype = ctypes.c_char_p
    assert L.csa_status_string(0) == b"ok"
    assert b"workspace" in L.csa_status_string(4)
    assert L.csa_status_string(99) == b"unknown status"


def test_validation_without_device(L):
    from compressed_sparse_long_02_b200 import binding as B
    P = ctypes.c_void_p
    # null configuration
    assert L.csa_compress(None, 1, 8, P(16), P(16), P(16), None, 2, None, None, None, None) == 1
    cfg = B._PoolCfg(4, 1, 96, 0, 1e-6, 0, 1e4, 0)  # C = 96 is not supported
    assert L.csa_compress(ctypes.byref(cfg), 1, 8, P(16), P(16), P(16), None, 2, None, None, None, None) == 3
    cfg = B._PoolCfg(4, 1, 128, 0, 1e-6, 3, 1e4, 0)  # odd rope dims
    assert L.csa_compress(ctypes.byref(cfg), 1, 8, P(16), P(16), P(16), None, 2, None, None, None, None) == 1
    cfg = B._PoolCfg(4, 1, 128, 0, 1e-6, 0, 1e4, 0)  # misaligned input pointer
    assert L.csa_compress(ctypes.byref(cfg), 1, 8, P(17), P(16), P(16), None, 2, None, None, None, None) == 2
    # decode-time compressor: no positions, misaligned rows, unsupported channels, nothing to do
    L.csa_compress_step.argtypes = [ctypes.POINTER(B._PoolCfg), ctypes.c_int, P, P, P, P, P, ctypes.c_int, P, P, P]
    cfg = B._PoolCfg(4, 1, 128, 0, 1e-6, 0, 1e4, 0)
    assert L.csa_compress_step(ctypes.byref(cfg), 2, None, P(16), P(16), P(16), P(16), 8, None, None, None) == 1
    assert L.csa_compress_step(ctypes.byref(cfg), 2, P(16), P(24), P(16), P(16), P(16), 8, None, None, None) == 2
    assert L.csa_compress_step(ctypes.byref(cfg), 2, P(16), P(16), P(16), P(16), P(16), 0, None, None, None) == 1
    assert L.csa_compress_step(ctypes.byref(cfg), 0, None, None, None, None, None, 8, None, None, None) == 0
    cfg = B._PoolCfg(4, 1, 96, 0, 1e-6, 0, 1e4, 0)
    assert L.csa_compress_step(ctypes.byref(cfg), 2, P(16), P(16), P(16), P(16), P(16), 8, None, None, None) == 3
    # quantiser: cols not a multiple of 32
    assert L.csa_quantize_mxfp4(P(16), 0, 4, 48, P(16), P(16), None) == 1
    # indexer: unsupported head dim, E_max not a multiple of 8, workspace too small
    assert L.csa_index_topk(1, 4, 96, 8, 4, *([P(16)] * 5), 1, 64, *([P(16)] * 5), None, P(16), 1 << 30,
                            None) == 3
    assert L.csa_index_topk(1, 4, 64, 8, 4, *([P(16)] * 5), 1, 60, *([P(16)] * 5), None, P(16), 1 << 30,
                            None) == 3
    assert L.csa_index_topk(1, 4, 64, 8, 4, *([P(16)] * 5), 1, 64, *([P(16)] * 5), None, P(16), 16, None) == 4
    # attention: only H = 64, D = 512
    assert L.csa_sparse_attn(1, 32, 512, 8, 128, ctypes.c_float(0.04), *([P(16)] * 3), 1, 64, P(16), P(16), P(16),
                             128, P(16), P(16), P(16), None, P(16), 1 << 30, None) == 3
    assert L.hca_attn(1, 64, 512, 0, 128, ctypes.c_float(0.04), *([P(16)] * 3), 1, 64, P(16), P(16), 128, P(16),
                      P(16), P(16), None, P(16), 1 << 30, None) == 1


def test_workspace_sizes(L):
    from compressed_sparse_long_02_b200 import binding as B
    assert B.csa_index_topk_workspace(32, 32768, 1024) >= 32 * 32768 * 4
    # one query per SM or more: no split, no partials
    assert B.csa_sparse_attn_workspace(8192, 64, 512, 512, 128) <= 256
    # decode: split partials of fp32 [splits, 64, 512] per query
    assert B.csa_sparse_attn_workspace(32, 64, 512, 1024, 128) >= 32 * 2 * 64 * 512 * 4


def test_batch_invariant_split_rule(L):
    """With the batch-invariant switch on, the attention split of a query depends on
    k + W only: the workspace per query (its partials) is the same for every batch size,
    the fewest power-of-two splits of at most 512 rows (at most 8).  Off, few queries are
    split more ways than many."""
    from compressed_sparse_long_02_b200 import binding as B

    def per_query_splits(Nq, k, W):
        ws = B.csa_sparse_attn_workspace(Nq, 64, 512, k, W)
        return 0 if ws <= 256 else round((ws - 512) / (Nq * 64 * (512 * 4 + 8)))

    try:
        B.csa_set_batch_invariant(True)
        for k, W, want in [(64, 128, 0), (448, 64, 0), (512, 128, 2), (1024, 128, 4), (2048, 128, 8),
                           (262144, 128, 8)]:
            got = {per_query_splits(Nq, k, W) for Nq in (1, 3, 32, 148, 8192)}
            assert got == {want}, f"k={k}, W={W}: splits {got}, expected {want} for every batch"
    finally:
        B.csa_set_batch_invariant(False)
    assert per_query_splits(1, 1024, 128) == 8 and per_query_splits(32, 1024, 128) == 4
    assert per_query_splits(8192, 1024, 128) == 0


def test_static_indexer_size_limit_boundary(L):
    """csa_index_topk_static holds Nq * round_up(E_max, 4) <= 2^21 scores.  The size check runs
    before any device work, so null pointers reach it: a call exactly at the limit passes it
    (and then stops at the null pointers), one row of 8 entries more is rejected as too large
    for the scratch, and E_max not a multiple of 8 is unsupported."""
    P, I = ctypes.c_void_p, ctypes.c_int
    L.csa_index_topk_static.argtypes = [I, I, I, I, I, P, P, P, P, P, I, I, P, P, P, P, P, P]
    L.csa_index_topk_static.restype = I

    def call(Nq, E_max):
        return L.csa_index_topk_static(Nq, 64, 128, 8, 4, *([None] * 5), 1, E_max, *([None] * 5), None)

    assert call(32, 65536) == 1          # 32 x 65536 = 2^21: within the limit, then INVALID_ARG
    assert call(32, 65544) == 4          # one more multiple of 8: CSA_ERR_WORKSPACE
    assert call(1, 1 << 21) == 1
    assert call(1, (1 << 21) + 8) == 4
    assert call(32, 65540) == 3          # E_max % 8 != 0: CSA_ERR_UNSUPPORTED


def test_index_fusion_switch_plan(L):
    """csa_index_topk's launch plan: two kernels by default; with the fusion switch on, one
    fused kernel for the 128K decode shape (32 queries, 32768 entries) and still two for
    rows too long for a cluster's slices (4 queries of 262144 entries)."""
    from compressed_sparse_long_02_b200 import binding as B
    assert B.csa_index_topk_launches(32, 64, 128, 32768, 1024) == 2
    try:
        B.csa_set_index_fusion(True)
        assert B.csa_index_topk_launches(32, 64, 128, 32768, 1024) == 1
        assert B.csa_index_topk_launches(4, 64, 128, 262144, 1024) == 2
        assert B.csa_index_topk_launches(32, 32, 128, 32768, 1024) == 2   # other head counts: not fused
        assert B.csa_index_topk_launches(0, 64, 128, 32768, 1024) == 0
    finally:
        B.csa_set_index_fusion(False)


def test_validation_of_the_newer_calls(L):
    """The multi-query indexer, the attention calls that prepare raw queries, and the grouped
    output projection reject what they do not support with a status, before any device
    work (null pointers past the checks stop at INVALID_ARG, never at a launch)."""
    from compressed_sparse_long_02_b200 import binding as B
    P = ctypes.c_void_p
    x = P(16)
    ws = 1 << 30

    def grouped(q_group, Nq, Hi, Di, E_max=64):
        return L.csa_index_topk_grouped(q_group, Nq, Hi, Di, 8, 4, x, x, x, x, x, 1, E_max, x, x, x, x, x, None, x, ws,
                                        None)

    assert grouped(3, 2, 64, 128) == 3     # only one or two query rows per group
    assert grouped(2, 2, 32, 128) == 3     # groups of two need 64 heads of 128 dims
    assert grouped(2, 2, 64, 64) == 3
    assert grouped(2, 2, 64, 128, E_max=60) == 3
    assert grouped(2, 0, 64, 128) == 0     # nothing to do
    assert L.csa_index_topk_grouped(2, 2, 64, 128, 8, 4, *([None] * 5), 1, 64, *([None] * 5), None, None, ws,
                                    None) == 1

    def attn_ex(rope_dims, eps=1e-6, theta=1e4, norm=1):
        prep = ctypes.byref(B._QPrep(norm, eps, rope_dims, theta))
        return L.csa_sparse_attn_ex(prep, 1, 64, 512, 8, 128, ctypes.c_float(0.04), x, x, x, 1, 64, x, x, x, 128, x, x,
                                    x, None, x, ws, None)

    for rd in (66, 3, -2):                 # RoPE on 0..64 even channels only
        assert attn_ex(rd) == 3
    assert attn_ex(64, eps=-1.0) == 1      # a negative epsilon
    assert attn_ex(64, theta=0.0) == 1     # RoPE without a base
    prep = ctypes.byref(B._QPrep(1, 1e-6, 66, 1e4))
    assert L.hca_attn_ex(prep, 1, 64, 512, 128, 128, ctypes.c_float(0.04), x, x, x, 1, 64, x, x, 128, x, x, x, None,
                         x, ws, None) == 3
    # grouped output projection: heads split evenly over groups, tile-friendly sizes
    assert L.csa_grouped_out_proj(16, 64, 512, 7, 1024, 4096, x, x, x, x, x, None) == 1
    assert L.csa_grouped_out_proj(16, 64, 512, 8, 1000, 4096, x, x, x, x, x, None) == 3
    assert L.csa_grouped_out_proj(16, 64, 512, 8, 1024, 4000, x, x, x, x, x, None) == 3
