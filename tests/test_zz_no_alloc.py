"""csa_index_topk_static -- the indexer + top-k for callers that cannot allocate device
memory (its score scratch is a fixed array inside the library) -- must give the same
indices and counts as csa_index_topk with a caller workspace, call after call.

Called straight through the C ABI (ctypes on libcsa.so).  Collected last so that a run
that stops at the first failure has already run every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

CSA_ERR_WORKSPACE = 4


@pytest.fixture(scope="module")
def lib(cuda):
    from compressed_sparse_long_02_b200 import binding
    L = binding.lib()
    P, I = ctypes.c_void_p, ctypes.c_int
    L.csa_index_topk_static.argtypes = [I, I, I, I, I, P, P, P, P, P, I, I, P, P, P, P, P, P]
    L.csa_index_topk_static.restype = I
    return L


def _case(seed, dev, B=4, E=4096, Hi=64, Di=128):
    from compressed_sparse_long_02_b200 import binding as Bd
    g = torch.Generator(device=dev)
    g.manual_seed(seed)
    keys = torch.randn((B, E, Di), generator=g, device=dev)
    keys[:, ::97] += 2.0
    qi = torch.randn((B, Hi, Di), generator=g, device=dev)
    kp, ks = Bd.csa_quantize_mxfp4(keys)
    qp, qs = Bd.csa_quantize_mxfp4(qi)
    w = torch.rand((B, Hi), generator=g, device=dev)
    n_ent = torch.tensor([E, E - 1000, E - 8, 777], dtype=torch.int32, device=dev)[:B]
    pos = (n_ent * 4 - 1).to(torch.int32)
    seq = torch.arange(B, dtype=torch.int32, device=dev)
    return dict(kp=kp, ks=ks, qp=qp, qs=qs, w=w, n_ent=n_ent, pos=pos, seq=seq, B=B, E=E, Hi=Hi, Di=Di)


def _static_call(L, c, k, idx, cnt):
    p = lambda t: ctypes.c_void_p(t.data_ptr())
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return L.csa_index_topk_static(c["B"], c["Hi"], c["Di"], k, 4, p(c["qp"]), p(c["qs"]), p(c["w"]), p(c["pos"]),
                                   p(c["seq"]), c["B"], c["E"], p(c["kp"]), p(c["ks"]), p(c["n_ent"]), p(idx), p(cnt),
                                   stream)


def test_static_scratch_matches_workspace_version_twice(lib, cuda):
    from compressed_sparse_long_02_b200 import binding as Bd
    k = 512
    for seed in (1, 2):  # two calls in a row share the library's scratch array
        c = _case(seed, cuda)
        idx_ref, cnt_ref, _ = Bd.csa_index_topk(c["qp"], c["qs"], c["w"], c["pos"], c["seq"], c["kp"], c["ks"],
                                                c["n_ent"], k=k, m=4)
        idx = torch.full((c["B"], k), -7, dtype=torch.int32, device=cuda)
        cnt = torch.full((c["B"],), -7, dtype=torch.int32, device=cuda)
        assert _static_call(lib, c, k, idx, cnt) == 0
        torch.cuda.synchronize()
        assert torch.equal(cnt, cnt_ref) and torch.equal(idx, idx_ref)
        assert Bd.csa_get_device_error() == 0


def test_static_scratch_rejects_oversize(lib, cuda):
    c = _case(3, cuda, B=4, E=4096)
    c["E"] = 1 << 20          # 4 x 2^20 scores > the 2^21 the array holds: rejected before any work
    idx = torch.empty((4, 8), dtype=torch.int32, device=cuda)
    cnt = torch.empty((4,), dtype=torch.int32, device=cuda)
    assert _static_call(lib, c, 8, idx, cnt) == CSA_ERR_WORKSPACE
