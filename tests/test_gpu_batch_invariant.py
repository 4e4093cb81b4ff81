"""Batch-invariant mode (`csa_set_batch_invariant`): a query's output is bitwise the same
whatever batch it is computed in, and the decode calls reproduce the prefill's outputs
bit for bit.

Without the mode the attention split count follows the batch (one query alone is split
eight ways, forty queries two ways), so partials and their merge order differ.  With
it, the split depends on k + W only.  Every other call is batch-invariant by
construction:
- indexer scores are a fixed per-pair chain, pinned bit-exact in both indexer kernels;
- top-k is exact;
- the decode-time compressor writes the whole-sequence entries.

The outputs computed with the mode on are also checked against the oracle (the
attention tolerance, and for the prefill rows the per-row index-set rule), so the
mode is not only self-consistent but correct.
"""
import numpy as np
import pytest
import torch

import oracle
from compressed_sparse_long_02_b200 import synth
from tests.helpers import assert_close_attn, check_csa_prefill_rows, t2np, to_dev, to_dev_bf16

pytestmark = pytest.mark.gpu


@pytest.fixture
def B(cuda):
    from compressed_sparse_long_02_b200 import binding
    binding.lib()
    binding.csa_set_batch_invariant(True)
    yield binding
    binding.csa_set_batch_invariant(False)


def _host(t: torch.Tensor) -> np.ndarray:
    if t.dtype == torch.bfloat16:
        return t.cpu().view(torch.int16).numpy().view(np.uint16)
    return t.cpu().numpy()


def _bits(x: torch.Tensor) -> torch.Tensor:
    return x.contiguous().view(torch.int16)


def test_sparse_attn_bitwise_across_batches(B, cuda):
    rng = np.random.default_rng(21)
    Nq, E, k, W, Tw, H, D = 40, 4096, 1024, 128, 8192, 64, 512
    ent_h = synth.to_dtype_np(rng.standard_normal((1, E, D)), "bf16")
    win_h = synth.to_dtype_np(rng.standard_normal((1, Tw, D)), "bf16")
    q_h = synth.to_dtype_np(rng.standard_normal((Nq, H, D)) * 0.3, "bf16")
    ent, win, q = to_dev_bf16(ent_h, cuda), to_dev_bf16(win_h, cuda), to_dev_bf16(q_h, cuda)
    pos = np.sort(rng.choice(np.arange(4 * k, Tw), Nq, replace=False)).astype(np.int32)
    n_vis = np.minimum((pos + 1) // 4, E)
    idx = np.stack([np.sort(rng.choice(int(n), k, replace=False)) for n in n_vis]).astype(np.int32)
    pos_d, idx_d = to_dev(pos, cuda), to_dev(idx, cuda)
    cnt_d = to_dev(np.full(Nq, k, np.int32), cuda)
    seq_d = to_dev(np.zeros(Nq, np.int32), cuda)
    zero = to_dev(np.zeros(1, np.int32), cuda)
    full, _ = B.csa_sparse_attn(q, pos_d, seq_d, ent, idx_d, cnt_d, win, zero, W=W)
    ref, _ = oracle.attention(q_h, pos, np.zeros(Nq, np.int32), ent_h, idx, np.full(Nq, k, np.int32), win_h,
                              np.zeros(1, np.int64), W)
    assert_close_attn(t2np(full), ref, "batch-invariant sparse attention vs the oracle")
    for a, b in [(0, 1), (5, 12), (20, 40), (39, 40)]:
        part, _ = B.csa_sparse_attn(q[a:b].contiguous(), pos_d[a:b], seq_d[a:b], ent, idx_d[a:b], cnt_d[a:b], win,
                                    zero, W=W)
        assert torch.equal(_bits(part), _bits(full[a:b])), f"queries {a}..{b - 1} differ from the 40-query batch"
    assert B.csa_get_device_error() == 0


def test_decode_calls_reproduce_prefill_bitwise(B, cuda):
    from compressed_sparse_long_02_b200 import layer
    wl = synth.WORKLOADS["csa_prefill_8k"].replace(T=1024, k=64)
    t = synth.prefill_inputs_torch(wl, cuda)
    r = layer.csa_prefill(wl, t)  # all 1024 rows in one batch
    rows = [64, 300, 777, 1023]
    pos = to_dev(np.array(rows, np.int32), cuda)
    seq = to_dev(np.zeros(len(rows), np.int32), cuda)
    zero = to_dev(np.zeros(1, np.int32), cuda)
    sel = torch.as_tensor(rows, device=cuda)
    scores = B.csa_index_score(r["q_fp4"][sel].contiguous(), r["q_scale"][sel].contiguous(), r["w"][sel].contiguous(),
                               pos, seq, r["k_fp4"], r["k_scale"], r["n_ent"], m=wl.m)
    idx, cnt = B.csa_topk_select(scores, pos, seq, r["n_ent"], k=wl.k, m=wl.m, E_max=r["k_fp4"].shape[1])
    out, _ = B.csa_sparse_attn(r["q"][sel].contiguous(), pos, seq, r["entries"], idx, cnt, r["window"], zero, W=wl.W,
                               prep=layer.q_prep(wl))
    assert torch.equal(idx, r["idx"][sel]) and torch.equal(cnt, r["cnt"][sel])
    assert torch.equal(_bits(out), _bits(r["out"][sel])), "decode calls differ from the prefill's rows"
    # and the prefill computed with the mode on is right on those rows
    host = {k: (_host(v) if k in ("bias", "bias_i") else _host(v)[0]) for k, v in t.items() if k not in ("q", "qi", "w")}
    for k in ("q", "qi", "w"):
        host[k] = _host(t[k][0][sel].contiguous())
    check_csa_prefill_rows(wl, host, r, np.array(rows))
    assert B.csa_get_device_error() == 0
