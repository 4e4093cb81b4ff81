"""GPU tests of the decode-time compressor (`csa_compress_step`) and of HCA attention at a
decode shape.

`csa_compress_step` must write, for each sequence whose newest token completes a group,
exactly the entry `csa_compress` writes for the whole sequence: the same pooling,
RMSNorm, RoPE and MXFP4 key, bit for bit (the two run the same arithmetic in the same
order; `csa_compress` itself is checked against the oracle in test_gpu_kernels.py).
Rows of tokens before position 0 must be ignored, sequences whose group is incomplete
must be left alone, and an entry index past E_max must be skipped and flagged.  The
entries it writes are also checked against the oracle directly: bf16 values within one
bf16 rounding of the float64 pooling, norm and RoPE, and MXFP4 keys equal to the oracle's
encoding except where a float64 value sits on a rounding or scale boundary.
"""
import numpy as np
import pytest
import torch

import oracle
from compressed_sparse_long_02_b200 import synth
from tests.helpers import assert_bf16_rounding, assert_close_attn, fp4_mismatch_justified, t2np, to_dev, to_dev_bf16

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def B(cuda):
    from compressed_sparse_long_02_b200 import binding
    binding.lib()
    return binding


def _dev_act(a, wl, dev):
    return to_dev_bf16(a, dev) if wl.dtype == "bf16" else to_dev(a, dev)


@pytest.mark.parametrize("name,T", [("csa_prefill_8k", 1024), ("tiny", 512), ("hca_prefill_64k", 1024)])
def test_compress_step_matches_whole_sequence(B, cuda, name, T):
    wl = synth.WORKLOADS[name]
    m, S = wl.m, (2 if wl.overlap else 1) * wl.m
    inp = synth.prefill_inputs(wl, T=T)
    E = T // m
    kw = dict(m=m, overlap=wl.overlap, norm=wl.norm, eps=wl.eps, rope_dims=wl.rope_dims, theta=wl.theta)
    kv, z, bias = _dev_act(inp["kv"], wl, cuda), _dev_act(inp["z"], wl, cuda), to_dev(inp["bias"], cuda)
    full = B.csa_compress(kv, z, bias, want_fp4=True, **kw)
    ent_full = full["entries"][0].view(torch.int16)
    fp4_full, sc_full = full["fp4"][0], full["fp4_scale"][0]

    # one row of the call per tested position of the same sequence: group-completing
    # tokens (entries 0, 1, a middle one, the last) and tokens inside a group
    done = [m - 1, 2 * m - 1, m * (E // 2) - 1, m * E - 1]
    inside = [0, m, m * 3 + 1, T - 2] if m > 1 else []
    pos = np.array(done + inside, np.int64)
    Bs = len(pos)
    kv_t, z_t = kv[0], z[0]
    ring_kv = torch.full((Bs, S, wl.C), 1e4, dtype=kv.dtype, device=cuda)  # rows before token 0: must be ignored
    ring_z = torch.full((Bs, S, wl.C), 1e4, dtype=z.dtype, device=cuda)
    for b, p in enumerate(pos):
        lo = p - S + 1
        for s in range(S):
            if lo + s >= 0:
                ring_kv[b, s] = kv_t[lo + s]
                ring_z[b, s] = z_t[lo + s]
    # the oracle's entries and MXFP4 keys of the same sequence (pooled before norm / RoPE)
    ent_ref = oracle.entries_rows(inp["kv"][0], inp["z"][0], inp["bias"], m, wl.overlap, wl.norm, wl.eps,
                                  wl.rope_dims, wl.theta)
    pool_ref = oracle.pool(inp["kv"][0], inp["z"][0], inp["bias"], m, wl.overlap)
    kp_ref, ks_ref = oracle.mxfp4_quantize(pool_ref.astype(np.float32))
    sentinel = 0x4444
    ent = torch.full((Bs, E, wl.C), sentinel, dtype=torch.int16, device=cuda)
    fp4 = torch.full((Bs, E, wl.C // 2), 0x55, dtype=torch.uint8, device=cuda)
    sc = torch.full((Bs, E, wl.C // 32), 0x66, dtype=torch.uint8, device=cuda)
    B.csa_compress_step(ring_kv, ring_z, bias, to_dev(pos.astype(np.int32), cuda), entries=ent.view(torch.bfloat16),
                        fp4=fp4, fp4_scale=sc, **kw)
    torch.cuda.synchronize()
    for b, p in enumerate(pos):
        rows = torch.ones(E, dtype=torch.bool, device=cuda)
        if (p + 1) % m == 0:
            j = (p + 1) // m - 1
            assert torch.equal(ent[b, j], ent_full[j]), f"{name}: entry {j} differs from the whole-sequence one"
            assert torch.equal(fp4[b, j], fp4_full[j]) and torch.equal(sc[b, j], sc_full[j]), f"{name}: fp4 key {j}"
            got = t2np(ent[b, j].view(torch.bfloat16))[None]
            assert_bf16_rounding(got, ent_ref[j][None], f"{name}: entry {j} vs the oracle")
            fp4_mismatch_justified(pool_ref[j][None], t2np(fp4[b, j])[None], t2np(sc[b, j])[None], kp_ref[j][None],
                                   ks_ref[j][None])
            rows[j] = False
        assert bool((ent[b][rows] == sentinel).all()), f"{name}: row {b} wrote outside its entry"
        assert bool((fp4[b][rows] == 0x55).all()) and bool((sc[b][rows] == 0x66).all())
    assert B.csa_get_device_error() == 0


def test_compress_step_entry_past_capacity_flagged(B, cuda):
    wl = synth.WORKLOADS["csa_prefill_8k"]
    m, S = wl.m, 2 * wl.m
    rng = np.random.default_rng(3)
    kv = to_dev_bf16(synth.to_dtype_np(rng.standard_normal((2, S, wl.C)), "bf16"), cuda)
    z = to_dev_bf16(synth.to_dtype_np(rng.standard_normal((2, S, wl.C)), "bf16"), cuda)
    bias = to_dev(np.zeros((S, wl.C), np.float32), cuda)
    E_max = 16
    ent = torch.full((2, E_max, wl.C), 0x4444, dtype=torch.int16, device=cuda)
    pos = to_dev(np.array([m * (E_max + 1) - 1, m * E_max - 1], np.int32), cuda)  # entry 16 (past) and entry 15
    B.csa_compress_step(kv, z, bias, pos, m=m, overlap=True, norm=True, eps=wl.eps, rope_dims=wl.rope_dims,
                        theta=wl.theta, entries=ent.view(torch.bfloat16))
    assert B.csa_get_device_error() == B.DEVERR_INDEX  # read and cleared
    assert bool((ent[0] == 0x4444).all())
    assert not bool((ent[1, E_max - 1] == 0x4444).all())


def test_hca_attn_decode_shape(B, cuda):
    """HCA at decode: one query per sequence at the end of a 64K context (512 entries),
    the 128 most recent raw rows as the window, several sequences of different lengths."""
    rng = np.random.default_rng(8)
    m, W, D, H = 128, 128, 512, 64
    L = np.array([65536, 40000, 129], np.int64)          # context lengths: entries 512, 312, 1
    Bs, E_max = len(L), 512
    ent = synth.to_dtype_np(rng.standard_normal((Bs, E_max, D)), "bf16")
    win = synth.to_dtype_np(rng.standard_normal((Bs, W, D)), "bf16")
    q = synth.to_dtype_np(rng.standard_normal((Bs, H, D)) * 0.3, "bf16")
    pos = L - 1
    seq = np.arange(Bs, dtype=np.int32)
    n_ent = (L // m).astype(np.int32)
    wbase = np.maximum(L - W, 0)
    idx, cnt = oracle.hca_select(pos, seq, n_ent, m)
    ref, lse_ref = oracle.attention(q, pos, seq, ent, idx, cnt, win, wbase, W)
    out, lse = B.hca_attn(to_dev_bf16(q, cuda), to_dev(pos.astype(np.int32), cuda), to_dev(seq, cuda),
                          to_dev_bf16(ent, cuda), to_dev(n_ent, cuda), to_dev_bf16(win, cuda),
                          to_dev(wbase.astype(np.int32), cuda), mprime=m, W=W, want_lse=True)
    assert_close_attn(t2np(out), ref, "hca attention, decode")
    np.testing.assert_allclose(t2np(lse), lse_ref, atol=2e-2)
    assert B.csa_get_device_error() == 0
