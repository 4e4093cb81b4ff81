"""GPU parity of the grouped output projection (`csa_grouped_out_proj`) against the oracle.

The oracle keeps the intermediate in float64; the GPU accumulates in float32 and rounds
the intermediate z to bf16 before the second product.  z must be within one bf16 rounding
of the oracle's; y, whose error also carries z's rounding, within the attention tolerance
(relative L2 1e-2, max-abs 3e-2).  Small shapes are compared in full; the full-size shape
(8192 tokens, 64 heads of 512, 8 groups, R = 1024, d_model = 4096) in the benchmark's
launch configuration on sampled rows, including the first and last rows of ragged tails.
"""
import numpy as np
import pytest
import torch

import oracle
from compressed_sparse_long_02_b200 import synth
from tests.helpers import assert_bf16_rounding, assert_close_attn, t2np, to_dev_bf16

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def B(cuda):
    from compressed_sparse_long_02_b200 import binding
    binding.lib()
    return binding


def _host(t):
    return t.cpu().view(torch.int16).numpy().view(np.uint16)


@pytest.mark.parametrize("T", [37, 128, 300])
def test_grouped_out_proj_small_full_compare(B, cuda, T):
    ps = synth.PROJ["tiny"]
    d = synth.proj_inputs(ps, T=T)
    z, y = B.csa_grouped_out_proj(to_dev_bf16(d["o"], cuda), to_dev_bf16(d["A"], cuda), to_dev_bf16(d["Bm"], cuda))
    z_ref, y_ref = oracle.grouped_out_proj(d["o"], d["A"], d["Bm"], ps.G)
    assert_bf16_rounding(t2np(z), z_ref, "grouped projection z", atol=1e-4)
    assert_close_attn(t2np(y), y_ref, "grouped projection y")
    assert B.csa_get_device_error() == 0


@pytest.mark.parametrize("T", [8192, 1000])
def test_grouped_out_proj_full_size_sampled(B, cuda, T):
    ps = synth.PROJ["csa_prefill_8k"]
    d = synth.proj_inputs_torch(ps, cuda, T=T)
    z, y = B.csa_grouped_out_proj(d["o"], d["A"], d["Bm"])
    torch.cuda.synchronize()
    rng = np.random.default_rng(T)
    rows = np.unique(np.concatenate([[0, 1, 127, 128, T - 129, T - 1], rng.choice(T, 10, replace=False)]))
    rows = rows[(rows >= 0) & (rows < T)]
    sel = torch.as_tensor(rows, device=cuda)
    o_h = _host(d["o"][sel].contiguous())
    z_ref, y_ref = oracle.grouped_out_proj(o_h, _host(d["A"]), _host(d["Bm"]), ps.G)
    assert_bf16_rounding(t2np(z[sel]), z_ref, "grouped projection z (full size)", atol=1e-4)
    assert_close_attn(t2np(y[sel]), y_ref, "grouped projection y (full size)")
    assert B.csa_get_device_error() == 0


def test_grouped_out_proj_empty_and_unsupported(B, cuda):
    ps = synth.PROJ["tiny"]
    e = torch.empty((0, ps.H, ps.D), dtype=torch.bfloat16, device=cuda)
    A = torch.zeros((ps.G, ps.R, (ps.H // ps.G) * ps.D), dtype=torch.bfloat16, device=cuda)
    Bm = torch.zeros((ps.d_model, ps.G * ps.R), dtype=torch.bfloat16, device=cuda)
    z, y = B.csa_grouped_out_proj(e, A, Bm)
    assert z.shape == (0, ps.G * ps.R) and y.shape == (0, ps.d_model)
    with pytest.raises(B.CsaError) as ex:  # R = 100 is not a multiple of 256
        B.csa_grouped_out_proj(torch.zeros((4, ps.H, ps.D), dtype=torch.bfloat16, device=cuda),
                               torch.zeros((ps.G, 100, (ps.H // ps.G) * ps.D), dtype=torch.bfloat16, device=cuda),
                               torch.zeros((ps.d_model, ps.G * 100), dtype=torch.bfloat16, device=cuda))
    assert ex.value.status == 3
    assert B.csa_get_device_error() == 0
