"""Failure detection on the GPU without a fault: the bounded pipeline waits.

Every wait of a kernel in the library on a pipeline barrier gives up after a bounded
number of SM cycles, records CSA_DEVERR_TIMEOUT in the device error word and releases
the kernel's other roles through a shared abort flag.  `csa_selftest_bounded_wait`
runs those waits against barriers that nothing ever completes: the test checks that the
first warp waited the full limit and timed out, that the second warp was released early
by the abort flag, that the host reads the timeout, and that the context still works.
No trap, no fault, no endless loop: the kernel ends by itself after about two seconds.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from tests.helpers import t2np, to_dev

pytestmark = pytest.mark.gpu

WAIT_LIMIT_CYCLES = 4_000_000_000  # the library's bound on one wait


@pytest.mark.parametrize("sleeping", [0, 1])
def test_bounded_wait_times_out_and_releases_the_other_roles(cuda, sleeping):
    from compressed_sparse_long_02_b200 import binding as B
    L = B.lib()
    L.csa_selftest_bounded_wait.argtypes = [ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p]
    L.csa_selftest_bounded_wait.restype = ctypes.c_int
    assert B.csa_get_device_error() == 0
    out = torch.full((4,), -1, dtype=torch.int64, device=cuda)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    assert L.csa_selftest_bounded_wait(sleeping, ctypes.c_void_p(out.data_ptr()), stream) == 0
    assert B.csa_get_device_error() == B.DEVERR_TIMEOUT      # read and cleared
    ok0, waited0, ok1, waited1 = out.cpu().tolist()
    assert ok0 == 0 and ok1 == 0, "a wait on a barrier nothing completes reported success"
    assert waited0 > WAIT_LIMIT_CYCLES, "the first role gave up before the limit"
    assert waited1 < WAIT_LIMIT_CYCLES, "the second role was not released by the abort flag"
    # the context is still usable: an ordinary call afterwards is right and raises nothing
    rng = np.random.default_rng(11)
    x = rng.standard_normal((256, 128)).astype(np.float32)
    pk, sc = B.csa_quantize_mxfp4(to_dev(x, cuda))
    rp, rs = oracle.mxfp4_quantize(x)
    assert np.array_equal(t2np(pk), rp) and np.array_equal(t2np(sc), rs)
    assert B.csa_get_device_error() == 0
