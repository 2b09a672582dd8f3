"""A bounded device wait that runs out, on the GPU, without a fault.

The product library's kernels bound every pipeline wait (2 s of %globaltimer) and,
when one expires, record the role in a device error word, let their in-flight copies
land, drain their tensor-core work, free their tensor memory and return.  This test
drives that path for real: a test-only build of the same sources (NVFP4_WAIT_TEST)
lets it shorten the limit to 2 ms and make the single-SM W4A4 kernel's MMA role wait
on a barrier nothing arrives on.  The kernel must return, report
NVFP4_ERR_DEVICE_TIMEOUT once (the word is cleared by the read), write nothing, and
leave the context usable: the next call of the same library, and one of the product
library, match the oracle."""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import block_scaled_precision_nvfp4_b200 as nv
from block_scaled_precision_nvfp4_b200 import _build
from block_scaled_precision_nvfp4_b200 import workloads as wl

from parity import bf16_to_f64, check

pytestmark = pytest.mark.gpu


def _wait_test_lib():
    lib = ctypes.CDLL(_build.build_wait_test())
    P, I, F = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
    lib.gemm_nvfp4_w4a4.restype = I
    lib.gemm_nvfp4_w4a4.argtypes = [P, P, F, P, P, F, P, I, I, I, P]
    lib.nvfp4_check_device_error.restype = I
    lib.nvfp4_check_device_error.argtypes = [P]
    lib.nvfp4_test_set_wait.restype = I
    lib.nvfp4_test_set_wait.argtypes = [ctypes.c_uint64, I]
    return lib


def test_product_library_has_no_test_switch():
    with pytest.raises(AttributeError):
        getattr(nv.load_library(), "nvfp4_test_set_wait")


def test_expired_wait_is_reported_and_the_context_stays_usable():
    lib = _wait_test_lib()
    t = wl.tiny_w4a4(0)
    d = lambda x: torch.from_numpy(np.ascontiguousarray(x)).cuda()
    A, sA, W, sW = d(t.A.codes), d(t.A.scales), d(t.W.codes), d(t.W.scales)
    stream = torch.cuda.current_stream().cuda_stream
    ref = oracle.gemm_w4a4(t.A.codes, t.A.scales, 1.0, t.W.codes, t.W.scales, 1.0, t.M, t.N, t.K)

    def call(y):
        return lib.gemm_nvfp4_w4a4(A.data_ptr(), sA.data_ptr(), 1.0, W.data_ptr(), sW.data_ptr(),
                                   1.0, y.data_ptr(), t.M, t.N, t.K, stream)

    assert lib.nvfp4_check_device_error(stream) == nv.Status.OK
    try:
        assert lib.nvfp4_test_set_wait(2_000_000, 1) == nv.Status.OK      # 2 ms, stall on
        y = torch.full((t.M, t.N), 7.0, dtype=torch.bfloat16, device="cuda")
        assert call(y) == nv.Status.OK                                     # enqueued
        assert lib.nvfp4_check_device_error(stream) == nv.Status.DEVICE_TIMEOUT
        assert lib.nvfp4_check_device_error(stream) == nv.Status.OK        # read clears it
        assert bool((y.float() == 7.0).all()), "the stalled kernel wrote output"
    finally:
        assert lib.nvfp4_test_set_wait(2_000_000_000, 0) == nv.Status.OK
    y = torch.empty((t.M, t.N), dtype=torch.bfloat16, device="cuda")
    assert call(y) == nv.Status.OK
    assert lib.nvfp4_check_device_error(stream) == nv.Status.OK
    check(bf16_to_f64(y), ref, "same library after the timeout")
    y2 = nv.gemm_nvfp4_w4a4(A, sA, 1.0, W, sW, 1.0)
    torch.cuda.synchronize()
    nv.nvfp4_check_device_error()
    check(bf16_to_f64(y2), ref, "product library after the timeout")
