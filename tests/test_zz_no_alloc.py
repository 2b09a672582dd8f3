"""The allocation-free quantiser entry point, through the C ABI.

nvfp4_quantize_bf16_noalloc serves callers that may not allocate device memory
(for example code running after an inference runtime has given all device
memory to its own pool, or a plugin step that must not allocate), by keeping
its scratch in a static device array inside the library.  Its results must be
the same bytes as nvfp4_quantize_bf16 with a caller workspace, call after call:
the second call here has a much smaller amax than the first, so a scratch word
left over from the first call would change every scale of the second.

This file is collected last, so that a run stopping at the first failure has
already run every other test; it also passes on its own in a fresh process
(the first call on the device sets up the array's address)."""
import ctypes

import numpy as np
import pytest
import torch

import block_scaled_precision_nvfp4_b200 as nv

pytestmark = pytest.mark.gpu


def _outputs(rows, K):
    # zero-filled, so that bytes neither call writes compare equal
    return (torch.zeros((rows, K // 2), dtype=torch.uint8, device="cuda"),
            torch.zeros((rows, K // 16), dtype=torch.uint8, device="cuda"),
            torch.zeros(nv.nvfp4_scale_layout_bytes(rows, K), dtype=torch.uint8, device="cuda"),
            torch.zeros(4, dtype=torch.float32, device="cuda"))


def _with_workspace(lib, x, out):
    rows, K = x.shape
    ws = torch.empty(int(lib.nvfp4_quantize_workspace_bytes()), dtype=torch.uint8, device="cuda")
    codes, scales, packed, g = out
    rc = lib.nvfp4_quantize_bf16(x.data_ptr(), rows, K, codes.data_ptr(), scales.data_ptr(),
                                 packed.data_ptr(), g.data_ptr(), ws.data_ptr(),
                                 ws.numel(), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == 0, lib.nvfp4_last_error()


def _no_alloc(lib, x, out):
    rows, K = x.shape
    codes, scales, packed, g = out
    rc = lib.nvfp4_quantize_bf16_noalloc(x.data_ptr(), rows, K, codes.data_ptr(), scales.data_ptr(),
                                         packed.data_ptr(), g.data_ptr(),
                                         ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == 0, lib.nvfp4_last_error()


def test_no_alloc_entry_point_matches_the_workspace_one_on_two_calls():
    lib = nv.load_library()
    rng = np.random.default_rng(11)
    shapes_scales = [((300, 1024), 50.0), ((130, 4160), 0.02)]   # the second amax is far smaller
    for (rows, K), scale in shapes_scales:
        x = (torch.from_numpy(rng.standard_normal((rows, K)).astype(np.float32) * np.float32(scale))
             .to(torch.bfloat16).cuda())
        ref, got = _outputs(rows, K), _outputs(rows, K)
        _with_workspace(lib, x, ref)
        _no_alloc(lib, x, got)
        torch.cuda.synchronize()
        assert lib.nvfp4_check_device_error(None) == 0
        for a, b in zip(ref, got):
            assert torch.equal(a, b)   # codes, scales, packed scales and g: exact
        assert float(got[3][0]) > 0
