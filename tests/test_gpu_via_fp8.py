"""The exact E2M1 -> E4M3 FP8 path: parity with the FP64 oracle (W4A4 definition), through the C ABI."""
import numpy as np
import pytest
import torch

import oracle
import block_scaled_precision_nvfp4_b200 as nv
from block_scaled_precision_nvfp4_b200 import workloads as wl

from parity import bf16_to_f64, check

pytestmark = pytest.mark.gpu


def _dev(x):
    return torch.from_numpy(np.ascontiguousarray(x)).cuda()


def _run(A, W, gA, gW, fn=None):
    fn = fn or nv.gemm_nvfp4_via_fp8
    y = fn(_dev(A.codes), _dev(A.scales), gA, _dev(W.codes), _dev(W.scales), gW)
    torch.cuda.synchronize()
    nv.nvfp4_check_device_error()
    return y


def test_tiny_workload():
    t = wl.tiny_w4a4(0)
    y = _run(t.A, t.W, 1.0, 1.0)
    ref = oracle.gemm_w4a4(t.A.codes, t.A.scales, 1.0, t.W.codes, t.W.scales, 1.0, t.M, t.N, t.K)
    check(bf16_to_f64(y), ref, "tiny via fp8")
    # every partial and scaled partial is exact: result is the BF16 rounding of the exact value
    yb = torch.from_numpy(ref).to(torch.bfloat16).double().numpy()
    assert np.mean(bf16_to_f64(y) == yb) > 0.999


def test_every_byte_converts_exactly():
    """One-hot weights read back every converted activation code: A holds all 256 packed
    byte values (both nibble positions), W row n selects k = n."""
    M, K = 8, 512
    N = 256
    codes = np.zeros((M, K), np.uint8)
    allbytes = np.arange(256, dtype=np.uint8)
    for m in range(M):
        codes[m, 0::2] = np.roll(allbytes, m) & 0xF
        codes[m, 1::2] = np.roll(allbytes, m) >> 4
    A = wl.Operand(wl.pack_codes(codes), np.full((M, K // 16), 0x38, np.uint8), 1.0)
    wc = np.zeros((N, K), np.uint8)
    wc[np.arange(N), np.arange(N)] = 0x2  # E2M1 1.0 at k = n
    W = wl.Operand(wl.pack_codes(wc), np.full((N, K // 16), 0x38, np.uint8), 1.0)
    for fn in (nv.gemm_nvfp4_via_fp8, nv.gemm_nvfp4_w4a4):
        y = bf16_to_f64(_run(A, W, 1.0, 1.0, fn))
        ref = oracle.gemm_w4a4(A.codes, A.scales, 1.0, W.codes, W.scales, 1.0, M, N, K)
        assert np.array_equal(y, ref), fn.__name__


SHAPES = [(1, 8, 256), (7, 24, 512), (128, 128, 256), (129, 264, 512), (300, 200, 1024),
          (513, 776, 768), (64, 1000, 2048)]


@pytest.mark.parametrize("M,N,K", SHAPES)
def test_ragged_shapes(M, N, K):
    rng = np.random.default_rng(M * 7919 + N * 31 + K + 5)
    A = wl.uniform_operand(rng, M, K)
    W = wl.uniform_operand(rng, N, K)
    y = _run(A, W, 0.75, 1.5)
    ref = oracle.gemm_w4a4(A.codes, A.scales, 0.75, W.codes, W.scales, 1.5, M, N, K)
    check(bf16_to_f64(y), ref, f"{M}x{N}x{K}")


def test_full_range_scales():
    rng = np.random.default_rng(78)
    M, N, K = 256, 384, 512
    A = wl.random_scale_operand(rng, M, K)
    W = wl.random_scale_operand(rng, N, K)
    y = _run(A, W, 1.0, 1.0)
    ref = oracle.gemm_w4a4(A.codes, A.scales, 1.0, W.codes, W.scales, 1.0, M, N, K)
    check(bf16_to_f64(y), ref, "full-range scales")


def test_ffn_down_full_size_against_w4a4_oracle():
    """Same shape and data as the FFN-down W4A4 workload; compared with that oracle."""
    t = wl.ffn_down_w4a4()
    y = _run(t.A, t.W, t.A.g, t.W.g)
    assert bool(torch.isfinite(y.float()).all())
    rng = np.random.default_rng(1)
    r = np.concatenate([np.repeat(rng.choice(t.M, 6, replace=False), t.N), rng.integers(0, t.M, 4096)])
    c = np.concatenate([np.tile(np.arange(t.N), 6), rng.integers(0, t.N, 4096)])
    ref = oracle.gemm_w4a4(t.A.codes, t.A.scales, t.A.g, t.W.codes, t.W.scales, t.W.g,
                           t.M, t.N, t.K, rows=r, cols=c)
    check(bf16_to_f64(y)[r, c], ref, "via fp8 ffn_down")


def test_agrees_with_w4a4_within_tolerance():
    rng = np.random.Generator(np.random.PCG64(9))
    M, N, K = 256, 512, 1024
    A = wl.quantize_nvfp4(rng.standard_normal((M, K), dtype=np.float32))
    W = wl.quantize_nvfp4(rng.standard_normal((N, K), dtype=np.float32) * np.float32(0.02))
    y8 = bf16_to_f64(_run(A, W, A.g, W.g))
    y4 = bf16_to_f64(_run(A, W, A.g, W.g, nv.gemm_nvfp4_w4a4))
    ref = oracle.gemm_w4a4(A.codes, A.scales, A.g, W.codes, W.scales, W.g, M, N, K)
    check(y8, ref, "via fp8")
    check(y4, ref, "w4a4")


def test_repeat_is_bitwise_deterministic():
    t = wl.tiny_w4a4(2, 200, 300, 1024)
    y1 = _run(t.A, t.W, 1.0, 1.0)
    y2 = _run(t.A, t.W, 1.0, 1.0)
    assert torch.equal(y1.view(torch.int16), y2.view(torch.int16))


def test_k_not_multiple_of_256_rejected():
    A = torch.zeros((4, 64), dtype=torch.uint8, device="cuda")
    sA = torch.zeros((4, 8), dtype=torch.uint8, device="cuda")
    with pytest.raises(nv.NvFp4Error) as e:
        nv.gemm_nvfp4_via_fp8(A, sA, 1.0, A, sA, 1.0)
    assert e.value.status == nv.Status.INVALID_ARG
