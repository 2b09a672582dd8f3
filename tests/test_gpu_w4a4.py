"""W4A4 (block-scaled FP4 MMA) parity against the FP64 oracle, through the C ABI."""
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


def _run(A, W, M, N, K, gA=None, gW=None, fn=None):
    fn = fn or nv.gemm_nvfp4_w4a4
    gA = A.g if gA is None else gA
    gW = W.g if gW is None else gW
    y = fn(_dev(A.codes), _dev(A.scales), gA, _dev(W.codes), _dev(W.scales), gW)
    torch.cuda.synchronize()
    nv.nvfp4_check_device_error()
    return y


def test_exec_of_on_this_device():
    assert nv.nvfp4_exec_of(torch.cuda.current_device(), nv.Fmt.NVFP4, nv.Fmt.NVFP4) \
        == nv.Exec.FP4_MMA


def test_tiny_workload():
    t = wl.tiny_w4a4(0)
    y = _run(t.A, t.W, t.M, t.N, t.K)
    ref = oracle.gemm_w4a4(t.A.codes, t.A.scales, 1.0, t.W.codes, t.W.scales, 1.0, t.M, t.N, t.K)
    rel, mx = check(bf16_to_f64(y), ref, "tiny")
    # every value is a multiple of 2^-10 well inside BF16 range: the result must be the
    # BF16 rounding of the exact value almost everywhere (FP32 accumulation is exact here)
    yb = torch.from_numpy(ref).to(torch.bfloat16).double().numpy()
    assert np.mean(bf16_to_f64(y) == yb) > 0.999


SHAPES = [(1, 8, 32), (7, 24, 64), (128, 256, 256), (129, 264, 288), (300, 200, 512),
          (256, 512, 1024), (130, 130, 96), (64, 1000, 2048), (1000, 72, 4096), (513, 776, 800)]


@pytest.mark.parametrize("M,N,K", SHAPES)
def test_ragged_shapes(M, N, K):
    rng = np.random.default_rng(M * 7919 + N * 31 + K)
    A = wl.uniform_operand(rng, M, K)
    W = wl.uniform_operand(rng, N, K)
    y = _run(A, W, M, N, K, 0.75, 1.5)
    ref = oracle.gemm_w4a4(A.codes, A.scales, 0.75, W.codes, W.scales, 1.5, M, N, K)
    check(bf16_to_f64(y), ref, f"{M}x{N}x{K}")


def test_full_range_scales():
    rng = np.random.default_rng(77)
    M, N, K = 256, 384, 512
    A = wl.random_scale_operand(rng, M, K)
    W = wl.random_scale_operand(rng, N, K)
    y = _run(A, W, M, N, K, 1.0, 1.0)
    ref = oracle.gemm_w4a4(A.codes, A.scales, 1.0, W.codes, W.scales, 1.0, M, N, K)
    check(bf16_to_f64(y), ref, "full-range scales")


def test_quantised_gaussian_medium():
    rng = np.random.Generator(np.random.PCG64(5))
    M, N, K = 384, 640, 2304
    A = wl.quantize_nvfp4(rng.standard_normal((M, K), dtype=np.float32))
    W = wl.quantize_nvfp4(rng.standard_normal((N, K), dtype=np.float32) * np.float32(0.02))
    y = _run(A, W, M, N, K)
    ref = oracle.gemm_w4a4(A.codes, A.scales, A.g, W.codes, W.scales, W.g, M, N, K)
    check(bf16_to_f64(y), ref, "gaussian")


def test_repeat_is_bitwise_deterministic():
    t = wl.tiny_w4a4(1, 300, 520, 768)
    y1 = _run(t.A, t.W, t.M, t.N, t.K)
    y2 = _run(t.A, t.W, t.M, t.N, t.K)
    assert torch.equal(y1.view(torch.int16), y2.view(torch.int16))


def test_empty_sizes_are_noops():
    z = torch.zeros((0, 16), dtype=torch.uint8, device="cuda")
    zs = torch.zeros((0, 2), dtype=torch.uint8, device="cuda")
    W = torch.zeros((8, 16), dtype=torch.uint8, device="cuda")
    sW = torch.zeros((8, 2), dtype=torch.uint8, device="cuda")
    y = nv.gemm_nvfp4_w4a4(z, zs, 1.0, W, sW, 1.0)
    assert y.shape == (0, 8)


def test_misaligned_pointer_rejected():
    buf = torch.zeros(64 * 17 + 1, dtype=torch.uint8, device="cuda")
    A = buf[1:1 + 64 * 16].view(64, 16)  # offset by one byte
    sA = torch.zeros((64, 2), dtype=torch.uint8, device="cuda")
    W = torch.zeros((8, 16), dtype=torch.uint8, device="cuda")
    sW = torch.zeros((8, 2), dtype=torch.uint8, device="cuda")
    with pytest.raises(nv.NvFp4Error) as e:
        nv.gemm_nvfp4_w4a4(A, sA, 1.0, W, sW, 1.0)
    assert e.value.status == nv.Status.MISALIGNED


def test_disabled_fp4_kernel_refuses_without_launch():
    nv.nvfp4_set_fp4_kernel_disabled(True)
    try:
        assert nv.nvfp4_exec_of(0, nv.Fmt.NVFP4, nv.Fmt.NVFP4) == nv.Exec.NO_FP4_KERNEL
        t = wl.tiny_w4a4(0)
        out = torch.full((t.M, t.N), 7.0, dtype=torch.bfloat16, device="cuda")
        with pytest.raises(nv.NvFp4Error) as e:
            nv.gemm_nvfp4_w4a4(_dev(t.A.codes), _dev(t.A.scales), 1.0, _dev(t.W.codes),
                               _dev(t.W.scales), 1.0, out=out)
        assert e.value.status == nv.Status.NO_FP4_KERNEL
        torch.cuda.synchronize()
        assert torch.all(out == 7.0)  # nothing was enqueued
    finally:
        nv.nvfp4_set_fp4_kernel_disabled(False)


def _sample_points(M, N, rng, rows=8, cols=8, points=2048):
    r = [np.repeat(rng.choice(M, rows, replace=False), N), np.repeat(np.arange(M), cols),
         rng.integers(0, M, points)]
    c = [np.tile(np.arange(N), rows), np.tile(rng.choice(N, cols, replace=False), M),
         rng.integers(0, N, points)]
    return np.concatenate(r), np.concatenate(c)


def test_ffn_down_full_size_sampled():
    """4096 x 5376 x 14336 as launched by the benchmark; sampled rows, columns and points."""
    t = wl.ffn_down_w4a4()
    y = _run(t.A, t.W, t.M, t.N, t.K)
    yf = y.float()
    assert bool(torch.isfinite(yf).all())
    rng = np.random.default_rng(0)
    r, c = _sample_points(t.M, t.N, rng)
    ref = oracle.gemm_w4a4(t.A.codes, t.A.scales, t.A.g, t.W.codes, t.W.scales, t.W.g,
                           t.M, t.N, t.K, rows=r, cols=c)
    got = bf16_to_f64(y)[r, c]
    check(got, ref, "ffn_down sampled")


@pytest.mark.parametrize("mode", ["unit", "row", "group", "both"])
def test_scale_structure(mode):
    """Localises a scale-layout error: unit scales (data path only), scales varying by row
    only, by group only, and both."""
    rng = np.random.default_rng(99)
    M, N, K = 256, 256, 512
    A = wl.uniform_operand(rng, M, K)
    W = wl.uniform_operand(rng, N, K)
    G = K // 16
    def mk(rows, kind):
        if kind == "unit":
            return np.full((rows, G), 0x38, np.uint8)
        if kind == "row":
            return np.repeat(((rng.integers(-4, 5, (rows, 1)) + 7) << 3).astype(np.uint8), G, 1)
        if kind == "group":
            return np.repeat(((rng.integers(-4, 5, (1, G)) + 7) << 3).astype(np.uint8), rows, 0)
        return ((rng.integers(-4, 5, (rows, G)) + 7) << 3).astype(np.uint8)
    kind = {"unit": "unit", "row": "row", "group": "group", "both": "both"}[mode]
    A.scales = mk(M, kind); W.scales = mk(N, kind)
    y = _run(A, W, M, N, K, 1.0, 1.0)
    ref = oracle.gemm_w4a4(A.codes, A.scales, 1.0, W.codes, W.scales, 1.0, M, N, K)
    check(bf16_to_f64(y), ref, mode)
