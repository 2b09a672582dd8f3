"""W4A8 (E4M3 activations under NVFP4 weights) on the exact E4M3 path: parity with the
FP64 oracle's W4A8 product, through the C ABI."""
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


def _run(A8, gA, W, gW=None):
    y = nv.gemm_nvfp4_w4a8(_dev(A8), gA, _dev(W.codes), _dev(W.scales), W.g if gW is None else gW)
    torch.cuda.synchronize()
    nv.nvfp4_check_device_error()
    return y


def _finite_e4m3(rng, shape):
    """Bytes uniform over every finite E4M3 value (0x7F and 0xFF are NaN)."""
    b = rng.integers(0, 254, size=shape, dtype=np.uint8)
    return np.where(b >= 0x7F, b + 1, b).astype(np.uint8)


def test_every_activation_byte_reads_exactly():
    """A holds every finite E4M3 byte; weight row n is E2M1 1.0 (scale 1.0) at k = n, so
    Y[m,n] is the activation byte's value, which BF16 holds exactly."""
    M, N, K = 8, 256, 512
    allb = np.arange(256, dtype=np.uint8)
    allb[0x7F], allb[0xFF] = 0x00, 0x80
    A8 = np.zeros((M, K), np.uint8)
    for m in range(M):
        A8[m, :256] = np.roll(allb, m)
    wc = np.zeros((N, K), np.uint8)
    wc[np.arange(N), np.arange(N)] = 0x2
    W = wl.Operand(wl.pack_codes(wc), np.full((N, K // 16), 0x38, np.uint8), 1.0)
    y = bf16_to_f64(_run(A8, 1.0, W))
    ref = oracle.gemm_w4a8(A8, 1.0, W.codes, W.scales, 1.0, M, N, K)
    assert np.array_equal(y, ref)


def test_every_weight_code_reads_exactly():
    """A row m is E4M3 1.0 at k = m; the weights hold all 16 codes under several scales,
    so Y[m,n] is the weight's code value times its group scale, exactly."""
    M, N, K = 256, 64, 256
    A8 = np.zeros((M, K), np.uint8)
    A8[np.arange(M), np.arange(M)] = 0x38
    codes = (np.arange(N)[:, None] + np.arange(K)[None, :]) % 16
    scales = np.tile(np.array([0x38, 0x30, 0x40, 0x08, 0x7E, 0x01], np.uint8),
                     (N, K // 16 // 6 + 1))[:, :K // 16]
    W = wl.Operand(wl.pack_codes(codes.astype(np.uint8)), np.ascontiguousarray(scales), 1.0)
    y = bf16_to_f64(_run(A8, 1.0, W))
    ref = oracle.gemm_w4a8(A8, 1.0, W.codes, W.scales, 1.0, M, N, K)
    assert np.array_equal(y, ref)


SHAPES = [(1, 8, 256), (1, 1, 256), (7, 24, 512), (128, 128, 256), (129, 264, 512),
          (300, 200, 1024), (513, 776, 768), (64, 1000, 2048)]


@pytest.mark.parametrize("M,N,K", SHAPES)
def test_ragged_shapes(M, N, K):
    """Activation bytes over the whole finite E4M3 range, weights with every code and
    power-of-two scales; ragged M and N tails."""
    rng = np.random.default_rng(M * 7919 + N * 31 + K + 8)
    A8 = _finite_e4m3(rng, (M, K))
    W = wl.uniform_operand(rng, N, K)
    y = _run(A8, 0.75, W, 1.5)
    ref = oracle.gemm_w4a8(A8, 0.75, W.codes, W.scales, 1.5, M, N, K)
    check(bf16_to_f64(y), ref, f"w4a8 {M}x{N}x{K}")


def test_full_range_weight_scales():
    rng = np.random.default_rng(81)
    M, N, K = 256, 384, 512
    A8 = _finite_e4m3(rng, (M, K))
    W = wl.random_scale_operand(rng, N, K)
    y = _run(A8, 1.0, W, 1.0)
    ref = oracle.gemm_w4a8(A8, 1.0, W.codes, W.scales, 1.0, M, N, K)
    check(bf16_to_f64(y), ref, "w4a8 full-range weight scales")


def test_per_tensor_fp8_activations():
    """The workload's recipe at a small size: N(0,1) activations as E4M3 with gA = amax/448."""
    rng = np.random.Generator(np.random.PCG64(5))
    M, N, K = 384, 640, 2048
    A8, gA = wl.fp8_per_tensor(rng, M, K)
    W = wl.quantize_nvfp4(rng.standard_normal((N, K), dtype=np.float32) * np.float32(0.02))
    y = _run(A8, gA, W)
    ref = oracle.gemm_w4a8(A8, gA, W.codes, W.scales, W.g, M, N, K)
    check(bf16_to_f64(y), ref, "w4a8 per-tensor fp8")


def test_ffn_down_full_size_sampled():
    """The FFN-down shape with FP8 activations (4096 x 5376 x 14336): six whole output rows
    and 4096 scattered elements against the oracle."""
    t = wl.w4a8_ffn_down()
    y = _run(t.A_fp8, t.gA, t.W)
    assert bool(torch.isfinite(y.float()).all())
    rng = np.random.default_rng(2)
    r = np.concatenate([np.repeat(rng.choice(t.M, 6, replace=False), t.N), rng.integers(0, t.M, 4096)])
    c = np.concatenate([np.tile(np.arange(t.N), 6), rng.integers(0, t.N, 4096)])
    ref = oracle.gemm_w4a8(t.A_fp8, t.gA, t.W.codes, t.W.scales, t.W.g, t.M, t.N, t.K,
                           rows=r, cols=c)
    check(bf16_to_f64(y)[r, c], ref, "w4a8 ffn_down")


def test_repeat_is_bitwise_deterministic():
    rng = np.random.default_rng(6)
    A8 = _finite_e4m3(rng, (200, 1024))
    W = wl.uniform_operand(rng, 300, 1024)
    y1 = _run(A8, 1.0, W, 1.0)
    y2 = _run(A8, 1.0, W, 1.0)
    assert torch.equal(y1.view(torch.int16), y2.view(torch.int16))


def test_empty_and_argument_errors():
    W = wl.uniform_operand(np.random.default_rng(0), 16, 256)
    y = nv.gemm_nvfp4_w4a8(torch.empty((0, 256), dtype=torch.uint8, device="cuda"), 1.0,
                           _dev(W.codes), _dev(W.scales), 1.0)
    torch.cuda.synchronize()
    assert y.shape == (0, 16)
    A = torch.zeros((4, 128), dtype=torch.uint8, device="cuda")
    W = wl.uniform_operand(np.random.default_rng(0), 4, 128)
    with pytest.raises(nv.NvFp4Error) as e:
        nv.gemm_nvfp4_w4a8(A, 1.0, _dev(W.codes), _dev(W.scales), 1.0)
    assert e.value.status == nv.Status.INVALID_ARG


def test_planner_names_the_exact_path_on_this_device():
    assert nv.nvfp4_exec_of(torch.cuda.current_device(), nv.Fmt.NVFP4, nv.Fmt.FP8_E4M3) \
        == nv.Exec.FP8_EXACT
