"""W4A16 (BF16 activations x NVFP4 weights widened in registers) parity, through the C ABI."""
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


def _run(A_bits, W, gW):
    a = _dev(A_bits.view(np.int16)).view(torch.bfloat16)
    y = nv.gemm_w4a16(a, _dev(W.codes), _dev(W.scales), gW)
    torch.cuda.synchronize()
    return y


def test_exec_of_bf16_widen():
    assert nv.nvfp4_exec_of(torch.cuda.current_device(), nv.Fmt.NVFP4, nv.Fmt.BF16) \
        == nv.Exec.BF16_WIDEN


def test_decode_workload_full_output():
    """16 x 5376 x 14336 as benchmarked: every output against the oracle."""
    t = wl.w4a16_decode()
    y = _run(t.A_bf16, t.W, t.W.g)
    ref = oracle.gemm_w4a16(t.A_bf16, t.W.codes, t.W.scales, t.W.g, t.M, t.N, t.K)
    check(bf16_to_f64(y), ref, "w4a16 decode")


# Rows spread over one wave of CTAs in blocks of 8: these shapes give 1 to 8
# blocks per CTA (and more CTAs than SMs for the tallest), odd N, a single row,
# K not a multiple of the 128-code span, and token counts around 16.
SHAPES = [(1, 8, 32), (1, 1, 32), (2, 101, 288), (3, 24, 96), (16, 100, 160),
          (16, 136, 1024), (5, 520, 4128), (7, 3000, 544), (17, 64, 256), (40, 200, 512),
          (16, 2048, 14336), (16, 12000, 256)]


@pytest.mark.parametrize("M,N,K", SHAPES)
def test_ragged_shapes(M, N, K):
    rng = np.random.default_rng(M * 1009 + N * 13 + K)
    A = wl.to_bf16_bits(rng.standard_normal((M, K), dtype=np.float32))
    W = wl.uniform_operand(rng, N, K)
    y = _run(A, W, 0.5)
    ref = oracle.gemm_w4a16(A, W.codes, W.scales, 0.5, M, N, K)
    check(bf16_to_f64(y), ref, f"{M}x{N}x{K}")


def test_every_code_and_every_scale_byte():
    """All 16 codes (incl. 0.5, whose widened BF16 pattern is subnormal) against all
    finite non-negative E4M3 scale bytes (incl. E4M3 subnormals and 448)."""
    rng = np.random.default_rng(3)
    M, N, K = 4, 127 * 2, 512
    A = wl.to_bf16_bits(rng.standard_normal((M, K), dtype=np.float32))
    codes = np.tile(np.arange(16, dtype=np.uint8), (N, K // 16))
    scales = np.tile(np.arange(127, dtype=np.uint8), 2)[:, None].repeat(K // 16, 1)
    W = wl.Operand(wl.pack_codes(codes), np.ascontiguousarray(scales), 1.0)
    y = _run(A, W, 1.0)
    ref = oracle.gemm_w4a16(A, W.codes, W.scales, 1.0, M, N, K)
    nz = np.abs(ref).max(axis=0) > 0
    check(bf16_to_f64(y)[:, nz], ref[:, nz], "codes x scales")
    assert np.all(bf16_to_f64(y)[:, ~nz] == 0)  # scale byte 0 rows give exact zeros


def test_one_hot_activations_pick_single_widened_weights():
    """A one-hot activation row reads back single weights exactly: the widening is exact."""
    rng = np.random.default_rng(4)
    N, K = 64, 256
    W = wl.random_scale_operand(rng, N, K)
    ks = rng.choice(K, 16, replace=False)
    A = np.zeros((16, K), np.float32)
    A[np.arange(16), ks] = 1.0
    y = bf16_to_f64(_run(wl.to_bf16_bits(A), W, 1.0))
    ref = oracle.gemm_w4a16(wl.to_bf16_bits(A), W.codes, W.scales, 1.0, 16, N, K)
    assert np.array_equal(y, torch.from_numpy(ref).to(torch.bfloat16).double().numpy())


def test_repeat_is_bitwise_deterministic():
    t = wl.w4a16_decode(N=1024, K=4096)
    y1 = _run(t.A_bf16, t.W, t.W.g)
    y2 = _run(t.A_bf16, t.W, t.W.g)
    assert torch.equal(y1.view(torch.int16), y2.view(torch.int16))


def test_w4a16_argument_errors():
    a = torch.zeros((2, 48), dtype=torch.bfloat16, device="cuda")
    W = torch.zeros((8, 24), dtype=torch.uint8, device="cuda")
    sW = torch.zeros((8, 3), dtype=torch.uint8, device="cuda")
    with pytest.raises(nv.NvFp4Error) as e:
        nv.gemm_w4a16(a, W, sW, 1.0)
    assert e.value.status == nv.Status.INVALID_ARG
