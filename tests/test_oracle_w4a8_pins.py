"""Pins of the oracle's W4A8 product (FP8 E4M3 activations under NVFP4 weights).

Y = gA*gW * sum_g sW[n,g] * sum_{k in g} e4m3(A[m,k]) * e2m1(W[n,k]); each pin ties
it to something other than itself: torch's float8_e4m3fn decode and numpy's matmul
(library routines), the W4A4 product on activations whose FP8 bytes hold E2M1
values exactly, and a flat brute-force sum over k."""
import numpy as np
import pytest
import torch

import oracle
from block_scaled_precision_nvfp4_b200 import workloads as wl

E2M1 = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


def e4m3_decode(b):
    return torch.from_numpy(np.ascontiguousarray(b, np.uint8)).view(torch.float8_e4m3fn).double().numpy()


def e2m1_decode(codes):
    return E2M1[codes & 7] * np.where(codes & 8, -1.0, 1.0)


def finite_fp8(rng, shape):
    b = rng.integers(0, 256, size=shape, dtype=np.uint8)
    return np.where((b & 0x7F) == 0x7F, b ^ 1, b).astype(np.uint8)   # no NaN bytes


def test_reduces_to_w4a4_when_the_activations_are_e2m1_values():
    rng = np.random.default_rng(0)
    M, N, K = 5, 7, 64
    a_codes = rng.integers(0, 16, size=(M, K), dtype=np.uint8)
    a8 = torch.from_numpy(e2m1_decode(a_codes).astype(np.float32)).to(torch.float8_e4m3fn).view(
        torch.uint8).numpy()
    W = wl.random_scale_operand(rng, N, K)
    got = oracle.gemm_w4a8(a8, 0.75, W.codes, W.scales, 1.5, M, N, K)
    ref = oracle.gemm_w4a4(wl.pack_codes(a_codes), np.full((M, K // 16), 0x38, np.uint8), 0.75,
                           W.codes, W.scales, 1.5, M, N, K)
    assert np.array_equal(got, ref)


def test_unit_scales_equal_numpy_matmul():
    rng = np.random.default_rng(1)
    M, N, K = 6, 9, 96
    a8 = finite_fp8(rng, (M, K))
    w_codes = rng.integers(0, 16, size=(N, K), dtype=np.uint8)
    got = oracle.gemm_w4a8(a8, 1.0, wl.pack_codes(w_codes), np.full((N, K // 16), 0x38, np.uint8),
                           1.0, M, N, K)
    ref = e4m3_decode(a8) @ e2m1_decode(w_codes).T
    assert np.array_equal(got, ref)


@pytest.mark.parametrize("K", [16, 32, 48])
def test_brute_force_flat_sum(K):
    rng = np.random.default_rng(K)
    M, N = 3, 4
    a8 = finite_fp8(rng, (M, K))
    W = wl.random_scale_operand(rng, N, K)
    wc = wl.unpack_codes(W.codes)
    gA, gW = 0.375, 3.0
    got = oracle.gemm_w4a8(a8, gA, W.codes, W.scales, gW, M, N, K)
    av = e4m3_decode(a8)
    sv = e4m3_decode(W.scales)
    for m in range(M):
        for n in range(N):
            tot = 0.0
            for k in range(K):
                tot += av[m, k] * E2M1[wc[n, k] & 7] * (-1.0 if wc[n, k] & 8 else 1.0) * sv[n, k // 16]
            # the sum's rounding order differs (flat here, per group there): FP64-tight
            assert abs(got[m, n] - gA * gW * tot) <= 1e-12 * max(1.0, abs(gA * gW * tot))


def test_bilinear_in_the_tensor_scales_and_sampled_matches_dense():
    rng = np.random.default_rng(2)
    M, N, K = 4, 5, 64
    a8 = finite_fp8(rng, (M, K))
    W = wl.random_scale_operand(rng, N, K)
    y1 = oracle.gemm_w4a8(a8, 1.0, W.codes, W.scales, 1.0, M, N, K)
    y2 = oracle.gemm_w4a8(a8, 0.5, W.codes, W.scales, 8.0, M, N, K)
    assert np.array_equal(y2, 4.0 * y1)
    r = np.array([0, 3, 1]); c = np.array([4, 0, 2])
    assert np.array_equal(oracle.gemm_w4a8(a8, 1.0, W.codes, W.scales, 1.0, M, N, K, rows=r, cols=c),
                          y1[r, c])
