"""Scales packed into the MMA's layout, and the pair-of-SMs W4A4 kernel that reads them."""
import numpy as np
import pytest
import torch

import oracle
import block_scaled_precision_nvfp4_b200 as nv
from block_scaled_precision_nvfp4_b200 import workloads as wl

from parity import bf16_to_f64, check, packed_reference

pytestmark = pytest.mark.gpu


def _dev(x):
    return torch.from_numpy(np.ascontiguousarray(x)).cuda()


@pytest.mark.parametrize("rows,K", [(1, 64), (128, 256), (130, 512), (300, 1024), (4096, 14336),
                                    (5376, 14336), (77, 192)])
def test_pack_layout_bit_exact(rows, K):
    rng = np.random.default_rng(rows + K)
    s = rng.integers(0, 0x7F, (rows, K // 16), dtype=np.uint8)
    p = nv.nvfp4_pack_scales(_dev(s), K)
    torch.cuda.synchronize()
    ref = packed_reference(s, K)
    assert nv.nvfp4_scale_layout_bytes(rows, K) == ref.size
    assert np.array_equal(p.cpu().numpy()[:ref.size], ref)


def _run_packed(A, W, gA, gW, K):
    sa = nv.nvfp4_pack_scales(_dev(A.scales), K)
    sw = nv.nvfp4_pack_scales(_dev(W.scales), K)
    y = nv.gemm_nvfp4_w4a4_packed(_dev(A.codes), sa, gA, _dev(W.codes), sw, gW)
    torch.cuda.synchronize()
    nv.nvfp4_check_device_error()
    return y


def test_tiny_workload():
    t = wl.tiny_w4a4(0)
    y = _run_packed(t.A, t.W, 1.0, 1.0, t.K)
    ref = oracle.gemm_w4a4(t.A.codes, t.A.scales, 1.0, t.W.codes, t.W.scales, 1.0, t.M, t.N, t.K)
    check(bf16_to_f64(y), ref, "tiny packed")
    yb = torch.from_numpy(ref).to(torch.bfloat16).double().numpy()
    assert np.mean(bf16_to_f64(y) == yb) > 0.999


SHAPES = [(1, 8, 256), (7, 24, 512), (256, 256, 256), (257, 264, 512), (300, 200, 768),
          (512, 512, 1024), (130, 130, 256), (64, 1000, 2048), (1000, 72, 4096), (513, 776, 1280)]


@pytest.mark.parametrize("M,N,K", SHAPES)
def test_ragged_shapes(M, N, K):
    rng = np.random.default_rng(M * 7919 + N * 31 + K + 17)
    A = wl.uniform_operand(rng, M, K)
    W = wl.uniform_operand(rng, N, K)
    y = _run_packed(A, W, 0.75, 1.5, K)
    ref = oracle.gemm_w4a4(A.codes, A.scales, 0.75, W.codes, W.scales, 1.5, M, N, K)
    check(bf16_to_f64(y), ref, f"packed {M}x{N}x{K}")


def test_full_range_scales():
    rng = np.random.default_rng(79)
    M, N, K = 512, 384, 512
    A = wl.random_scale_operand(rng, M, K)
    W = wl.random_scale_operand(rng, N, K)
    y = _run_packed(A, W, 1.0, 1.0, K)
    ref = oracle.gemm_w4a4(A.codes, A.scales, 1.0, W.codes, W.scales, 1.0, M, N, K)
    check(bf16_to_f64(y), ref, "packed full-range scales")


def test_ffn_down_full_size_sampled():
    t = wl.ffn_down_w4a4()
    y = _run_packed(t.A, t.W, t.A.g, t.W.g, t.K)
    assert bool(torch.isfinite(y.float()).all())
    rng = np.random.default_rng(3)
    r = np.concatenate([np.repeat(rng.choice(t.M, 8, replace=False), t.N), rng.integers(0, t.M, 4096)])
    c = np.concatenate([np.tile(np.arange(t.N), 8), rng.integers(0, t.N, 4096)])
    ref = oracle.gemm_w4a4(t.A.codes, t.A.scales, t.A.g, t.W.codes, t.W.scales, t.W.g,
                           t.M, t.N, t.K, rows=r, cols=c)
    check(bf16_to_f64(y)[r, c], ref, "packed ffn_down sampled")


def test_agrees_with_plain_scale_entry():
    rng = np.random.Generator(np.random.PCG64(12))
    M, N, K = 640, 768, 2048
    A = wl.quantize_nvfp4(rng.standard_normal((M, K), dtype=np.float32))
    W = wl.quantize_nvfp4(rng.standard_normal((N, K), dtype=np.float32) * np.float32(0.02))
    yp = bf16_to_f64(_run_packed(A, W, A.g, W.g, K))
    y = bf16_to_f64(nv.gemm_nvfp4_w4a4(_dev(A.codes), _dev(A.scales), A.g, _dev(W.codes),
                                       _dev(W.scales), W.g))
    ref = oracle.gemm_w4a4(A.codes, A.scales, A.g, W.codes, W.scales, W.g, M, N, K)
    check(yp, ref, "packed")
    check(y, ref, "plain")


def test_repeat_is_bitwise_deterministic():
    t = wl.tiny_w4a4(3, 600, 520, 1024)
    y1 = _run_packed(t.A, t.W, 1.0, 1.0, t.K)
    y2 = _run_packed(t.A, t.W, 1.0, 1.0, t.K)
    assert torch.equal(y1.view(torch.int16), y2.view(torch.int16))


def test_packed_rejects_k_not_multiple_of_256():
    A = torch.zeros((4, 64), dtype=torch.uint8, device="cuda")
    s = torch.zeros(4096, dtype=torch.uint8, device="cuda")
    with pytest.raises(nv.NvFp4Error) as e:
        nv.gemm_nvfp4_w4a4_packed(A, s, 1.0, A, s, 1.0)
    assert e.value.status == nv.Status.INVALID_ARG
