"""Grouped (MoE) W4A4 on pairs of SMs with per-expert packed scales: the grouped
packing layout bit for bit, and parity with the FP64 oracle through the C ABI."""
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


def _packed_block_reference(s, K):
    """packed[rb][ks][i][j][t] = s[rb*128 + 32j + i][4ks + t], zero rows past the end."""
    rows = s.shape[0]
    rb_n = (rows + 127) // 128
    pad = np.zeros((rb_n * 128, K // 16), np.uint8)
    pad[:rows] = s
    v = pad.reshape(rb_n, 4, 32, K // 64, 4)          # [rb][j][i][ks][t]
    return np.ascontiguousarray(v.transpose(0, 3, 2, 1, 4)).ravel()


def grouped_packed_reference(s, offsets, K):
    """Each group's rows packed on their own, groups laid end to end."""
    parts = [_packed_block_reference(s[offsets[g]:offsets[g + 1]], K)
             for g in range(len(offsets) - 1)]
    return np.concatenate(parts) if parts else np.zeros(0, np.uint8)


@pytest.mark.parametrize("counts,K", [
    ([1], 64), ([0, 5, 0, 128, 129, 300], 256), ([127, 1, 256], 192), ([3278, 1473, 977], 4096),
])
def test_grouped_pack_layout_bit_exact(counts, K):
    rng = np.random.default_rng(sum(counts) + K)
    off = np.concatenate([[0], np.cumsum(counts)]).astype(np.int64)
    s = rng.integers(0, 0x7F, (int(off[-1]), K // 16), dtype=np.uint8)
    p = nv.nvfp4_pack_scales_grouped(_dev(s), list(off), K)
    torch.cuda.synchronize()
    ref = grouped_packed_reference(s, off, K)
    assert nv.nvfp4_grouped_scale_layout_bytes(list(off), K) == ref.size
    assert np.array_equal(p.cpu().numpy()[:ref.size], ref)


def _run(A, Wc, Ws, gA, gW, offsets):
    E, N, K = Wc.shape[0], Wc.shape[1], 2 * Wc.shape[2]
    sa = nv.nvfp4_pack_scales_grouped(_dev(A.scales), list(offsets), K)
    sw = nv.nvfp4_pack_scales_grouped(_dev(Ws.reshape(E * N, K // 16)),
                                      [e * N for e in range(E + 1)], K)
    y = nv.gemm_nvfp4_w4a4_grouped_packed(_dev(A.codes), sa, gA, _dev(Wc), sw, list(gW),
                                          list(offsets))
    torch.cuda.synchronize()
    nv.nvfp4_check_device_error()
    return y


def _random_grouped(counts, N, K, seed):
    rng = np.random.default_rng(seed)
    off = np.concatenate([[0], np.cumsum(counts)]).astype(np.int64)
    A = wl.uniform_operand(rng, int(off[-1]), K)
    Ws = [wl.uniform_operand(rng, N, K) for _ in counts]
    Wc = np.stack([w.codes for w in Ws]); Wsc = np.stack([w.scales for w in Ws])
    gW = rng.choice([0.25, 0.5, 1.0, 2.0], len(counts))
    return A, Wc, Wsc, gW, off


@pytest.mark.parametrize("counts,N,K", [
    ([1, 8, 17, 64, 127, 128], 520, 512),      # every expert swapped, N not a multiple of 256
    ([0, 130, 0, 1, 256, 300], 264, 256),      # empty experts, full blocks, ragged tails
    ([127, 128, 129, 383, 384, 385], 136, 768),
    ([16], 1000, 1024),
    ([200, 3, 50, 513], 256, 4096),
    ([40] * 20, 384, 256),                     # many small experts
    ([5, 300, 129, 64], 100, 256),             # N % 8 != 0: plain copy-out instead of TMA stores
])
def test_forced_ragged_experts(counts, N, K):
    A, Wc, Ws, gW, off = _random_grouped(counts, N, K, sum(counts) + N + K)
    y = _run(A, Wc, Ws, 1.5, gW, off)
    ref = oracle.gemm_grouped_w4a4(A.codes, A.scales, 1.5, Wc, Ws, gW, off, N, K)
    check(bf16_to_f64(y), ref, f"grouped packed {counts}")


def test_single_expert_matches_dense_packed():
    """E = 1 with 512 rows runs only unswapped 256-token tiles: the same MMA
    sequence as the dense pair kernel, so the two agree bit for bit."""
    rng = np.random.default_rng(6)
    M, N, K = 512, 512, 1024
    A = wl.uniform_operand(rng, M, K); W = wl.uniform_operand(rng, N, K)
    yg = _run(A, W.codes[None], W.scales[None], 1.0, [1.0], [0, M])
    yd = nv.gemm_nvfp4_w4a4_packed(_dev(A.codes), nv.nvfp4_pack_scales(_dev(A.scales), K), 1.0,
                                   _dev(W.codes), nv.nvfp4_pack_scales(_dev(W.scales), K), 1.0)
    torch.cuda.synchronize()
    ref = oracle.gemm_w4a4(A.codes, A.scales, 1.0, W.codes, W.scales, 1.0, M, N, K)
    check(bf16_to_f64(yg), ref, "grouped packed E=1")
    assert torch.equal(yg.view(torch.int16), yd.view(torch.int16))


def test_full_range_scales():
    rng = np.random.default_rng(81)
    counts, N, K = [100, 300], 384, 512
    off = np.array([0, 100, 400])
    A = wl.random_scale_operand(rng, 400, K)
    Ws = [wl.random_scale_operand(rng, N, K) for _ in counts]
    Wc = np.stack([w.codes for w in Ws]); Wsc = np.stack([w.scales for w in Ws])
    y = _run(A, Wc, Wsc, 1.0, [1.0, 1.0], off)
    ref = oracle.gemm_grouped_w4a4(A.codes, A.scales, 1.0, Wc, Wsc, np.ones(2), off, N, K)
    check(bf16_to_f64(y), ref, "grouped packed full-range scales")


def test_moe_workload_full_size_sampled():
    """8 experts of W [14336, 4096], 8192 tokens routed top-1 with Zipf(1.1) popularity."""
    t = wl.grouped_w4a4()
    Wc, Ws, gW = wl.stack_experts(t)
    y = _run(t.A, Wc, Ws, t.A.g, gW, t.offsets)
    assert bool(torch.isfinite(y.float()).all())
    rng = np.random.default_rng(4)
    rows, cols = [], []
    for e in range(t.E):
        lo, hi = int(t.offsets[e]), int(t.offsets[e + 1])
        for r in (lo, hi - 1):  # first row, and a row of the ragged (possibly swapped) tail
            rows.append(np.full(512, r)); cols.append(rng.choice(t.N, 512, replace=False))
    rows.append(rng.integers(0, t.M, 4096)); cols.append(rng.integers(0, t.N, 4096))
    r = np.concatenate(rows); c = np.concatenate(cols)
    ref = oracle.gemm_grouped_w4a4(t.A.codes, t.A.scales, t.A.g, Wc, Ws, gW.astype(np.float64),
                                   t.offsets, t.N, t.K, rows=r, cols=c)
    check(bf16_to_f64(y)[r, c], ref, "moe packed sampled")


def test_repeat_is_bitwise_deterministic():
    A, Wc, Ws, gW, off = _random_grouped([70, 300, 5], 384, 512, 11)
    y1 = _run(A, Wc, Ws, 1.0, gW, off)
    y2 = _run(A, Wc, Ws, 1.0, gW, off)
    assert torch.equal(y1.view(torch.int16), y2.view(torch.int16))


def test_grouped_packed_rejects_bad_arguments():
    A = torch.zeros((4, 64), dtype=torch.uint8, device="cuda")
    W = torch.zeros((1, 8, 64), dtype=torch.uint8, device="cuda")
    s = torch.zeros(4096, dtype=torch.uint8, device="cuda")
    with pytest.raises(nv.NvFp4Error) as e:   # K = 128 is not a multiple of 256
        nv.gemm_nvfp4_w4a4_grouped_packed(A, s, 1.0, W, s, [1.0], [0, 4])
    assert e.value.status == nv.Status.INVALID_ARG
    with pytest.raises(ValueError):
        nv.gemm_nvfp4_w4a4_grouped_packed(A, s, 1.0, W, s, [1.0], [0, 3])
