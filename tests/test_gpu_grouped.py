"""Grouped (MoE) W4A4 with swap-AB for small experts: parity with the FP64 oracle, via the C ABI."""
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


def _run(A, Wc, Ws, gA, gW, offsets):
    y = nv.gemm_nvfp4_w4a4_grouped(_dev(A.codes), _dev(A.scales), gA, _dev(Wc), _dev(Ws),
                                   list(gW), list(offsets))
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
    ([1, 8, 17, 64, 127], 520, 512),           # every expert swapped
    ([0, 130, 0, 1, 256, 300], 264, 256),      # empty experts, full blocks, ragged tails
    ([127, 128, 129], 136, 768),
    ([16], 1000, 1024),
    ([200, 3, 50], 256, 4096),
])
def test_forced_ragged_experts(counts, N, K):
    A, Wc, Ws, gW, off = _random_grouped(counts, N, K, sum(counts) + N + K)
    y = _run(A, Wc, Ws, 1.5, gW, off)
    ref = oracle.gemm_grouped_w4a4(A.codes, A.scales, 1.5, Wc, Ws, gW, off, N, K)
    check(bf16_to_f64(y), ref, f"grouped {counts}")


def test_single_expert_matches_dense_w4a4():
    rng = np.random.default_rng(5)
    M, N, K = 300, 512, 1024
    A = wl.uniform_operand(rng, M, K); W = wl.uniform_operand(rng, N, K)
    yg = _run(A, W.codes[None], W.scales[None], 1.0, [1.0], [0, M])
    yd = nv.gemm_nvfp4_w4a4(_dev(A.codes), _dev(A.scales), 1.0, _dev(W.codes), _dev(W.scales), 1.0)
    torch.cuda.synchronize()
    ref = oracle.gemm_w4a4(A.codes, A.scales, 1.0, W.codes, W.scales, 1.0, M, N, K)
    check(bf16_to_f64(yg), ref, "grouped E=1")
    # the full 128-row blocks run the same MMA sequence as the dense kernel
    assert torch.equal(yg[:256].view(torch.int16), yd[:256].view(torch.int16))


def test_moe_workload_full_size_sampled():
    """8 experts of W [14336, 4096], 8192 tokens routed top-1 with Zipf(1.1) popularity."""
    t = wl.grouped_w4a4()
    Wc, Ws, gW = wl.stack_experts(t)
    y = _run(t.A, Wc, Ws, t.A.g, gW, t.offsets)
    assert bool(torch.isfinite(y.float()).all())
    rng = np.random.default_rng(2)
    rows, cols = [], []
    for e in range(t.E):
        lo, hi = int(t.offsets[e]), int(t.offsets[e + 1])
        last = hi - 1  # a row of the ragged (swapped) tail
        for r in (lo, last):
            rows.append(np.full(512, r)); cols.append(rng.choice(t.N, 512, replace=False))
    rows.append(rng.integers(0, t.M, 4096)); cols.append(rng.integers(0, t.N, 4096))
    r = np.concatenate(rows); c = np.concatenate(cols)
    ref = oracle.gemm_grouped_w4a4(t.A.codes, t.A.scales, t.A.g, Wc, Ws, gW.astype(np.float64),
                                   t.offsets, t.N, t.K, rows=r, cols=c)
    check(bf16_to_f64(y)[r, c], ref, "moe sampled")


def test_repeat_is_bitwise_deterministic():
    A, Wc, Ws, gW, off = _random_grouped([70, 300, 5], 384, 512, 11)
    y1 = _run(A, Wc, Ws, 1.0, gW, off)
    y2 = _run(A, Wc, Ws, 1.0, gW, off)
    assert torch.equal(y1.view(torch.int16), y2.view(torch.int16))


def test_offsets_must_cover_all_rows():
    A, Wc, Ws, gW, off = _random_grouped([4, 4], 64, 256, 1)
    with pytest.raises(ValueError):
        nv.gemm_nvfp4_w4a4_grouped(_dev(A.codes), _dev(A.scales), 1.0, _dev(Wc), _dev(Ws),
                                   [1.0, 1.0], [0, 4, 7])
