"""Every output element of the full-size workloads against the oracle.

The FFN-down product (4096 x 5376 x 14336) through every entry point that computes
it -- the plain-scale single-SM kernel, the SM-pair kernel with whole tiles and with
the last waves cut between pairs (the benchmark's launch), and the exact FP8 path --
the W4A8 product on the same shape, and the 8-expert grouped product (8192 routed
tokens, 14336 x 4096 experts) through the host-planned and the device-offset entry
points, and the activation quantiser on the FFN-down activations.  Each oracle
result is computed once per session and shared; each comparison asserts that all
outputs were compared."""
import functools

import numpy as np
import pytest
import torch

import oracle
import block_scaled_precision_nvfp4_b200 as nv
from block_scaled_precision_nvfp4_b200 import workloads as wl

from parity import Accum

pytestmark = pytest.mark.gpu
CHUNK = 512  # rows moved to the host and compared at a time


def _dev(x):
    return torch.from_numpy(np.ascontiguousarray(x)).cuda()


def _compare_all(y, ref_rows, M, N, what):
    """ref_rows(r0, r1) -> the FP64 reference of rows r0..r1-1."""
    acc = Accum(what)
    for r0 in range(0, M, CHUNK):
        r1 = min(M, r0 + CHUNK)
        got = y[r0:r1].float().cpu().numpy().astype(np.float64)
        acc.add(got, ref_rows(r0, r1))
    return acc.finish(M * N)


@functools.lru_cache(maxsize=None)
def _ffn():
    t = wl.ffn_down_w4a4()
    ref = oracle.gemm_w4a4(t.A.codes, t.A.scales, t.A.g, t.W.codes, t.W.scales, t.W.g,
                           t.M, t.N, t.K)
    return t, ref


@pytest.mark.parametrize("path", ["plain", "pair", "pair_stream_k", "via_fp8"])
def test_ffn_down_every_output(path):
    t, ref = _ffn()
    A, sA, W, sW = _dev(t.A.codes), _dev(t.A.scales), _dev(t.W.codes), _dev(t.W.scales)
    if path == "plain":
        y = nv.gemm_nvfp4_w4a4(A, sA, t.A.g, W, sW, t.W.g)
    elif path == "via_fp8":
        y = nv.gemm_nvfp4_via_fp8(A, sA, t.A.g, W, sW, t.W.g)
    else:
        sa, sw = nv.nvfp4_prepare_scales(sA), nv.nvfp4_prepare_scales(sW)
        ws = nv.w4a4_packed_workspace(t.M, t.N, t.K) if path == "pair_stream_k" else None
        if path == "pair_stream_k":
            assert ws is not None, "the benchmark's shape must cut its last waves"
        y = nv.gemm_nvfp4_w4a4_packed(A, sa, t.A.g, W, sw, t.W.g, workspace=ws)
    torch.cuda.synchronize()
    nv.nvfp4_check_device_error()
    _compare_all(y, lambda r0, r1: ref[r0:r1], t.M, t.N, f"ffn_down {path}")


def test_w4a8_every_output():
    t = wl.w4a8_ffn_down()
    y = nv.gemm_nvfp4_w4a8(_dev(t.A_fp8), t.gA, _dev(t.W.codes), _dev(t.W.scales), t.W.g)
    torch.cuda.synchronize()
    nv.nvfp4_check_device_error()
    ref = oracle.gemm_w4a8(t.A_fp8, t.gA, t.W.codes, t.W.scales, t.W.g, t.M, t.N, t.K)
    _compare_all(y, lambda r0, r1: ref[r0:r1], t.M, t.N, "w4a8 ffn_down")


@functools.lru_cache(maxsize=None)
def _grouped():
    t = wl.grouped_w4a4()
    Wc, Ws, gW = wl.stack_experts(t)
    off = t.offsets
    # per-expert FP64 references (the grouped definition is the per-expert product)
    refs = []
    for e in range(t.E):
        r0, r1 = int(off[e]), int(off[e + 1])
        refs.append(oracle.gemm_w4a4(t.A.codes[r0:r1], t.A.scales[r0:r1], t.A.g, Wc[e], Ws[e],
                                     float(gW[e]), r1 - r0, t.N, t.K) if r1 > r0 else None)
    return t, Wc, Ws, gW, refs


@pytest.mark.parametrize("path", ["host_planned_pair", "device_offsets"])
def test_grouped_every_output(path):
    t, Wc, Ws, gW, refs = _grouped()
    off = t.offsets
    A, sA = _dev(t.A.codes), _dev(t.A.scales)
    if path == "device_offsets":
        y = nv.gemm_nvfp4_w4a4_grouped(A, sA, t.A.g, _dev(Wc), _dev(Ws), list(gW),
                                       _dev(off.astype(np.int32)))
    else:
        sw = nv.nvfp4_pack_scales_grouped(_dev(Ws.reshape(t.E * t.N, -1)),
                                          [e * t.N for e in range(t.E + 1)], t.K)
        sa = nv.nvfp4_pack_scales_grouped(sA, list(off), t.K)
        y = nv.gemm_nvfp4_w4a4_grouped_packed(A, sa, t.A.g, _dev(Wc), sw, list(gW), list(off))
    torch.cuda.synchronize()
    nv.nvfp4_check_device_error()
    acc = Accum(f"grouped {path}")
    for e in range(t.E):
        r0, r1 = int(off[e]), int(off[e + 1])
        for c0 in range(r0, r1, CHUNK):
            c1 = min(r1, c0 + CHUNK)
            acc.add(y[c0:c1].float().cpu().numpy().astype(np.float64), refs[e][c0 - r0:c1 - r0])
    acc.finish(t.M * t.N)


def test_quantiser_every_element_full_size():
    """The FFN-down activations (4096 x 14336 BF16): every code, every plain and packed
    scale byte and g, bit for bit against the oracle's quantiser.  The tensor holds a
    few -0 inputs inside groups with a nonzero scale, whose codes must keep the sign."""
    from oracle import quantize as oq
    from parity import packed_reference
    t = wl.activations_bf16()
    bits = t.A_bf16.view(np.uint16)
    x = _dev(bits.view(np.int16)).view(torch.bfloat16)
    codes, s, sp, g = nv.nvfp4_quantize_bf16(x, plain=True, packed=True)
    torch.cuda.synchronize()
    nv.nvfp4_check_device_error()
    rc, rs, rg = oq.quantize_nvfp4_bf16(bits)
    assert float(g.cpu().numpy()[0]) == float(rg)
    got = codes.cpu().numpy()
    assert got.shape == rc.shape
    bad = np.argwhere(got != rc)
    assert bad.size == 0, f"{len(bad)} code bytes differ, first {bad[:5]}"
    assert np.array_equal(s.cpu().numpy(), rs)
    ref = packed_reference(rs, bits.shape[1])
    assert np.array_equal(sp.cpu().numpy()[:ref.size], ref)
