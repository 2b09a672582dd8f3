"""The pair kernel with its last waves balanced over the pairs (stream-K): parity with
the oracle on shapes whose tiles do not divide among the pairs, cut at many different
K-blocks; a fixed output from run to run; the workspace's tickets back at zero after
every call; the full FFN-down shape on sampled outputs."""
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


def _sms():
    return torch.cuda.get_device_properties(0).multi_processor_count


def _pairs(M, N, max_pairs):
    tiles = -(-M // 256) * -(-N // 256)
    p = min(tiles, _sms() // 2)
    return min(p, max_pairs) if max_pairs else p


def _run(A, W, gA, gW, K, max_pairs, ws="alloc"):
    M, N = A.codes.shape[0], W.codes.shape[0]
    sa = nv.nvfp4_pack_scales(_dev(A.scales), K)
    sw = nv.nvfp4_pack_scales(_dev(W.scales), K)
    if ws == "alloc":
        ws = nv.w4a4_packed_workspace(M, N, K, max_pairs)
    y = nv.gemm_nvfp4_w4a4_packed(_dev(A.codes), sa, gA, _dev(W.codes), sw, gW, workspace=ws,
                                  max_pairs=max_pairs)
    torch.cuda.synchronize()
    nv.nvfp4_check_device_error()
    return y, ws


# (M, N, K, max_pairs): tiles = ceil(M/256) * ceil(N/256) that leave a part-full
# last wave on that many pairs, so the last waves are cut into K-block ranges
SPLIT = [(768, 1024, 1024, 5),      # 12 tiles on 5 pairs: 5 whole, 7 cut over 4 K-blocks each
         (513, 776, 1280, 5),       # ragged M and N, 5 K-blocks
         (300, 1000, 2304, 6),      # 8 tiles on 6 pairs, 9 K-blocks
         (1000, 72, 4096, 3),       # 4 tiles on 3 pairs: every pair cuts
         (64, 1000, 2048, 3),       # M below one tile
         (2560, 2048, 512, 0),      # 80 tiles on all pairs (74 on a 148-SM part), 2 K-blocks
         (1280, 1536, 768, 7),      # 30 tiles on 7 pairs, 3 K-blocks
         (512, 520, 3072, 4)]       # 6 tiles on 4 pairs, N tail of 8 columns


@pytest.mark.parametrize("M,N,K,max_pairs", SPLIT)
def test_split_parity(M, N, K, max_pairs):
    assert nv.nvfp4_w4a4_packed_workspace_bytes(M, N, K, max_pairs) > 0, "shape does not split"
    rng = np.random.default_rng(M * 131 + N * 7 + K + max_pairs)
    A = wl.uniform_operand(rng, M, K)
    W = wl.uniform_operand(rng, N, K)
    y, ws = _run(A, W, 0.75, 1.5, K, max_pairs)
    ref = oracle.gemm_w4a4(A.codes, A.scales, 0.75, W.codes, W.scales, 1.5, M, N, K)
    check(bf16_to_f64(y), ref, f"split {M}x{N}x{K} on {max_pairs} pairs")
    # every ticket is back at zero, ready for the next call
    assert int(ws[:(_pairs(M, N, max_pairs) - 1) * 64].count_nonzero()) == 0
    # a second call with the same workspace gives the same bytes
    y2, _ = _run(A, W, 0.75, 1.5, K, max_pairs, ws=ws)
    assert torch.equal(y.view(torch.int16), y2.view(torch.int16))


def test_split_and_whole_tiles_agree_closely():
    """Cutting a tile's K range changes only where FP32 accumulation is split: the two
    entries agree to within the BF16 rounding of the output."""
    rng = np.random.Generator(np.random.PCG64(12))
    M, N, K = 768, 1024, 4096
    A = wl.quantize_nvfp4(rng.standard_normal((M, K), dtype=np.float32))
    W = wl.quantize_nvfp4(rng.standard_normal((N, K), dtype=np.float32) * np.float32(0.02))
    ys, _ = _run(A, W, A.g, W.g, K, 5)
    yw = nv.gemm_nvfp4_w4a4_packed(_dev(A.codes), nv.nvfp4_pack_scales(_dev(A.scales), K), A.g,
                                   _dev(W.codes), nv.nvfp4_pack_scales(_dev(W.scales), K), W.g)
    torch.cuda.synchronize()
    a, b = bf16_to_f64(ys), bf16_to_f64(yw)
    # one BF16 step of the larger, plus FP32 reassociation noise far below it (outputs
    # that cancel to near zero are where the split's rounding can show)
    tol = 2.0 ** -7 * np.maximum(np.abs(a), np.abs(b)) + 2.0 ** -12 * np.max(np.abs(b))
    assert np.all(np.abs(a - b) <= tol)
    assert np.mean(a == b) > 0.9
    ref = oracle.gemm_w4a4(A.codes, A.scales, A.g, W.codes, W.scales, W.g, M, N, K)
    check(a, ref, "split")


def test_even_tiles_need_no_workspace():
    # 4 tiles on 4 pairs, 8 on 4, 2 on 2: whole waves, nothing to balance
    assert nv.nvfp4_w4a4_packed_workspace_bytes(512, 512, 1024, 4) == 0
    assert nv.nvfp4_w4a4_packed_workspace_bytes(1024, 512, 1024, 4) == 0
    assert nv.nvfp4_w4a4_packed_workspace_bytes(256, 512, 1024, 0) == 0
    # a single K-block cannot be cut
    assert nv.nvfp4_w4a4_packed_workspace_bytes(768, 1024, 256, 5) == 0
    # 9 tiles on 5 pairs: the last wave is 80 % full and stays whole; 8 on 5 is cut
    assert nv.nvfp4_w4a4_packed_workspace_bytes(768, 768, 1024, 5) == 0
    assert nv.nvfp4_w4a4_packed_workspace_bytes(512, 1024, 1024, 5) > 0


def test_workspace_size_of_the_ffn_down_shape():
    P = _sms() // 2
    slots = P - 1
    need = (slots * 64 + 255) // 256 * 256 + slots * 2 * 2 * 8 * 32 * 128 * 4
    assert nv.nvfp4_w4a4_packed_workspace_bytes(4096, 5376, 14336, 0) == need


def test_too_small_workspace_is_refused():
    M, N, K = 768, 1024, 1024
    need = nv.nvfp4_w4a4_packed_workspace_bytes(M, N, K, 5)
    A = torch.zeros((M, K // 2), dtype=torch.uint8, device="cuda")
    W = torch.zeros((N, K // 2), dtype=torch.uint8, device="cuda")
    sa = torch.zeros(nv.nvfp4_scale_layout_bytes(M, K), dtype=torch.uint8, device="cuda")
    sw = torch.zeros(nv.nvfp4_scale_layout_bytes(N, K), dtype=torch.uint8, device="cuda")
    ws = torch.zeros(need - 16, dtype=torch.uint8, device="cuda")
    with pytest.raises(nv.NvFp4Error) as e:
        nv.gemm_nvfp4_w4a4_packed(A, sa, 1.0, W, sw, 1.0, workspace=ws, max_pairs=5)
    assert e.value.status == nv.Status.INVALID_ARG


def test_ffn_down_full_size_split_sampled():
    """The bench's launch: 4096 x 5376 x 14336 with the balanced last waves."""
    t = wl.ffn_down_w4a4()
    assert nv.nvfp4_w4a4_packed_workspace_bytes(t.M, t.N, t.K) > 0
    y, ws = _run(t.A, t.W, t.A.g, t.W.g, t.K, 0)
    assert bool(torch.isfinite(y.float()).all())
    rng = np.random.default_rng(5)
    # whole rows of 8 random tokens, plus 4096 scattered outputs
    r = np.concatenate([np.repeat(rng.choice(t.M, 8, replace=False), t.N), rng.integers(0, t.M, 4096)])
    c = np.concatenate([np.tile(np.arange(t.N), 8), rng.integers(0, t.N, 4096)])
    ref = oracle.gemm_w4a4(t.A.codes, t.A.scales, t.A.g, t.W.codes, t.W.scales, t.W.g,
                           t.M, t.N, t.K, rows=r, cols=c)
    check(bf16_to_f64(y)[r, c], ref, "split ffn_down sampled")
    assert int(ws[:(_sms() // 2 - 1) * 64].count_nonzero()) == 0
