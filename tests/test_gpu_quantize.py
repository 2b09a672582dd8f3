"""GPU NVFP4 activation quantiser: bit-exact against the oracle's quantiser, through the C ABI.

Codes, scale bytes, the packed scale layout and g are integer / byte / exact
results, so every comparison is exact."""
import numpy as np
import pytest
import torch

import oracle
from oracle import quantize as oq
import block_scaled_precision_nvfp4_b200 as nv

from parity import bf16_to_f64, check, packed_reference

pytestmark = pytest.mark.gpu


def _bits(x):
    return torch.from_numpy(np.asarray(x, np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def _gpu(bits, plain=True, packed=True):
    x = torch.from_numpy(bits.view(np.int16)).cuda().view(torch.bfloat16)
    codes, s, sp, g = nv.nvfp4_quantize_bf16(x, plain=plain, packed=packed)
    torch.cuda.synchronize()
    nv.nvfp4_check_device_error()
    return (codes.cpu().numpy(), None if s is None else s.cpu().numpy(),
            None if sp is None else sp.cpu().numpy(), float(g.cpu().numpy()[0]))


def _expect_equal(bits, K, plain=True, packed=True):
    c, s, sp, g = _gpu(bits, plain, packed)
    rc, rs, rg = oq.quantize_nvfp4_bf16(bits)
    assert g == float(rg)
    assert np.array_equal(c, rc), f"codes differ at {np.argwhere(c != rc)[:5]}"
    if plain:
        assert np.array_equal(s, rs), f"scales differ at {np.argwhere(s != rs)[:5]}"
    if packed:
        ref = packed_reference(rs, K)
        assert np.array_equal(sp[:ref.size], ref)


SHAPES = [(1, 16), (3, 48), (1, 64), (130, 320), (128, 256), (257, 1024), (64, 4160),
          (1000, 2048)]


@pytest.mark.parametrize("rows,K", SHAPES)
def test_random_shapes_bit_exact(rows, K):
    rng = np.random.default_rng(rows * 7919 + K)
    bits = _bits(rng.standard_normal((rows, K)).astype(np.float32) * np.float32(rng.uniform(0.01, 30)))
    _expect_equal(bits, K, plain=True, packed=(K % 64 == 0))


def test_plain_only_and_packed_only():
    rng = np.random.default_rng(1)
    bits = _bits(rng.standard_normal((200, 512)).astype(np.float32))
    _expect_equal(bits, 512, plain=True, packed=False)
    _expect_equal(bits, 512, plain=False, packed=True)


def test_special_values():
    """Zero rows and blocks, -0 (alone and inside a block with a nonzero scale), tiny
    values that give E4M3-subnormal and zero block scales or quotients that underflow,
    the BF16 extremes, and values at E2M1 midpoints of their block."""
    rng = np.random.default_rng(2)
    x = rng.standard_normal((8, 256)).astype(np.float32)
    x[0] = 0.0                                  # a zero row
    x[1, :16] = -0.0                            # a block of -0
    x[2, 16:32] = 1e-30                         # underflows to a zero scale against the amax
    x[3, :16] = np.float32(3e38)                # the tensor amax near the BF16 maximum
    x[3, 16:32] = -np.float32(3e38)
    x[4, 32:48] = np.float32(1e-5) * rng.standard_normal(16)   # subnormal E4M3 scales
    x[6, 16:32] = rng.standard_normal(16)
    x[6, 17] = -0.0                             # -0 and quotients that underflow, in a
    x[6, 20] = -1e-38                           # group with a nonzero scale: codes -0
    x[6, 21] = 1e-38
    base = np.float32(2.0 ** -3)
    x[5, :16] = base * np.array([6, 0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5, -0.25, -0.75,
                                 -1.25, -1.75, -2.5, -3.5, -5, 0], np.float32)
    _expect_equal(_bits(x), 256)


def test_all_zero_tensor_and_empty():
    _expect_equal(np.zeros((4, 64), np.uint16), 64)
    x = torch.empty((0, 64), dtype=torch.bfloat16, device="cuda")
    codes, s, sp, g = nv.nvfp4_quantize_bf16(x)
    torch.cuda.synchronize()
    assert codes.numel() == 0 and float(g.cpu()[0]) == 1.0


def test_ffn_down_activations_full_size_sampled():
    """The FFN-down activations (4096 x 14336, N(0,1)): the whole GPU result against the
    oracle on sampled rows, with the tensor's amax."""
    rng = np.random.default_rng(0)
    M, K = 4096, 14336
    xb = _bits(rng.standard_normal((M, K), dtype=np.float32))
    c, s, sp, g = _gpu(xb)
    amax = np.max(np.abs(oq.bf16_to_f32(xb)))
    rows = np.concatenate([np.arange(4), rng.choice(M, 60, replace=False), [M - 1]])
    rc, rs, rg = oq.quantize_nvfp4_bf16(xb[rows], amax=amax)
    assert g == float(rg)
    assert np.array_equal(c[rows], rc) and np.array_equal(s[rows], rs)
    ref = packed_reference(s, K)       # the packed copy holds exactly the plain bytes
    assert np.array_equal(sp[:ref.size], ref)


def test_quantised_activations_feed_the_w4a4_product():
    """GPU quantiser -> packed W4A4 product: the result matches the oracle's product of
    the same bytes (the quantiser's packed scales are consumed as they are)."""
    rng = np.random.default_rng(3)
    M, N, K = 300, 256, 1024
    xb = _bits(rng.standard_normal((M, K), dtype=np.float32))
    x = torch.from_numpy(xb.view(np.int16)).cuda().view(torch.bfloat16)
    codes, s, sp, g = nv.nvfp4_quantize_bf16(x)
    from block_scaled_precision_nvfp4_b200 import workloads as wl
    W = wl.quantize_nvfp4(rng.standard_normal((N, K), dtype=np.float32) * np.float32(0.02))
    wd = torch.from_numpy(W.codes).cuda()
    swp = nv.nvfp4_pack_scales(torch.from_numpy(W.scales).cuda(), K)
    gA = float(g.cpu()[0])
    y = nv.gemm_nvfp4_w4a4_packed(codes, sp, gA, wd, swp, W.g)
    torch.cuda.synchronize()
    ref = oracle.gemm_w4a4(codes.cpu().numpy(), s.cpu().numpy(), gA, W.codes, W.scales, W.g, M, N, K)
    check(bf16_to_f64(y), ref, "quantise -> W4A4")


def test_repeat_is_deterministic_and_workspace_reusable():
    rng = np.random.default_rng(4)
    bits = _bits(rng.standard_normal((256, 512)).astype(np.float32))
    x = torch.from_numpy(bits.view(np.int16)).cuda().view(torch.bfloat16)
    ws = torch.full((16,), 0xAB, dtype=torch.uint8, device="cuda")   # garbage: the call clears it
    a = nv.nvfp4_quantize_bf16(x, workspace=ws)
    b = nv.nvfp4_quantize_bf16(x, workspace=ws)
    torch.cuda.synchronize()
    assert all(torch.equal(p, q) for p, q in zip(a, b))


def test_argument_errors():
    x = torch.zeros((4, 40), dtype=torch.bfloat16, device="cuda")   # K % 16 != 0
    with pytest.raises(nv.NvFp4Error) as e:
        nv.nvfp4_quantize_bf16(x)
    assert e.value.status == nv.Status.INVALID_ARG
    x = torch.zeros((4, 48), dtype=torch.bfloat16, device="cuda")   # packed needs K % 64
    with pytest.raises(nv.NvFp4Error) as e:
        nv.nvfp4_quantize_bf16(x, packed=True)
    assert e.value.status == nv.Status.INVALID_ARG


@pytest.mark.parametrize("dist", ["normal", "uniform", "cauchy", "wide"])
def test_every_element_bit_exact_over_distributions(dist):
    """8.4M elements compared one by one: the division by each group's s*g is the
    correctly rounded FP32 quotient, so every code equals the oracle's."""
    rng = np.random.default_rng({"normal": 1, "uniform": 2, "cauchy": 3, "wide": 4}[dist])
    rows, K = 1024, 8192
    if dist == "normal":
        x = rng.standard_normal((rows, K)).astype(np.float32)
    elif dist == "uniform":
        x = rng.uniform(-3, 3, (rows, K)).astype(np.float32)
    elif dist == "cauchy":
        x = np.clip(rng.standard_cauchy((rows, K)), -1e30, 1e30).astype(np.float32)
    else:   # blocks spread over 2^-100 .. 2^100
        x = (rng.standard_normal((rows, K)) *
             np.exp2(rng.integers(-100, 100, size=(rows, K // 16))).repeat(16, axis=1)).astype(np.float32)
    _expect_equal(_bits(x), K)


def _groups_with_maxima(maxima, K, rng):
    """One 16-group per entry of `maxima` (BF16 magnitude bits), row-major over rows of
    K columns, zero-padded: each group holds its maximum once (random place and sign)
    and 15 magnitudes drawn uniformly from [0, maximum]."""
    n = maxima.size
    gpr = K // 16
    rows = -(-n // gpr)
    mx = np.zeros(rows * gpr, np.uint32)
    mx[:n] = maxima
    mags = np.floor(rng.random((rows * gpr, 16)) * (mx[:, None] + 1)).astype(np.uint32)
    mags = np.minimum(mags, mx[:, None])
    mags[np.arange(rows * gpr), rng.integers(0, 16, rows * gpr)] = mx
    sign = rng.integers(0, 2, (rows * gpr, 16)).astype(np.uint32) << 15
    return ((mags | sign).astype(np.uint16)).reshape(rows, K)


@pytest.mark.parametrize("top", [0x7F7F, 0x4700, 0x3F80, 0x2D00, 0x2000, 0x1E00, 0x0400, 0x0100])
def test_every_bf16_group_maximum_bit_exact(top):
    """Every BF16 magnitude up to the tensor's maximum `top` is one group's maximum, so
    each scale quotient amax_b / (6 g) the tensor can produce is taken once and compared
    with the oracle's.  The maxima span both sides of the kernel's range test on 6g
    (448 * 2^-60 and 448 * 2^60 lie between the chosen tops), subnormal group maxima
    included."""
    rng = np.random.default_rng(top)
    maxima = np.arange(0, top + 1, dtype=np.uint32)
    rng.shuffle(maxima)
    K = 1024
    bits = _groups_with_maxima(maxima, K, rng)
    _expect_equal(bits, K)


def test_unaligned_tensor_takes_the_128bit_loads():
    """A tensor that starts 16 bytes past a 32-byte boundary is read with 128-bit loads
    instead of 256-bit ones; the results are the same bytes."""
    rng = np.random.default_rng(77)
    rows, K = 300, 1024
    bits = _bits(rng.standard_normal((rows, K)).astype(np.float32))
    base = torch.zeros(rows * K + 8, dtype=torch.int16, device="cuda")
    base[8:] = torch.from_numpy(bits.view(np.int16).reshape(-1)).cuda()
    x = base[8:].view(torch.bfloat16).view(rows, K)
    assert x.data_ptr() % 32 == 16
    codes, s, sp, g = nv.nvfp4_quantize_bf16(x, plain=True, packed=True)
    torch.cuda.synchronize()
    nv.nvfp4_check_device_error()
    rc, rs, rg = oq.quantize_nvfp4_bf16(bits)
    assert float(g.cpu().numpy()[0]) == float(rg)
    assert np.array_equal(codes.cpu().numpy(), rc)
    assert np.array_equal(s.cpu().numpy(), rs)
    ref = packed_reference(rs, K)
    assert np.array_equal(sp.cpu().numpy()[:ref.size], ref)


@pytest.mark.parametrize("rows,K,E,k", [(1000, 2048, 8, 1), (300, 512, 4, 2), (257, 4160, 8, 1),
                                         (64, 96, 3, 3)])
def test_routed_quantiser_writes_the_dispatch_order(rows, K, E, k):
    """nvfp4_quantize_bf16_routed with the route's dest equals the plain quantiser
    followed by the route's row permutation (out[dest[p]] = row p // k), bit for bit,
    with the same g."""
    rng = np.random.default_rng(rows + K + E + k)
    bits = _bits(rng.standard_normal((rows, K)).astype(np.float32) * np.float32(3.0))
    x = torch.from_numpy(bits.view(np.int16)).cuda().view(torch.bfloat16)
    ids = torch.from_numpy(rng.integers(0, E, size=(rows, k)).astype(np.int32)).cuda()
    off, dest, src = nv.moe_route(ids, E)
    codes, scales, g = nv.nvfp4_quantize_bf16_routed(x, dest, k)
    rc, rs, _, rg = nv.nvfp4_quantize_bf16(x, plain=True, packed=False)
    torch.cuda.synchronize()
    nv.nvfp4_check_device_error()
    assert float(g.cpu()[0]) == float(rg.cpu()[0])
    d = dest.cpu().numpy()
    assert sorted(d.tolist()) == list(range(rows * k))
    rows_of = np.arange(rows * k) // k
    want_c = np.empty((rows * k, K // 2), np.uint8)
    want_s = np.empty((rows * k, K // 16), np.uint8)
    want_c[d] = rc.cpu().numpy()[rows_of]
    want_s[d] = rs.cpu().numpy()[rows_of]
    assert np.array_equal(codes.cpu().numpy(), want_c)
    assert np.array_equal(scales.cpu().numpy(), want_s)


def test_routed_quantiser_skips_pairs_placed_nowhere():
    """A destination outside [0, rows k) (the route's -1) writes nothing: that output
    row keeps what was there, and every other row is the quantised source row."""
    rng = np.random.default_rng(11)
    rows, K, k = 96, 256, 2
    bits = _bits(rng.standard_normal((rows, K)).astype(np.float32))
    x = torch.from_numpy(bits.view(np.int16)).cuda().view(torch.bfloat16)
    d = rng.permutation(rows * k).astype(np.int32)
    hole = int(d[7])
    d[7] = -1
    dest = torch.from_numpy(d).cuda()
    codes = torch.full((rows * k, K // 2), 0xAB, dtype=torch.uint8, device="cuda")
    scales = torch.full((rows * k, K // 16), 0xCD, dtype=torch.uint8, device="cuda")
    g = torch.empty(4, dtype=torch.float32, device="cuda")
    nv.nvfp4_quantize_bf16_routed(x, dest, k, out=(codes, scales, g))
    rc, rs, _, _ = nv.nvfp4_quantize_bf16(x, plain=True, packed=False)
    torch.cuda.synchronize()
    nv.nvfp4_check_device_error()
    c, s = codes.cpu().numpy(), scales.cpu().numpy()
    assert np.all(c[hole] == 0xAB) and np.all(s[hole] == 0xCD)
    rc, rs = rc.cpu().numpy(), rs.cpu().numpy()
    for p in range(rows * k):
        if d[p] >= 0:
            assert np.array_equal(c[d[p]], rc[p // k]) and np.array_equal(s[d[p]], rs[p // k])


def test_routed_quantiser_argument_errors():
    x = torch.zeros((4, 64), dtype=torch.bfloat16, device="cuda")
    dest = torch.arange(4 * 9, dtype=torch.int32, device="cuda")
    with pytest.raises(nv.NvFp4Error) as e:   # k above 8
        nv.nvfp4_quantize_bf16_routed(x, dest, 9)
    assert e.value.status == nv.Status.INVALID_ARG
