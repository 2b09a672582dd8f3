"""Pins of the FP64 oracle against things other than itself (CPU only).

Every oracle function is checked against what the formats and the mathematics
fix: a library decode (torch's float8_e4m3fn), the page-1 bit identity over all
16 codes, brute-force triple loops written here with their own decode, an
int64 evaluation that is exact for the tiny workload, a numpy matmul for the
unit-scale special case, and invariants (scale linearity, bilinearity in the
per-tensor scales, sign symmetry, K permutations, -0 == +0).  Each is chosen so
that a dropped term, a wrong sign or index, or a transposed operand in the
oracle fails at least one of them.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from block_scaled_precision_nvfp4_b200 import workloads as wl

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")


# --- independent decoders, written from the bit-field definitions ----------------

def e2m1_fields(c: int) -> float:
    s, e, m = (c >> 3) & 1, (c >> 1) & 3, c & 1
    mag = 0.5 * m if e == 0 else 2.0 ** (e - 1) * (1 + m / 2)
    return -mag if s else mag


def e4m3_torch(b: np.ndarray) -> np.ndarray:
    return torch.from_numpy(np.ascontiguousarray(b, dtype=np.uint8)).view(
        torch.float8_e4m3fn).double().numpy()


def decode_codes(packed: np.ndarray) -> np.ndarray:
    tab = np.array([e2m1_fields(c) for c in range(16)])
    return tab[wl.unpack_codes(packed)]


def brute_w4a4(A, sA, gA, W, sW, gW, M, N, K):
    """Flat triple loop: sum over k of (a*sA)*(w*sW), no group partials."""
    a = decode_codes(A); w = decode_codes(W)
    sa = e4m3_torch(sA); sw = e4m3_torch(sW)
    Y = np.zeros((M, N))
    for m in range(M):
        for n in range(N):
            t = 0.0
            for k in range(K):
                t += (a[m, k] * sa[m, k // 16]) * (w[n, k] * sw[n, k // 16])
            Y[m, n] = float(np.float32(gA)) * float(np.float32(gW)) * t
    return Y


# --- tables ----------------------------------------------------------------------

def test_e4m3_table_matches_library():
    ours = np.array([oracle.e4m3_value(b) for b in range(256)])
    ref = e4m3_torch(np.arange(256, dtype=np.uint8))
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(ours), nan)
    assert nan.sum() == 2 and nan[0x7F] and nan[0xFF]
    assert np.array_equal(ours[~nan], ref[~nan])
    assert oracle.e4m3_value(0x7E) == 448.0 and oracle.e4m3_value(0x01) == 2.0 ** -9


def test_e2m1_table_by_field_definition():
    for c in range(16):
        assert oracle.e2m1_value(c) == e2m1_fields(c)
        assert math.copysign(1.0, oracle.e2m1_value(c)) == (-1.0 if c >= 8 else 1.0)


def test_e2m1_table_by_page_identity():
    """metrale_circuit hardware::exec module doc, bullet 2: the converted byte is value*2^-6
    for all 16 codes (E4M3 decode from the library, not from the oracle)."""
    for c in range(16):
        q = c << 4
        b = oracle.e2m1_to_e4m3_word(q) & 0xFF
        assert e4m3_torch(np.array([b], np.uint8))[0] * 64.0 == oracle.e2m1_value(c)


def test_identity_acts_bytewise_on_words():
    rng = np.random.default_rng(5)
    for q in rng.integers(0, 2 ** 32, size=2000, dtype=np.uint64):
        q = int(q)
        out = oracle.e2m1_to_e4m3_word(q)
        for i in range(4):
            byte = (q >> (8 * i)) & 0xFF
            expect = (byte & 0x80) | ((byte & 0x70) >> 2)
            assert (out >> (8 * i)) & 0xFF == expect


def test_e2m1_matches_torch_fp4_if_available():
    if not hasattr(torch, "float4_e2m1fn_x2"):
        pytest.skip("torch has no float4_e2m1fn_x2")
    try:
        packed = torch.arange(256, dtype=torch.uint8).view(torch.float4_e2m1fn_x2)
        vals = packed.to(torch.float32)  # may be unimplemented
    except Exception:
        pytest.skip("torch cannot convert float4_e2m1fn_x2")
    del vals


# --- GEMM definition -------------------------------------------------------------

@pytest.mark.parametrize("M,N,K", [(1, 1, 16), (2, 3, 32), (4, 4, 48), (3, 2, 64)])
def test_brute_force_tiny(M, N, K):
    rng = np.random.default_rng(M * 100 + N * 10 + K)
    A = wl.random_scale_operand(rng, M, K)
    W = wl.random_scale_operand(rng, N, K)
    gA, gW = 0.75, 1.25
    Y = oracle.gemm_w4a4(A.codes, A.scales, gA, W.codes, W.scales, gW, M, N, K)
    ref = brute_w4a4(A.codes, A.scales, gA, W.codes, W.scales, gW, M, N, K)
    assert np.array_equal(Y, ref)


def _int64_exact(A, W, M, N, K):
    """Y * 2^10 for codes in E2M1 and scales 2^k (k in [-4,4]): an exact integer sum."""
    twice = np.array([int(round(2 * e2m1_fields(c))) for c in range(16)], dtype=np.int64)
    a = twice[wl.unpack_codes(A.codes)]
    w = twice[wl.unpack_codes(W.codes)]
    ka = (A.scales.astype(np.int64) >> 3) - 7 + 4  # 2^(k+4), integer in [1, 256]
    kw = (W.scales.astype(np.int64) >> 3) - 7 + 4
    sa = np.left_shift(1, ka).repeat(16, axis=1)
    sw = np.left_shift(1, kw).repeat(16, axis=1)
    return (a * sa) @ (w * sw).T  # int64 matmul: exact


def test_tiny_workload_exact_int64():
    t = wl.tiny_w4a4(seed=0)
    Y = oracle.gemm_w4a4(t.A.codes, t.A.scales, t.A.g, t.W.codes, t.W.scales, t.W.g,
                         t.M, t.N, t.K)
    exact = _int64_exact(t.A, t.W, t.M, t.N, t.K)
    assert np.array_equal(Y * 1024.0, exact.astype(np.float64))
    assert np.abs(exact).max() < 2 ** 53 and np.any(exact != 0)


def test_unit_scales_reduce_to_library_matmul():
    rng = np.random.default_rng(11)
    M, N, K = 33, 17, 96
    A = wl.uniform_operand(rng, M, K, 0, 0)
    W = wl.uniform_operand(rng, N, K, 0, 0)
    assert np.all(A.scales == 0x38) and np.all(W.scales == 0x38)  # E4M3 1.0
    Y = oracle.gemm_w4a4(A.codes, A.scales, 1.0, W.codes, W.scales, 1.0, M, N, K)
    ref = decode_codes(A.codes) @ decode_codes(W.codes).T
    assert np.array_equal(Y, ref)


def test_transposed_operand_is_caught():
    """Y must be A.W^T (W stored [N,K]); swapping the operand roles gives Y^T, not Y."""
    rng = np.random.default_rng(12)
    M = N = 8
    K = 64
    A = wl.uniform_operand(rng, M, K); W = wl.uniform_operand(rng, N, K)
    Y = oracle.gemm_w4a4(A.codes, A.scales, 1, W.codes, W.scales, 1, M, N, K)
    Yt = oracle.gemm_w4a4(W.codes, W.scales, 1, A.codes, A.scales, 1, N, M, K)
    assert np.array_equal(Y, Yt.T)
    ref = _int64_exact(A, W, M, N, K) / 1024.0
    assert np.array_equal(Y, ref) and not np.array_equal(Y, ref.T)


# --- invariants --------------------------------------------------------------------

def _tiny(seed=3, M=6, N=5, K=64):
    rng = np.random.default_rng(seed)
    return wl.uniform_operand(rng, M, K), wl.uniform_operand(rng, N, K), M, N, K


def test_scale_linearity_per_group():
    A, W, M, N, K = _tiny()
    Y0 = oracle.gemm_w4a4(A.codes, A.scales, 1, W.codes, W.scales, 1, M, N, K)
    m, g = 2, 1
    s2 = A.scales.copy(); s2[m, g] += 8  # exponent + 1: scale doubles exactly
    Y1 = oracle.gemm_w4a4(A.codes, s2, 1, W.codes, W.scales, 1, M, N, K)
    only = np.zeros_like(A.scales); only[m, g] = A.scales[m, g]  # zero bytes elsewhere
    Yg = oracle.gemm_w4a4(A.codes, only, 1, W.codes, W.scales, 1, M, N, K)
    assert np.array_equal(Y1 - Y0, Yg)
    assert np.array_equal(np.delete(Y1, m, 0), np.delete(Y0, m, 0))
    assert np.any(Yg[m] != 0)


def test_bilinear_in_tensor_scales():
    A, W, M, N, K = _tiny(4)
    Y = oracle.gemm_w4a4(A.codes, A.scales, 1, W.codes, W.scales, 1, M, N, K)
    Y2 = oracle.gemm_w4a4(A.codes, A.scales, 2.0, W.codes, W.scales, 0.375, M, N, K)
    assert np.array_equal(Y2, Y * 0.75)


def test_sign_symmetry_row():
    A, W, M, N, K = _tiny(5)
    Y = oracle.gemm_w4a4(A.codes, A.scales, 1, W.codes, W.scales, 1, M, N, K)
    c2 = A.codes.copy(); c2[1] ^= 0x88  # flip both sign bits of every byte of row 1
    Yn = oracle.gemm_w4a4(c2, A.scales, 1, W.codes, W.scales, 1, M, N, K)
    assert np.array_equal(Yn[1], -Y[1] + 0.0)
    assert np.array_equal(np.delete(Yn, 1, 0), np.delete(Y, 1, 0))


def test_joint_permutation_within_group_and_of_groups():
    A, W, M, N, K = _tiny(6)
    Y = oracle.gemm_w4a4(A.codes, A.scales, 1, W.codes, W.scales, 1, M, N, K)
    rng = np.random.default_rng(7)
    ca, cw = wl.unpack_codes(A.codes), wl.unpack_codes(W.codes)
    perm = np.concatenate([16 * g + rng.permutation(16) for g in range(K // 16)])
    Yp = oracle.gemm_w4a4(wl.pack_codes(ca[:, perm]), A.scales, 1, wl.pack_codes(cw[:, perm]),
                          W.scales, 1, M, N, K)
    assert np.array_equal(Yp, Y)
    gp = rng.permutation(K // 16)
    kp = np.concatenate([np.arange(16 * g, 16 * g + 16) for g in gp])
    Yg = oracle.gemm_w4a4(wl.pack_codes(ca[:, kp]), A.scales[:, gp], 1,
                          wl.pack_codes(cw[:, kp]), W.scales[:, gp], 1, M, N, K)
    assert np.array_equal(Yg, Y)
    # permuting A alone (not W) must change the result
    Yb = oracle.gemm_w4a4(wl.pack_codes(ca[:, perm]), A.scales, 1, W.codes, W.scales, 1, M, N, K)
    assert not np.array_equal(Yb, Y)


def test_negative_zero_code():
    A, W, M, N, K = _tiny(8)
    ca = wl.unpack_codes(A.codes)
    z = ca.copy(); z[ca == 8] = 0
    Y = oracle.gemm_w4a4(A.codes, A.scales, 1, W.codes, W.scales, 1, M, N, K)
    Yz = oracle.gemm_w4a4(wl.pack_codes(z), A.scales, 1, W.codes, W.scales, 1, M, N, K)
    assert np.array_equal(Y, Yz)


def test_nibble_order_matters_for_one_operand():
    """Even k sits in the low nibble: swapping the nibbles of A alone pairs each A code
    with the wrong W code and changes Y; swapping both operands leaves Y unchanged."""
    A, W, M, N, K = _tiny(9)
    sw = ((A.codes & 0x0F) << 4) | (A.codes >> 4)
    Y = oracle.gemm_w4a4(A.codes, A.scales, 1, W.codes, W.scales, 1, M, N, K)
    Ys = oracle.gemm_w4a4(sw, A.scales, 1, W.codes, W.scales, 1, M, N, K)
    assert not np.array_equal(Y, Ys)
    # swapping both operands' nibbles permutes k within each pair: Y unchanged
    sww = ((W.codes & 0x0F) << 4) | (W.codes >> 4)
    assert np.array_equal(Y, oracle.gemm_w4a4(sw, A.scales, 1, sww, W.scales, 1, M, N, K))


# --- the sibling paths -----------------------------------------------------------

@pytest.mark.parametrize("seed", [0, 1, 2])
def test_via_fp8_equals_w4a4_exactly(seed):
    """hardware::exec bullet 2: 'the same products as the declared W4A4'."""
    rng = np.random.default_rng(seed)
    M, N, K = 9, 13, 128
    A = wl.random_scale_operand(rng, M, K); W = wl.random_scale_operand(rng, N, K)
    Y = oracle.gemm_w4a4(A.codes, A.scales, 0.5, W.codes, W.scales, 3.0, M, N, K)
    Y8 = oracle.gemm_via_fp8(A.codes, A.scales, 0.5, W.codes, W.scales, 3.0, M, N, K)
    assert np.array_equal(Y, Y8)


def test_w4a16_brute_force():
    rng = np.random.default_rng(21)
    M, N, K = 3, 4, 48
    A = wl.to_bf16_bits(rng.standard_normal((M, K), dtype=np.float32))
    W = wl.random_scale_operand(rng, N, K)
    Y = oracle.gemm_w4a16(A, W.codes, W.scales, 0.625, M, N, K)
    a = torch.from_numpy(A.view(np.int16)).view(torch.bfloat16).double().numpy()
    w = decode_codes(W.codes) * e4m3_torch(W.scales).repeat(16, axis=1)
    ref = np.zeros((M, N))
    for m in range(M):
        for n in range(N):
            ref[m, n] = 0.625 * sum(a[m, k] * w[n, k] for k in range(K))
    np.testing.assert_allclose(Y, ref, rtol=1e-13, atol=1e-300)


def test_w4a16_reduces_to_w4a4_when_activations_are_nvfp4_values():
    """BF16 activations equal to e2m1*sA (exact in BF16) make W4A16 == W4A4 exactly."""
    rng = np.random.default_rng(22)
    M, N, K = 7, 9, 64
    A = wl.uniform_operand(rng, M, K); W = wl.random_scale_operand(rng, N, K)
    vals = decode_codes(A.codes) * e4m3_torch(A.scales).repeat(16, axis=1)
    bits = wl.to_bf16_bits(vals.astype(np.float32))
    back = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).double().numpy()
    assert np.array_equal(back, vals)
    Y16 = oracle.gemm_w4a16(bits, W.codes, W.scales, 1.5, M, N, K)
    Y4 = oracle.gemm_w4a4(A.codes, A.scales, 1.0, W.codes, W.scales, 1.5, M, N, K)
    assert np.array_equal(Y16, Y4)


def test_grouped_equals_per_expert_calls():
    rng = np.random.default_rng(31)
    E, N, K = 4, 12, 64
    counts = [5, 0, 9, 3]
    off = np.concatenate([[0], np.cumsum(counts)]).astype(np.int64)
    M = int(off[-1])
    A = wl.uniform_operand(rng, M, K)
    Ws = [wl.random_scale_operand(rng, N, K) for _ in range(E)]
    gW = np.array([0.5, 1.0, 2.0, 0.25])
    Y = oracle.gemm_grouped_w4a4(A.codes, A.scales, 1.5, np.stack([w.codes for w in Ws]),
                                 np.stack([w.scales for w in Ws]), gW, off, N, K)
    for e in range(E):
        r0, r1 = off[e], off[e + 1]
        if r1 == r0:
            continue
        ref = oracle.gemm_w4a4(A.codes[r0:r1], A.scales[r0:r1], 1.5, Ws[e].codes, Ws[e].scales,
                               gW[e], r1 - r0, N, K)
        assert np.array_equal(Y[r0:r1], ref)


def test_sampled_equals_dense():
    t = wl.tiny_w4a4(seed=0)
    Y = oracle.gemm_w4a4(t.A.codes, t.A.scales, 1, t.W.codes, t.W.scales, 1, t.M, t.N, t.K)
    rng = np.random.default_rng(0)
    r = rng.integers(0, t.M, 300); c = rng.integers(0, t.N, 300)
    s = oracle.gemm_w4a4(t.A.codes, t.A.scales, 1, t.W.codes, t.W.scales, 1, t.M, t.N, t.K,
                         rows=r, cols=c)
    assert np.array_equal(s, Y[r, c])
    s8 = oracle.gemm_via_fp8(t.A.codes, t.A.scales, 1, t.W.codes, t.W.scales, 1, t.M, t.N, t.K,
                             rows=r, cols=c)
    assert np.array_equal(s8, Y[r, c])


def test_oracle_rejects_bad_shapes():
    with pytest.raises(ValueError):
        oracle.gemm_w4a4(np.zeros((1, 4), np.uint8), np.zeros((1, 0), np.uint8), 1,
                         np.zeros((1, 4), np.uint8), np.zeros((1, 0), np.uint8), 1, 1, 1, 8)
