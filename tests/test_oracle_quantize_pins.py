"""Pins of the oracle's NVFP4 quantiser (CPU only).

Each pin ties the quantiser to something other than itself: a library routine
(torch's float8_e4m3fn cast), the formats' midpoint tables, exact round trips
of values that are representable by construction, and invariants that any
correct implementation keeps (power-of-two scaling, sign symmetry, block
permutations, zero blocks)."""
import numpy as np
import pytest
import torch

import oracle
from oracle import quantize as oq

E2M1 = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]


def f32(x):
    return np.asarray(x, dtype=np.float32)


def to_bf16_bits(x):
    return torch.from_numpy(f32(x)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def test_tables_are_the_decoders():
    e4, e2 = oq._tables()
    assert list(e2) == E2M1
    assert e4[0] == 0.0 and e4[0x7E] == 448.0 and e4[1] == 2.0 ** -9 and np.all(np.diff(e4) > 0)


def test_e4m3_encoder_matches_torch_cast():
    """Nearest-even E4M3 against torch's float8_e4m3fn cast (a library routine), on a
    sweep holding every value, every midpoint between neighbours (ties), points just
    off the midpoints, subnormals and values up to the saturation point."""
    e4, _ = oq._tables()
    mids = (e4[:-1] + e4[1:]) / 2
    q = np.concatenate([e4, mids, np.nextafter(f32(mids), f32(0)), np.nextafter(f32(mids), f32(1e9)),
                        np.geomspace(1e-6, 447.9, 20000)]).astype(np.float32)
    q = q[(q >= 0) & (q <= 448)]
    ref = torch.from_numpy(q).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(oq.e4m3_rne_satfinite(q), ref)


def test_e4m3_encoder_saturates():
    assert np.all(oq.e4m3_rne_satfinite(f32([448.0, 460.0, 479.9, 480.0, 1e6])) == 0x7E)
    assert oq.e4m3_rne_satfinite(f32([0.0]))[0] == 0


def test_e2m1_midpoints_go_to_even():
    # 0.25 -> 0, 0.75 -> 1, 1.25 -> 1, 1.75 -> 2, 2.5 -> 2, 3.5 -> 4, 5 -> 4
    mids = f32([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0])
    assert [E2M1[c] for c in oq.e2m1_rne_satfinite(mids)] == [0.0, 1.0, 1.0, 2.0, 2.0, 4.0, 4.0]
    below = np.nextafter(mids, f32(0))
    above = np.nextafter(mids, f32(100))
    assert [E2M1[c] for c in oq.e2m1_rne_satfinite(below)] == [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0]
    assert [E2M1[c] for c in oq.e2m1_rne_satfinite(above)] == [0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]


def test_e2m1_signs_and_saturation():
    c = oq.e2m1_rne_satfinite(f32([-0.0, 0.0, -0.1, -6.0, -7.5, 1e9, -1e9, 6.0]))
    assert list(c) == [8, 0, 8, 15, 15, 7, 15, 7]
    # every exact value maps to its own code, both signs
    for code, v in enumerate(E2M1):
        assert oq.e2m1_rne_satfinite(f32([v]))[0] == code
        assert oq.e2m1_rne_satfinite(f32([-v]))[0] == code | 8


def _rand_bf16(rng, rows, K, scale=1.0):
    return to_bf16_bits(rng.standard_normal((rows, K)).astype(np.float32) * np.float32(scale))


def test_global_scale_is_amax_over_2688_in_fp32():
    rng = np.random.default_rng(0)
    x = _rand_bf16(rng, 8, 64)
    _, _, g = oq.quantize_nvfp4_bf16(x)
    amax = np.max(np.abs(oq.bf16_to_f32(x)))
    assert g == np.float32(amax) / np.float32(2688.0)
    _, s, g0 = oq.quantize_nvfp4_bf16(np.zeros((3, 32), np.uint16))
    assert g0 == 1.0 and np.all(s == 0)


def test_representable_blocks_round_trip_exactly():
    """Blocks built as s * e2m1 with the block maximum at 6 s, in a tensor whose
    amax is 2688 (so g = 1): the block scale comes back as s and every code exactly."""
    rng = np.random.default_rng(1)
    e4, _ = oq._tables()
    rows, K = 6, 256
    codes = rng.integers(0, 16, size=(rows, K)).astype(np.uint8)
    codes[:, ::16] = 7                         # each block holds a +6
    sbytes = rng.integers(0x08, 0x70, size=(rows, K // 16)).astype(np.uint8)   # normal scales
    sbytes[0, 0] = 0x7E                        # one block at 448: 6 * 448 = 2688 = amax
    vals = np.array([E2M1[c & 7] * (-1.0 if c & 8 else 1.0) for c in codes.ravel()]).reshape(rows, K)
    x = vals * np.repeat(e4[sbytes], 16, axis=1)
    bits = to_bf16_bits(x)
    assert np.array_equal(oq.bf16_to_f32(bits), x.astype(np.float32))   # exact in BF16
    packed, s, g = oq.quantize_nvfp4_bf16(bits)
    assert g == 1.0
    assert np.array_equal(s, sbytes)
    want = np.where(codes == 8, 8, codes)      # -0 stays -0
    assert np.array_equal(packed, (want[:, 0::2] | (want[:, 1::2] << 4)).astype(np.uint8))


def test_codes_are_nearest_and_scales_are_nearest():
    """Brute force on a small random tensor: every code is a nearest E2M1 magnitude to
    |t| (ties to the even one) and every scale byte a nearest E4M3 value to q."""
    rng = np.random.default_rng(2)
    bits = _rand_bf16(rng, 4, 64, 3.0)
    packed, s, g = oq.quantize_nvfp4_bf16(bits)
    e4, _ = oq._tables()
    x = oq.bf16_to_f32(bits).reshape(4, 4, 16)
    amax_b = np.abs(x).max(axis=2)
    q = (amax_b / np.float32(np.float32(6.0) * g)).astype(np.float32)
    for (i, j), qq in np.ndenumerate(q):
        d = np.abs(e4 - float(qq))
        best = np.flatnonzero(d == d.min())
        assert s[i, j] in best and (len(best) == 1 or s[i, j] % 2 == 0)
    codes = np.empty((4, 64), np.uint8)
    codes[:, 0::2] = packed & 15
    codes[:, 1::2] = packed >> 4
    den = (e4[s].astype(np.float32) * g).astype(np.float32)
    t = (x / den[:, :, None]).astype(np.float32).reshape(4, 64)
    for (i, k), tt in np.ndenumerate(t):
        d = np.abs(np.array(E2M1) - abs(float(tt)))
        best = np.flatnonzero(d == d.min())
        c = codes[i, k]
        assert (c & 7) in best and (len(best) == 1 or (c & 7) % 2 == 0)
        assert bool(c & 8) == bool(np.signbit(tt))


@pytest.mark.parametrize("k", [-3, 2, 7])
def test_power_of_two_scaling_moves_only_g(k):
    rng = np.random.default_rng(3)
    bits = _rand_bf16(rng, 5, 128)
    p0, s0, g0 = oq.quantize_nvfp4_bf16(bits)
    scaled = to_bf16_bits(oq.bf16_to_f32(bits) * np.float32(2.0 ** k))
    p1, s1, g1 = oq.quantize_nvfp4_bf16(scaled)
    assert np.array_equal(p0, p1) and np.array_equal(s0, s1) and g1 == g0 * np.float32(2.0 ** k)


def test_negation_flips_only_the_sign_bits():
    rng = np.random.default_rng(4)
    bits = _rand_bf16(rng, 5, 96)
    p0, s0, g0 = oq.quantize_nvfp4_bf16(bits)
    p1, s1, g1 = oq.quantize_nvfp4_bf16(bits ^ np.uint16(0x8000))
    assert np.array_equal(s0, s1) and g0 == g1 and np.array_equal(p1, p0 ^ np.uint8(0x88))


def test_permuting_a_block_permutes_its_codes():
    rng = np.random.default_rng(5)
    bits = _rand_bf16(rng, 3, 48)
    perm = rng.permutation(16)
    pb = bits.reshape(3, 3, 16)[:, :, perm].reshape(3, 48)
    p0, s0, _ = oq.quantize_nvfp4_bf16(bits)
    p1, s1, _ = oq.quantize_nvfp4_bf16(pb)
    c0 = np.empty((3, 48), np.uint8); c0[:, 0::2] = p0 & 15; c0[:, 1::2] = p0 >> 4
    c1 = np.empty((3, 48), np.uint8); c1[:, 0::2] = p1 & 15; c1[:, 1::2] = p1 >> 4
    assert np.array_equal(s0, s1)
    assert np.array_equal(c0.reshape(3, 3, 16)[:, :, perm].reshape(3, 48), c1)


def test_zero_block_in_a_live_tensor():
    rng = np.random.default_rng(6)
    bits = _rand_bf16(rng, 2, 64)
    bits[1, 16:32] = 0
    p, s, _ = oq.quantize_nvfp4_bf16(bits)
    assert s[1, 1] == 0 and np.all(p[1, 8:16] == 0)


def test_dequantised_error_within_half_a_code_step():
    """|x - value(code) * s * g| <= half the E2M1 step at the chosen code (in units of
    s * g), up to FP32 rounding of t: a bound any nearest-rounding quantiser meets."""
    rng = np.random.default_rng(7)
    bits = _rand_bf16(rng, 16, 256, 0.7)
    p, s, g = oq.quantize_nvfp4_bf16(bits)
    e4, _ = oq._tables()
    codes = np.empty((16, 256), np.uint8); codes[:, 0::2] = p & 15; codes[:, 1::2] = p >> 4
    mag = np.array(E2M1)[codes & 7] * np.where(codes & 8, -1.0, 1.0)
    sg = np.repeat(e4[s], 16, axis=1) * float(g)
    x = oq.bf16_to_f32(bits).astype(np.float64)
    half_step = np.array([0.25, 0.25, 0.25, 0.25, 0.5, 0.5, 1.0, 1.0])[codes & 7]
    assert np.all(np.abs(x - mag * sg) <= half_step * sg * (1 + 2.0 ** -20) + 1e-30)


def test_signed_zero_codes_inside_a_live_block():
    """In a block with a nonzero scale, -0 and a negative value whose quotient rounds to
    zero both give the code -0 (nibble 8), their positive twins +0: the code is the
    signed E2M1 rounding of the IEEE quotient, and x / (s g) keeps x's sign."""
    x = np.zeros(16, np.float32)
    x[0] = 1.0                      # the block maximum: a nonzero scale
    x[1] = -0.0
    x[2] = np.float32(-1e-38)       # BF16 subnormal; the quotient underflows to -0
    x[3] = np.float32(1e-38)
    x[4] = np.float32(-0.01)        # rounds to zero against 1/6 of the max
    bits = to_bf16_bits(x[None, :])
    p, s, g = oq.quantize_nvfp4_bf16(bits)
    assert s[0, 0] != 0
    nib = [(int(p[0, e >> 1]) >> (4 * (e & 1))) & 0xF for e in range(16)]
    assert nib[1] == 8 and nib[2] == 8 and nib[4] == 8
    assert nib[3] == 0 and all(n == 0 for n in nib[5:])
    assert nib[0] != 0
