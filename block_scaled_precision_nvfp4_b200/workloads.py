"""Seeded synthetic NVFP4 workloads (input generation only).

This module produces the bytes that BOTH the GPU library and the FP64 oracle
consume: packed E2M1 codes ``uint8[rows, K/2]`` (even k in the low nibble),
E4M3 group scales ``uint8[rows, K/16]`` and FP32 per-tensor scales.  It holds
none of the matmul's arithmetic: it draws random numbers and encodes them to
NVFP4 with the standard two-level recipe, and nothing here decodes a code.

Quantisation recipe (two-level NVFP4; the per-16 scale and per-tensor scale of
the FFN-down workload description):
    g   = amax(|X|) / (6 * 448)                    (FP32; 1.0 if amax == 0)
    s_b = E4M3_RNE(min(amax_b / (6 g), 448))       (per 16 consecutive k)
    c   = E2M1_RNE_satfinite(x / (s_b g))          (0 where s_b == 0)
with round-to-nearest-even at the E2M1 midpoints 0.25, 0.75, 1.25, 1.75, 2.5,
3.5 and 5.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np
import torch

E4M3_MAX = 448.0
E2M1_MAX = 6.0


@dataclass
class Operand:
    """One NVFP4 operand: packed codes [rows, K/2], E4M3 scales [rows, K/16], FP32 scale."""
    codes: np.ndarray
    scales: np.ndarray
    g: float

    @property
    def rows(self) -> int:
        return self.codes.shape[0]


@dataclass
class Workload:
    name: str
    M: int
    N: int
    K: int
    A: Operand | None = None          # NVFP4 activations (W4A4 paths)
    W: Operand | None = None          # NVFP4 weights [N, K]
    A_bf16: np.ndarray | None = None  # uint16 BF16 bit patterns [M, K] (W4A16)
    A_fp8: np.ndarray | None = None   # uint8 E4M3 bytes [M, K] (W4A8)
    expert_ids: np.ndarray | None = None  # int32 [T, k] top-k routing (MoE layer)
    gA: float = 1.0                   # FP32 per-tensor scale of A_fp8
    # grouped
    E: int = 0
    offsets: np.ndarray | None = None  # int64 [E+1]
    W_e: list = field(default_factory=list)  # per-expert Operand, each [N, K]
    notes: str = ""


# --- encoders --------------------------------------------------------------------

def e4m3_rne(x: np.ndarray) -> np.ndarray:
    """FP32 -> E4M3 byte, round-to-nearest-even, saturated to 448 (torch's cast is RNE)."""
    x = np.clip(np.asarray(x, dtype=np.float32), -E4M3_MAX, E4M3_MAX)
    return torch.from_numpy(np.ascontiguousarray(x)).to(torch.float8_e4m3fn).view(
        torch.uint8).numpy()


def e2m1_rne(t: np.ndarray) -> np.ndarray:
    """FP32 -> 4-bit E2M1 code (sign in bit 3), RNE, saturating at 6."""
    t = np.asarray(t, dtype=np.float32)
    a = np.abs(t)
    mag = ((a > 0.25).astype(np.uint8) + (a >= 0.75) + (a > 1.25) + (a >= 1.75)
           + (a > 2.5) + (a >= 3.5) + (a > 5.0)).astype(np.uint8)
    sign = (np.signbit(t) & (mag > 0)).astype(np.uint8) << 3
    return mag | sign


def pack_codes(codes: np.ndarray) -> np.ndarray:
    """[rows, K] 4-bit codes -> [rows, K/2] bytes, even k in the low nibble."""
    codes = np.asarray(codes, dtype=np.uint8)
    return np.ascontiguousarray(codes[:, 0::2] | (codes[:, 1::2] << 4))


def unpack_codes(packed: np.ndarray) -> np.ndarray:
    """Inverse of pack_codes (bit shuffling only)."""
    packed = np.asarray(packed, dtype=np.uint8)
    out = np.empty((packed.shape[0], packed.shape[1] * 2), dtype=np.uint8)
    out[:, 0::2] = packed & 0x0F
    out[:, 1::2] = packed >> 4
    return out


def quantize_nvfp4(x: np.ndarray) -> Operand:
    """Two-level NVFP4 quantisation of an FP32 [rows, K] matrix (K % 16 == 0)."""
    x = np.asarray(x, dtype=np.float32)
    rows, K = x.shape
    assert K % 16 == 0
    amax = float(np.max(np.abs(x))) if x.size else 0.0
    g = np.float32(amax / (6.0 * E4M3_MAX)) if amax > 0 else np.float32(1.0)
    xb = x.reshape(rows, K // 16, 16)
    amax_b = np.max(np.abs(xb), axis=2)
    s_bytes = e4m3_rne(amax_b / (np.float32(6.0) * g))
    s_vals = torch.from_numpy(s_bytes).view(torch.float8_e4m3fn).float().numpy()
    denom = (s_vals * g)[:, :, None]
    with np.errstate(divide="ignore", invalid="ignore"):
        t = np.where(denom > 0, xb / np.where(denom > 0, denom, 1.0), 0.0).astype(np.float32)
    codes = e2m1_rne(t).reshape(rows, K)
    return Operand(pack_codes(codes), np.ascontiguousarray(s_bytes), float(g))


def quantize_nvfp4_chunked(rng: np.random.Generator, rows: int, K: int, std: float,
                           chunk_rows: int = 2048) -> Operand:
    """N(0, std) [rows, K] drawn and quantised in row chunks (bounded memory).

    The per-tensor scale needs the global amax first, so the rows are drawn
    twice from the same seed state: once for amax, once for the codes.
    """
    state = rng.bit_generator.state
    amax = 0.0
    for r0 in range(0, rows, chunk_rows):
        r1 = min(rows, r0 + chunk_rows)
        amax = max(amax, float(np.max(np.abs(
            rng.standard_normal((r1 - r0, K), dtype=np.float32) * np.float32(std)))))
    rng.bit_generator.state = state
    g = np.float32(amax / (6.0 * E4M3_MAX)) if amax > 0 else np.float32(1.0)
    codes = np.empty((rows, K // 2), dtype=np.uint8)
    scales = np.empty((rows, K // 16), dtype=np.uint8)
    for r0 in range(0, rows, chunk_rows):
        r1 = min(rows, r0 + chunk_rows)
        x = rng.standard_normal((r1 - r0, K), dtype=np.float32) * np.float32(std)
        xb = x.reshape(r1 - r0, K // 16, 16)
        s_bytes = e4m3_rne(np.max(np.abs(xb), axis=2) / (np.float32(6.0) * g))
        s_vals = torch.from_numpy(s_bytes).view(torch.float8_e4m3fn).float().numpy()
        denom = (s_vals * g)[:, :, None]
        with np.errstate(divide="ignore", invalid="ignore"):
            t = np.where(denom > 0, xb / np.where(denom > 0, denom, 1.0), 0.0).astype(np.float32)
        codes[r0:r1] = pack_codes(e2m1_rne(t).reshape(r1 - r0, K))
        scales[r0:r1] = s_bytes
    return Operand(codes, scales, float(g))


def to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """FP32 -> BF16 bit patterns (uint16), round-to-nearest-even (torch's cast)."""
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(
        torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


# --- uniform-code generators (tiny / parity sweeps) ---------------------------------

def uniform_operand(rng: np.random.Generator, rows: int, K: int, kmin: int = -4,
                    kmax: int = 4) -> Operand:
    """Codes uniform over all 16 values; scales 2^k, k uniform in [kmin, kmax], g = 1."""
    codes = rng.integers(0, 16, size=(rows, K), dtype=np.uint8)
    k = rng.integers(kmin, kmax + 1, size=(rows, K // 16))
    return Operand(pack_codes(codes), ((k + 7) << 3).astype(np.uint8), 1.0)


def random_scale_operand(rng: np.random.Generator, rows: int, K: int) -> Operand:
    """Codes uniform; scale bytes uniform over all finite non-negative E4M3 (0x00..0x7E)."""
    codes = rng.integers(0, 16, size=(rows, K), dtype=np.uint8)
    scales = rng.integers(0, 0x7F, size=(rows, K // 16), dtype=np.uint8)
    return Operand(pack_codes(codes), scales, 1.0)


# --- the five workloads -----------------------------------------------------------

def tiny_w4a4(seed: int = 0, M: int = 128, N: int = 256, K: int = 256) -> Workload:
    """Uniform codes, scales 2^U{-4..4}, g = 1; one stream: A codes, W codes, sA, sW."""
    rng = np.random.Generator(np.random.PCG64(seed))
    a = rng.integers(0, 16, size=(M, K), dtype=np.uint8)
    w = rng.integers(0, 16, size=(N, K), dtype=np.uint8)
    ka = rng.integers(-4, 5, size=(M, K // 16))
    kw = rng.integers(-4, 5, size=(N, K // 16))
    A = Operand(pack_codes(a), ((ka + 7) << 3).astype(np.uint8), 1.0)
    W = Operand(pack_codes(w), ((kw + 7) << 3).astype(np.uint8), 1.0)
    return Workload("tiny_w4a4_128x256x256", M, N, K, A=A, W=W,
                    notes="codes U{0..15}, scales 2^U{-4..4}, g=1, seed %d" % seed)


def ffn_down_w4a4(M: int = 4096, N: int = 5376, K: int = 14336, seed_a: int = 0,
                  seed_w: int = 1) -> Workload:
    """FFN down projection: A ~ N(0,1) [M,K] (seed 0), W ~ N(0,0.02) [N,K] (seed 1)."""
    A = quantize_nvfp4_chunked(np.random.Generator(np.random.PCG64(seed_a)), M, K, 1.0)
    W = quantize_nvfp4_chunked(np.random.Generator(np.random.PCG64(seed_w)), N, K, 0.02)
    return Workload(f"ffn_down_w4a4_{M}x{N}x{K}", M, N, K, A=A, W=W,
                    notes="A~N(0,1) seed %d, W~N(0,0.02) seed %d, two-level NVFP4" % (
                        seed_a, seed_w))


def w4a16_decode(M: int = 16, N: int = 5376, K: int = 14336, seed_a: int = 0,
                 seed_w: int = 1) -> Workload:
    """W4A16 decode: BF16 A ~ N(0,1) [M,K] (seed 0); W as the FFN-down weights (seed 1)."""
    rng = np.random.Generator(np.random.PCG64(seed_a))
    A = to_bf16_bits(rng.standard_normal((M, K), dtype=np.float32))
    W = quantize_nvfp4_chunked(np.random.Generator(np.random.PCG64(seed_w)), N, K, 0.02)
    return Workload(f"w4a16_decode_{M}x{N}x{K}", M, N, K, W=W, A_bf16=A,
                    notes="A bf16 N(0,1) seed %d, W~N(0,0.02) seed %d" % (seed_a, seed_w))


def activations_bf16(M: int = 4096, K: int = 14336, seed: int = 0) -> Workload:
    """The FFN-down activations before quantisation: BF16 N(0,1) [M,K] (seed 0)."""
    rng = np.random.Generator(np.random.PCG64(seed))
    A = to_bf16_bits(rng.standard_normal((M, K), dtype=np.float32))
    return Workload(f"quantize_bf16_{M}x{K}", M, 0, K, A_bf16=A,
                    notes="X bf16 N(0,1) seed %d" % seed)


def fp8_per_tensor(rng: np.random.Generator, rows: int, K: int, std: float = 1.0,
                   chunk_rows: int = 2048) -> tuple[np.ndarray, float]:
    """N(0, std) [rows, K] as E4M3 bytes with one FP32 per-tensor scale gA = amax/448
    (x / gA rounded to nearest even by torch's cast), drawn in row chunks."""
    state = rng.bit_generator.state
    amax = 0.0
    for r0 in range(0, rows, chunk_rows):
        r1 = min(rows, r0 + chunk_rows)
        amax = max(amax, float(np.max(np.abs(
            rng.standard_normal((r1 - r0, K), dtype=np.float32) * np.float32(std)))))
    rng.bit_generator.state = state
    g = np.float32(amax / E4M3_MAX) if amax > 0 else np.float32(1.0)
    out = np.empty((rows, K), dtype=np.uint8)
    for r0 in range(0, rows, chunk_rows):
        r1 = min(rows, r0 + chunk_rows)
        x = rng.standard_normal((r1 - r0, K), dtype=np.float32) * np.float32(std)
        out[r0:r1] = e4m3_rne(x / g)
    return out, float(g)


def w4a8_ffn_down(M: int = 4096, N: int = 5376, K: int = 14336, seed_a: int = 0,
                  seed_w: int = 1) -> Workload:
    """FFN down projection with FP8 activations: A ~ N(0,1) [M,K] (seed 0) as E4M3 bytes
    with a per-tensor scale; W as the FFN-down NVFP4 weights (seed 1)."""
    A8, gA = fp8_per_tensor(np.random.Generator(np.random.PCG64(seed_a)), M, K)
    W = quantize_nvfp4_chunked(np.random.Generator(np.random.PCG64(seed_w)), N, K, 0.02)
    return Workload(f"w4a8_ffn_down_{M}x{N}x{K}", M, N, K, W=W, A_fp8=A8, gA=gA,
                    notes="A e4m3 N(0,1)/gA seed %d, gA=amax/448; W~N(0,0.02) seed %d" % (
                        seed_a, seed_w))


def zipf_routing(tokens: int, E: int, s: float, seed: int) -> np.ndarray:
    """Top-1 expert per token from a multinomial with p_e proportional to (e+1)^-s."""
    p = (np.arange(1, E + 1, dtype=np.float64)) ** (-s)
    p /= p.sum()
    rng = np.random.Generator(np.random.PCG64(seed))
    return rng.choice(E, size=tokens, p=p)


def grouped_w4a4(E: int = 8, tokens: int = 8192, N: int = 14336, K: int = 4096,
                 seed_a: int = 0, seed_w: int = 1, seed_route: int = 2,
                 counts: list[int] | None = None) -> Workload:
    """Grouped MoE W4A4: per-expert W_e [N,K] ~ N(0,0.02), tokens ~ N(0,1) routed top-1
    with Zipf(1.1) popularity, grouped by expert in ascending token order.  ``counts``
    overrides the routing (forced ragged / small-M cases)."""
    if counts is None:
        ids = zipf_routing(tokens, E, 1.1, seed_route)
        counts = np.bincount(ids, minlength=E).tolist()
    assert len(counts) == E
    offsets = np.zeros(E + 1, dtype=np.int64)
    offsets[1:] = np.cumsum(counts)
    M = int(offsets[-1])
    A = quantize_nvfp4_chunked(np.random.Generator(np.random.PCG64(seed_a)), M, K, 1.0) \
        if M > 0 else Operand(np.zeros((0, K // 2), np.uint8), np.zeros((0, K // 16), np.uint8),
                              1.0)
    rngw = np.random.Generator(np.random.PCG64(seed_w))
    W_e = [quantize_nvfp4_chunked(rngw, N, K, 0.02) for _ in range(E)]
    return Workload(f"grouped_w4a4_E{E}_T{M}_{N}x{K}", M, N, K, A=A, E=E, offsets=offsets,
                    W_e=W_e, notes="counts %s" % list(counts))


def moe_layer(E: int = 8, tokens: int = 8192, N: int = 14336, K: int = 4096, seed_a: int = 0,
              seed_w: int = 1, seed_route: int = 2) -> Workload:
    """One MoE layer from BF16 tokens: X ~ N(0,1) [T,K] in token order (seed 0), top-1
    Zipf(1.1) routing (seed 2), the grouped workload's expert weights (seed 1)."""
    rng = np.random.Generator(np.random.PCG64(seed_a))
    X = to_bf16_bits(rng.standard_normal((tokens, K), dtype=np.float32))
    ids = zipf_routing(tokens, E, 1.1, seed_route).astype(np.int32).reshape(tokens, 1)
    rngw = np.random.Generator(np.random.PCG64(seed_w))
    W_e = [quantize_nvfp4_chunked(rngw, N, K, 0.02) for _ in range(E)]
    return Workload(f"moe_layer_E{E}_T{tokens}_{N}x{K}", tokens, N, K, A_bf16=X, E=E, W_e=W_e,
                    expert_ids=ids, notes="X bf16 N(0,1) seed %d, top-1 Zipf(1.1) seed %d, "
                                          "W_e~N(0,0.02) seed %d" % (seed_a, seed_route, seed_w))


def stack_experts(wl: Workload):
    """[E,N,K/2] codes, [E,N,K/16] scales and [E] FP32 scales of a grouped workload."""
    codes = np.stack([w.codes for w in wl.W_e])
    scales = np.stack([w.scales for w in wl.W_e])
    g = np.array([w.g for w in wl.W_e], dtype=np.float32)
    return codes, scales, g
