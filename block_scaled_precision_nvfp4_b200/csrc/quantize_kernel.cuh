// quantize_kernel.cuh -- BF16 activations -> NVFP4 (E2M1 codes, E4M3 group
// scales, FP32 per-tensor scale): the step ahead of the W4A4 matmul.
//
// Two-level recipe of the FFN-down workload: each run of 16 elements gets an E4M3
// scale from its largest magnitude over 6, taken relative to an FP32 per-tensor
// scale from the tensor's largest magnitude over 6 x 448.  Every step is an IEEE
// FP32 operation rounded to nearest even, in this order:
//     g      = amax|X| / 2688                         (1 when amax = 0)
//     q      = amax_b / (6 * g)                       per 16 consecutive k
//     s_b    = E4M3(q), nearest even, satfinite       (cvt.rn.satfinite)
//     t      = x / (s * g)                            (+-0 when s = 0)
//     code   = sign(t) | E2M1(|t|), nearest even, satfinite
// Two launches: a reduction of amax into a caller-owned scratch word (the
// magnitude bits of BF16 order like the values, so the maximum is an integer
// maximum), then the quantiser proper, one CTA per 128 rows x 256 columns,
// which also writes the scales in the block-scaled MMA's packed layout
// (pack_scales_kernel.cuh) so the matmul needs no separate packing pass.
#pragma once
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cstdint>

#include "ptx.cuh"

namespace nvfp4 {
namespace quant {

constexpr int AMAX_THREADS = 512;
constexpr int TILE_ROWS = 128;   // one packed 128-row block
constexpr int TILE_COLS = 256;   // 16 groups: four K = 64 steps
constexpr int THREADS = 256;     // 8 warps x 16 rows
constexpr int QB = 4;            // row pairs of a warp in flight at once

// max over |x| as BF16 magnitude bits (15 bits), into *amax_bits (atomic max)
__global__ void __launch_bounds__(AMAX_THREADS)
amax_bf16_kernel(const uint4* __restrict__ x, size_t n16, const uint16_t* __restrict__ tail,
                 int ntail, unsigned* amax_bits) {
    // the quantiser launched after this kernel may start now: it reads X ahead and
    // waits for this grid (griddepcontrol.wait) before it reads the maximum
    grid_dependents_launch();
    unsigned m = 0;
    for (size_t i = blockIdx.x * (size_t)AMAX_THREADS + threadIdx.x; i < n16;
         i += (size_t)gridDim.x * AMAX_THREADS) {
        const uint4 v = __ldcs(x + i);
        const unsigned a = __vmaxu2(v.x & 0x7FFF7FFFu, v.y & 0x7FFF7FFFu);
        const unsigned b = __vmaxu2(v.z & 0x7FFF7FFFu, v.w & 0x7FFF7FFFu);
        const unsigned c = __vmaxu2(a, b);
        m = max(m, max(c & 0xFFFFu, c >> 16));
    }
    if (blockIdx.x == 0)
        for (int i = threadIdx.x; i < ntail; i += AMAX_THREADS) m = max(m, (unsigned)(tail[i] & 0x7FFFu));
    m = __reduce_max_sync(0xffffffffu, m);
    __shared__ unsigned wmax[AMAX_THREADS / 32];
    if ((threadIdx.x & 31) == 0) wmax[threadIdx.x >> 5] = m;
    __syncthreads();
    if (threadIdx.x < 32) {
        unsigned v = threadIdx.x < AMAX_THREADS / 32 ? wmax[threadIdx.x] : 0u;
        v = __reduce_max_sync(0xffffffffu, v);
        if (threadIdx.x == 0 && v != 0) atomicMax(amax_bits, v);
    }
}

__device__ __forceinline__ float global_scale(unsigned amax_bits) {
    const float amax = __uint_as_float(amax_bits << 16);
    return amax > 0.f ? __fdiv_rn(amax, 2688.0f) : 1.0f;
}

// q >= 0 -> E4M3 byte, nearest even, saturating at 448
__device__ __forceinline__ uint32_t e4m3_satfinite(float q) {
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(q), "f"(q));
    return r & 0xFFu;
}
// E4M3 byte -> its value (exact)
__device__ __forceinline__ float e4m3_value(uint32_t b) {
    uint32_t h2;
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"((uint16_t)(b | (b << 8))));
    return __half2float(__ushort_as_half((uint16_t)(h2 & 0xFFFFu)));
}
// two FP32 lanes at once: d = RN(a*b), d = RN(a*b + c) per lane
__device__ __forceinline__ uint64_t mul_f32x2(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ uint64_t fma_f32x2(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}

// eight values t0 .. t7 -> eight signed E2M1 codes (the sign of t kept, -0 and
// values that round to zero included), packed with element 2j in the low nibble
// of byte j (cvt puts its first operand in the high nibble)
__device__ __forceinline__ uint32_t e2m1x8(const float (&t)[8]) {
    uint32_t r;
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
        "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
        : "=r"(r)
        : "f"(t[0]), "f"(t[1]), "f"(t[2]), "f"(t[3]), "f"(t[4]), "f"(t[5]), "f"(t[6]), "f"(t[7]));
    return r;
}

// The sixteen BF16 values of one group, as eight words (element 2j in the low half
// of word j).  V8: one 256-bit load (the row start is 32-byte aligned); otherwise two
// 128-bit loads.  Streaming: X is read once more by nobody.
template <bool V8>
__device__ __forceinline__ void load_group(const __nv_bfloat16* p, uint32_t (&w)[8]) {
    if constexpr (V8) {
        asm("ld.global.cs.v8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
            : "=r"(w[0]), "=r"(w[1]), "=r"(w[2]), "=r"(w[3]), "=r"(w[4]), "=r"(w[5]), "=r"(w[6]),
              "=r"(w[7])
            : "l"(p));
    } else {
        const uint4 a = __ldcs(reinterpret_cast<const uint4*>(p));
        const uint4 b = __ldcs(reinterpret_cast<const uint4*>(p) + 1);
        w[0] = a.x; w[1] = a.y; w[2] = a.z; w[3] = a.w;
        w[4] = b.x; w[5] = b.y; w[6] = b.z; w[7] = b.w;
    }
}

// a / b by Markstein's correction from y = RN(1/b), for b in [2^-60, 2^60] and
// 0 <= a / b <= 2^68: q = RN(a*y), r = a - b*q (exact by FMA), RN(q + r*y).  That is
// RN(a / b) whenever a >= 2^-100, where no step underflows; below that the result
// can be off in its last (subnormal) places or be -0.
__device__ __forceinline__ float div_markstein(float a, float b, float y) {
    const float q = __fmul_rn(a, y);
    const float r = __fmaf_rn(-b, q, a);
    return __fmaf_rn(r, y, q);
}

// prmt.b32 in its generic mode: a selector nibble with bit 3 set fills the byte
// with the sign (bit 7) of the selected source byte.
__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
    uint32_t r;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(sel));
    return r;
}

// Eight codes (element 2j in the low nibble of byte j) with each sign bit set from
// x's own sign, the eight BF16 values being w0 .. w3 (element 2j in the low half of
// word j).  A correctly rounded x / den with den > 0 has x's sign, -0 and values that
// round to zero included; the corrected quotient can lose that sign only where it
// underflows, which is far below the smallest nonzero code.
__device__ __forceinline__ uint32_t with_signs(uint32_t code, uint32_t w0, uint32_t w1, uint32_t w2,
                                               uint32_t w3) {
    const uint32_t a = prmt(w0, w1, 0xFDB9u);    // bytes 0x00/0xFF: signs of elements 0..3
    const uint32_t b = prmt(w2, w3, 0xFDB9u);    // elements 4..7
    const uint32_t even = prmt(a, b, 0x6420u);   // elements 0, 2, 4, 6
    const uint32_t odd = prmt(a, b, 0x7531u);    // elements 1, 3, 5, 7
    return (code & 0x77777777u) | (even & 0x08080808u) | (odd & 0x80808080u);
}

// One CTA: rows [128*blockIdx.x, +128) x columns [256*blockIdx.y, +256).
// One lane per 16-group: lanes 16h .. 16h+15 of warp w take the 16 groups of row
// 16w + 2i + h (i = 0 .. 7), so a warp instruction covers two rows of the tile.
// ROUTED: row r's codes and plain scales go to rows dest[r k + j] (j < k) of the
// outputs instead of row r, which is the row permutation of an MoE dispatch done as
// the rows are written (no packed scales then); a destination outside [0, rows k)
// (-1: a pair the route placed nowhere) is skipped.
template <bool V8, bool ROUTED>
__global__ void __launch_bounds__(THREADS, 4)
quantize_bf16_kernel(const __nv_bfloat16* __restrict__ X, int rows, int K,
                     const unsigned* __restrict__ amax_bits, uint8_t* __restrict__ codes,
                     uint8_t* __restrict__ scales, uint8_t* __restrict__ scales_packed,
                     float* __restrict__ g_out, const int32_t* __restrict__ dest, int k) {
    __shared__ uint32_t sc[TILE_ROWS][TILE_COLS / 64 + 1];  // [row][K=64 step] four scale bytes
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int r0 = blockIdx.x * TILE_ROWS, c0 = blockIdx.y * TILE_COLS;
    const int gi = lane & 15, half = lane >> 4;  // group of the tile row; which row of the pair
    const int col = c0 + 16 * gi;
    const bool col_ok = col < K;  // K % 16 == 0: a group is all in or all out

    constexpr int PAIRS = TILE_ROWS / 16;  // row pairs per warp
    uint32_t vin[QB][8];
    auto load_rows = [&](int i0) {
#pragma unroll
        for (int i = 0; i < QB; ++i) {
            const int row = r0 + warp * 16 + 2 * (i0 + i) + half;
            if (col_ok && row < rows) {
                load_group<V8>(X + (size_t)row * K + col, vin[i]);
            } else {
#pragma unroll
                for (int j = 0; j < 8; ++j) vin[i][j] = 0u;
            }
        }
    };
    // The first rows are read while the amax kernel before this one may still run
    // (programmatic launch); the maximum is read only after that grid has completed.
    load_rows(0);
    grid_dependency_wait();
    const float g = global_scale(__ldcg(amax_bits));
    const float d6 = __fmul_rn(6.0f, g);
    const bool fast6 = d6 >= 0x1p-60f && d6 <= 0x1p60f;  // the same for the whole tensor
    const float y6 = __frcp_rn(d6);
    if (blockIdx.x == 0 && blockIdx.y == 0 && threadIdx.x == 0) *g_out = g;
    uint8_t* scb = reinterpret_cast<uint8_t*>(&sc[0][0]);
#pragma unroll 1
    for (int i0 = 0; i0 < PAIRS; i0 += QB) {
        if (i0 > 0) load_rows(i0);
#pragma unroll
        for (int i = 0; i < QB; ++i) {
            const int rl = warp * 16 + 2 * (i0 + i) + half;
            const int row = r0 + rl;
            const bool ok = col_ok && row < rows;
            const uint32_t(&w)[8] = vin[i];
            // group amax (integer max of the magnitude bits; they order like the values)
            const unsigned a01 = __vmaxu2(w[0] & 0x7FFF7FFFu, w[1] & 0x7FFF7FFFu);
            const unsigned a23 = __vmaxu2(w[2] & 0x7FFF7FFFu, w[3] & 0x7FFF7FFFu);
            const unsigned a45 = __vmaxu2(w[4] & 0x7FFF7FFFu, w[5] & 0x7FFF7FFFu);
            const unsigned a67 = __vmaxu2(w[6] & 0x7FFF7FFFu, w[7] & 0x7FFF7FFFu);
            const unsigned a = __vmaxu2(__vmaxu2(a01, a23), __vmaxu2(a45, a67));
            const float amax_b = __uint_as_float(max(a & 0xFFFFu, a >> 16) << 16);
            // s_b = E4M3(RN(amax_b / (6g))); amax_b <= amax makes the quotient <= 448
            // (|.|: the corrected quotient may come out as -0 where it underflows; the
            // scale byte is 0 there either way)
            const float qs = fast6 ? fabsf(div_markstein(amax_b, d6, y6)) : __fdiv_rn(amax_b, d6);
            const uint32_t sb = e4m3_satfinite(qs);
            const float den = __fmul_rn(e4m3_value(sb), g);
            float t[16];
            // t = x / den, correctly rounded.  The divisor is shared by the group, so its
            // correctly rounded reciprocal is taken once and each quotient is finished by
            // Markstein's correction on packed f32x2 lanes (two elements per instruction,
            // each lane one IEEE RN operation).  For den in [2^-60, 2^60] that is RN(x/den)
            // wherever x / den >= 2^-3 in magnitude (every step stays normal; |t| < 7 by
            // the choice of s); smaller quotients give a zero code whatever their last
            // places, and with_signs gives it x's sign.  Other groups, and den == 0, keep
            // the plain division.
            if (den >= 0x1p-60f && den <= 0x1p60f) {
                const float y = __frcp_rn(den);
                const uint64_t y2 = ((uint64_t)__float_as_uint(y) << 32) | __float_as_uint(y);
                const uint64_t nd2 = ((uint64_t)__float_as_uint(-den) << 32) | __float_as_uint(-den);
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const uint64_t x2 = ((uint64_t)(w[j] & 0xFFFF0000u) << 32) | (uint64_t)(w[j] << 16);
                    const uint64_t q2 = mul_f32x2(x2, y2);
                    const uint64_t t2 = fma_f32x2(fma_f32x2(q2, nd2, x2), y2, q2);
                    t[2 * j] = __uint_as_float((uint32_t)t2);
                    t[2 * j + 1] = __uint_as_float((uint32_t)(t2 >> 32));
                }
            } else {
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    // element e is half (e & 1) of word e >> 1
                    const uint32_t h = (e & 1) ? (w[e >> 1] & 0xFFFF0000u) : (w[e >> 1] << 16);
                    const float xe = __uint_as_float(h);
                    t[e] = den > 0.f ? __fdiv_rn(xe, den) : xe * 0.0f;
                }
            }
            const float(&tlo)[8] = *reinterpret_cast<const float(*)[8]>(&t[0]);
            const float(&thi)[8] = *reinterpret_cast<const float(*)[8]>(&t[8]);
            if (ok) {
                const uint2 cv = make_uint2(with_signs(e2m1x8(tlo), w[0], w[1], w[2], w[3]),
                                            with_signs(e2m1x8(thi), w[4], w[5], w[6], w[7]));
                if (ROUTED) {
                    for (int j = 0; j < k; ++j) {
                        // a pair the route placed nowhere (-1) is skipped
                        const int d = __ldg(dest + (size_t)row * k + j);
                        if ((unsigned)d < (unsigned)(rows * k))
                            *reinterpret_cast<uint2*>(codes + (size_t)d * (K / 2) + col / 2) = cv;
                    }
                } else {
                    *reinterpret_cast<uint2*>(codes + (size_t)row * (K / 2) + col / 2) = cv;
                }
            }
            // the group's scale byte (group gi of the row is byte gi of the row's words)
            scb[rl * (TILE_COLS / 64 + 1) * 4 + gi] = ok ? (uint8_t)sb : (uint8_t)0;
        }
    }
    __syncthreads();

    const int nks = min(TILE_COLS / 64, (K - c0 + 63) / 64);  // K = 64 steps of this tile
    if (scales) {
        // plain [rows][K/16]: each row's 4..16 bytes of this tile
        for (int idx = threadIdx.x; idx < TILE_ROWS * (TILE_COLS / 64); idx += THREADS) {
            const int rl = idx >> 2, ks = idx & 3, row = r0 + rl;
            const int g0 = c0 / 16 + 4 * ks;  // first group of the word
            if (row < rows && g0 < K / 16) {
                const uint32_t wv = sc[rl][ks];
                const int n = min(4, K / 16 - g0);
                for (int j = 0; j < (ROUTED ? k : 1); ++j) {
                    const int drow = ROUTED ? __ldg(dest + (size_t)row * k + j) : row;
                    if (ROUTED && (unsigned)drow >= (unsigned)(rows * k)) continue;
                    uint8_t* dst = scales + (size_t)drow * (K / 16) + g0;
                    if (n == 4 && (K / 16) % 4 == 0) {
                        *reinterpret_cast<uint32_t*>(dst) = wv;  // 4-byte aligned
                    } else {
                        for (int b = 0; b < n; ++b) dst[b] = (uint8_t)(wv >> (8 * b));
                    }
                }
            }
        }
    }
    if (!ROUTED && scales_packed && K % 64 == 0) {
        // packed[rb][ks][i][j][t] = s[128 rb + 32 j + i][4 ks + t]: this tile's nks atoms,
        // contiguous, one 16-byte line (i) per thread and step
        const int ksteps = K / 64, ks0 = c0 / 64;
        uint4* dst = reinterpret_cast<uint4*>(scales_packed + ((size_t)blockIdx.x * ksteps + ks0) * 512);
        for (int line = threadIdx.x; line < nks * 32; line += THREADS) {
            const int ksl = line >> 5, i = line & 31;
            dst[line] = make_uint4(sc[i][ksl], sc[i + 32][ksl], sc[i + 64][ksl], sc[i + 96][ksl]);
        }
    }
}

}  // namespace quant
}  // namespace nvfp4
