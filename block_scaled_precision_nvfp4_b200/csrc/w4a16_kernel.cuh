// w4a16_kernel.cuh -- BF16 activations x NVFP4 weights widened in registers.
//
// The BF16 row of the metrale_circuit `hardware::exec` module doc, bullet 1
// (BF16 activations on the BF16 MMA, the weights widened to BF16 in registers
// whatever their format), for the decode shape (a handful of tokens, HBM-bound
// on the weight stream).
//
// Design (one wave of CTAs, one per SM, no cluster, no workspace):
//  * the weight rows are cut into blocks of 8 (the MMA's N); CTA c takes a
//    contiguous range of LDG_MAX_NB or fewer blocks, over the whole of K;
//  * every weight byte travels global -> registers in one 128-bit load: lane
//    (g, t) of a warp holds, for each of the CTA's blocks, the 32 codes of row
//    8b + g at code 128 j + 32 t of span j, and their two group scales;
//  * a code is widened with two shifts and one LOP3 per pair into BF16 bits
//    worth e2m1 * 2^-126, then multiplied (bf16x2, exact) by the group scale
//    pre-multiplied by 2^119, so each weight is e2m1 * s * 2^-7 exactly;
//  * the MMA is mma.sync m16n8k16 BF16 with the 16 tokens on M and the block's
//    8 weight rows on N; K is permuted inside each lane's 32 codes and the
//    lane's activation fragments are built in the same order;
//  * the warps' partial sums meet in shared memory and are added in a fixed
//    warp order (deterministic), scaled by 2^7 * gW and rounded to BF16.
#pragma once
#include <cuda_bf16.h>
#include <cstdint>

#include "ptx.cuh"

namespace nvfp4 {
namespace w4a16 {

constexpr int TOK = 16;        // tokens per launch (the MMA's M)
constexpr int SPAN = 128;      // codes per span (4 lanes x 32 codes per row)
constexpr int ROWS = 8;        // weight rows per block (the MMA's N)

__device__ __forceinline__ uint4 ldg_stream(const void* p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
    return v;
}

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
    uint32_t d;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
    return d;
}

__device__ __forceinline__ uint32_t mul_bf16x2(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

// E4M3 scale byte (0x00..0x7E) -> BF16 bits of s * 2^119, packed twice.  For a
// normal byte (exponent field E >= 1) the BF16 exponent is E + 239 and the
// three mantissa bits move up by four, i.e. (b << 4) + (239 << 7); the
// subnormal bytes (and zero) take the float route.
__device__ __forceinline__ uint32_t scale_pair(uint32_t b) {
    uint32_t h;
    if (b >= 8u) h = (b << 4) + (239u << 7);
    else h = __float_as_uint((float)b * 0x1p110f) >> 16;
    return h * 0x10001u;
}

// Eight codes of one word -> four BF16 pairs worth e2m1 * 2^-126, as
// (code u, code u+4) for u = 0, 1, 2, 3, then times the scale pair.
__device__ __forceinline__ void widen8(uint32_t q, uint32_t ss, uint32_t (&p)[4]) {
    constexpr uint32_t MAG = 0x01C001C0u, SGN = 0x80008000u;
    p[0] = mul_bf16x2(((q << 6) & MAG) | ((q << 12) & SGN), ss);  // codes 0, 4
    p[1] = mul_bf16x2(((q << 2) & MAG) | ((q << 8) & SGN), ss);   // codes 1, 5
    p[2] = mul_bf16x2(((q >> 2) & MAG) | ((q << 4) & SGN), ss);   // codes 2, 6
    p[3] = mul_bf16x2(((q >> 6) & MAG) | (q & SGN), ss);          // codes 3, 7
}

__device__ __forceinline__ void mma_bf16(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                         uint32_t a3, uint32_t b0, uint32_t b1) {
    asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
        "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// ---------------------------------------------------------------------------------
// The kernel.  CTA c owns a contiguous range of up to LDG_MAX_NB blocks of 8 weight
// rows over all of K.  Its 8 warps take the 128-code spans of K in turn (warp w: spans
// w, w + 8, ...), so at any moment the CTA reads 512 contiguous bytes of each of its
// rows.  Lane (g, t) of a warp loads, for every block b of the CTA, the 16 bytes (32
// codes) of row 8b + g at code 128 j + 32 t, and its two group-scale bytes; and the
// 16 tokens' activations of the same 32 codes (tokens g and g + 8: four 16-byte loads
// each, from L2).  Span j + 8's loads are issued before span j is widened and
// multiplied, so a warp keeps about 100 bytes in flight per lane.
constexpr int LDG_WARPS = 8;
constexpr int LDG_THREADS = 32 * LDG_WARPS;
constexpr int LDG_MAX_NB = 6;

template <int NB>
struct SpanRegs {
    uint4 a[8];        // tokens g (0..3) and g + 8 (4..7): 4 x 8 BF16 each
    uint4 w[NB];       // 32 codes of row 8b + g
    uint32_t s[NB];    // their two group-scale bytes
};

template <int NB>
__device__ __forceinline__ void load_span(SpanRegs<NB>& r, const uint16_t* __restrict__ A,
                                          const uint8_t* __restrict__ W,
                                          const uint8_t* __restrict__ sW, int j, int nspan,
                                          int rowbase, int nb, int M, int N, int K, int g, int t) {
    const int k0 = j * SPAN + 32 * t;
    const bool kok = j < nspan && k0 < K;  // K % 32 == 0: a lane's 32 codes are all in or out
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const int tok = g + 8 * h;
        const bool ok = kok && tok < M;
        const uint16_t* src = A + (size_t)tok * K + k0;
#pragma unroll
        for (int m = 0; m < 4; ++m)
            r.a[h * 4 + m] = ok ? __ldg(reinterpret_cast<const uint4*>(src + 8 * m)) : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int b = 0; b < NB; ++b) {
        const int row = rowbase + 8 * b + g;
        const bool ok = kok && b < nb && row < N;
        r.w[b] = ok ? ldg_stream(W + (size_t)row * (K / 2) + k0 / 2) : make_uint4(0u, 0u, 0u, 0u);
        r.s[b] = ok ? (uint32_t)__ldg(reinterpret_cast<const uint16_t*>(sW + (size_t)row * (K / 16) + k0 / 16)) : 0u;
    }
}

template <int NB>
__device__ __forceinline__ void mma_span(const SpanRegs<NB>& r, float (&acc)[NB][4], int nb) {
    // the lane's activation fragments, in the K order of widen8 (K-step 2v + h)
    uint32_t af[8][4];
#pragma unroll
    for (int v = 0; v < 4; ++v) {
        const uint4 x0 = r.a[v], x1 = r.a[4 + v];  // tokens g, g+8
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const uint32_t lo0 = h ? x0.y : x0.x, hi0 = h ? x0.w : x0.z;
            const uint32_t lo1 = h ? x1.y : x1.x, hi1 = h ? x1.w : x1.z;
            af[2 * v + h][0] = prmt(lo0, hi0, 0x5410);
            af[2 * v + h][1] = prmt(lo1, hi1, 0x5410);
            af[2 * v + h][2] = prmt(lo0, hi0, 0x7632);
            af[2 * v + h][3] = prmt(lo1, hi1, 0x7632);
        }
    }
#pragma unroll
    for (int b = 0; b < NB; ++b) {
        if (b >= nb) break;
        const uint32_t s0 = scale_pair(r.s[b] & 0xFFu), s1 = scale_pair((r.s[b] >> 8) & 0xFFu);
        const uint32_t wq[4] = {r.w[b].x, r.w[b].y, r.w[b].z, r.w[b].w};
#pragma unroll
        for (int v = 0; v < 4; ++v) {
            uint32_t p[4];
            widen8(wq[v], v < 2 ? s0 : s1, p);
#pragma unroll
            for (int h = 0; h < 2; ++h)
                mma_bf16(acc[b], af[2 * v + h][0], af[2 * v + h][1], af[2 * v + h][2],
                         af[2 * v + h][3], p[2 * h], p[2 * h + 1]);
        }
    }
}

template <int NB>
__global__ void __launch_bounds__(LDG_THREADS, 1)
w4a16_ldg_kernel(const uint16_t* __restrict__ A, const uint8_t* __restrict__ W,
                 const uint8_t* __restrict__ sW, __nv_bfloat16* __restrict__ Y, int M, int N, int K,
                 float out_scale, int nrb) {
    __shared__ float4 red[LDG_WARPS][NB][32];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;
    const int G = gridDim.x;
    const int rb0 = (int)((long long)blockIdx.x * nrb / G);
    const int nb = (int)((long long)(blockIdx.x + 1) * nrb / G) - rb0;  // <= NB
    const int rowbase = rb0 * ROWS;
    const int nspan = (K + SPAN - 1) / SPAN;

    float acc[NB][4];
#pragma unroll
    for (int b = 0; b < NB; ++b) acc[b][0] = acc[b][1] = acc[b][2] = acc[b][3] = 0.f;
    SpanRegs<NB> cur, nxt;
    int j = warp;
    load_span<NB>(cur, A, W, sW, j, nspan, rowbase, nb, M, N, K, g, t);
    for (; j < nspan; j += LDG_WARPS) {
        load_span<NB>(nxt, A, W, sW, j + LDG_WARPS, nspan, rowbase, nb, M, N, K, g, t);
        mma_span<NB>(cur, acc, nb);
        cur = nxt;
    }

    // the warps' partial sums meet in shared memory and are added in a fixed warp order
#pragma unroll
    for (int b = 0; b < NB; ++b) red[warp][b][lane] = make_float4(acc[b][0], acc[b][1], acc[b][2], acc[b][3]);
    __syncthreads();
    // D[tok][n] of lane l (tokens l/4 and l/4 + 8, columns 2(l%4) and 2(l%4)+1) -> Y[tok][8b + n]
    for (int idx = threadIdx.x; idx < nb * 128; idx += LDG_THREADS) {
        const int b = idx >> 7, l = (idx >> 2) & 31, e = idx & 3;
        float sum = 0.f;
#pragma unroll
        for (int ww = 0; ww < LDG_WARPS; ++ww) {
            const float4 v = red[ww][b][l];
            sum += e == 0 ? v.x : e == 1 ? v.y : e == 2 ? v.z : v.w;
        }
        const int tok = (l >> 2) + 8 * (e >> 1);
        const int row = rowbase + 8 * b + 2 * (l & 3) + (e & 1);
        if (tok < M && row < N) Y[(size_t)tok * N + row] = __float2bfloat16_rn(sum * out_scale);
    }
}

}  // namespace w4a16
}  // namespace nvfp4
