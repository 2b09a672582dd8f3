// w4a16_kernel.cuh -- BF16 activations x NVFP4 weights widened in registers.
//
// The "BF16 activations: BF16 MMA, any weight format widened in registers"
// row of the metrale_circuit `hardware::exec` module doc, bullet 1, for the
// decode shape (a handful of tokens, HBM-bound on the weight stream).
//
// Design:
//  * one warp owns 16 weight rows; a cluster of 8 CTAs splits K into 8
//    slices (CTA rank = slice), each CTA's 8 warps cover the cluster's 8
//    16-row blocks;
//  * weights stream from HBM with 128-bit ld.global.nc (each lane 32 codes of
//    one row per 128-code span, four spans in flight), never through smem;
//  * a code is widened with two shifts and one LOP3 per pair into BF16 bits
//    worth e2m1 * 2^-126, then multiplied (bf16x2, exact) by the group scale
//    pre-multiplied by 2^119, so each weight is e2m1 * s * 2^-7 exactly;
//  * the MMA is mma.sync m16n8k16 BF16 with weight rows on M and tokens on N
//    (two N tiles = 16 tokens); K is permuted inside each lane's 32 codes,
//    and the activations are staged in shared memory in the same permuted
//    order (conflict-free 64-bit reads);
//  * the 8 K-slice partials are reduced in a fixed order through distributed
//    shared memory (no global workspace), scaled by 2^7 * gW, rounded to BF16.
#pragma once
#include <cuda_bf16.h>
#include <cooperative_groups.h>
#include <cstdint>

namespace nvfp4 {
namespace w4a16 {

constexpr int TOK = 16;       // tokens per launch (two N = 8 MMA tiles)
constexpr int SPAN = 128;     // codes per span (4 lanes x 32 codes per row)
constexpr int WARPS = 8;      // 16-row blocks per CTA
constexpr int CLUSTER = 8;    // K slices per cluster
constexpr int THREADS = 32 * WARPS;
constexpr int PF = 4;         // spans in flight per lane

static_assert(CLUSTER == WARPS, "each CTA of a cluster reduces one warp's row block");

__host__ __device__ constexpr int act_row_bytes(int spans_per_slice) {
    return spans_per_slice * 256 + 32;  // row stride = 32 mod 128: conflict-free reads
}
__host__ __device__ constexpr size_t smem_bytes(int spans_per_slice) {
    return (size_t)TOK * act_row_bytes(spans_per_slice) + (size_t)WARPS * 16 * TOK * 4;
}

__device__ __forceinline__ uint4 ldg_stream(const void* p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
    return v;
}

__device__ __forceinline__ uint32_t mul_bf16x2(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

// E4M3 scale byte (non-negative) -> BF16 bits of s * 2^119, packed twice.
__device__ __forceinline__ uint32_t scale_pair(uint32_t b) {
    const uint32_t E = (b >> 3) & 15u, M = b & 7u;
    uint32_t h;
    if (E != 0) h = ((E + 239u) << 7) | (M << 4);
    else h = __float_as_uint((float)M * 0x1p110f) >> 16;
    return h | (h << 16);
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
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
        "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

struct Span {
    uint4 q0, q1;      // 32 codes of row g and of row g+8
    uint32_t s0, s1;   // their two group-scale bytes (low byte: codes 0-15)
};

__global__ void __launch_bounds__(THREADS, 1)
w4a16_kernel(const uint16_t* __restrict__ A, const uint8_t* __restrict__ W,
             const uint8_t* __restrict__ sW, __nv_bfloat16* __restrict__ Y, int M, int N, int K,
             float out_scale, int spans_per_slice) {
    namespace cg = cooperative_groups;
    cg::cluster_group cluster = cg::this_cluster();
    extern __shared__ __align__(128) uint8_t smem[];
    const int row_bytes = act_row_bytes(spans_per_slice);
    uint8_t* act = smem;
    float* part = reinterpret_cast<float*>(smem + (size_t)TOK * row_bytes);

    const int slice = (int)cluster.block_rank();
    const int cluster_id = blockIdx.x / CLUSTER;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;
    const int span0 = slice * spans_per_slice;
    const int total_spans = (K + SPAN - 1) / SPAN;
    const int nspans = max(0, min(spans_per_slice, total_spans - span0));

    // ---- stage this slice's activations, permuted to the MMA's K order
    for (int c = threadIdx.x; c < TOK * spans_per_slice * 4; c += THREADS) {
        const int tt = c & 3, sp = (c >> 2) % spans_per_slice, n = c / (4 * spans_per_slice);
        const int k = (span0 + sp) * SPAN + 32 * tt;
        uint32_t a[16];
        if (n < M && sp < nspans && k < K) {
            const uint4* src = reinterpret_cast<const uint4*>(A + (size_t)n * K + k);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                uint4 v = __ldg(src + j);
                a[4 * j] = v.x; a[4 * j + 1] = v.y; a[4 * j + 2] = v.z; a[4 * j + 3] = v.w;
            }
        } else {
#pragma unroll
            for (int j = 0; j < 16; ++j) a[j] = 0u;
        }
        // a[] holds 32 bf16: element e is half (e & 1) of a[e >> 1]
        auto el = [&](int e) -> uint32_t { return (a[e >> 1] >> (16 * (e & 1))) & 0xFFFFu; };
        uint8_t* dst = act + (size_t)n * row_bytes + sp * 256 + tt * 8;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int w8 = 8 * (i >> 1) + 2 * (i & 1);
            uint2 v;
            v.x = el(w8) | (el(w8 + 4) << 16);
            v.y = el(w8 + 1) | (el(w8 + 5) << 16);
            *reinterpret_cast<uint2*>(dst + i * 32) = v;
        }
    }
    __syncthreads();

    // ---- stream this warp's 16 weight rows over the slice
    const int rb = cluster_id * WARPS + warp;
    const int r0 = rb * 16 + g, r1 = r0 + 8;
    const size_t row_stride = (size_t)K / 2, srow_stride = (size_t)K / 16;
    const bool ok0 = r0 < N, ok1 = r1 < N;
    float acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};

    auto load = [&](int sp, Span& s) {
        const int k = (span0 + sp) * SPAN + 32 * t;
        const bool in = sp < nspans && k < K;
        s.q0 = make_uint4(0u, 0u, 0u, 0u);
        s.q1 = s.q0;
        s.s0 = s.s1 = 0u;
        if (in && ok0) {
            s.q0 = ldg_stream(W + r0 * row_stride + k / 2);
            s.s0 = __ldg(reinterpret_cast<const uint16_t*>(sW + r0 * srow_stride + k / 16));
        }
        if (in && ok1) {
            s.q1 = ldg_stream(W + r1 * row_stride + k / 2);
            s.s1 = __ldg(reinterpret_cast<const uint16_t*>(sW + r1 * srow_stride + k / 16));
        }
    };

    auto compute = [&](int sp, const Span& s) {
        const uint32_t sa0 = scale_pair(s.s0 & 0xFFu), sb0 = scale_pair((s.s0 >> 8) & 0xFFu);
        const uint32_t sa1 = scale_pair(s.s1 & 0xFFu), sb1 = scale_pair((s.s1 >> 8) & 0xFFu);
        const uint32_t w0[4] = {s.q0.x, s.q0.y, s.q0.z, s.q0.w};
        const uint32_t w1[4] = {s.q1.x, s.q1.y, s.q1.z, s.q1.w};
        const uint8_t* arow0 = act + (size_t)g * row_bytes + sp * 256 + t * 8;
        const uint8_t* arow1 = arow0 + (size_t)8 * row_bytes;
#pragma unroll
        for (int w = 0; w < 4; ++w) {
            uint32_t p0[4], p1[4];
            widen8(w0[w], w < 2 ? sa0 : sb0, p0);
            widen8(w1[w], w < 2 ? sa1 : sb1, p1);
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int i = 2 * w + h;
                const uint2 b0 = *reinterpret_cast<const uint2*>(arow0 + i * 32);
                const uint2 b1 = *reinterpret_cast<const uint2*>(arow1 + i * 32);
                mma_bf16(acc[0], p0[2 * h], p1[2 * h], p0[2 * h + 1], p1[2 * h + 1], b0.x, b0.y);
                mma_bf16(acc[1], p0[2 * h], p1[2 * h], p0[2 * h + 1], p1[2 * h + 1], b1.x, b1.y);
            }
        }
    };

    Span buf[PF];
#pragma unroll
    for (int p = 0; p < PF; ++p) load(p, buf[p]);
    for (int sp = 0; sp < nspans; sp += PF) {
#pragma unroll
        for (int p = 0; p < PF; ++p) {
            const Span cur = buf[p];
            load(sp + p + PF, buf[p]);
            if (sp + p < nspans) compute(sp + p, cur);
        }
    }

    // ---- partial sums of this slice: part[warp][row][token]
    float* pw = part + warp * 16 * TOK;
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
        const int tok = 8 * nt + 2 * t;
        pw[g * TOK + tok] = acc[nt][0];
        pw[g * TOK + tok + 1] = acc[nt][1];
        pw[(g + 8) * TOK + tok] = acc[nt][2];
        pw[(g + 8) * TOK + tok + 1] = acc[nt][3];
    }
    cluster.sync();

    // ---- CTA `slice` reduces row block `slice` of the cluster over all slices
    {
        const int row = threadIdx.x / TOK, tok = threadIdx.x % TOK;
        const int rrb = cluster_id * WARPS + slice;
        const int n = rrb * 16 + row;
        float* mine = part + slice * 16 * TOK + row * TOK + tok;
        float s = 0.f;
#pragma unroll
        for (int c = 0; c < CLUSTER; ++c) s += *cluster.map_shared_rank(mine, c);
        if (n < N && tok < M) Y[(size_t)tok * N + n] = __float2bfloat16_rn(s * out_scale);
    }
    cluster.sync();
}

}  // namespace w4a16
}  // namespace nvfp4
