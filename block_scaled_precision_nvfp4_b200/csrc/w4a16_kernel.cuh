// w4a16_kernel.cuh -- BF16 activations x NVFP4 weights widened in registers.
//
// The "BF16 activations: BF16 MMA, any weight format widened in registers"
// row of the metrale_circuit `hardware::exec` module doc, bullet 1, for the
// decode shape (a handful of tokens, HBM-bound on the weight stream).
//
// Design (one wave of CTAs, one per SM, no cluster, no workspace):
//  * the weight rows are cut into blocks of 8 (the MMA's N); CTA c takes a
//    contiguous range of NB or fewer blocks, over the whole of K;
//  * a producer warp streams the CTA's codes and group scales through a ring
//    of shared-memory stages with TMA (1024 codes of K per stage: four
//    128-byte-wide, 128-byte-swizzled boxes of all the CTA's rows, and one box
//    of their scales), so many bytes stay in flight without registers;
//  * 8 consumer warps split each stage's K: warp w takes the stage's w-th
//    128-code span for every row block, so its activation fragments serve NB
//    blocks; the activations arrive by cp.async into per-lane slots;
//  * a code is widened with two shifts and one LOP3 per pair into BF16 bits
//    worth e2m1 * 2^-126, then multiplied (bf16x2, exact) by the group scale
//    pre-multiplied by 2^119, so each weight is e2m1 * s * 2^-7 exactly;
//  * the MMA is mma.sync m16n8k16 BF16 with the 16 tokens on M and 8 weight
//    rows on N (column n of the block holding row PERM(n), which makes the
//    swizzled reads conflict-free); K is permuted inside each lane's 32 codes
//    and the lane's activation fragments are built in the same order;
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
constexpr int CONSUMERS = 8;   // K splits of a stage (one span each)
constexpr int THREADS = 32 * (CONSUMERS + 1);  // + one producer warp
constexpr int ROWS = 8;        // weight rows per block (the MMA's N)
constexpr int MAX_NB = 8;      // row blocks per CTA at most
constexpr int STAGE_K = CONSUMERS * SPAN;      // 1024 codes of K per stage
constexpr int NA = 2;          // activation spans per warp in shared memory (cp.async slots)
constexpr int SLOT_U4 = 8 * 32;  // one span's activation chunks of a warp, in uint4

// One stage: codes [4 column boxes][NB * 8 rows][128 B], then scales [NB * 8 rows][64 B].
__host__ __device__ constexpr uint32_t stage_code_bytes(int nb) { return (uint32_t)nb * 4096u; }
// (a multiple of 1024 bytes: each 128-byte-swizzled box starts on a 1024-byte boundary)
__host__ __device__ constexpr uint32_t stage_bytes(int nb) { return ((uint32_t)nb * 4608u + 1023u) & ~1023u; }
// roles recorded in the device error word when a wait expires
constexpr int ROLE_W16_PRODUCER = 9, ROLE_W16_CONSUMER = 10;
// as many stages as fit in about 150 KB, between 2 and 8
__host__ __device__ constexpr int stages_for(int nb) {
    return 150 * 1024 / (int)stage_bytes(nb) > 8 ? 8
           : (150 * 1024 / (int)stage_bytes(nb) < 2 ? 2 : 150 * 1024 / (int)stage_bytes(nb));
}
__host__ __device__ constexpr size_t a_ring_bytes() { return (size_t)CONSUMERS * NA * SLOT_U4 * 16; }
__host__ __device__ constexpr size_t smem_bytes(int nb) {
    return 1024 + (size_t)stages_for(nb) * stage_bytes(nb) + a_ring_bytes() + 2 * 8 * 8;
}
// the weight row (within its block of 8) held by MMA column n
__host__ __device__ constexpr int perm_row(int n) { return (n >> 1) | ((n & 1) << 2); }

__device__ __forceinline__ uint4 ldg_stream(const void* p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
    return v;
}

// 16-byte asynchronous copy global -> shared through L1 (a lane's four copies
// of one 128-byte line land in it back to back, so each 32-byte sector leaves
// L2 once); `src_bytes` = 0 writes zeros.
__device__ __forceinline__ void cp_async16(void* smem_dst, const void* gsrc, uint32_t src_bytes) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 16, %2;"
                 ::"r"(static_cast<uint32_t>(__cvta_generic_to_shared(smem_dst))), "l"(gsrc),
                   "r"(src_bytes)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

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

// NB: row blocks per CTA at most; SF_TMA: the group scales travel by TMA with
// the codes (needs the scale row pitch K/16 to be a multiple of 16 bytes);
// otherwise each lane loads its two scale bytes itself, one stage ahead.
template <int NB, bool SF_TMA>
__global__ void __launch_bounds__(THREADS, 1)
w4a16_kernel(const __grid_constant__ CUtensorMap tmW,   // codes [N][K/2], box 128 B x 8*NB rows, 128B swizzle
             const __grid_constant__ CUtensorMap tmW1,  // the same with a box of 8*(NB-1) rows
             const __grid_constant__ CUtensorMap tmS,   // scales [N][K/16], box 64 B x 8*NB rows (SF_TMA)
             const __grid_constant__ CUtensorMap tmS1,  // the same with a box of 8*(NB-1) rows
             const uint16_t* __restrict__ A, const uint8_t* __restrict__ sW,
             __nv_bfloat16* __restrict__ Y, int M, int N, int K, float out_scale, int nrb) {
    constexpr int STAGES = stages_for(NB);
    constexpr uint32_t STAGE_BYTES = stage_bytes(NB);
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~uintptr_t(1023));
    uint8_t* stages = smem;                                          // 1024-aligned stages
    uint4* aring = reinterpret_cast<uint4*>(smem + (size_t)STAGES * STAGE_BYTES);
    uint64_t* full = reinterpret_cast<uint64_t*>(reinterpret_cast<uint8_t*>(aring) + a_ring_bytes());
    uint64_t* empty = full + 8;
    __shared__ int abort_flag;
    volatile int* abort = &abort_flag;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int G = gridDim.x;
    const int rb0 = (int)((long long)blockIdx.x * nrb / G);
    const int nb = (int)((long long)(blockIdx.x + 1) * nrb / G) - rb0;  // <= NB
    const int nst = (K + STAGE_K - 1) / STAGE_K;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], CONSUMERS);
        }
        abort_flag = 0;
        fence_mbarrier_init();
    }
    __syncthreads();

    if (warp == CONSUMERS) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            // a CTA owns NB or NB - 1 row blocks: the box of the matching height
            const CUtensorMap* mw = nb == NB ? &tmW : &tmW1;
            const CUtensorMap* ms = nb == NB ? &tmS : &tmS1;
            tma_prefetch_desc(mw);
            if (SF_TMA) tma_prefetch_desc(ms);
            const uint32_t bytes = (uint32_t)nb * ROWS * (512u + (SF_TMA ? 64u : 0u));
            const int y = rb0 * ROWS;
            int i = 0;
            for (; i < nst; ++i) {
                const int s = i % STAGES;
                if (!mbar_wait(&empty[s], ((i / STAGES) & 1) ^ 1, abort, ROLE_W16_PRODUCER)) break;
                uint8_t* st = stages + (size_t)s * STAGE_BYTES;
                mbar_arrive_expect_tx(&full[s], bytes);
#pragma unroll
                for (int c = 0; c < 4; ++c)
                    tma_load_2d(st + c * (NB * 1024), mw, &full[s], i * (STAGE_K / 2) + c * 128, y);
                if (SF_TMA) tma_load_2d(st + stage_code_bytes(NB), ms, &full[s], i * (STAGE_K / 16), y);
            }
            // copies still in flight land before the CTA can leave
            for (int j = (i > STAGES ? i - STAGES : 0); j < i; ++j) {
                const uint64_t t0 = globaltimer_ns();
                while (!mbar_try_wait(&full[j % STAGES], (j / STAGES) & 1) &&
                       globaltimer_ns() - t0 < kWaitLimitNs) {
                }
            }
        }
        return;  // the producer takes no part in the epilogue
    }

    // ---------------------------------------------------------------- consumers
    const int w = warp, g = lane >> 2, t = lane & 3;
    const int prow = perm_row(g);  // this lane's weight row within a block
    uint4* aslot = aring + (size_t)w * NA * SLOT_U4 + lane;

    // cp.async of stage i's span-w activations for this lane: tokens g and g+8, its 32 codes
    auto issue_a = [&](int i) {
        if (i < nst) {
            const int k0 = i * STAGE_K + w * SPAN + 32 * t;
            uint4* dst = aslot + (i % NA) * SLOT_U4;
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int tok = g + 8 * h;
                const bool ok = k0 < K && tok < M;
                const uint16_t* src = ok ? A + (size_t)tok * K + k0 : A;
#pragma unroll
                for (int m = 0; m < 4; ++m)
                    cp_async16(dst + (h * 4 + m) * 32, ok ? src + 8 * m : A, ok ? 16u : 0u);
            }
        }
        cp_async_commit();  // one group per stage, empty past the end
    };
    // lane's own scale bytes of stage i, block b (the path without scale TMA)
    auto scale_g = [&](int i, int b) -> uint32_t {
        const int row = (rb0 + b) * ROWS + prow;
        const int k0 = i * STAGE_K + w * SPAN + 32 * t;
        if (i >= nst || b >= nb || row >= N || k0 >= K) return 0u;
        return __ldg(reinterpret_cast<const uint16_t*>(sW + (size_t)row * (K / 16) + k0 / 16));
    };

    float acc[NB][4];
#pragma unroll
    for (int b = 0; b < NB; ++b) acc[b][0] = acc[b][1] = acc[b][2] = acc[b][3] = 0.f;
    uint32_t sc_next[NB];
    if (!SF_TMA) {
#pragma unroll
        for (int b = 0; b < NB; ++b) sc_next[b] = scale_g(0, b);
    }
#pragma unroll
    for (int a = 0; a < NA - 1; ++a) issue_a(a);

    for (int i = 0; i < nst; ++i) {
        const int s = i % STAGES;
        // this stage's activation fragments (K-step 2v + h, see the file comment)
        uint32_t af[8][4];
        cp_async_wait<NA - 2>();
        {
            const uint4* src = aslot + (i % NA) * SLOT_U4;
#pragma unroll
            for (int v = 0; v < 4; ++v) {
                const uint4 x0 = src[v * 32], x1 = src[(4 + v) * 32];  // tokens g, g+8
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const uint32_t lo0 = h ? x0.y : x0.x, hi0 = h ? x0.w : x0.z;
                    const uint32_t lo1 = h ? x1.y : x1.x, hi1 = h ? x1.w : x1.z;
                    af[2 * v + h][0] = prmt(lo0, hi0, 0x5410);  // codes 2h, 2h+4 of token g
                    af[2 * v + h][1] = prmt(lo1, hi1, 0x5410);  // the same of token g+8
                    af[2 * v + h][2] = prmt(lo0, hi0, 0x7632);  // codes 2h+1, 2h+5
                    af[2 * v + h][3] = prmt(lo1, hi1, 0x7632);
                }
            }
        }
        issue_a(i + NA - 1);
        uint32_t sc[NB];
        if (!SF_TMA) {
#pragma unroll
            for (int b = 0; b < NB; ++b) {
                sc[b] = sc_next[b];
                sc_next[b] = scale_g(i + 1, b);
            }
        }
        {
            int ok = 1;
            if (lane == 0) ok = mbar_wait(&full[s], (i / STAGES) & 1, abort, ROLE_W16_CONSUMER) ? 1 : 0;
            if (!__shfl_sync(0xffffffffu, ok, 0)) break;
            // complete already: every lane's own wait orders its reads after the copy
            while (!mbar_try_wait(&full[s], (i / STAGES) & 1)) {
            }
        }
        const uint8_t* st = stages + (size_t)s * STAGE_BYTES;
        // all of this lane's codes and scales of the stage first, then the MMAs
        // interleaved across the row blocks (independent accumulators back to back)
        uint32_t wq[NB][4], ss[NB][2];
#pragma unroll
        for (int b = 0; b < NB; ++b) {
            uint4 q = make_uint4(0u, 0u, 0u, 0u);
            uint32_t sb2 = 0u;
            if (b < nb) {
                q = *reinterpret_cast<const uint4*>(
                    st + ((w >> 1) * NB * 8 + b * 8 + prow) * 128 + ((((w & 1) * 4 + t) ^ prow) << 4));
                sb2 = SF_TMA ? (uint32_t)*reinterpret_cast<const uint16_t*>(
                                   st + stage_code_bytes(NB) + (b * 8 + prow) * 64 + w * 8 + t * 2)
                             : sc[b];
            }
            wq[b][0] = q.x; wq[b][1] = q.y; wq[b][2] = q.z; wq[b][3] = q.w;
            ss[b][0] = scale_pair(sb2 & 0xFFu);
            ss[b][1] = scale_pair((sb2 >> 8) & 0xFFu);
        }
#pragma unroll
        for (int v = 0; v < 4; ++v) {
            uint32_t p[NB][4];
#pragma unroll
            for (int b = 0; b < NB; ++b) widen8(wq[b][v], ss[b][v >> 1], p[b]);
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const uint32_t(&a)[4] = af[2 * v + h];
#pragma unroll
                for (int b = 0; b < NB; ++b)
                    if (b < nb) mma_bf16(acc[b], a[0], a[1], a[2], a[3], p[b][2 * h], p[b][2 * h + 1]);
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[s]);  // this warp has read the stage
    }
    cp_async_wait<0>();

    // ---- the warps' partials meet in the (now idle) activation slots: red[w][b][lane][4]
    named_bar_sync(1, 32 * CONSUMERS);
    float* red = reinterpret_cast<float*>(aring);
#pragma unroll
    for (int b = 0; b < NB; ++b)
        if (b < nb)
            *reinterpret_cast<float4*>(red + ((size_t)(w * NB + b) * 32 + lane) * 4) =
                make_float4(acc[b][0], acc[b][1], acc[b][2], acc[b][3]);
    named_bar_sync(1, 32 * CONSUMERS);

    // ---- fixed-order sum over the warps; D[tok][n] of lane l -> Y[tok][block row PERM(n)]
    for (int idx = threadIdx.x; idx < nb * 128; idx += 32 * CONSUMERS) {
        const int b = idx >> 7, l = (idx >> 2) & 31, e = idx & 3;
        float sum = 0.f;
#pragma unroll
        for (int ww = 0; ww < CONSUMERS; ++ww) sum += red[((size_t)(ww * NB + b) * 32 + l) * 4 + e];
        const int tok = (l >> 2) + 8 * (e >> 1);
        const int row = (rb0 + b) * ROWS + perm_row(2 * (l & 3) + (e & 1));
        if (tok < M && row < N) Y[(size_t)tok * N + row] = __float2bfloat16_rn(sum * out_scale);
    }
}

}  // namespace w4a16
}  // namespace nvfp4
