// via_fp8_kernel.cuh -- the NVFP4 matmul through the exact E2M1 -> E4M3
// conversion on the FP8 tensor-core MMA (metrale_circuit `hardware::exec`
// module doc, bullet 2).
//
// Each code is placed in the high nibble of a byte and converted by the page's
// identity (q & 0x80808080) | ((q & 0x70707070) >> 2), an E4M3 byte worth the
// code's value times 2^-6.  For every 16-group g an FP8 MMA (kind::f8f6f4,
// E4M3 x E4M3 -> FP32, K = 32) forms the exact partial
//     P_g[m,n] = sum_{k in g} a8[m,k] * w8[n,k]
// (products lie on a 2^-14 grid, |P_g| <= 576 * 2^-12: exact in FP32), and the
// block scales with the folded 2^6 are applied in FP32 per K = 16 step:
//     acc[m,n] += P_g[m,n] * ((sA[m,g] * 2^6) * (sW[n,g] * 2^6))
// where the scale product (8 significant bits) and the scaled partial are
// exact, so the only rounding is the FP32 accumulation, as on the W4A4 path.
//
// One K = 32 MMA covers one group: the A operand's second 16-byte K chunk (for
// an even group) or first chunk (odd group) is a shared all-zero tile, reached
// through the smem descriptor's leading byte offset -- no zeros are copied.
//
// Roles (one persistent CTA per SM, 20 warps, 128 x 128 output tiles):
//   warp 0      TMA producer: packed FP4 A/W K-blocks (256 codes, 128-byte
//               swizzle) and their raw [rows][16 B] scale tiles.
//   warp 1      TMEM owner, MMA issuer: one MMA per group into a 4-deep ring
//               of 128-column FP32 partial buffers.
//   warps 2-3   converters: FP4 -> E4M3 by the identity, into per-group
//               [rows][16 B] operand tiles; scales -> FP32 (x 2^6).
//   warps 4-19  scale-apply + epilogue: warp w reads TMEM lane quarter w % 4
//               (32 rows) and column slab (w - 4) / 4 (32 columns) of every
//               partial, and adds P * (sA*64)(sW*64) with packed f32x2 FMAs into
//               32 FP32 accumulators per thread; at the end of a tile, x alpha,
//               BF16 RNE, store.
// Every 16-group's 128 x 128 FP32 partial leaves TMEM to be scaled: two FP32
// operations per output element per group (the scale product and the FMA), which
// the FP32 pipe bounds, not the FP8 tensor pipe.  Sixteen apply warps keep four
// TMEM reads and their arithmetic in flight per scheduler.  Requires
// K % 256 == 0 (TMA of the scale tiles).
#pragma once
#include <cuda_bf16.h>
#include <cstdint>

#include "ptx.cuh"

namespace nvfp4 {
namespace via_fp8 {

constexpr int BM = 128, BN = 128;
constexpr int BK = 256;              // codes per raw K-block
constexpr int RSTAGES = 4;           // raw K-block ring
constexpr int NSLOTS = 4;            // converted group-pair ring
constexpr int NPART = 4;             // TMEM partial buffers (128 columns each)
constexpr int CONV_WARPS = 2, APPLY_WARPS = 16;
constexpr int FIRST_APPLY = 2 + CONV_WARPS;       // a multiple of 4: warp % 4 = lane quarter
constexpr int SLAB = BN / (APPLY_WARPS / 4);      // columns per apply warp (32)
constexpr int NUM_THREADS = 32 * (2 + CONV_WARPS + APPLY_WARPS);
static_assert(FIRST_APPLY % 4 == 0 && SLAB == 32, "apply warps: 4 per lane quarter, 32 columns each");
constexpr int GROUP_M = 8;

enum Role { ROLE_PRODUCER = 1, ROLE_MMA = 2, ROLE_CONV = 3, ROLE_APPLY = 4, ROLE_DRAIN = 5 };

struct Smem {
    alignas(1024) uint8_t raw_a[RSTAGES][BM * 128];   // 128-byte swizzled rows
    alignas(1024) uint8_t raw_b[RSTAGES][BN * 128];
    alignas(16) uint8_t raw_sa[RSTAGES][BM * 16];     // [row][16 groups]
    alignas(16) uint8_t raw_sb[RSTAGES][BN * 16];
    alignas(128) uint8_t zlo[BM * 16];                // zero tile below every a8 tile
    alignas(128) uint8_t a8[NSLOTS][2][BM * 16];      // [slot][group of pair][row][16 B]
    alignas(128) uint8_t b8[NSLOTS][2][BN * 16];
    alignas(128) uint8_t zhi[BM * 16];                // zero tile above every a8 tile
    alignas(16) float sa_f[NSLOTS][2][BM];            // sA * 2^6
    alignas(16) float sw_f[NSLOTS][2][BN];            // sW * 2^6
    uint64_t raw_full[RSTAGES], raw_empty[RSTAGES];
    uint64_t slot_full[NSLOTS], slot_empty[NSLOTS];
    uint64_t part_full[NPART], part_empty[NPART];
    uint64_t drain;
    uint32_t tmem_base;
    int abort;
};
constexpr size_t SMEM_BYTES = sizeof(Smem) + 1024;
constexpr uint32_t RAW_BYTES = (BM + BN) * 128 + (BM + BN) * 16;

__device__ __forceinline__ void tile_coords(int tile, int num_m, int num_n, int& mb, int& nb) {
    const int per_group = GROUP_M * num_n;
    const int first_m = (tile / per_group) * GROUP_M;
    const int gsize = min(num_m - first_m, GROUP_M);
    const int in_group = tile % per_group;
    mb = first_m + in_group % gsize;
    nb = in_group / gsize;
}

__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort,
                                          int role) {
    int ok = 1;
    if ((threadIdx.x & 31) == 0) ok = mbar_wait(bar, parity, abort, role) ? 1 : 0;
    return __shfl_sync(0xffffffffu, ok, 0) != 0;
}

// The page's identity on four codes held in the high nibbles of q.
__device__ __forceinline__ uint32_t e2m1_hi_to_e4m3(uint32_t q) {
    return (q & 0x80808080u) | ((q & 0x70707070u) >> 2);
}

// Eight packed codes (even k in the low nibble) -> eight E4M3 bytes in k order.
__device__ __forceinline__ uint2 convert8(uint32_t w) {
    const uint32_t lo = e2m1_hi_to_e4m3((w << 4) & 0xF0F0F0F0u);  // k = 0, 2, 4, 6
    const uint32_t hi = e2m1_hi_to_e4m3(w & 0xF0F0F0F0u);         // k = 1, 3, 5, 7
    return make_uint2(__byte_perm(lo, hi, 0x5140), __byte_perm(lo, hi, 0x7362));
}

// Word i (0..3) of four held in registers, without indexing local memory.
__device__ __forceinline__ uint32_t pick4(const uint32_t (&a)[4], int i) {
    const uint32_t lo = (i & 1) ? a[1] : a[0], hi = (i & 1) ? a[3] : a[2];
    return (i & 2) ? hi : lo;
}

// Non-negative E4M3 scale byte -> its value times 2^6, as FP32 (exact).
__device__ __forceinline__ float scale_x64(uint32_t b) {
    const uint32_t E = (b >> 3) & 15u, M = b & 7u;
    if (E == 0) return (float)M * 0.125f;
    return __uint_as_float(((E + 126u) << 23) | (M << 20));
}

__device__ __forceinline__ uint64_t fma2(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}
__device__ __forceinline__ uint64_t mul2(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ uint64_t pack2(uint32_t lo, uint32_t hi) {
    return (uint64_t)lo | ((uint64_t)hi << 32);
}

__global__ void __launch_bounds__(NUM_THREADS, 1)
via_fp8_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
               const __grid_constant__ CUtensorMap tmSA, const __grid_constant__ CUtensorMap tmSB,
               __nv_bfloat16* __restrict__ Y, int M, int N, int K, float alpha) {
    extern __shared__ uint8_t smem_raw[];
    Smem& sm = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                        ~uintptr_t(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int num_m = (M + BM - 1) / BM, num_n = (N + BN - 1) / BN;
    const int tiles = num_m * num_n;
    const int num_kb = K / BK;
    volatile int* abort = &sm.abort;

    if (threadIdx.x == 0) {
        for (int s = 0; s < RSTAGES; ++s) {
            mbar_init(&sm.raw_full[s], 1);
            mbar_init(&sm.raw_empty[s], CONV_WARPS);
        }
        for (int s = 0; s < NSLOTS; ++s) {
            mbar_init(&sm.slot_full[s], CONV_WARPS);
            mbar_init(&sm.slot_empty[s], 1 + APPLY_WARPS);
        }
        for (int p = 0; p < NPART; ++p) {
            mbar_init(&sm.part_full[p], 1);
            mbar_init(&sm.part_empty[p], APPLY_WARPS);
        }
        mbar_init(&sm.drain, 1);
        sm.abort = 0;
        fence_mbarrier_init();
        tma_prefetch_desc(&tmA);
        tma_prefetch_desc(&tmB);
        tma_prefetch_desc(&tmSA);
        tma_prefetch_desc(&tmSB);
    }
    for (int i = threadIdx.x; i < BM * 16 / 4; i += NUM_THREADS) {
        reinterpret_cast<uint32_t*>(sm.zlo)[i] = 0u;
        reinterpret_cast<uint32_t*>(sm.zhi)[i] = 0u;
    }
    fence_proxy_async_smem();
    if (warp == 1) {
        tmem_alloc(&sm.tmem_base, NPART * 128);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem_base;

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        // The whole warp walks the loop (converged); one elected lane issues.
        int it = 0;
        bool ok = true;
        for (int tile = blockIdx.x; tile < tiles && ok; tile += gridDim.x) {
            int mb, nb;
            tile_coords(tile, num_m, num_n, mb, nb);
            for (int kb = 0; kb < num_kb; ++kb, ++it) {
                const int r = it % RSTAGES;
                if (!warp_wait(&sm.raw_empty[r], ((it / RSTAGES) & 1) ^ 1, abort, ROLE_PRODUCER)) {
                    ok = false;
                    break;
                }
                if (elect_one()) {
                    mbar_arrive_expect_tx(&sm.raw_full[r], RAW_BYTES);
                    tma_load_2d(sm.raw_a[r], &tmA, &sm.raw_full[r], kb * 128, mb * BM);
                    tma_load_2d(sm.raw_b[r], &tmB, &sm.raw_full[r], kb * 128, nb * BN);
                    tma_load_2d(sm.raw_sa[r], &tmSA, &sm.raw_full[r], kb * 16, mb * BM);
                    tma_load_2d(sm.raw_sb[r], &tmSB, &sm.raw_full[r], kb * 16, nb * BN);
                }
                __syncwarp();
            }
        }
        if (!ok && lane == 0) {
            // every copy this warp started lands before the CTA can exit
            for (int j = max(0, it - RSTAGES); j < it; ++j) {
                const uint64_t t0 = globaltimer_ns();
                while (!mbar_try_wait(&sm.raw_full[j % RSTAGES], (j / RSTAGES) & 1) &&
                       globaltimer_ns() - t0 < kWaitLimitNs) {
                }
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        // The whole warp walks the loop (converged, as tcgen05 issue wants it); the
        // same elected lane issues every MMA and every commit that tracks them.
        const uint32_t idesc = idesc_f8f6f4_e4m3(BM, BN);
        const uint32_t zlo = smem_u32(sm.zlo), zhi = smem_u32(sm.zhi);
        int pc = 0, gc = 0;
        bool ok = true;
        for (int tile = blockIdx.x; tile < tiles && ok; tile += gridDim.x) {
            for (int pair = 0; pair < num_kb * 8 && ok; ++pair, ++pc) {
                const int sl = pc % NSLOTS;
                if (!warp_wait(&sm.slot_full[sl], (pc / NSLOTS) & 1, abort, ROLE_MMA)) { ok = false; break; }
                const uint32_t a_even = smem_u32(sm.a8[sl][0]), a_odd = smem_u32(sm.a8[sl][1]);
                const uint32_t b0 = smem_u32(sm.b8[sl][0]), b1 = smem_u32(sm.b8[sl][1]);
                // B: the K = 32 slice holding both groups of the pair
                const uint64_t bdesc = smem_desc(b0, b1 - b0, 128, 0);
#pragma unroll
                for (int gi = 0; gi < 2; ++gi, ++gc) {
                    const int p = gc % NPART;
                    if (!warp_wait(&sm.part_empty[p], ((gc / NPART) & 1) ^ 1, abort, ROLE_MMA)) { ok = false; break; }
                    tc_fence_after();
                    if (elect_one()) {
                        // A: this group's 16 bytes in one K chunk, the other chunk all zero
                        const uint64_t adesc = gi == 0 ? smem_desc(a_even, zhi - a_even, 128, 0)
                                                       : smem_desc(zlo, a_odd - zlo, 128, 0);
                        mma_f8f6f4(tmem + p * 128, adesc, bdesc, idesc, 0u);
                        mma_commit(&sm.part_full[p]);
                    }
                    __syncwarp();
                }
                if (ok && elect_one()) mma_commit(&sm.slot_empty[sl]);
                __syncwarp();
            }
        }
        // every MMA issued completes before TMEM is freed
        if (elect_one()) {
            mma_commit(&sm.drain);
            const uint64_t t0 = globaltimer_ns();
            while (!mbar_try_wait(&sm.drain, 0)) {
                if (globaltimer_ns() - t0 > kWaitLimitNs) {
                    atomicOr(&g_device_error, 1 | (ROLE_DRAIN << 8));
                    break;
                }
            }
        }
        __syncwarp();
    } else if (warp < 2 + CONV_WARPS) {
        // ------------------------------------------------------------ converters
        const int ctid = threadIdx.x - 64;  // 0..63: rows ctid and ctid + 64 of A and of W
        int it = 0, pc = 0;
        for (int tile = blockIdx.x; tile < tiles; tile += gridDim.x) {
            bool ok = true;
            for (int kb = 0; kb < num_kb && ok; ++kb, ++it) {
                const int r = it % RSTAGES;
                if (!warp_wait(&sm.raw_full[r], (it / RSTAGES) & 1, abort, ROLE_CONV)) { ok = false; break; }
                uint32_t saw[2][4], sbw[2][4];
#pragma unroll
                for (int rr = 0; rr < 2; ++rr) {
                    const uint4 a = *reinterpret_cast<const uint4*>(sm.raw_sa[r] + (ctid + 64 * rr) * 16);
                    const uint4 b = *reinterpret_cast<const uint4*>(sm.raw_sb[r] + (ctid + 64 * rr) * 16);
                    saw[rr][0] = a.x; saw[rr][1] = a.y; saw[rr][2] = a.z; saw[rr][3] = a.w;
                    sbw[rr][0] = b.x; sbw[rr][1] = b.y; sbw[rr][2] = b.z; sbw[rr][3] = b.w;
                }
#pragma unroll 1
                for (int h = 0; h < 8; ++h, ++pc) {
                    const int sl = pc % NSLOTS;
                    if (!warp_wait(&sm.slot_empty[sl], ((pc / NSLOTS) & 1) ^ 1, abort, ROLE_CONV)) { ok = false; break; }
#pragma unroll
                    for (int rr = 0; rr < 2; ++rr) {
                        const int row = ctid + 64 * rr;
                        // 16-byte chunk h of the row (groups 2h, 2h+1) under the 128-byte swizzle
                        const int off = row * 128 + ((h ^ (row & 7)) << 4);
                        const uint4 qa = *reinterpret_cast<const uint4*>(sm.raw_a[r] + off);
                        const uint4 qb = *reinterpret_cast<const uint4*>(sm.raw_b[r] + off);
                        const uint2 a0 = convert8(qa.x), a1 = convert8(qa.y), a2 = convert8(qa.z), a3 = convert8(qa.w);
                        const uint2 b0 = convert8(qb.x), b1 = convert8(qb.y), b2 = convert8(qb.z), b3 = convert8(qb.w);
                        *reinterpret_cast<uint4*>(sm.a8[sl][0] + row * 16) = make_uint4(a0.x, a0.y, a1.x, a1.y);
                        *reinterpret_cast<uint4*>(sm.a8[sl][1] + row * 16) = make_uint4(a2.x, a2.y, a3.x, a3.y);
                        *reinterpret_cast<uint4*>(sm.b8[sl][0] + row * 16) = make_uint4(b0.x, b0.y, b1.x, b1.y);
                        *reinterpret_cast<uint4*>(sm.b8[sl][1] + row * 16) = make_uint4(b2.x, b2.y, b3.x, b3.y);
                        // scale bytes g0 = 2h and g1 = 2h + 1: bytes 2(h&1), 2(h&1)+1 of word h/2
                        const uint32_t wa = pick4(saw[rr], h >> 1) >> (16 * (h & 1));
                        const uint32_t wb = pick4(sbw[rr], h >> 1) >> (16 * (h & 1));
                        sm.sa_f[sl][0][row] = scale_x64(wa & 0xFFu);
                        sm.sa_f[sl][1][row] = scale_x64((wa >> 8) & 0xFFu);
                        sm.sw_f[sl][0][row] = scale_x64(wb & 0xFFu);
                        sm.sw_f[sl][1][row] = scale_x64((wb >> 8) & 0xFFu);
                    }
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&sm.slot_full[sl]);
                }
                __syncwarp();
                if (ok && lane == 0) mbar_arrive(&sm.raw_empty[r]);
            }
            if (!ok) break;
        }
    } else {
        // ------------------------------------------------------------ scale-apply + epilogue
        const int q = warp & 3;                    // TMEM lane quarter
        const int slab = (warp - FIRST_APPLY) >> 2;  // 32-column slab of the tile
        const int trow = 32 * q + lane;            // row within the tile
        const bool vec_ok = (N % 8) == 0;
        int pc = 0, gc = 0;
        for (int tile = blockIdx.x; tile < tiles; tile += gridDim.x) {
            int mb, nb;
            tile_coords(tile, num_m, num_n, mb, nb);
            uint64_t acc[SLAB / 2];  // FP32 pairs
#pragma unroll
            for (int j = 0; j < SLAB / 2; ++j) acc[j] = 0ull;
            bool ok = true;
            for (int pair = 0; pair < num_kb * 8 && ok; ++pair, ++pc) {
                const int sl = pc % NSLOTS;
                if (!warp_wait(&sm.slot_full[sl], (pc / NSLOTS) & 1, abort, ROLE_APPLY)) { ok = false; break; }
#pragma unroll
                for (int gi = 0; gi < 2; ++gi, ++gc) {
                    const int p = gc % NPART;
                    if (!warp_wait(&sm.part_full[p], (gc / NPART) & 1, abort, ROLE_APPLY)) { ok = false; break; }
                    tc_fence_after();
                    uint32_t v[32];
                    tmem_ld_32x32b_x32(tmem + ((uint32_t)(32 * q) << 16) + p * 128 + slab * SLAB, v);
                    tmem_ld_wait();
                    reg_fence(v);
                    // the partial is in registers: hand its columns back to the MMA
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&sm.part_empty[p]);
                    // acc += P * ((sA*64) * (sW*64)): the scale product has at most 8
                    // significant bits and P*S at most 22, so both are exact and the FMA
                    // rounds once, into the accumulator (packed f32x2 lanes)
                    const float sa = sm.sa_f[sl][gi][trow];
                    const uint64_t sa2 = pack2(__float_as_uint(sa), __float_as_uint(sa));
                    const float4* sw4 = reinterpret_cast<const float4*>(&sm.sw_f[sl][gi][slab * SLAB]);
#pragma unroll
                    for (int i = 0; i < SLAB / 4; ++i) {
                        const float4 w4 = sw4[i];
                        const uint64_t s01 = mul2(sa2, pack2(__float_as_uint(w4.x), __float_as_uint(w4.y)));
                        const uint64_t s23 = mul2(sa2, pack2(__float_as_uint(w4.z), __float_as_uint(w4.w)));
                        acc[2 * i] = fma2(pack2(v[4 * i], v[4 * i + 1]), s01, acc[2 * i]);
                        acc[2 * i + 1] = fma2(pack2(v[4 * i + 2], v[4 * i + 3]), s23, acc[2 * i + 1]);
                    }
                }
                __syncwarp();
                if (ok && lane == 0) mbar_arrive(&sm.slot_empty[sl]);
            }
            if (!ok) break;
            // epilogue: x alpha, BF16 RNE, store this thread's 32 columns
            const int row = mb * BM + trow;
            const int col0 = nb * BN + slab * SLAB;
            if (row < M) {
                uint32_t packed[SLAB / 2];
#pragma unroll
                for (int j = 0; j < SLAB / 2; ++j) {
                    __nv_bfloat162 h2 = __floats2bfloat162_rn(__fmul_rn(__uint_as_float((uint32_t)acc[j]), alpha),
                                                              __fmul_rn(__uint_as_float((uint32_t)(acc[j] >> 32)), alpha));
                    packed[j] = *reinterpret_cast<uint32_t*>(&h2);
                }
                __nv_bfloat16* yrow = Y + (size_t)row * N;
                if (vec_ok && col0 + SLAB <= N) {
                    uint4* dst = reinterpret_cast<uint4*>(yrow + col0);
#pragma unroll
                    for (int j = 0; j < SLAB / 8; ++j)
                        dst[j] = make_uint4(packed[4 * j], packed[4 * j + 1], packed[4 * j + 2], packed[4 * j + 3]);
                } else {
                    uint16_t* y16 = reinterpret_cast<uint16_t*>(yrow);
#pragma unroll
                    for (int j = 0; j < SLAB; ++j)
                        if (col0 + j < N) y16[col0 + j] = (uint16_t)(packed[j >> 1] >> (16 * (j & 1)));
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem, NPART * 128);
}

}  // namespace via_fp8
}  // namespace nvfp4
