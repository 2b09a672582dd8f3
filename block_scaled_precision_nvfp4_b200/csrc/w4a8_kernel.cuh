// w4a8_kernel.cuh -- FP8 (E4M3) activations under NVFP4 weights on the exact
// E4M3 path (metrale_circuit `hardware::exec`, exec_of: "NVFP4 weights under
// FP8 activations (W4A8 with group-16 E4M3 scales) have no single-instruction
// MMA ...; they take the exact E4M3 path").
//
//     Y[m,n] = gA*gW * sum_g sW[n,g] * sum_{k in g} a8[m,k] * e2m1(W[n,k])
//
// The weights go through the page's identity (each code in the high nibble of
// a byte: (q & 0x80808080) | ((q & 0x70707070) >> 2), an E4M3 byte worth the
// code's value times 2^-6); the activations are E4M3 already.  For every
// 16-group an FP8 MMA (kind::f8f6f4, E4M3 x E4M3 -> FP32, K = 32) forms the
// group's partial, and the weights' group scale with the folded 2^6 is applied
// in FP32 per K = 16 step:  acc[m,n] += P_g[m,n] * (sW[n,g] * 2^6).
// Each product has at most 6 significant bits, so P_g is exact in FP32 unless
// the group's nonzero products span more than 2^15 in magnitude; the scale
// apply is one fused multiply-add.
//
// One K = 32 MMA covers one group: A's K = 32 slice (two groups) comes straight
// from the TMA-loaded, 128-byte-swizzled activation tile, and B holds the group
// in one 16-byte K chunk and a shared all-zero tile in the other (reached
// through the smem descriptor's leading byte offset), so the other group of
// the slice contributes nothing.
//
// Roles (one persistent CTA per SM, 12 warps, 128 x 128 output tiles), as on
// the W4A4 exact path (via_fp8_kernel.cuh):
//   warp 0      TMA producer: E4M3 activation K-blocks (256 bytes of a row as
//               two 128-byte swizzled boxes), packed FP4 weight K-blocks and
//               the weights' raw [rows][16 B] scale tiles.
//   warp 1      TMEM owner, MMA issuer: one MMA per group into a 4-deep ring of
//               128-column FP32 partial buffers; it also releases the raw stage
//               (its MMAs read the activations there).
//   warps 2-3   converters: weight codes -> E4M3 per-group [rows][16 B] tiles;
//               weight scales -> FP32 (x 2^6).
//   warps 4-11  scale-apply + epilogue: per group, partial TMEM -> registers,
//               acc += P * (sW*64) with packed f32x2 FMAs; at the end of a
//               tile, x alpha, BF16 RNE, store.
// Requires K % 256 == 0 (TMA of the scale tiles).
#pragma once
#include <cuda_bf16.h>
#include <cstdint>

#include "ptx.cuh"
#include "via_fp8_kernel.cuh"

namespace nvfp4 {
namespace w4a8 {

using via_fp8::convert8;
using via_fp8::fma2;
using via_fp8::pack2;
using via_fp8::scale_x64;
using via_fp8::tile_coords;
using via_fp8::warp_wait;

constexpr int BM = 128, BN = 128;
constexpr int BK = 256;              // codes per raw K-block (16 groups)
constexpr int RSTAGES = 3;           // raw K-block ring
constexpr int NSLOTS = 4;            // converted group-pair ring
constexpr int NPART = 4;             // TMEM partial buffers (128 columns each)
constexpr int CONV_WARPS = 2, APPLY_WARPS = 8;
constexpr int NUM_THREADS = 32 * (2 + CONV_WARPS + APPLY_WARPS);

enum Role { ROLE_PRODUCER = 1, ROLE_MMA = 2, ROLE_CONV = 3, ROLE_APPLY = 4, ROLE_DRAIN = 5 };

struct Smem {
    alignas(1024) uint8_t raw_a[RSTAGES][2][BM * 128];  // E4M3 activations, two swizzled boxes
    alignas(1024) uint8_t raw_b[RSTAGES][BN * 128];     // packed FP4 weights, swizzled
    alignas(16) uint8_t raw_sb[RSTAGES][BN * 16];       // weight scales [row][16 groups]
    alignas(128) uint8_t zlo[BN * 16];                  // zero tile below every b8 tile
    alignas(128) uint8_t b8[NSLOTS][2][BN * 16];        // [slot][group of pair][row][16 B]
    alignas(128) uint8_t zhi[BN * 16];                  // zero tile above every b8 tile
    alignas(16) float sw_f[NSLOTS][2][BN];              // sW * 2^6
    uint64_t raw_full[RSTAGES], raw_empty[RSTAGES];
    uint64_t slot_full[NSLOTS], slot_empty[NSLOTS];
    uint64_t part_full[NPART], part_empty[NPART];
    uint64_t drain;
    uint32_t tmem_base;
    int abort;
};
constexpr size_t SMEM_BYTES = sizeof(Smem) + 1024;
constexpr uint32_t RAW_BYTES = BM * 256 + BN * 128 + BN * 16;

__global__ void __launch_bounds__(NUM_THREADS, 1)
w4a8_kernel(const __grid_constant__ CUtensorMap tmA,   // E4M3 [M][K], box 128 B x 128 rows
            const __grid_constant__ CUtensorMap tmB,   // packed W [N][K/2], box 128 B x 128 rows
            const __grid_constant__ CUtensorMap tmSB,  // sW [N][K/16], box 16 B x 128 rows
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
            mbar_init(&sm.raw_empty[s], CONV_WARPS + 1);  // converters + the MMA's commit
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
        tma_prefetch_desc(&tmSB);
    }
    for (int i = threadIdx.x; i < BN * 16 / 4; i += NUM_THREADS) {
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
        if (lane == 0) {
            int it = 0;
            for (int tile = blockIdx.x; tile < tiles && !*abort; tile += gridDim.x) {
                int mb, nb;
                tile_coords(tile, num_m, num_n, mb, nb);
                for (int kb = 0; kb < num_kb; ++kb, ++it) {
                    const int r = it % RSTAGES;
                    if (!mbar_wait(&sm.raw_empty[r], ((it / RSTAGES) & 1) ^ 1, abort, ROLE_PRODUCER))
                        goto producer_done;
                    mbar_arrive_expect_tx(&sm.raw_full[r], RAW_BYTES);
                    tma_load_2d(sm.raw_a[r][0], &tmA, &sm.raw_full[r], kb * 256, mb * BM);
                    tma_load_2d(sm.raw_a[r][1], &tmA, &sm.raw_full[r], kb * 256 + 128, mb * BM);
                    tma_load_2d(sm.raw_b[r], &tmB, &sm.raw_full[r], kb * 128, nb * BN);
                    tma_load_2d(sm.raw_sb[r], &tmSB, &sm.raw_full[r], kb * 16, nb * BN);
                }
            }
        producer_done:
            if (*abort) {
                for (int j = max(0, it - RSTAGES); j < it; ++j) {
                    const uint64_t t0 = globaltimer_ns();
                    while (!mbar_try_wait(&sm.raw_full[j % RSTAGES], (j / RSTAGES) & 1) &&
                           globaltimer_ns() - t0 < kWaitLimitNs) {
                    }
                }
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            const uint32_t idesc = idesc_f8f6f4_e4m3(BM, BN);
            const uint32_t zlo = smem_u32(sm.zlo), zhi = smem_u32(sm.zhi);
            int pc = 0, gc = 0, it = 0;
            bool ok = true;
            for (int tile = blockIdx.x; tile < tiles && ok; tile += gridDim.x) {
                for (int kb = 0; kb < num_kb && ok; ++kb, ++it) {
                    const int r = it % RSTAGES;
                    // the activations are read from the raw stage itself: wait for its
                    // TMA bytes here too (the stage cannot be refilled before this
                    // K-block's commit below, so the phase cannot run ahead)
                    if (!mbar_wait(&sm.raw_full[r], (it / RSTAGES) & 1, abort, ROLE_MMA)) { ok = false; break; }
                    for (int h = 0; h < 8 && ok; ++h, ++pc) {
                        const int sl = pc % NSLOTS;
                        if (!mbar_wait(&sm.slot_full[sl], (pc / NSLOTS) & 1, abort, ROLE_MMA)) { ok = false; break; }
                        // A: the pair's 32 bytes of the row (groups 2h, 2h+1), straight from
                        // the swizzled activation box
                        const uint64_t adesc =
                            desc_kmajor_sw128(smem_u32(sm.raw_a[r][h >> 2]) + (h & 3) * 32);
                        const uint32_t b0 = smem_u32(sm.b8[sl][0]), b1 = smem_u32(sm.b8[sl][1]);
#pragma unroll
                        for (int gi = 0; gi < 2; ++gi, ++gc) {
                            const int p = gc % NPART;
                            if (!mbar_wait(&sm.part_empty[p], ((gc / NPART) & 1) ^ 1, abort, ROLE_MMA)) { ok = false; break; }
                            tc_fence_after();
                            // B: the group in its own K chunk, the other chunk all zero
                            const uint64_t bdesc = gi == 0 ? smem_desc(b0, zhi - b0, 128, 0)
                                                           : smem_desc(zlo, b1 - zlo, 128, 0);
                            mma_f8f6f4(tmem + p * 128, adesc, bdesc, idesc, 0u);
                            mma_commit(&sm.part_full[p]);
                        }
                        if (ok) mma_commit(&sm.slot_empty[sl]);
                    }
                    if (ok) mma_commit(&sm.raw_empty[r]);  // the activations of this stage are read
                }
            }
            mma_commit(&sm.drain);
            const uint64_t t0 = globaltimer_ns();
            while (!mbar_try_wait(&sm.drain, 0)) {
                if (globaltimer_ns() - t0 > kWaitLimitNs) {
                    atomicOr(&g_device_error, 1 | (ROLE_DRAIN << 8));
                    break;
                }
            }
        }
    } else if (warp < 2 + CONV_WARPS) {
        // ------------------------------------------------------------ converters (weights)
        const int ctid = threadIdx.x - 64;  // 0..63: weight rows ctid and ctid + 64
        int it = 0, pc = 0;
        bool ok = true;
        for (int tile = blockIdx.x; tile < tiles && ok; tile += gridDim.x) {
            for (int kb = 0; kb < num_kb && ok; ++kb, ++it) {
                const int r = it % RSTAGES;
                if (!warp_wait(&sm.raw_full[r], (it / RSTAGES) & 1, abort, ROLE_CONV)) { ok = false; break; }
                uint32_t sbw[2][4];
#pragma unroll
                for (int rr = 0; rr < 2; ++rr) {
                    const uint4 b = *reinterpret_cast<const uint4*>(sm.raw_sb[r] + (ctid + 64 * rr) * 16);
                    sbw[rr][0] = b.x; sbw[rr][1] = b.y; sbw[rr][2] = b.z; sbw[rr][3] = b.w;
                }
#pragma unroll 1
                for (int h = 0; h < 8; ++h, ++pc) {
                    const int sl = pc % NSLOTS;
                    if (!warp_wait(&sm.slot_empty[sl], ((pc / NSLOTS) & 1) ^ 1, abort, ROLE_CONV)) { ok = false; break; }
                    const int g0 = 2 * h, g1 = 2 * h + 1;
#pragma unroll
                    for (int rr = 0; rr < 2; ++rr) {
                        const int row = ctid + 64 * rr;
                        // 16-byte chunk h of the row (groups 2h, 2h+1) under the 128-byte swizzle
                        const uint4 qb = *reinterpret_cast<const uint4*>(
                            sm.raw_b[r] + row * 128 + ((h ^ (row & 7)) << 4));
                        const uint2 b0 = convert8(qb.x), b1 = convert8(qb.y), b2 = convert8(qb.z),
                                    b3 = convert8(qb.w);
                        *reinterpret_cast<uint4*>(sm.b8[sl][0] + row * 16) = make_uint4(b0.x, b0.y, b1.x, b1.y);
                        *reinterpret_cast<uint4*>(sm.b8[sl][1] + row * 16) = make_uint4(b2.x, b2.y, b3.x, b3.y);
                        sm.sw_f[sl][0][row] = scale_x64((sbw[rr][g0 >> 2] >> (8 * (g0 & 3))) & 0xFFu);
                        sm.sw_f[sl][1][row] = scale_x64((sbw[rr][g1 >> 2] >> (8 * (g1 & 3))) & 0xFFu);
                    }
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&sm.slot_full[sl]);
                }
                __syncwarp();
                if (ok && lane == 0) mbar_arrive(&sm.raw_empty[r]);
            }
        }
    } else {
        // ------------------------------------------------------------ scale-apply + epilogue
        const int q = warp & 3;                         // TMEM lane quarter
        const int half = (warp - 2 - CONV_WARPS) >> 2;  // column half
        const int trow = 32 * q + lane;                 // row within the tile
        const bool vec_ok = (N % 8) == 0;
        int pc = 0, gc = 0;
        bool ok = true;
        for (int tile = blockIdx.x; tile < tiles && ok; tile += gridDim.x) {
            int mb, nb;
            tile_coords(tile, num_m, num_n, mb, nb);
            uint64_t acc[32];
#pragma unroll
            for (int j = 0; j < 32; ++j) acc[j] = 0ull;
            for (int pair = 0; pair < num_kb * 8 && ok; ++pair, ++pc) {
                const int sl = pc % NSLOTS;
                if (!warp_wait(&sm.slot_full[sl], (pc / NSLOTS) & 1, abort, ROLE_APPLY)) { ok = false; break; }
#pragma unroll
                for (int gi = 0; gi < 2; ++gi, ++gc) {
                    const int p = gc % NPART;
                    if (!warp_wait(&sm.part_full[p], (gc / NPART) & 1, abort, ROLE_APPLY)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t ta = tmem + ((uint32_t)(32 * q) << 16) + p * 128 + half * 64;
                    const float4* sw4 = reinterpret_cast<const float4*>(&sm.sw_f[sl][gi][half * 64]);
#pragma unroll
                    for (int c = 0; c < 2; ++c) {
                        uint32_t v[32];
                        tmem_ld_32x32b_x32(ta + 32 * c, v);
                        tmem_ld_wait();
                        reg_fence(v);
                        if (c == 1) {  // the whole partial is in registers: release it
                            tc_fence_before();
                            __syncwarp();
                            if (lane == 0) mbar_arrive(&sm.part_empty[p]);
                        }
#pragma unroll
                        for (int j = 0; j < 8; ++j) {
                            const float4 w4 = sw4[8 * c + j];
                            acc[16 * c + 2 * j] = fma2(pack2(v[4 * j], v[4 * j + 1]),
                                                       pack2(__float_as_uint(w4.x), __float_as_uint(w4.y)),
                                                       acc[16 * c + 2 * j]);
                            acc[16 * c + 2 * j + 1] = fma2(pack2(v[4 * j + 2], v[4 * j + 3]),
                                                           pack2(__float_as_uint(w4.z), __float_as_uint(w4.w)),
                                                           acc[16 * c + 2 * j + 1]);
                        }
                    }
                }
                __syncwarp();
                if (ok && lane == 0) mbar_arrive(&sm.slot_empty[sl]);
            }
            if (!ok) break;
            // epilogue: x alpha, BF16 RNE, store this thread's 64 columns
            const int row = mb * BM + trow;
            const int col0 = nb * BN + half * 64;
            if (row < M) {
                uint32_t packed[32];
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                    const float lo = __uint_as_float((uint32_t)acc[j]) * alpha;
                    const float hi = __uint_as_float((uint32_t)(acc[j] >> 32)) * alpha;
                    __nv_bfloat162 h2 = __floats2bfloat162_rn(lo, hi);
                    packed[j] = *reinterpret_cast<uint32_t*>(&h2);
                }
                __nv_bfloat16* yrow = Y + (size_t)row * N;
                if (vec_ok && col0 + 64 <= N) {
                    uint4* dst = reinterpret_cast<uint4*>(yrow + col0);
#pragma unroll
                    for (int j = 0; j < 8; ++j)
                        dst[j] = make_uint4(packed[4 * j], packed[4 * j + 1], packed[4 * j + 2], packed[4 * j + 3]);
                } else {
                    uint16_t* y16 = reinterpret_cast<uint16_t*>(yrow);
#pragma unroll
                    for (int j = 0; j < 64; ++j)
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

}  // namespace w4a8
}  // namespace nvfp4
