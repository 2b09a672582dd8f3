// grouped_kernel.cuh -- grouped (mixture-of-experts) NVFP4 W4A4 matmul.
//
// Expert e multiplies its contiguous token rows A[row_start[e] .. row_start[e+1])
// by its own weights W_e [N][K] (block-scaled FP4 MMA, per-expert alpha =
// gA * gW_e).  The tile list spans all experts:
//   * every full 128-token block of an expert is a normal 128 x 256 tile
//     (tokens on the MMA's M side, weight rows on N);
//   * the ragged remainder of an expert (fewer than 128 tokens, which is the
//     whole expert when it is small) runs with the operands swapped:
//     Y_e^T = W_e . A_e^T, 128 weight rows on the MMA's M side and the tokens on
//     its N side (rounded up to a multiple of 16), so the MMA's 128-row side is
//     always full; the epilogue writes the transposed accumulator.
// The swap-AB layout for small M follows the prior-art MegaMoE kernel the
// pages describe (flashinfer swapab_cutedsl_megakernel skill doc, Layout).
//
// Warp roles, pipeline, scale handling and bounded waits are those of
// w4a4_kernel.cuh (TMA producer, MMA issuer, scale-factor transposer, eight
// epilogue warps); K % 256 == 0 is required (scale tiles by TMA).
#pragma once
#include <cuda_bf16.h>
#include <cstdint>

#include "ptx.cuh"
#include "w4a4_kernel.cuh"

namespace nvfp4 {
namespace grouped {

using w4a4::BM;
using w4a4::BK;
using w4a4::BKB;
using w4a4::KSTEPS;
using w4a4::NUM_EPI_WARPS;
using w4a4::NUM_THREADS;

constexpr int BN = 256;      // normal tiles: weight rows per tile
constexpr int SBN = 128;     // swapped tiles: weight rows per tile (MMA M)
constexpr int STAGES = 4;
constexpr int MAX_EXPERTS = 256;

struct Params {
    int E, N, K;
    int tile_start[MAX_EXPERTS + 1];  // prefix sums of tiles per expert
    int row_start[MAX_EXPERTS + 1];   // token offsets
    float alpha[MAX_EXPERTS];         // gA * gW_e
};

using S = w4a4::Smem<BN, STAGES>;
using C = w4a4::Cfg<BN, STAGES>;

struct Tile {
    int e;        // expert
    bool swap;
    int m0;       // first token row of the tile (global row of A and of Y)
    int rows;     // valid token rows (128 for normal tiles)
    int n0;       // first weight row within the expert
    int n_mma;    // MMA N: 256 (normal) or the token count rounded up to 16
};

__host__ __device__ inline int tiles_of_expert(int Me, int N) {
    const int full = Me / BM, rem = Me % BM;
    return full * ((N + BN - 1) / BN) + (rem ? (N + SBN - 1) / SBN : 0);
}

__device__ __forceinline__ Tile decode(const Params& p, int t) {
    int lo = 0, hi = p.E;  // last e with tile_start[e] <= t
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (p.tile_start[mid] <= t) lo = mid; else hi = mid;
    }
    while (lo + 1 < p.E && p.tile_start[lo + 1] <= t) ++lo;
    Tile tl;
    tl.e = lo;
    const int local = t - p.tile_start[lo];
    const int r0 = p.row_start[lo], Me = p.row_start[lo + 1] - r0;
    const int full = Me / BM;
    const int nbn = (p.N + BN - 1) / BN;
    if (local < full * nbn) {
        tl.swap = false;
        tl.m0 = r0 + (local % full) * BM;
        tl.rows = BM;
        tl.n0 = (local / full) * BN;
        tl.n_mma = BN;
    } else {
        const int rem = Me - full * BM;
        tl.swap = true;
        tl.m0 = r0 + full * BM;
        tl.rows = rem;
        tl.n0 = (local - full * nbn) * SBN;
        tl.n_mma = (rem + 15) & ~15;
    }
    return tl;
}

__global__ void __launch_bounds__(NUM_THREADS, 1)
grouped_kernel(const __grid_constant__ CUtensorMap tmA,      // A codes, box 128 rows
               const __grid_constant__ CUtensorMap tmW256,   // W codes [E*N rows], box 256
               const __grid_constant__ CUtensorMap tmW128,   // W codes, box 128
               const __grid_constant__ CUtensorMap tmSA,     // A scales, box 128 rows
               const __grid_constant__ CUtensorMap tmSW256,  // W scales, box 256
               const __grid_constant__ CUtensorMap tmSW128,  // W scales, box 128
               const __grid_constant__ Params p, __nv_bfloat16* __restrict__ Y) {
    using namespace w4a4;
    constexpr int NRB = C::NRB;
    extern __shared__ uint8_t smem_raw[];
    S& sm = *reinterpret_cast<S*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int N = p.N, K = p.K;
    const int tiles = p.tile_start[p.E];
    const int num_kb = K / BK;
    volatile int* abort = &sm.abort;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&sm.tma_full[s], 1);
            mbar_init(&sm.sf_full[s], 1);
            mbar_init(&sm.empty[s], 1);
        }
        mbar_init(&sm.acc_full, 1);
        mbar_init(&sm.acc_empty, NUM_EPI_WARPS);
        mbar_init(&sm.drain, 1);
        sm.abort = 0;
        fence_mbarrier_init();
    }
    if (warp == 1) {
        tmem_alloc(&sm.tmem_base, C::TMEM_COLS);
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
            for (int t = blockIdx.x; t < tiles && !*abort; t += gridDim.x) {
                const Tile tl = decode(p, t);
                const int wrow = tl.e * N + tl.n0;  // row in the [E*N] weight view
                const uint32_t bytes = tl.swap ? (BM + SBN) * (BKB + 16) : C::BYTES_A + C::BYTES_B + C::BYTES_SF;
                for (int kb = 0; kb < num_kb; ++kb, ++it) {
                    const int s = it % STAGES;
                    if (!mbar_wait(&sm.empty[s], ((it / STAGES) & 1) ^ 1, abort, ROLE_PRODUCER))
                        goto producer_done;
                    mbar_arrive_expect_tx(&sm.tma_full[s], bytes);
                    if (!tl.swap) {
                        tma_load_2d(sm.a[s], &tmA, &sm.tma_full[s], kb * BKB, tl.m0);
                        tma_load_2d(sm.b[s], &tmW256, &sm.tma_full[s], kb * BKB, wrow);
                        tma_load_2d(sm.sfa[s], &tmSA, &sm.tma_full[s], kb * 16, tl.m0);
                        tma_load_2d(sm.sfb[s], &tmSW256, &sm.tma_full[s], kb * 16, wrow);
                    } else {
                        // MMA A side: 128 weight rows; MMA B side: the tokens
                        tma_load_2d(sm.a[s], &tmW128, &sm.tma_full[s], kb * BKB, wrow);
                        tma_load_2d(sm.b[s], &tmA, &sm.tma_full[s], kb * BKB, tl.m0);
                        tma_load_2d(sm.sfa[s], &tmSW128, &sm.tma_full[s], kb * 16, wrow);
                        tma_load_2d(sm.sfb[s], &tmSA, &sm.tma_full[s], kb * 16, tl.m0);
                    }
                }
            }
        producer_done:
            if (*abort) {
                for (int j = max(0, it - STAGES); j < it; ++j) {
                    const uint64_t t0 = globaltimer_ns();
                    while (!mbar_try_wait(&sm.tma_full[j % STAGES], (j / STAGES) & 1) &&
                           globaltimer_ns() - t0 < kWaitLimitNs) {
                    }
                }
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            int it = 0, tc = 0;
            for (int t = blockIdx.x; t < tiles; t += gridDim.x, ++tc) {
                const Tile tl = decode(p, t);
                const uint32_t idesc = idesc_mxf4nvf4(BM, tl.n_mma);
                if (!mbar_wait(&sm.acc_empty, (tc & 1) ^ 1, abort, ROLE_MMA)) break;
                tc_fence_after();
                bool ok = true;
                for (int kb = 0; kb < num_kb; ++kb, ++it) {
                    const int s = it % STAGES;
                    const uint32_t ph = (it / STAGES) & 1;
                    if (!mbar_wait(&sm.tma_full[s], ph, abort, ROLE_MMA) ||
                        !mbar_wait(&sm.sf_full[s], ph, abort, ROLE_MMA)) { ok = false; break; }
                    tc_fence_after();
#pragma unroll
                    for (int ks = 0; ks < KSTEPS; ++ks)
                        tmem_cp_32x128b_x4(tmem + C::sfa_col(s) + ks * 4,
                                           desc_sf_32x16(smem_u32(&sm.sfa[s][ks * 128])));
                    const int nrb = tl.swap ? 1 : NRB;
                    for (int ks = 0; ks < KSTEPS; ++ks)
                        for (int rb = 0; rb < nrb; ++rb)
                            tmem_cp_32x128b_x4(tmem + C::sfb_col(s) + (ks * NRB + rb) * 4,
                                               desc_sf_32x16(smem_u32(&sm.sfb[s][(ks * NRB + rb) * 128])));
                    const uint32_t a0 = smem_u32(sm.a[s]), b0 = smem_u32(sm.b[s]);
#pragma unroll
                    for (int ks = 0; ks < KSTEPS; ++ks)
                        mma_mxf4nvf4(tmem, desc_kmajor_sw128(a0 + ks * 32),
                                     desc_kmajor_sw128(b0 + ks * 32), idesc,
                                     tmem + C::sfa_col(s) + ks * 4,
                                     tmem + C::sfb_col(s) + ks * NRB * 4, (kb | ks) != 0);
                    mma_commit(&sm.empty[s]);
                }
                if (!ok) break;
                mma_commit(&sm.acc_full);
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
    } else if (warp == 2) {
        // ------------------------------------------------------------ scale factors
        int it = 0;
        for (int t = blockIdx.x; t < tiles; t += gridDim.x) {
            const Tile tl = decode(p, t);
            const int nblk = tl.swap ? 2 : 1 + NRB;  // 128-row blocks present in this stage
            bool ok = true;
            for (int kb = 0; kb < num_kb; ++kb, ++it) {
                const int s = it % STAGES;
                if (!warp_wait(&sm.tma_full[s], (it / STAGES) & 1, abort, ROLE_SF)) { ok = false; break; }
                uint4 v[4 * (1 + NRB)];
#pragma unroll
                for (int i = 0; i < 4 * (1 + NRB); ++i) {
                    const int blk = i / 4;
                    const int rr = 32 * (lane >> 3) + 8 * (i & 3) + (lane & 7);
                    const uint4* raw = blk == 0
                        ? reinterpret_cast<const uint4*>(sm.sfa[s]) + rr
                        : reinterpret_cast<const uint4*>(sm.sfb[s]) + (blk - 1) * 128 + rr;
                    v[i] = blk < nblk ? *raw : make_uint4(0u, 0u, 0u, 0u);
                }
                __syncwarp();
#pragma unroll
                for (int i = 0; i < 4 * (1 + NRB); ++i) {
                    const int blk = i / 4;
                    if (blk >= nblk) continue;
                    const int rr = 32 * (lane >> 3) + 8 * (i & 3) + (lane & 7);
                    const int word = (rr & 31) * 4 + (rr >> 5);
                    if (blk == 0) {
                        sm.sfa[s][0 * 128 + word] = v[i].x;
                        sm.sfa[s][1 * 128 + word] = v[i].y;
                        sm.sfa[s][2 * 128 + word] = v[i].z;
                        sm.sfa[s][3 * 128 + word] = v[i].w;
                    } else {
                        const int rb = blk - 1;
                        sm.sfb[s][(0 * NRB + rb) * 128 + word] = v[i].x;
                        sm.sfb[s][(1 * NRB + rb) * 128 + word] = v[i].y;
                        sm.sfb[s][(2 * NRB + rb) * 128 + word] = v[i].z;
                        sm.sfb[s][(3 * NRB + rb) * 128 + word] = v[i].w;
                    }
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(&sm.sf_full[s]);
            }
            if (!ok) break;
        }
    } else if (warp >= 4) {
        // ------------------------------------------------------------ epilogue
        const int q = warp & 3, half = (warp - 4) >> 2;
        const bool vec_ok = (N % 8) == 0;
        int tc = 0;
        for (int t = blockIdx.x; t < tiles; t += gridDim.x, ++tc) {
            const Tile tl = decode(p, t);
            const float alpha = p.alpha[tl.e];
            if (!warp_wait(&sm.acc_full, tc & 1, abort, ROLE_EPI)) break;
            tc_fence_after();
            const uint32_t lane_base = tmem + ((uint32_t)(32 * q) << 16);
            if (!tl.swap) {
                constexpr int COLS = BN / 2;
                uint32_t packed[COLS / 2];
#pragma unroll
                for (int c = 0; c < COLS / 32; ++c) {
                    uint32_t r[32];
                    tmem_ld_32x32b_x32(lane_base + half * COLS + c * 32, r);
                    tmem_ld_wait();
                    reg_fence(r);
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        __nv_bfloat162 h = __floats2bfloat162_rn(__uint_as_float(r[2 * j]) * alpha,
                                                                 __uint_as_float(r[2 * j + 1]) * alpha);
                        packed[c * 16 + j] = *reinterpret_cast<uint32_t*>(&h);
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&sm.acc_empty);
                const int row = tl.m0 + 32 * q + lane;
                const int col0 = tl.n0 + half * COLS;
                __nv_bfloat16* yrow = Y + (size_t)row * N;
                if (vec_ok && col0 + COLS <= N) {
                    uint4* dst = reinterpret_cast<uint4*>(yrow + col0);
#pragma unroll
                    for (int j = 0; j < COLS / 8; ++j)
                        dst[j] = make_uint4(packed[4 * j], packed[4 * j + 1], packed[4 * j + 2],
                                            packed[4 * j + 3]);
                } else {
                    uint16_t* y16 = reinterpret_cast<uint16_t*>(yrow);
#pragma unroll
                    for (int j = 0; j < COLS; ++j)
                        if (col0 + j < N) y16[col0 + j] = (uint16_t)(packed[j >> 1] >> (16 * (j & 1)));
                }
            } else {
                // lanes are weight rows, columns are tokens: Y[m0 + tok][n]
                const int n = tl.n0 + 32 * q + lane;
                const bool nok = n < N;
                uint16_t* ycol = reinterpret_cast<uint16_t*>(Y) + (size_t)tl.m0 * N + n;
                uint32_t r[2][32];
#pragma unroll
                for (int c = 0; c < 2; ++c) {
                    const int tok0 = half * 64 + c * 32;
                    if (tok0 < tl.n_mma) {  // warp-uniform
                        tmem_ld_32x32b_x32(lane_base + tok0, r[c]);
                        tmem_ld_wait();
                        reg_fence(r[c]);
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&sm.acc_empty);
#pragma unroll
                for (int c = 0; c < 2; ++c) {
                    const int tok0 = half * 64 + c * 32;
#pragma unroll
                    for (int j = 0; j < 32; ++j) {
                        if (nok && tok0 + j < tl.rows)
                            ycol[(size_t)(tok0 + j) * N] =
                                __bfloat16_as_ushort(__float2bfloat16_rn(__uint_as_float(r[c][j]) * alpha));
                    }
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem, C::TMEM_COLS);
}

}  // namespace grouped
}  // namespace nvfp4
