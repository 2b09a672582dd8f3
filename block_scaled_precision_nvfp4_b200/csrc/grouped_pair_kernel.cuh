// grouped_pair_kernel.cuh -- grouped (mixture-of-experts) NVFP4 W4A4 matmul on
// pairs of SMs, with scales packed in the MMA's layout per expert.
//
// Expert e multiplies its contiguous token rows A[row_start[e] .. row_start[e+1])
// by its own weights W_e [N][K] with alpha_e = gA * gW_e.  The tile list spans
// all experts, 256 weight rows (N) per tile, ordered within an expert as the
// dense pair kernel orders its tiles:
//   * normal tiles: 256 tokens of one expert on the MMA's M side (128 per CTA,
//     the last block of an expert may be partly beyond its rows), weight rows
//     on N -- tcgen05.mma.cta_group::2 M=256 N=256;
//   * swapped tiles, for an expert's last 1..128 tokens (all of a small
//     expert): Y_e^T = W_e . A_e^T, 256 weight rows on the MMA's M side (128
//     per CTA) and 128 token slots on N (64 loaded by each CTA), so the MMA's
//     wide side stays full; the epilogue stores the transposed accumulator.
// The swap-AB layout for small M follows the prior-art MegaMoE kernel the
// pages describe (flashinfer swapab_cutedsl_megakernel skill doc, Layout).
//
// Packed scales (pack_scales_kernel.cuh) start every expert on a 128-row block
// boundary (block_start[e]), so every tile's scales are whole 512-byte atoms
// reached by plain TMA tile loads.  Pipeline, barriers, bounded waits and the
// TMA-store epilogue are those of w4a4_pair_kernel.cuh; a warp whose 32 rows
// are not all inside the expert stores its rows with plain stores, so that no
// row of the next expert is touched.
#pragma once
#include <cuda_bf16.h>
#include <cstdint>

#include "ptx.cuh"
#include "w4a4_pair_kernel.cuh"
#include "pack_scales_kernel.cuh"

namespace nvfp4 {
namespace grouped_pair {

using w4a4::BK;
using w4a4::BKB;
using w4a4::KSTEPS;
using w4a4::ROLE_DRAIN;
using w4a4::ROLE_EPI;
using w4a4::ROLE_MMA;
using w4a4::ROLE_PRODUCER;
using w4a4::warp_wait;
using w4a4_pair::BM;
using w4a4_pair::BN;
using w4a4_pair::BNH;
using w4a4_pair::FIRST_EPI_WARP;
using w4a4_pair::NRB;
using w4a4_pair::NUM_EPI_WARPS;
using w4a4_pair::NUM_THREADS;
using w4a4_pair::sfa_col;
using w4a4_pair::sfb_col;
using w4a4_pair::Smem;
using w4a4_pair::SMEM_BYTES;
using w4a4_pair::STAGES;
using w4a4_pair::TILE_M;
using w4a4_pair::TMEM_COLS;
using w4a4_pair::store_slab;
using w4a4_pair::tma_load_3d_pair;

constexpr int MAX_EXPERTS = 256;
constexpr int SWAP_N = 128;            // token slots of a swapped tile (MMA N)
constexpr int SWAP_HALF = SWAP_N / 2;  // token rows loaded by each CTA

struct Params {
    int E, N, K;
    int tile_start[MAX_EXPERTS + 1];   // prefix sums of tiles per expert
    int row_start[MAX_EXPERTS + 1];    // token offsets
    int block_start[MAX_EXPERTS + 1];  // first packed 128-row block of each expert's sA
    float alpha[MAX_EXPERTS];          // gA * gW_e
};

__host__ __device__ inline int normal_blocks(int Me) {  // 256-token blocks run unswapped
    return Me / TILE_M + ((Me % TILE_M) > SWAP_N ? 1 : 0);
}
__host__ __device__ inline int swapped_blocks(int Me) {
    const int rem = Me % TILE_M;
    return (rem > 0 && rem <= SWAP_N) ? 1 : 0;
}
__host__ __device__ inline int tiles_of_expert(int Me, int N) {
    return (normal_blocks(Me) + swapped_blocks(Me)) * ((N + BN - 1) / BN);
}

struct Tile {
    int e;
    bool swap;
    int mblk;   // 256-token block index within the expert
    int m0;     // first token row (global) of the tile
    int rows;   // valid token rows from m0
    int n0;     // first weight row within the expert
};

__device__ __forceinline__ Tile decode(const Params& p, int t) {
    int lo = 0, hi = p.E;
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (p.tile_start[mid] <= t) lo = mid; else hi = mid;
    }
    Tile tl;
    tl.e = lo;
    const int local = t - p.tile_start[lo];
    const int r0 = p.row_start[lo], Me = p.row_start[lo + 1] - r0;
    // within the expert, groups of GROUP_M token blocks sweep N together, so the
    // clusters running at one time share weight tiles through L2
    const int nbn = (p.N + BN - 1) / BN;
    const int nmb = normal_blocks(Me) + swapped_blocks(Me);
    int mblk, nb;
    w4a4_pair::tile_coords(local, nmb, nbn, mblk, nb);
    tl.mblk = mblk;
    tl.n0 = nb * BN;
    tl.swap = mblk >= normal_blocks(Me);
    tl.m0 = r0 + mblk * TILE_M;
    tl.rows = min(TILE_M, Me - mblk * TILE_M);
    return tl;
}

constexpr int BAD_DEST = 0x40000;  // device error bit: a grouped row's Y row outside [0, dest_rows)

// The Y row and output factor of one grouped row, for a fused combine: row `dest`
// (the grouped row's index on entry) goes to Y row row_dest[dest], scaled by
// alpha * row_w[that row].  A row outside [0, dest_rows) is recorded in the device
// error word and left out (dest = -1); rows past the tile (`valid` false) are not read.
__device__ __forceinline__ void row_target(const int32_t* __restrict__ row_dest,
                                           const float* __restrict__ row_w, int dest_rows,
                                           bool valid, float alpha, int& dest, float& f) {
    if (!valid) {
        dest = -1;
        return;
    }
    const int d = __ldg(row_dest + dest);
    if ((unsigned)d >= (unsigned)dest_rows) {
        atomicOr(&g_device_error, BAD_DEST);
        dest = -1;
        return;
    }
    dest = d;
    if (row_w) f = alpha * __ldg(row_w + d);
}

// store_slab for scattered rows: the warp's 32 rows x 128 columns (packed BF16
// pairs, lane = row) pass through the warp's staging buffer one 64-column box at a
// time, and each row leaves as one 128-byte store to Y row `dest` of its lane
// (rows with dest < 0, rows past `nrows` and columns past N are not written).
// N must be even.
__device__ __forceinline__ void scatter_slab(uint8_t* stage, const uint32_t (&packed)[64], int dest,
                                             int nrows, int col0, int N, __nv_bfloat16* __restrict__ Y) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        if (lane == 0) bulk_wait_read_all();  // no TMA store still reads the buffer
        __syncwarp();
        uint8_t* rowp = stage + lane * 128;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
            const int w = h * 32 + c * 4;
            *reinterpret_cast<uint4*>(rowp + ((c ^ (lane & 7)) << 4)) =
                make_uint4(packed[w], packed[w + 1], packed[w + 2], packed[w + 3]);
        }
        __syncwarp();
        const int x = col0 + h * 64 + 2 * lane;  // this lane's two columns
        for (int r = 0; r < nrows; ++r) {
            const int d = __shfl_sync(0xffffffffu, dest, r);
            const uint32_t v = *reinterpret_cast<const uint32_t*>(
                stage + r * 128 + (((lane >> 2) ^ (r & 7)) << 4) + (lane & 3) * 4);
            if (d >= 0 && x < N)
                *reinterpret_cast<uint32_t*>(reinterpret_cast<uint16_t*>(Y) + (size_t)d * N + x) = v;
        }
        __syncwarp();  // the box is read before the next one overwrites it
    }
}

// One stage's scale copies and MMAs (issued by one thread of the leader):
// sA of the MMA's M rows (this CTA's 128), sB of its N side in NB 128-row
// blocks, then four K = 64 block-scaled MMAs.  Unrolled for each NB so the
// issuing thread keeps ahead of the tensor pipe.
template <int NB>
__device__ __forceinline__ void issue_stage(Smem& sm, int s, uint32_t tmem, uint32_t idesc,
                                            bool accumulate) {
#pragma unroll
    for (int ks = 0; ks < KSTEPS; ++ks)
        tmem_cp_32x128b_x4_pair(tmem + sfa_col(s) + ks * 4,
                                desc_sf_32x16(smem_u32(&sm.sfa[s][ks * 128])));
#pragma unroll
    for (int ks = 0; ks < KSTEPS; ++ks)
#pragma unroll
        for (int rb = 0; rb < NB; ++rb)
            tmem_cp_32x128b_x4_pair(tmem + sfb_col(s) + (ks * NRB + rb) * 4,
                                    desc_sf_32x16(smem_u32(&sm.sfb[s][(rb * KSTEPS + ks) * 128])));
    const uint32_t a0 = smem_u32(sm.a[s]), b0 = smem_u32(sm.b[s]);
#pragma unroll
    for (int ks = 0; ks < KSTEPS; ++ks)
        mma_mxf4nvf4_pair(tmem, desc_kmajor_sw128(a0 + ks * 32), desc_kmajor_sw128(b0 + ks * 32),
                          idesc, tmem + sfa_col(s) + ks * 4, tmem + sfb_col(s) + ks * NRB * 4,
                          accumulate || ks != 0);
}

__global__ void __launch_bounds__(NUM_THREADS, 1)
grouped_pair_kernel(const __grid_constant__ CUtensorMap tmA,    // A codes, box 128 rows
                    const __grid_constant__ CUtensorMap tmA64,  // A codes, box 64 rows (swapped B side)
                    const __grid_constant__ CUtensorMap tmW,    // W codes [E*N rows], box 128 rows
                    const __grid_constant__ CUtensorMap tmSA,   // grouped-packed sA, box (128,16,1)
                    const __grid_constant__ CUtensorMap tmSW2,  // packed sW, box (128,16,2)
                    const __grid_constant__ CUtensorMap tmSW1,  // packed sW, box (128,16,1)
                    const __grid_constant__ CUtensorMap tmY,    // Y bf16 [M][N], box 64 x 32, 128B swizzle
                    int tma_out,                                // tmY is valid (N % 8 == 0)
                    const __grid_constant__ Params p_param,
                    const Params* __restrict__ p_dev,           // schedule in device memory, or null
                    __nv_bfloat16* __restrict__ Y,
                    // with row_dest: grouped row r goes to Y row row_dest[r] (of dest_rows),
                    // times row_w[row_dest[r]] when row_w is given (a fused top-1 combine)
                    const int32_t* __restrict__ row_dest, const float* __restrict__ row_w,
                    int dest_rows) {
    // the tile schedule: kernel parameters planned on the host, or device memory
    // written by grouped_schedule_kernel from device-resident expert offsets
    const Params& p = p_dev ? *p_dev : p_param;
    extern __shared__ uint8_t smem_raw[];
    Smem& sm = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                        ~uintptr_t(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const bool leader = rank == 0;
    const int cid = blockIdx.x >> 1, nclusters = gridDim.x >> 1;
    volatile int* abort = &sm.abort;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&sm.full[s], 1);
            mbar_init(&sm.empty[s], 1);
        }
        mbar_init(&sm.acc_full, 1);
        mbar_init(&sm.acc_empty, 2 * NUM_EPI_WARPS);
        mbar_init(&sm.drain, 1);
        sm.abort = 0;
        fence_mbarrier_init();
    }
    if (warp == 1) {
        tmem_alloc_pair(&sm.tmem_base, TMEM_COLS);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    cluster_sync();
    tc_fence_after();
    const uint32_t tmem = sm.tmem_base;
    // the set-up above overlaps the kernel before this one (scale packing or the
    // schedule, when launched programmatically); their output -- the packed scales
    // and, with p_dev, the schedule itself -- is read only from here
    grid_dependency_wait();
    const int N = p.N, K = p.K;
    const int tiles = p.tile_start[p.E];
    const int num_kb = K / BK;
    const int wblocks = (N + 127) / 128;  // packed 128-row blocks of one expert's sW

    if (warp == 0) {
        // ------------------------------------------------------------ producer (both CTAs)
        int it = 0;
        bool ok = true;
        for (int t = cid; t < tiles && ok; t += nclusters) {
            const Tile tl = decode(p, t);
            const int wrow = tl.e * N + tl.n0 + (int)rank * BNH;  // this CTA's 128 weight rows
            const int wblk = tl.e * wblocks + tl.n0 / 128;       // packed sW block of the tile
            const int ablk = p.block_start[tl.e] + 2 * tl.mblk;  // packed sA block of the tile
            const uint32_t bytes = tl.swap
                ? 2u * ((BNH + SWAP_HALF) * BKB + (BNH + 128) * 16)
                : 2u * ((BM + BNH) * BKB + (BM + BN) * 16);
            for (int kb = 0; kb < num_kb; ++kb, ++it) {
                const int s = it % STAGES;
                if (!warp_wait(&sm.empty[s], ((it / STAGES) & 1) ^ 1, abort, ROLE_PRODUCER, 32)) {
                    ok = false;
                    break;
                }
                if (elect_one()) {
                    if (leader) mbar_arrive_expect_tx(&sm.full[s], bytes);
                    const uint32_t full0 = map_to_rank(&sm.full[s], 0);
                    if (!tl.swap) {
                        tma_load_2d_pair(sm.a[s], &tmA, full0, kb * BKB, tl.m0 + (int)rank * BM);
                        tma_load_2d_pair(sm.b[s], &tmW, full0, kb * BKB, wrow);
                        tma_load_3d_pair(sm.sfa[s], &tmSA, full0, 0, kb * 16, ablk + (int)rank);
                        tma_load_3d_pair(sm.sfb[s], &tmSW2, full0, 0, kb * 16, wblk);
                    } else {
                        // MMA A side: this CTA's 128 weight rows; B side: 64 of the tokens
                        tma_load_2d_pair(sm.a[s], &tmW, full0, kb * BKB, wrow);
                        tma_load_2d_pair(sm.b[s], &tmA64, full0, kb * BKB, tl.m0 + (int)rank * SWAP_HALF);
                        tma_load_3d_pair(sm.sfa[s], &tmSW1, full0, 0, kb * 16, wblk + (int)rank);
                        tma_load_3d_pair(sm.sfb[s], &tmSA, full0, 0, kb * 16, ablk);
                    }
                }
                __syncwarp();
            }
        }
        if (!ok && leader && lane == 0) {
            for (int j = max(0, it - STAGES); j < it; ++j) {
                const uint64_t t0 = globaltimer_ns();
                while (!mbar_try_wait(&sm.full[j % STAGES], (j / STAGES) & 1) &&
                       globaltimer_ns() - t0 < kWaitLimitNs) {
                }
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer (leader)
        if (leader) {
            int it = 0, tc = 0;
            bool ok = true;
            for (int t = cid; t < tiles && ok; t += nclusters, ++tc) {
                const Tile tl = decode(p, t);
                if (!warp_wait(&sm.acc_empty, (tc & 1) ^ 1, abort, ROLE_MMA)) { ok = false; break; }
                tc_fence_after();
                for (int kb = 0; kb < num_kb; ++kb, ++it) {
                    const int s = it % STAGES;
                    if (!warp_wait(&sm.full[s], (it / STAGES) & 1, abort, ROLE_MMA)) { ok = false; break; }
                    tc_fence_after();
                    if (elect_one()) {
                        if (tl.swap)
                            issue_stage<1>(sm, s, tmem, idesc_mxf4nvf4(TILE_M, SWAP_N), kb != 0);
                        else
                            issue_stage<NRB>(sm, s, tmem, idesc_mxf4nvf4(TILE_M, BN), kb != 0);
                        mma_commit_pair(&sm.empty[s], 0x3);
                    }
                    __syncwarp();
                }
                if (!ok) break;
                if (elect_one()) mma_commit_pair(&sm.acc_full, 0x3);
                __syncwarp();
            }
            if (elect_one()) {
                mma_commit_pair(&sm.drain, 0x1);
                const uint64_t t0 = globaltimer_ns();
                while (!mbar_try_wait(&sm.drain, 0)) {
                    if (globaltimer_ns() - t0 > kWaitLimitNs) {
                        atomicOr(&g_device_error, 1 | (ROLE_DRAIN << 8));
                        break;
                    }
                }
            }
            __syncwarp();
        }
    } else {
        // ------------------------------------------------------------ epilogue (both CTAs)
        const int q = warp & 3, half = (warp - FIRST_EPI_WARP) >> 2;
        constexpr int COLS = BN / 2, CHUNKS = COLS / 32;
        uint8_t* stage = sm.out[warp - FIRST_EPI_WARP];
        const uint32_t lane_base = tmem + ((uint32_t)(32 * q) << 16);
        int tc = 0;
        for (int t = cid; t < tiles; t += nclusters, ++tc) {
            const Tile tl = decode(p, t);
            const float alpha = p.alpha[tl.e];
            if (!tl.swap) {
                const int rbase = (int)rank * BM + 32 * q;  // the warp's first row within the tile
                // this lane's row: its Y row and factor (read before the accumulator is ready)
                int dest = tl.m0 + rbase + lane;
                float f = alpha;
                if (row_dest) row_target(row_dest, row_w, dest_rows, rbase + lane < tl.rows, alpha, dest, f);
                if (!warp_wait(&sm.acc_full, tc & 1, abort, ROLE_EPI)) break;
                tc_fence_after();
                uint32_t packed[COLS / 2];
#pragma unroll
                for (int c = 0; c < CHUNKS; ++c) {
                    uint32_t r[32];
                    tmem_ld_32x32b_x32(lane_base + half * COLS + c * 32, r);
                    tmem_ld_wait();
                    reg_fence(r);
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        __nv_bfloat162 h = __floats2bfloat162_rn(__uint_as_float(r[2 * j]) * f,
                                                                 __uint_as_float(r[2 * j + 1]) * f);
                        packed[c * 16 + j] = *reinterpret_cast<uint32_t*>(&h);
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive_remote(&sm.acc_empty, 0);
                const int col0 = tl.n0 + half * COLS;
                if (rbase < tl.rows) {
                    if (row_dest)
                        scatter_slab(stage, packed, dest, min(32, tl.rows - rbase), col0, N, Y);
                    else
                        store_slab(&tmY, tma_out != 0 && rbase + 32 <= tl.rows, stage, packed,
                                   tl.m0 + rbase, min(32, tl.rows - rbase), col0, N, Y);
                }
            } else {
                // lanes are this CTA's weight rows, columns are the tile's token slots; this
                // lane holds the Y row and factor of token slots lane and 32 + lane
                const int n = tl.n0 + (int)rank * BNH + 32 * q + lane;
                const bool nok = n < N;
                const int tok0 = half * 64;
                int d0 = tl.m0 + tok0 + lane, d1 = d0 + 32;
                float f0 = alpha, f1 = alpha;
                if (row_dest) {
                    row_target(row_dest, row_w, dest_rows, tok0 + lane < tl.rows, alpha, d0, f0);
                    row_target(row_dest, row_w, dest_rows, tok0 + 32 + lane < tl.rows, alpha, d1, f1);
                }
                if (!warp_wait(&sm.acc_full, tc & 1, abort, ROLE_EPI)) break;
                tc_fence_after();
                uint32_t tok2[32];  // BF16 pairs of consecutive tokens
#pragma unroll
                for (int c = 0; c < 2; ++c) {
                    uint32_t r[32];
                    tmem_ld_32x32b_x32(lane_base + half * 64 + c * 32, r);
                    tmem_ld_wait();
                    reg_fence(r);
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        // token slots 32c + 2j and 32c + 2j + 1; their factors sit in lanes 2j, 2j + 1
                        const float fa = __shfl_sync(0xffffffffu, c ? f1 : f0, 2 * j);
                        const float fb = __shfl_sync(0xffffffffu, c ? f1 : f0, 2 * j + 1);
                        __nv_bfloat162 h = __floats2bfloat162_rn(__uint_as_float(r[2 * j]) * fa,
                                                                 __uint_as_float(r[2 * j + 1]) * fb);
                        tok2[c * 16 + j] = *reinterpret_cast<uint32_t*>(&h);
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive_remote(&sm.acc_empty, 0);
                uint16_t* y16 = reinterpret_cast<uint16_t*>(Y);
#pragma unroll
                for (int j = 0; j < 64; ++j) {
                    const int d = __shfl_sync(0xffffffffu, j < 32 ? d0 : d1, j & 31);
                    if (nok && tok0 + j < tl.rows && d >= 0)
                        y16[(size_t)d * N + n] = (uint16_t)(tok2[j >> 1] >> (16 * (j & 1)));
                }
            }
        }
        if (lane == 0) bulk_wait_all();  // staging buffers stay alive until the stores are done
    }

    tc_fence_before();
    cluster_sync();
    tc_fence_after();
    if (warp == 1) tmem_dealloc_pair(tmem, TMEM_COLS);
}

// The tile schedule from device-resident expert offsets (one thread; E <= 256):
// what the host-planned entry point computes, written to device memory, plus
// the grouped packing map of the activations' scales.  Offsets that are not a
// non-decreasing run from 0 to M give an empty schedule and a device error bit.
constexpr int BAD_OFFSETS = 0x20000;
struct GwArray {
    float v[MAX_EXPERTS];
};

__global__ void grouped_schedule_kernel(const int32_t* __restrict__ offsets, int E, int M, int N,
                                        int K, const float* __restrict__ gA_dev, float gA_host,
                                        const __grid_constant__ GwArray gw, Params* __restrict__ out,
                                        pack::GroupedPack* __restrict__ pk) {
    if (threadIdx.x != 0 || blockIdx.x != 0) return;
    const float gA = gA_dev ? *gA_dev : gA_host;
    bool ok = offsets[0] == 0 && offsets[E] == M;
    for (int e = 0; e < E && ok; ++e) ok = offsets[e + 1] >= offsets[e];
    out->E = E;
    out->N = N;
    out->K = K;
    pk->groups_n = E;
    int total = 0, blocks = 0;
    for (int e = 0; e <= E; ++e) {
        const int r = ok ? offsets[e] : 0;
        out->tile_start[e] = total;
        out->row_start[e] = r;
        out->block_start[e] = blocks;
        pk->row_start[e] = r;
        pk->block_start[e] = blocks;
        if (e < E) {
            out->alpha[e] = gA * gw.v[e];
            const int Me = ok ? offsets[e + 1] - offsets[e] : 0;
            total += tiles_of_expert(Me, N);
            blocks += (Me + 127) / 128;
        }
    }
    if (!ok) atomicOr(&g_device_error, BAD_OFFSETS);
}

}  // namespace grouped_pair
}  // namespace nvfp4
