// w4a4_kernel.cuh -- NVFP4 W4A4 matmul on the sm_100a block-scaled FP4 MMA.
//
// Computes Y = BF16(alpha * (A.sA)(W.sW)^T): the "NVFP4: the block-scaled FP4
// MMA" row of the metrale_circuit `hardware::exec` module doc, bullet 1.
//
// Design (one persistent CTA per SM, 12 warps):
//   warp 0      TMA producer: 128-byte K-slices (256 codes) of the A and W
//               tiles, 128-byte swizzle, into a STAGES-deep ring, and (when the
//               scale row pitch allows) the matching raw [rows][16 B] scale tiles.
//   warp 1      TMEM owner + MMA issuer (one elected lane of the converged
//               warp -- a warp that issues tcgen05 work keeps its lanes
//               together instead of parking 31 of them): per stage copies the
//               stage's scale factors smem -> TMEM (tcgen05.cp) and issues four
//               tcgen05.mma kind::mxf4nvf4 scale_vec::4X (K = 64 each) into an
//               FP32 accumulator in TMEM; commits free the stage.
//   warp 2      scale-factor warp: rewrites the stage's plain row-major E4M3
//               scales in place into the MMA's scale layout (per 128 rows and
//               K = 64: 32 lines of 16 bytes, line i holding rows i, i+32, i+64,
//               i+96), so callers pass plain [rows][K/16] scales and no
//               reordering pass over global memory is needed.
//   warps 4-11  epilogue: TMEM -> registers (tcgen05.ld), x alpha, BF16 RNE,
//               stores to global; the accumulator is released as soon as it is
//               in registers so the next tile's MMAs overlap the stores.
// Every wait is bounded (see ptx.cuh); a CTA that gives up drains its own
// in-flight copies and MMAs, frees its TMEM and exits.
#pragma once
#include <cuda_bf16.h>
#include <cstdint>

#include "ptx.cuh"

namespace nvfp4 {
namespace w4a4 {

constexpr int BM = 128;          // rows of A per tile (MMA M)
constexpr int BK = 256;          // codes per K-block
constexpr int BKB = BK / 2;      // bytes per row per K-block (= the 128-byte swizzle span)
constexpr int KSTEPS = BK / 64;  // MMAs per K-block
constexpr int NUM_EPI_WARPS = 8;
constexpr int NUM_THREADS = 32 * (4 + NUM_EPI_WARPS);
constexpr int GROUP_M = 8;       // tile rasterisation: 8 row-blocks share a sweep over N

enum Role { ROLE_PRODUCER = 1, ROLE_MMA = 2, ROLE_SF = 3, ROLE_EPI = 4, ROLE_DRAIN = 5 };

template <int BN, int STAGES>
struct Smem {
    static constexpr int NRB = BN / 128;  // 128-row blocks of W per tile
    alignas(1024) uint8_t a[STAGES][BM * BKB];
    alignas(1024) uint8_t b[STAGES][BN * BKB];
    alignas(16) uint32_t sfa[STAGES][KSTEPS * 128];        // [ks][512 B atom]
    alignas(16) uint32_t sfb[STAGES][KSTEPS * NRB * 128];  // [ks][rb][512 B atom]
    uint64_t tma_full[STAGES];
    uint64_t sf_full[STAGES];
    uint64_t empty[STAGES];
    uint64_t acc_full;
    uint64_t acc_empty;
    uint64_t drain;
#ifdef NVFP4_WAIT_TEST
    uint64_t never;  // test-only: a barrier nothing arrives on
#endif
    uint32_t tmem_base;
    int abort;
};

template <int BN, int STAGES>
struct Cfg {
    static constexpr int NRB = BN / 128;
    static constexpr int SFA_COLS = KSTEPS * 4;
    static constexpr int SFB_COLS = KSTEPS * NRB * 4;
    static constexpr int TMEM_USED = BN + STAGES * (SFA_COLS + SFB_COLS);
    static constexpr int TMEM_COLS = TMEM_USED <= 32 ? 32 : TMEM_USED <= 64 ? 64
                                   : TMEM_USED <= 128 ? 128 : TMEM_USED <= 256 ? 256 : 512;
    static_assert(TMEM_USED <= 512, "TMEM budget exceeded");
    static constexpr uint32_t BYTES_A = BM * BKB;
    static constexpr uint32_t BYTES_B = BN * BKB;
    static constexpr uint32_t BYTES_SF = (BM + BN) * 16;  // raw scale tiles per stage
    static constexpr size_t SMEM_BYTES = sizeof(Smem<BN, STAGES>) + 1024;
    __host__ __device__ static constexpr uint32_t sfa_col(int s) { return BN + s * (SFA_COLS + SFB_COLS); }
    __host__ __device__ static constexpr uint32_t sfb_col(int s) { return sfa_col(s) + SFA_COLS; }
};

__device__ __forceinline__ void tile_coords(int tile, int num_m, int num_n, int& mb, int& nb) {
    const int per_group = GROUP_M * num_n;
    const int group = tile / per_group;
    const int first_m = group * GROUP_M;
    const int gsize = min(num_m - first_m, GROUP_M);
    const int in_group = tile % per_group;
    mb = first_m + in_group % gsize;
    nb = in_group / gsize;
}

__device__ __forceinline__ uint4 ld_nc_v4(const void* p) {
    uint4 v;
    asm volatile("ld.global.nc.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
    return v;
}

// Warp-uniform bounded wait: lane 0 waits, the verdict is broadcast.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort,
                                          int role, uint32_t backoff_ns = 0) {
    const int lane = threadIdx.x & 31;
    int ok = 1;
    if (lane == 0) ok = mbar_wait(bar, parity, abort, role, backoff_ns) ? 1 : 0;
    return __shfl_sync(0xffffffffu, ok, 0) != 0;
}

// 16 scale bytes (one K-block) of global row `grow`, zero outside [0,rows) x [0,K/16).
__device__ __forceinline__ uint4 load_sf16(const uint8_t* __restrict__ s, int grow, int rows,
                                           int kb, int G, bool fast) {
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if (grow >= rows) return v;
    const uint8_t* p = s + (size_t)grow * G + (size_t)kb * 16;
    if (fast) return ld_nc_v4(p);
    uint32_t w[4] = {0u, 0u, 0u, 0u};
#pragma unroll
    for (int j = 0; j < 16; ++j)
        if (kb * 16 + j < G) w[j >> 2] |= (uint32_t)__ldg(p + j) << (8 * (j & 3));
    return make_uint4(w[0], w[1], w[2], w[3]);
}

// SF_TMA: the scale tiles arrive by TMA with the operand tiles (needs the scale
// row pitch K/16 to be a multiple of 16 bytes, i.e. K % 256 == 0) and the
// scale-factor warp only transposes them in shared memory; otherwise the
// scale-factor warp reads them from global memory itself.
template <int BN, int STAGES, bool SF_TMA>
__global__ void __launch_bounds__(NUM_THREADS, 1)
w4a4_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
            const __grid_constant__ CUtensorMap tmSA, const __grid_constant__ CUtensorMap tmSB,
            const uint8_t* __restrict__ sA, const uint8_t* __restrict__ sW,
            __nv_bfloat16* __restrict__ Y, int M, int N, int K, float alpha) {
    using C = Cfg<BN, STAGES>;
    using S = Smem<BN, STAGES>;
    constexpr int NRB = C::NRB;
    extern __shared__ uint8_t smem_raw[];
    S& sm = *reinterpret_cast<S*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int num_m = (M + BM - 1) / BM;
    const int num_n = (N + BN - 1) / BN;
    const int tiles = num_m * num_n;
    const int num_kb = (K + BK - 1) / BK;
    const int G = K / 16;
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
#ifdef NVFP4_WAIT_TEST
        mbar_init(&sm.never, 1);
#endif
        sm.abort = 0;
        fence_mbarrier_init();
        tma_prefetch_desc(&tmA);
        tma_prefetch_desc(&tmB);
        if (SF_TMA) {
            tma_prefetch_desc(&tmSA);
            tma_prefetch_desc(&tmSB);
        }
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
        // The whole warp walks the loop (converged); one elected lane issues.
        int it = 0;
        bool ok = true;
        for (int tile = blockIdx.x; tile < tiles && ok; tile += gridDim.x) {
            int mb, nb;
            tile_coords(tile, num_m, num_n, mb, nb);
            for (int kb = 0; kb < num_kb; ++kb, ++it) {
                const int s = it % STAGES;
                const uint32_t ph = (it / STAGES) & 1;
                if (!warp_wait(&sm.empty[s], ph ^ 1, abort, ROLE_PRODUCER)) { ok = false; break; }
                if (elect_one()) {
                    mbar_arrive_expect_tx(&sm.tma_full[s], C::BYTES_A + C::BYTES_B +
                                                               (SF_TMA ? C::BYTES_SF : 0u));
                    tma_load_2d(sm.a[s], &tmA, &sm.tma_full[s], kb * BKB, mb * BM);
                    tma_load_2d(sm.b[s], &tmB, &sm.tma_full[s], kb * BKB, nb * BN);
                    if (SF_TMA) {
                        // raw [rows][16 B] scale tiles, transposed in place by warp 2
                        tma_load_2d(sm.sfa[s], &tmSA, &sm.tma_full[s], kb * 16, mb * BM);
                        tma_load_2d(sm.sfb[s], &tmSB, &sm.tma_full[s], kb * 16, nb * BN);
                    }
                }
                __syncwarp();
            }
        }
        if (!ok && lane == 0) {
            // Let every copy this warp started land before the CTA exits.
            for (int j = max(0, it - STAGES); j < it; ++j) {
                uint64_t* bar = &sm.tma_full[j % STAGES];
                const uint64_t t0 = globaltimer_ns();
                while (!mbar_try_wait(bar, (j / STAGES) & 1) && globaltimer_ns() - t0 < kWaitLimitNs) {
                }
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        // Converged warp; the elected lane (the same lane every time) issues the
        // scale copies, the MMAs and the commits that track them.
        const uint32_t idesc = idesc_mxf4nvf4(BM, BN);
        int it = 0, tc = 0;
        bool ok = true;
#ifdef NVFP4_WAIT_TEST
        // test-only: wait on a barrier nothing arms, so that this bounded wait
        // expires and every role of the CTA takes its abort path
        if (g_wait_test_stall && !warp_wait(&sm.never, 0, abort, ROLE_MMA)) ok = false;
#endif
        for (int tile = blockIdx.x; tile < tiles && ok; tile += gridDim.x, ++tc) {
            if (!warp_wait(&sm.acc_empty, (tc & 1) ^ 1, abort, ROLE_MMA)) { ok = false; break; }
            tc_fence_after();
            for (int kb = 0; kb < num_kb; ++kb, ++it) {
                const int s = it % STAGES;
                const uint32_t ph = (it / STAGES) & 1;
                if (!warp_wait(&sm.tma_full[s], ph, abort, ROLE_MMA) ||
                    !warp_wait(&sm.sf_full[s], ph, abort, ROLE_MMA)) { ok = false; break; }
                tc_fence_after();
                if (elect_one()) {
#pragma unroll
                    for (int ks = 0; ks < KSTEPS; ++ks)
                        tmem_cp_32x128b_x4(tmem + C::sfa_col(s) + ks * 4,
                                           desc_sf_32x16(smem_u32(&sm.sfa[s][ks * 128])));
#pragma unroll
                    for (int j = 0; j < KSTEPS * NRB; ++j)
                        tmem_cp_32x128b_x4(tmem + C::sfb_col(s) + j * 4,
                                           desc_sf_32x16(smem_u32(&sm.sfb[s][j * 128])));
                    const uint32_t a0 = smem_u32(sm.a[s]);
                    const uint32_t b0 = smem_u32(sm.b[s]);
#pragma unroll
                    for (int ks = 0; ks < KSTEPS; ++ks)
                        mma_mxf4nvf4(tmem, desc_kmajor_sw128(a0 + ks * 32),
                                     desc_kmajor_sw128(b0 + ks * 32), idesc,
                                     tmem + C::sfa_col(s) + ks * 4,
                                     tmem + C::sfb_col(s) + ks * NRB * 4, (kb | ks) != 0);
                    mma_commit(&sm.empty[s]);
                }
                __syncwarp();
            }
            if (!ok) break;
            if (elect_one()) mma_commit(&sm.acc_full);
            __syncwarp();
        }
        // Every MMA and copy issued completes before TMEM is freed.
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
    } else if (warp == 2) {
        // ------------------------------------------------------------ scale factors
        // Row rr of a 128-row block goes to word (rr%32)*4 + rr/32 of each
        // k-step's 512-byte atom.  The lane -> row choice keeps the 32 stores of
        // one instruction in 32 distinct banks and the 16-byte reads of each
        // quarter-warp on 8 consecutive rows.
        const bool fast = (K % BK) == 0;
        int it = 0;
        for (int tile = blockIdx.x; tile < tiles; tile += gridDim.x) {
            int mb, nb;
            tile_coords(tile, num_m, num_n, mb, nb);
            bool ok = true;
            for (int kb = 0; kb < num_kb; ++kb, ++it) {
                const int s = it % STAGES;
                const uint32_t ph = (it / STAGES) & 1;
                uint4 v[4 * (1 + NRB)];
                if (SF_TMA) {
                    if (!warp_wait(&sm.tma_full[s], ph, abort, ROLE_SF)) { ok = false; break; }
#pragma unroll
                    for (int i = 0; i < 4 * (1 + NRB); ++i) {
                        const int blk = i / 4;
                        const int rr = 32 * (lane >> 3) + 8 * (i & 3) + (lane & 7);
                        const uint4* raw = blk == 0
                            ? reinterpret_cast<const uint4*>(sm.sfa[s]) + rr
                            : reinterpret_cast<const uint4*>(sm.sfb[s]) + (blk - 1) * 128 + rr;
                        v[i] = *raw;
                    }
                    __syncwarp();
                } else {
                    if (!warp_wait(&sm.empty[s], ph ^ 1, abort, ROLE_SF)) { ok = false; break; }
#pragma unroll
                    for (int i = 0; i < 4 * (1 + NRB); ++i) {
                        const int blk = i / 4;
                        const int rr = 32 * (lane >> 3) + 8 * (i & 3) + (lane & 7);
                        v[i] = blk == 0 ? load_sf16(sA, mb * BM + rr, M, kb, G, fast)
                                        : load_sf16(sW, nb * BN + (blk - 1) * 128 + rr, N, kb, G, fast);
                    }
                }
#pragma unroll
                for (int i = 0; i < 4 * (1 + NRB); ++i) {
                    const int blk = i / 4;
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
        const int q = warp & 3;                 // TMEM lane quarter this warp may access
        const int half = (warp - 4) >> 2;       // which half of the BN columns
        constexpr int COLS = BN / 2;
        constexpr int CHUNKS = COLS / 32;
        const bool vec_ok = (N % 8) == 0;
        int tc = 0;
        for (int tile = blockIdx.x; tile < tiles; tile += gridDim.x, ++tc) {
            int mb, nb;
            tile_coords(tile, num_m, num_n, mb, nb);
            if (!warp_wait(&sm.acc_full, tc & 1, abort, ROLE_EPI)) break;
            tc_fence_after();
            uint32_t packed[COLS / 2];
#pragma unroll
            for (int c = 0; c < CHUNKS; ++c) {
                uint32_t r[32];
                tmem_ld_32x32b_x32(tmem + ((uint32_t)(32 * q) << 16) + half * COLS + c * 32, r);
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

            const int row = mb * BM + 32 * q + lane;
            const int col0 = nb * BN + half * COLS;
            if (row < M) {
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
                    for (int j = 0; j < COLS; ++j) {
                        if (col0 + j < N)
                            y16[col0 + j] = (uint16_t)(packed[j >> 1] >> (16 * (j & 1)));
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

}  // namespace w4a4
}  // namespace nvfp4
