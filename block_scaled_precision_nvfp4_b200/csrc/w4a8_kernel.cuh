// w4a8_kernel.cuh -- FP8 (E4M3) activations under NVFP4 weights on the FP8
// tensor-core MMA, exactly (metrale_circuit `hardware::exec`, exec_of: W4A8
// with group-16 E4M3 weight scales has no single-instruction MMA and takes the
// exact E4M3 path):
//
//     Y[m,n] = gA*gW * sum_g sW[n,g] * sum_{k in g} a8[m,k] * e2m1(W[n,k])
//
// The activations go to the FP8 MMA as they are.  The weights go through an
// exact conversion that carries the group scale inside the operand, so the
// FP32 accumulator stays in tensor memory for the whole of K (no per-group
// partial leaves TMEM):
//
//  * a scale byte s is x * 2^b with x an integer in 0..15 (x = 8 + mantissa,
//    b = E - 10 for a normal byte; x = mantissa, b = -9 for a subnormal one);
//  * x is written in non-adjacent form, x = sum_i sigma_i * 2^t_i with at most
//    three nonzero signed digits (x3 = x + (x >> 1), c = (x >> 1) ^ x3: the
//    positive digits are x3 & c, the negative ones (x >> 1) & c);
//  * plane i of a weight is sigma_i * e2m1(w) * 2^(t_i + b), an E5M2 byte: an
//    E2M1 value has two significant bits, and |t_i + b| <= 9 keeps every value
//    inside E5M2's normal range, so the byte is exact;
//  * sum_i plane_i = e2m1(w) * s, so three E4M3 x E5M2 MMAs per K step, one per
//    plane, accumulate sum_k a8 * w * s in FP32 exactly as the declared W4A4
//    block-scaled product would (each product exact, FP32 accumulation).
//
// Operand placement: the weight planes are the MMA's A operand (M = 128 weight
// rows) and live in tensor memory, written there by the converter warps with
// tcgen05.st straight from registers; the activations are the B operand
// (N = 256 tokens), 128-byte-swizzled tiles loaded by TMA.  The accumulator is
// D[weight row][token]; the epilogue writes Y[token][weight row].
//
// Roles (one persistent CTA per SM, 16 warps, tiles of 128 weight rows x 256
// tokens):
//   warp 0      activation producer: TMA of 128-byte-wide boxes of the tile's
//               256 token rows into a 4-stage ring released by MMA commits.
//   warp 1      TMEM owner (512 columns: accumulator 256, plane ring 8 x 24),
//               MMA issuer.
//   warp 2      weight producer: packed weight K-blocks and their raw scale
//               tiles into a 4-stage ring released by the converters, so the
//               weights run ahead of the activations.
//   warps 4-11  converters, one weight row per thread (TMEM lane), two warps
//               per lane quarter taking the even and the odd K steps: per step,
//               32 codes -> three planes of 32 E5M2 bytes -> tcgen05.st.  The
//               plane tables of every scale byte are built once per CTA in
//               shared memory.
//   warps 12-15 epilogue: TMEM -> registers, x alpha, BF16 RNE, store.
// Requires K % 256 == 0 (TMA of the scale tiles).
#pragma once
#include <cuda_bf16.h>
#include <cstdint>

#include "ptx.cuh"
#include "via_fp8_kernel.cuh"

namespace nvfp4 {
namespace w4a8 {

using via_fp8::tile_coords;
using via_fp8::warp_wait;

constexpr int BW = 128;               // weight rows per tile (TMEM lanes, the MMA's M)
constexpr int BT = 256;               // tokens per tile (the MMA's N)
constexpr int BK = 256;               // codes per weight K-block
constexpr int STEPS = BK / 32;        // K = 32 MMA steps per weight K-block
constexpr int ASTAGES = 4;            // activation ring, 128 bytes of K (4 steps) per stage
constexpr int WSTAGES = 4;            // weight ring, one K-block per stage
constexpr int PLANES = 3;             // signed digits of a scale, at most
constexpr int NSLOT = 8;              // TMEM plane-slot ring, one K step each
constexpr int SLOT_COLS = PLANES * 8; // 32 bytes of K per lane = 8 columns per plane
constexpr int ACC_COLS = BT;          // FP32 accumulator columns
constexpr int TMEM_COLS = 512;
constexpr int CONV_WARPS = 8, EPI_WARPS = 4;  // two converter warps per TMEM lane quarter
constexpr int CONV_PER_Q = CONV_WARPS / 4;    // ... taking every CONV_PER_Q-th K step
constexpr int FIRST_CONV = 4;                 // warps 0-3: producers, MMA, one spare
constexpr int NUM_THREADS = 32 * (FIRST_CONV + CONV_WARPS + EPI_WARPS);
static_assert(ACC_COLS + NSLOT * SLOT_COLS <= TMEM_COLS, "TMEM budget");
static_assert(NSLOT == STEPS, "one TMEM slot per K step of a block");

enum Role { ROLE_PRODUCER = 1, ROLE_MMA = 2, ROLE_CONV = 3, ROLE_EPI = 4, ROLE_DRAIN = 5 };

struct Smem {
    alignas(1024) uint8_t act[ASTAGES][BT * 128];     // E4M3 activations, 128-byte swizzled
    alignas(1024) uint8_t w[WSTAGES][BW * 128];       // packed FP4 weights, swizzled
    alignas(16) uint8_t sw[WSTAGES][BW * 16];         // weight scales [row][16 groups]
    uint4 ptab01[128];                                // plane tables per scale byte: planes 0, 1
    uint2 ptab2[128];                                 // ... and plane 2
    uint64_t act_full[ASTAGES], act_empty[ASTAGES];
    uint64_t w_full[WSTAGES], w_empty[WSTAGES];
    uint64_t slot_full[NSLOT], slot_empty[NSLOT];
    uint64_t acc_full, acc_empty;
    uint64_t drain;
    uint32_t tmem_base;
    int abort;
};
constexpr size_t SMEM_BYTES = sizeof(Smem) + 1024;
constexpr uint32_t ACT_BYTES = BT * 128;
constexpr uint32_t W_BYTES = BW * 128 + BW * 16;

// kind::f8f6f4 instruction descriptor: F32 accumulator, A and B formats
// (0 = E4M3, 1 = E5M2), both K-major, M x N.
__host__ __device__ constexpr uint32_t idesc_f8f6f4(uint32_t M, uint32_t N, uint32_t afmt,
                                                    uint32_t bfmt) {
    return (1u << 4) | (afmt << 7) | (bfmt << 10) | ((N >> 3) << 17) | ((M >> 4) << 24);
}

// D (TMEM) += A (TMEM, K-major: row i in lane i, K bytes along the columns) x B (smem).
__device__ __forceinline__ void mma_f8f6f4_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                              uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], [%1], %2, %3, p;\n\t}"
        ::"r"(d_tmem), "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// This warp's 32 lanes x 8 consecutive 32-bit columns from registers.
__device__ __forceinline__ void tmem_st_32x32b_x8(uint32_t taddr, const uint32_t (&r)[8]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};"
        ::"r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]),
          "r"(r[7])
        : "memory");
}
__device__ __forceinline__ void tmem_st_wait() {
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// One plane of one group: an 8-entry byte table T[c] = E5M2(sigma * e2m1(c) *
// 2^p) for the magnitude codes c = 0..7, as two words for byte_perm.  With
// base = (p + 14) << 2 the E5M2 magnitudes are
//   c=0: 0                  c=1 (0.5): base      c=2 (1): base + 4
//   c=3 (1.5): base + 6     c=4 (2): base + 8    c=5 (3): base + 10
//   c=6 (4): base + 12      c=7 (6): base + 14
// (exponent field p + 14 + e2m1 exponent, mantissa bit of the code in bit 1),
// and the digit's sign sigma sits in bit 7 of every entry (so T[0] may be -0).
// A plane the scale does not use is all 0x80: -0 for every code.  The code's
// own sign is XORed in afterwards.
struct PlaneTable {
    uint32_t lo, hi;
};

__device__ __forceinline__ void plane_tables(uint32_t sb, PlaneTable (&t)[PLANES]) {
    const uint32_t E = (sb >> 3) & 15u, mt = sb & 7u;
    const uint32_t x = E ? (8u | mt) : mt;
    const int b = E ? (int)E - 10 : -9;
    const uint32_t xh = x >> 1, x3 = x + xh, c = xh ^ x3;
    const uint32_t neg = xh & c;
    uint32_t d = (x3 & c) | neg;  // digit positions, at most three
#pragma unroll
    for (int i = 0; i < PLANES; ++i) {
        if (d) {
            const int ti = __ffs(d) - 1;
            d &= d - 1;
            const uint32_t base = (uint32_t)(ti + b + 14) << 2;
            const uint32_t sgn = ((neg >> ti) & 1u) ? 0x80808080u : 0u;
            t[i].lo = (base * 0x01010100u + 0x06040000u) | sgn;
            t[i].hi = (base * 0x01010101u + 0x0E0C0A08u) | sgn;
        } else {
            t[i].lo = 0x80808080u;
            t[i].hi = 0x80808080u;
        }
    }
}

// Eight packed codes (code j in nibble j) -> for each plane, two words of E5M2
// bytes in k order (byte j of the first word = code j).
__device__ __forceinline__ void convert8_planes(uint32_t w, const PlaneTable (&t)[PLANES],
                                                uint32_t (&out)[PLANES][2]) {
    // byte_perm reads the low 16 bits of its selector: four nibbles
    const uint32_t sel_lo = w & 0x77777777u, sel_hi = sel_lo >> 16;
    // 0x80 in byte j where code j is negative: byte_perm of (byte 0 = 0, byte 1 = 0x80)
    const uint32_t sgn = (w >> 3) & 0x11111111u;
    const uint32_t sg_lo = __byte_perm(0x8000u, 0u, sgn);
    const uint32_t sg_hi = __byte_perm(0x8000u, 0u, sgn >> 16);
#pragma unroll
    for (int i = 0; i < PLANES; ++i) {
        out[i][0] = __byte_perm(t[i].lo, t[i].hi, sel_lo) ^ sg_lo;
        out[i][1] = __byte_perm(t[i].lo, t[i].hi, sel_hi) ^ sg_hi;
    }
}

// A producer that has given up waits (bounded) for the copies it started.
__device__ __forceinline__ void drain_copies(uint64_t* full, int stages, int it) {
    for (int j = max(0, it - stages); j < it; ++j) {
        const uint64_t t0 = globaltimer_ns();
        while (!mbar_try_wait(&full[j % stages], (j / stages) & 1) &&
               globaltimer_ns() - t0 < kWaitLimitNs) {
        }
    }
}

__global__ void __launch_bounds__(NUM_THREADS, 1)
w4a8_kernel(const __grid_constant__ CUtensorMap tmA,   // E4M3 [M][K], box 128 B x 256 rows
            const __grid_constant__ CUtensorMap tmB,   // packed W [N][K/2], box 128 B x 128 rows
            const __grid_constant__ CUtensorMap tmSB,  // sW [N][K/16], box 16 B x 128 rows
            __nv_bfloat16* __restrict__ Y, int M, int N, int K, float alpha) {
    extern __shared__ uint8_t smem_raw[];
    Smem& sm = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                        ~uintptr_t(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int num_t = (M + BT - 1) / BT, num_w = (N + BW - 1) / BW;
    const int tiles = num_t * num_w;
    const int num_kb = K / BK;
    volatile int* abort = &sm.abort;

    if (threadIdx.x == 0) {
        for (int s = 0; s < ASTAGES; ++s) {
            mbar_init(&sm.act_full[s], 1);
            mbar_init(&sm.act_empty[s], 1);           // the MMA's commit
        }
        for (int s = 0; s < WSTAGES; ++s) {
            mbar_init(&sm.w_full[s], 1);
            mbar_init(&sm.w_empty[s], CONV_WARPS);    // every converter warp
        }
        for (int s = 0; s < NSLOT; ++s) {
            mbar_init(&sm.slot_full[s], 4);  // the step's converter warp of each lane quarter
            mbar_init(&sm.slot_empty[s], 1);
        }
        mbar_init(&sm.acc_full, 1);
        mbar_init(&sm.acc_empty, EPI_WARPS);
        mbar_init(&sm.drain, 1);
        sm.abort = 0;
        fence_mbarrier_init();
        tma_prefetch_desc(&tmA);
        tma_prefetch_desc(&tmB);
        tma_prefetch_desc(&tmSB);
    }
    if (threadIdx.x < 128) {  // the plane tables of scale byte threadIdx.x
        PlaneTable t[PLANES];
        plane_tables(threadIdx.x, t);
        sm.ptab01[threadIdx.x] = make_uint4(t[0].lo, t[0].hi, t[1].lo, t[1].hi);
        sm.ptab2[threadIdx.x] = make_uint2(t[2].lo, t[2].hi);
    }
    if (warp == 1) {
        tmem_alloc(&sm.tmem_base, TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem_base;

    if (warp == 0) {
        // ------------------------------------------------------------ activation producer
        if (lane == 0) {
            int it = 0;
            for (int tile = blockIdx.x; tile < tiles && !*abort; tile += gridDim.x) {
                int tt, tw;
                tile_coords(tile, num_t, num_w, tt, tw);
                for (int j = 0; j < 2 * num_kb; ++j, ++it) {
                    const int a = it % ASTAGES;
                    if (!mbar_wait(&sm.act_empty[a], ((it / ASTAGES) & 1) ^ 1, abort, ROLE_PRODUCER))
                        goto act_done;
                    mbar_arrive_expect_tx(&sm.act_full[a], ACT_BYTES);
                    tma_load_2d(sm.act[a], &tmA, &sm.act_full[a], j * 128, tt * BT);
                }
            }
        act_done:
            if (*abort) drain_copies(sm.act_full, ASTAGES, it);
        }
    } else if (warp == 2) {
        // ------------------------------------------------------------ weight producer
        if (lane == 0) {
            int it = 0;
            for (int tile = blockIdx.x; tile < tiles && !*abort; tile += gridDim.x) {
                int tt, tw;
                tile_coords(tile, num_t, num_w, tt, tw);
                for (int kb = 0; kb < num_kb; ++kb, ++it) {
                    const int r = it % WSTAGES;
                    if (!mbar_wait(&sm.w_empty[r], ((it / WSTAGES) & 1) ^ 1, abort, ROLE_PRODUCER))
                        goto w_done;
                    mbar_arrive_expect_tx(&sm.w_full[r], W_BYTES);
                    tma_load_2d(sm.w[r], &tmB, &sm.w_full[r], kb * 128, tw * BW);
                    tma_load_2d(sm.sw[r], &tmSB, &sm.w_full[r], kb * 16, tw * BW);
                }
            }
        w_done:
            if (*abort) drain_copies(sm.w_full, WSTAGES, it);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        // The whole warp walks the loop (converged, as tcgen05 issue wants it); the
        // same elected lane issues every MMA and every commit that tracks them.
        const uint32_t idesc = idesc_f8f6f4(BW, BT, /*A E5M2*/ 1u, /*B E4M3*/ 0u);
        // descriptor of stage 0's first K slice; stage a and slice hh add their offsets
        // (in 16-byte units) to the start-address field
        const uint64_t bdesc0 = desc_kmajor_sw128(smem_u32(sm.act[0]));
        int ait = 0, it = 0, tc = 0;
        bool ok = true;
        for (int tile = blockIdx.x; tile < tiles && ok; tile += gridDim.x, ++tc) {
            // the epilogue has read the previous tile's accumulator
            if (!warp_wait(&sm.acc_empty, (tc & 1) ^ 1, abort, ROLE_MMA)) { ok = false; break; }
            tc_fence_after();
            for (int kb = 0; kb < num_kb && ok; ++kb, ++it) {
                for (int half = 0; half < 2 && ok; ++half, ++ait) {
                    const int a = ait % ASTAGES;
                    if (!warp_wait(&sm.act_full[a], (ait / ASTAGES) & 1, abort, ROLE_MMA)) { ok = false; break; }
                    for (int hh = 0; hh < 4; ++hh) {
                        const int h = 4 * half + hh;  // K step of the block = TMEM slot
                        if (!warp_wait(&sm.slot_full[h], it & 1, abort, ROLE_MMA)) { ok = false; break; }
                        tc_fence_after();
                        if (elect_one()) {
                            // B: the K = 32 slice of the 256 activation rows (128-byte swizzle)
                            const uint64_t bdesc = bdesc0 + (uint64_t)(a * (BT * 128 / 16) + hh * 2);
                            const uint32_t a0 = tmem + ACC_COLS + h * SLOT_COLS;
#pragma unroll
                            for (int i = 0; i < PLANES; ++i)
                                mma_f8f6f4_ts(tmem, a0 + i * 8, bdesc, idesc, (kb | h | i) != 0);
                            mma_commit(&sm.slot_empty[h]);
                        }
                        __syncwarp();
                    }
                    if (ok && elect_one()) mma_commit(&sm.act_empty[a]);  // this stage's activations are read
                    __syncwarp();
                }
            }
            if (ok && elect_one()) mma_commit(&sm.acc_full);
            __syncwarp();
        }
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
    } else if (warp >= FIRST_CONV && warp < FIRST_CONV + CONV_WARPS) {
        // ------------------------------------------------------------ converters
        const int q = warp & 3;                      // TMEM lane quarter this warp may access
        const int par = (warp - FIRST_CONV) >> 2;    // K steps h = par, par + CONV_PER_Q, ...
        const int row = 32 * q + lane;               // weight row within the tile
        const uint32_t tq = tmem + ((uint32_t)(32 * q) << 16) + ACC_COLS;
        int it = 0;
        bool ok = true;
        for (int tile = blockIdx.x; tile < tiles && ok; tile += gridDim.x) {
            for (int kb = 0; kb < num_kb && ok; ++kb, ++it) {
                const int r = it % WSTAGES;
                if (!warp_wait(&sm.w_full[r], (it / WSTAGES) & 1, abort, ROLE_CONV)) { ok = false; break; }
                const uint4 sbq = *reinterpret_cast<const uint4*>(sm.sw[r] + row * 16);
                const uint32_t sbw[4] = {sbq.x, sbq.y, sbq.z, sbq.w};
#pragma unroll 1
                for (int h = par; h < STEPS; h += CONV_PER_Q) {
                    // K step h of the block uses TMEM slot h (STEPS == NSLOT): codes
                    // 32h .. 32h+31 of the row, 16 bytes, chunk h of the 128-byte swizzled
                    // row; groups 2h and 2h+1
                    const uint4 qb = *reinterpret_cast<const uint4*>(
                        sm.w[r] + row * 128 + ((h ^ (row & 7)) << 4));
                    const uint32_t sb0 = (sbw[h >> 1] >> (16 * (h & 1))) & 0x7Fu;
                    const uint32_t sb1 = (sbw[h >> 1] >> (16 * (h & 1) + 8)) & 0x7Fu;
                    PlaneTable t0[PLANES], t1[PLANES];
                    {
                        const uint4 a01 = sm.ptab01[sb0], b01 = sm.ptab01[sb1];
                        const uint2 a2 = sm.ptab2[sb0], b2 = sm.ptab2[sb1];
                        t0[0] = {a01.x, a01.y}; t0[1] = {a01.z, a01.w}; t0[2] = {a2.x, a2.y};
                        t1[0] = {b01.x, b01.y}; t1[1] = {b01.z, b01.w}; t1[2] = {b2.x, b2.y};
                    }
                    uint32_t o0[PLANES][2], o1[PLANES][2], o2[PLANES][2], o3[PLANES][2];
                    convert8_planes(qb.x, t0, o0);
                    convert8_planes(qb.y, t0, o1);
                    convert8_planes(qb.z, t1, o2);
                    convert8_planes(qb.w, t1, o3);
                    if (!warp_wait(&sm.slot_empty[h], (it & 1) ^ 1, abort, ROLE_CONV)) { ok = false; break; }
                    tc_fence_after();
#pragma unroll
                    for (int i = 0; i < PLANES; ++i) {
                        const uint32_t v[8] = {o0[i][0], o0[i][1], o1[i][0], o1[i][1],
                                               o2[i][0], o2[i][1], o3[i][0], o3[i][1]};
                        tmem_st_32x32b_x8(tq + h * SLOT_COLS + i * 8, v);
                    }
                    tmem_st_wait();
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&sm.slot_full[h]);
                }
                __syncwarp();
                if (ok && lane == 0) mbar_arrive(&sm.w_empty[r]);  // this K-block's weights are read
            }
        }
    } else if (warp >= FIRST_CONV + CONV_WARPS) {
        // ------------------------------------------------------------ epilogue
        const int q = warp & 3;
        const uint32_t tq = tmem + ((uint32_t)(32 * q) << 16);
        int tc = 0;
        for (int tile = blockIdx.x; tile < tiles; tile += gridDim.x, ++tc) {
            int tt, tw;
            tile_coords(tile, num_t, num_w, tt, tw);
            if (!warp_wait(&sm.acc_full, tc & 1, abort, ROLE_EPI)) break;
            tc_fence_after();
            const int n = tw * BW + 32 * q + lane;   // this thread's weight row = output column
            const int m0 = tt * BT;
#pragma unroll 1
            for (int c = 0; c < BT / 32; ++c) {
                uint32_t v[32];
                tmem_ld_32x32b_x32(tq + 32 * c, v);
                tmem_ld_wait();
                reg_fence(v);
                if (c == BT / 32 - 1) {  // the whole accumulator is read: release it
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&sm.acc_empty);
                }
                if (n < N) {
                    // token m0 + 32c + j; the warp's 32 lanes write 64 contiguous bytes
#pragma unroll
                    for (int j = 0; j < 32; ++j) {
                        const int m = m0 + 32 * c + j;
                        if (m < M)
                            Y[(size_t)m * N + n] = __float2bfloat16_rn(__uint_as_float(v[j]) * alpha);
                    }
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem, TMEM_COLS);
}

}  // namespace w4a8
}  // namespace nvfp4
