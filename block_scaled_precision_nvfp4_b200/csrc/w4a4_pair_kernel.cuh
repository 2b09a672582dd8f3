// w4a4_pair_kernel.cuh -- NVFP4 W4A4 matmul on pairs of SMs (tcgen05 cta_group::2)
// with scales already in the MMA's scale layout (pack_scales_kernel.cuh).
//
// Same product as w4a4_kernel.cuh (metrale_circuit `hardware::exec` module doc,
// bullet 1, the NVFP4 row), with 256 x 256 output tiles computed by a cluster
// of two CTAs on two SMs:
//   * each CTA loads, with plain TMA tile loads, its own 128 rows of A, its own
//     128 rows of W (half of the tile's N), the packed scales of its A rows and
//     the packed scales of all 256 W rows; completion of both CTAs' loads is
//     counted on one barrier in the leader CTA (rank 0), armed for both;
//   * the leader's MMA thread copies both CTAs' scales to their TMEM
//     (tcgen05.cp.cta_group::2: one instruction serves both SMs) and issues
//     tcgen05.mma.cta_group::2 kind::mxf4nvf4 M=256 N=256 K=64; its commits
//     free the stage in both CTAs;
//   * each CTA's epilogue reads its own 128 x 256 accumulator, releases it,
//     and writes the BF16 tile through shared memory with TMA bulk stores
//     (one 32-row x 128-byte box per store): a plain store from each thread's
//     accumulator row would touch 32 rows per instruction, and those scattered
//     stores compete with the tensor core for the shared-memory data path.
// Against one SM per 128 x 256 tile, every SM reads half as many W bytes per
// flop and the pair issues half as many scale copies per flop; with the
// scales packed ahead there is no shared-memory rewrite or cross-CTA hand-off
// on the critical path.  All waits are bounded; both CTAs meet at a cluster
// barrier before the pair's TMEM is freed.
//
// Load balance (stream-K over the last waves): when the tiles do not divide
// evenly among the pairs, the last wave of whole tiles would leave most pairs
// idle.  With a workspace, the tiles are then handed out in two parts:
//   * the K-blocks of the last one-and-a-half waves of tiles, laid end to end,
//     are cut into one contiguous range per pair, so every pair multiplies the
//     same number of K-blocks (give or take one).  A range is at least one tile
//     long, so a tile cut by a range boundary has exactly two contributors;
//   * the other tiles go whole to the pairs in turn, after each pair's range
//     (so the partial-sum exchange below is hidden behind them).
// Each epilogue warp of a cut tile takes a ticket in the workspace: the first of
// the two contributors to arrive writes its FP32 partial sums there, and the
// second adds them to its own and writes the BF16 output.  Nobody waits for
// anybody, and the sum of two FP32 terms is the same in either order, so the
// output does not depend on which contributor comes first.  The second one
// resets the ticket, so the workspace is ready for the next launch.
#pragma once
#include <cuda_bf16.h>
#include <cstdint>

#include "ptx.cuh"
#include "w4a4_kernel.cuh"

namespace nvfp4 {
namespace w4a4_pair {

using w4a4::BK;
using w4a4::BKB;
using w4a4::KSTEPS;
using w4a4::ROLE_DRAIN;
using w4a4::ROLE_EPI;
using w4a4::ROLE_MMA;
using w4a4::ROLE_PRODUCER;
using w4a4::warp_wait;

constexpr int BM = 128;        // rows of A per CTA (the pair covers 256)
constexpr int TILE_M = 256;
constexpr int BN = 256;        // tile columns (rows of W) per pair
constexpr int BNH = 128;       // rows of W loaded by each CTA
constexpr int NRB = BN / 128;  // 128-row scale blocks of W per tile
constexpr int STAGES = 5;
constexpr int NUM_EPI_WARPS = 8;
constexpr int NUM_THREADS = 32 * (2 + NUM_EPI_WARPS);
constexpr int FIRST_EPI_WARP = 2;
constexpr int GROUP_M = 16;

struct Smem {
    alignas(1024) uint8_t a[STAGES][BM * BKB];
    alignas(1024) uint8_t b[STAGES][BNH * BKB];
    alignas(128) uint32_t sfa[STAGES][KSTEPS * 128];        // [ks][512-byte atom]
    alignas(128) uint32_t sfb[STAGES][NRB * KSTEPS * 128];  // [rb][ks][512-byte atom]
    alignas(1024) uint8_t out[NUM_EPI_WARPS][32 * 128];     // each epilogue warp's staging box
    uint64_t full[STAGES];   // leader: every byte of the stage, both CTAs
    uint64_t empty[STAGES];  // each CTA: stage free (commit from the leader)
    uint64_t acc_full;       // each CTA: accumulator ready (commit from the leader)
    uint64_t acc_empty;      // leader: both CTAs' epilogues have read TMEM
    uint64_t drain;
    uint32_t tmem_base;
    int abort;
};

// one CTA's bytes per stage: A, half of W, sA of its rows, sW of all 256 rows
constexpr uint32_t BYTES_CTA = (BM + BNH) * BKB + (BM + BN) * 16;
constexpr int SFA_COLS = KSTEPS * 4, SFB_COLS = KSTEPS * NRB * 4;
constexpr int TMEM_COLS = 512;
static_assert(BN + STAGES * (SFA_COLS + SFB_COLS) <= TMEM_COLS, "TMEM budget exceeded");
constexpr size_t SMEM_BYTES = sizeof(Smem) + 1024;
__host__ __device__ constexpr uint32_t sfa_col(int s) { return BN + s * (SFA_COLS + SFB_COLS); }
__host__ __device__ constexpr uint32_t sfb_col(int s) { return sfa_col(s) + SFA_COLS; }

constexpr int SLAB_COLS = 64;  // columns of one output store box (128 bytes)

// ---- stream-K workspace: per cut tile ("slot"), a ticket for each epilogue warp of
// each CTA, and the two contributors' FP32 partials of that warp's 32 x 128 block,
// stored as [32 column quads][32 lanes] float4 (a warp's store of one quad is 512
// contiguous bytes).
constexpr int PART_FLOATS = 32 * (BN / 2);
constexpr int TICKETS_PER_SLOT = 2 * NUM_EPI_WARPS;
__host__ __device__ constexpr size_t part_offset(int slot, int side, int rank, int w) {
    return ((((size_t)slot * 2 + side) * 2 + rank) * NUM_EPI_WARPS + w) * PART_FLOATS;
}
// bytes of tickets (rounded up to 256) and partials for `slots` cut tiles
__host__ __device__ constexpr size_t ticket_bytes(int slots) {
    return ((size_t)slots * TICKETS_PER_SLOT * 4 + 255) & ~(size_t)255;
}
__host__ __device__ constexpr size_t split_workspace_bytes(int slots) {
    return ticket_bytes(slots) + part_offset(slots, 0, 0, 0) * sizeof(float);
}

// One unit of a pair's work: K-blocks [kb0, kb1) of one output tile.
struct Segment {
    int tile, kb0, kb1;
    int slot;  // -1: the tile is this pair's alone; else its partial-sum slot
    int side;  // 0: the tile's first K-blocks, 1: its last ones
};

// The j-th segment of pair `cid` of `P`: first this pair's range of the K-blocks
// of the tiles from dp_tiles on (range c is [c*S/P, (c+1)*S/P) of the S K-blocks
// laid end to end), then the tiles below dp_tiles whole, in turn (cid, cid + P,
// ...).  The cut tiles come first, the shorter cut before the longer and both
// before the range's whole tiles: the epilogue of a cut segment exchanges partial
// sums, and what follows it on the MMA should be long enough to hide that (with a
// single accumulator, a late epilogue holds up the MMAs of the segment after
// next).  The cut at the start of range c (c >= 1) is slot c - 1.  False past the
// pair's last segment.
__device__ __forceinline__ bool segment_of(int j, int cid, int P, int tiles, int dp_tiles,
                                           int num_kb, Segment& sg) {
    const long long S = (long long)(tiles - dp_tiles) * num_kb;
    const long long b = S * cid / P, e = S * (cid + 1) / P;
    const int n_sk = S > 0 ? (int)((e - 1) / num_kb - b / num_kb + 1) : 0;
    sg.slot = -1;
    sg.side = 0;
    if (j >= n_sk) {
        const int jd = j - n_sk;
        const int n_dp = cid < dp_tiles ? (dp_tiles - cid + P - 1) / P : 0;
        if (jd >= n_dp) return false;
        sg.tile = cid + jd * P;
        sg.kb0 = 0;
        sg.kb1 = num_kb;
        return true;
    }
    // the range's segments in K order are 0 .. n_sk-1; 0 is cut when b is inside a
    // tile, n_sk-1 when e is (a range of at least one tile has two distinct ends)
    const int head = (int)(b % num_kb), tail = (int)(e % num_kb);
    int k = j;
    if (head && tail) {
        const bool head_shorter = num_kb - head <= tail;
        k = j == 0 ? (head_shorter ? 0 : n_sk - 1) : j == 1 ? (head_shorter ? n_sk - 1 : 0) : j - 1;
    } else if (tail) {
        k = j == 0 ? n_sk - 1 : j - 1;
    }
    const long long t = b / num_kb + k;  // among the tiles from dp_tiles on
    const long long t0 = t * num_kb;     // its first K-block, end to end
    sg.tile = dp_tiles + (int)t;
    sg.kb0 = b > t0 ? (int)(b - t0) : 0;
    sg.kb1 = e - t0 < num_kb ? (int)(e - t0) : num_kb;
    if (sg.kb0 > 0) {
        sg.slot = cid - 1;
        sg.side = 1;
    } else if (sg.kb1 < num_kb) {
        sg.slot = cid;
        sg.side = 0;
    }
    return true;
}

__device__ __forceinline__ uint32_t ld_acquire_gpu(const unsigned* p) {
    uint32_t v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// A cut tile's epilogue warp, holding its own FP32 partial sums in r (column
// 32c + k in r[c][k]).  Returns false when it is the first contributor to arrive:
// its partial is then left in the workspace.  Returns true when it is the second:
// r then holds the sum of both partials, and the ticket is back at zero.
__device__ __forceinline__ bool combine_partial(float* __restrict__ ws, unsigned* __restrict__ tickets,
                                                const Segment& sg, int rank, int w,
                                                uint32_t (&r)[4][32]) {
    const int lane = threadIdx.x & 31;
    unsigned* tk = tickets + (sg.slot * 2 + rank) * NUM_EPI_WARPS + w;
    unsigned seen = 0;
    if (lane == 0) seen = ld_acquire_gpu(tk);
    seen = __shfl_sync(0xffffffffu, seen, 0);
    if (seen == 0) {
        float4* mine = reinterpret_cast<float4*>(ws + part_offset(sg.slot, sg.side, rank, w)) + lane;
#pragma unroll
        for (int i = 0; i < 32; ++i)
            __stcg(mine + i * 32, make_float4(__uint_as_float(r[i >> 3][(i & 7) * 4]),
                                              __uint_as_float(r[i >> 3][(i & 7) * 4 + 1]),
                                              __uint_as_float(r[i >> 3][(i & 7) * 4 + 2]),
                                              __uint_as_float(r[i >> 3][(i & 7) * 4 + 3])));
        __threadfence();
        __syncwarp();
        if (lane == 0) seen = atomicAdd(tk, 1u);
        seen = __shfl_sync(0xffffffffu, seen, 0);
        if (seen == 0) return false;
    }
    // lane 0 saw the other contributor's ticket (an acquire load, or the add followed
    // by this fence); the warp barrier then orders every lane's reads after it
    __threadfence();
    __syncwarp();
    const float4* other =
        reinterpret_cast<const float4*>(ws + part_offset(sg.slot, sg.side ^ 1, rank, w)) + lane;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
#pragma unroll
        for (int q = 0; q < 8; ++q) {
            const float4 o = __ldcg(other + (c * 8 + q) * 32);
            r[c][4 * q] = __float_as_uint(__uint_as_float(r[c][4 * q]) + o.x);
            r[c][4 * q + 1] = __float_as_uint(__uint_as_float(r[c][4 * q + 1]) + o.y);
            r[c][4 * q + 2] = __float_as_uint(__uint_as_float(r[c][4 * q + 2]) + o.z);
            r[c][4 * q + 3] = __float_as_uint(__uint_as_float(r[c][4 * q + 3]) + o.w);
        }
        reg_fence(r[c]);
    }
    __syncwarp();
    if (lane == 0) atomicExch(tk, 0u);
    return true;
}

// One epilogue warp's 32 rows (lane = row) x 128 columns, held as packed BF16
// pairs, stored through the warp's 4 KB staging buffer as two 32 x 64 boxes.
// The buffer holds the 128-byte swizzle of the box (16-byte chunk c of row r
// at chunk c ^ (r & 7)), which makes the warp's shared-memory writes
// conflict-free.  With `tma` (a valid output map, and all 32 rows of the slab
// belonging to this output) each box leaves by one TMA bulk store, clipped at
// N and at the map's last row; otherwise the warp copies the first `nrows`
// rows of the box out with plain stores (rows of the slab past `nrows`, and
// columns past N, are not written).
__device__ __forceinline__ void store_slab(const CUtensorMap* tmY, bool tma, uint8_t* stage,
                                           const uint32_t (&packed)[64], int row0, int nrows,
                                           int col0, int N, __nv_bfloat16* __restrict__ Y) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        if (lane == 0) bulk_wait_read_all();  // the previous box has left the buffer
        __syncwarp();
        uint8_t* rowp = stage + lane * 128;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
            const int w = h * 32 + c * 4;
            *reinterpret_cast<uint4*>(rowp + ((c ^ (lane & 7)) << 4)) =
                make_uint4(packed[w], packed[w + 1], packed[w + 2], packed[w + 3]);
        }
        const int x = col0 + h * SLAB_COLS;
        if (tma) {
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0 && x < N) {
                tma_store_2d(tmY, stage, x, row0);
                bulk_commit_group();
            }
        } else {
            __syncwarp();
            uint16_t* y16 = reinterpret_cast<uint16_t*>(Y);
            for (int r = 0; r < nrows; ++r) {
                const uint8_t* src = stage + r * 128;
                for (int c = lane; c < SLAB_COLS; c += 32)
                    if (x + c < N)
                        y16[(size_t)(row0 + r) * N + x + c] = *reinterpret_cast<const uint16_t*>(
                            src + ((((c >> 3) ^ (r & 7))) << 4) + (c & 7) * 2);
            }
            __syncwarp();  // the box is read before the next one overwrites it
        }
    }
}

__device__ __forceinline__ void tile_coords(int tile, int num_m, int num_n, int& mb, int& nb) {
    const int per_group = GROUP_M * num_n;
    const int first_m = (tile / per_group) * GROUP_M;
    const int gsize = min(num_m - first_m, GROUP_M);
    const int in_group = tile % per_group;
    mb = first_m + in_group % gsize;
    nb = in_group / gsize;
}

__device__ __forceinline__ void tma_load_3d_pair(void* smem_dst, const CUtensorMap* map,
                                                 uint32_t bar_cluster, int32_t x, int32_t y,
                                                 int32_t z) {
    asm volatile(
        "cp.async.bulk.tensor.3d.cta_group::2.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4, %5}], [%2];"
        ::"r"(smem_u32(smem_dst)), "l"(reinterpret_cast<uint64_t>(map)), "r"(bar_cluster),
          "r"(x), "r"(y), "r"(z)
        : "memory");
}

__global__ void __launch_bounds__(NUM_THREADS, 1)
w4a4_pair_kernel(const __grid_constant__ CUtensorMap tmA,   // A codes, box 128 B x 128 rows
                 const __grid_constant__ CUtensorMap tmB,   // W codes, box 128 B x 128 rows
                 const __grid_constant__ CUtensorMap tmSA,  // packed sA: [rb][ks*4][128 B], box (128, 16, 1)
                 const __grid_constant__ CUtensorMap tmSB,  // packed sW: same view, box (128, 16, 2)
                 const __grid_constant__ CUtensorMap tmY,   // Y bf16 [M][N], box 64 x 32, 128B swizzle
                 int tma_out,                               // tmY is valid (N % 8 == 0)
                 __nv_bfloat16* __restrict__ Y, int M, int N, int K, float alpha,
                 int dp_tiles,                     // tiles handed out whole (all of them: no split)
                 float* __restrict__ ws,           // partial sums of cut tiles (split only)
                 unsigned* __restrict__ tickets) { // one per epilogue warp of a cut tile, zero between launches
    extern __shared__ uint8_t smem_raw[];
    Smem& sm = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                        ~uintptr_t(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const bool leader = rank == 0;
    const int cid = blockIdx.x >> 1, nclusters = gridDim.x >> 1;
    const int num_m = (M + TILE_M - 1) / TILE_M, num_n = (N + BN - 1) / BN;
    const int tiles = num_m * num_n;
    const int num_kb = K / BK;
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
        tma_prefetch_desc(&tmA);
        tma_prefetch_desc(&tmB);
        tma_prefetch_desc(&tmSA);
        tma_prefetch_desc(&tmSB);
    }
    if (warp == 1) {
        tmem_alloc_pair(&sm.tmem_base, TMEM_COLS);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    cluster_sync();  // both CTAs' barriers exist before any remote arrive
    tc_fence_after();
    const uint32_t tmem = sm.tmem_base;
    // the set-up above overlaps the kernel before this one (the activations' scale
    // packing, when launched programmatically); its output is read only from here
    grid_dependency_wait();

    if (warp == 0) {
        // ------------------------------------------------------------ producer (both CTAs)
        int it = 0;
        bool ok = true;
        Segment sg;
        for (int j = 0; ok && segment_of(j, cid, nclusters, tiles, dp_tiles, num_kb, sg); ++j) {
            int mb, nb;
            tile_coords(sg.tile, num_m, num_n, mb, nb);
            const int arb = mb * 2 + (int)rank;  // this CTA's 128-row block of A
            for (int kb = sg.kb0; kb < sg.kb1; ++kb, ++it) {
                const int s = it % STAGES;
                if (!warp_wait(&sm.empty[s], ((it / STAGES) & 1) ^ 1, abort, ROLE_PRODUCER, 32)) {
                    ok = false;
                    break;
                }
                if (elect_one()) {
                    if (leader) mbar_arrive_expect_tx(&sm.full[s], 2 * BYTES_CTA);
                    const uint32_t full0 = map_to_rank(&sm.full[s], 0);
                    tma_load_2d_pair(sm.a[s], &tmA, full0, kb * BKB, arb * BM);
                    tma_load_2d_pair(sm.b[s], &tmB, full0, kb * BKB, nb * BN + (int)rank * BNH);
                    tma_load_3d_pair(sm.sfa[s], &tmSA, full0, 0, kb * 16, arb);
                    tma_load_3d_pair(sm.sfb[s], &tmSB, full0, 0, kb * 16, nb * NRB);
                }
                __syncwarp();
            }
        }
        if (!ok && leader && lane == 0) {
            // every copy of this pair lands before either CTA leaves
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
            const uint32_t idesc = idesc_mxf4nvf4(TILE_M, BN);
            int it = 0, tc = 0;
            bool ok = true;
            Segment sg;
            for (int j = 0; ok && segment_of(j, cid, nclusters, tiles, dp_tiles, num_kb, sg);
                 ++j, ++tc) {
                if (!warp_wait(&sm.acc_empty, (tc & 1) ^ 1, abort, ROLE_MMA)) { ok = false; break; }
                tc_fence_after();
                for (int kb = sg.kb0; kb < sg.kb1; ++kb, ++it) {
                    const int s = it % STAGES;
                    if (!warp_wait(&sm.full[s], (it / STAGES) & 1, abort, ROLE_MMA)) { ok = false; break; }
                    tc_fence_after();
                    if (elect_one()) {
#pragma unroll
                        for (int ks = 0; ks < KSTEPS; ++ks)
                            tmem_cp_32x128b_x4_pair(tmem + sfa_col(s) + ks * 4,
                                                    desc_sf_32x16(smem_u32(&sm.sfa[s][ks * 128])));
#pragma unroll
                        for (int ks = 0; ks < KSTEPS; ++ks)
#pragma unroll
                            for (int rb = 0; rb < NRB; ++rb)
                                tmem_cp_32x128b_x4_pair(
                                    tmem + sfb_col(s) + (ks * NRB + rb) * 4,
                                    desc_sf_32x16(smem_u32(&sm.sfb[s][(rb * KSTEPS + ks) * 128])));
                        const uint32_t a0 = smem_u32(sm.a[s]), b0 = smem_u32(sm.b[s]);
#pragma unroll
                        for (int ks = 0; ks < KSTEPS; ++ks)
                            mma_mxf4nvf4_pair(tmem, desc_kmajor_sw128(a0 + ks * 32),
                                              desc_kmajor_sw128(b0 + ks * 32), idesc,
                                              tmem + sfa_col(s) + ks * 4,
                                              tmem + sfb_col(s) + ks * NRB * 4,
                                              kb != sg.kb0 || ks != 0);
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
        static_assert(COLS == 128, "one epilogue warp stores 128 columns");
        uint8_t* stage = sm.out[warp - FIRST_EPI_WARP];
        int tc = 0;
        Segment sg;
        for (int j = 0; segment_of(j, cid, nclusters, tiles, dp_tiles, num_kb, sg); ++j, ++tc) {
            int mb, nb;
            tile_coords(sg.tile, num_m, num_n, mb, nb);
            if (!warp_wait(&sm.acc_full, tc & 1, abort, ROLE_EPI)) break;
            tc_fence_after();
            // the whole accumulator block behind one wait, then TMEM goes back to the MMA
            uint32_t r[CHUNKS][32];
#pragma unroll
            for (int c = 0; c < CHUNKS; ++c)
                tmem_ld_32x32b_x32(tmem + ((uint32_t)(32 * q) << 16) + half * COLS + c * 32, r[c]);
            tmem_ld_wait();
#pragma unroll
            for (int c = 0; c < CHUNKS; ++c) reg_fence(r[c]);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_remote(&sm.acc_empty, 0);
            if (sg.slot >= 0 &&
                !combine_partial(ws, tickets, sg, (int)rank, warp - FIRST_EPI_WARP, r))
                continue;  // the other contributor of this cut tile finishes it
            uint32_t packed[COLS / 2];
#pragma unroll
            for (int c = 0; c < CHUNKS; ++c)
#pragma unroll
                for (int k = 0; k < 16; ++k) {
                    __nv_bfloat162 h = __floats2bfloat162_rn(__uint_as_float(r[c][2 * k]) * alpha,
                                                             __uint_as_float(r[c][2 * k + 1]) * alpha);
                    packed[c * 16 + k] = *reinterpret_cast<uint32_t*>(&h);
                }

            const int row0 = mb * TILE_M + (int)rank * BM + 32 * q;
            const int col0 = nb * BN + half * COLS;
            if (row0 < M)
                store_slab(&tmY, tma_out != 0, stage, packed, row0, min(32, M - row0), col0, N, Y);
        }
        if (lane == 0) bulk_wait_all();  // staging buffers stay alive until the stores are done
    }

    // No CTA of the pair leaves (or frees TMEM) while the other may still use it.
    tc_fence_before();
    cluster_sync();
    tc_fence_after();
    if (warp == 1) tmem_dealloc_pair(tmem, TMEM_COLS);
}

}  // namespace w4a4_pair
}  // namespace nvfp4
