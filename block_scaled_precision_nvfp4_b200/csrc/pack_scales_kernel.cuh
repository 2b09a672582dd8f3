// pack_scales_kernel.cuh -- plain E4M3 group scales -> the block-scaled MMA's
// scale layout, so the matmul can move them with plain TMA tile loads.
//
// Plain layout: s[rows][K/16], one byte per (row, 16-group).
// Packed layout (per 128-row block rb and K = 64 step ks, a 512-byte atom):
//     packed[rb][ks][i][j][t] = s[rb*128 + 32*j + i][4*ks + t]
// for i < 32, j < 4, t < 4: atom line i holds rows i, i+32, i+64, i+96, four
// scale bytes each.  Rows past `rows` (past a group's end) are zero.  This is the layout in which
// one tcgen05.cp 32x128b.warpx4 puts a K = 64 step's scales for 128 rows into
// TMEM.  The rearrangement is pure data movement (HBM-bound).
#pragma once
#include "ptx.cuh"
#include <cstdint>

namespace nvfp4 {
namespace pack {

constexpr int ROWS = 128;  // one row block per CTA
constexpr int KCHUNK = 8;  // K = 64 steps per CTA (32 scale bytes of each row)

// One 128-row block of one K chunk: `src` is the plain scales of the block's
// first row, `valid` how many of its 128 rows exist, `dst` the block's packed
// atoms.  Reads the 32-byte segment of each row (one row per thread, whole
// sectors), transposes through shared memory, and writes the KCHUNK
// consecutive 512-byte atoms [8*kc .. 8*kc+7] as one contiguous 4 KB run.
__device__ __forceinline__ void pack_block(const uint8_t* __restrict__ src, int valid,
                                           uint8_t* __restrict__ dst_block, int groups,
                                           int ksteps, int kc) {
    __shared__ uint32_t tile[ROWS][KCHUNK + 1];  // +1 word: conflict-free column reads
    const int t = threadIdx.x;
    const int ks0 = kc * KCHUNK;
    const int nks = min(KCHUNK, ksteps - ks0);
    const uint8_t* row = src + (long long)t * groups + 4 * ks0;
    if (t < valid && (groups % 16) == 0 && nks == KCHUNK) {
        const uint4 a = *reinterpret_cast<const uint4*>(row);
        const uint4 b = *reinterpret_cast<const uint4*>(row + 16);
        tile[t][0] = a.x; tile[t][1] = a.y; tile[t][2] = a.z; tile[t][3] = a.w;
        tile[t][4] = b.x; tile[t][5] = b.y; tile[t][6] = b.z; tile[t][7] = b.w;
    } else {
#pragma unroll
        for (int w = 0; w < KCHUNK; ++w)
            tile[t][w] = (t < valid && w < nks) ? *reinterpret_cast<const uint32_t*>(row + 4 * w) : 0u;
    }
    __syncthreads();
    uint4* dst = reinterpret_cast<uint4*>(dst_block + (long long)ks0 * 512);
    for (int line = t; line < nks * 32; line += ROWS) {
        const int ksl = line >> 5, i = line & 31;
        dst[line] = make_uint4(tile[i][ksl], tile[i + 32][ksl], tile[i + 64][ksl], tile[i + 96][ksl]);
    }
}

// CTA (rb, kc) packs block rb of a [rows][groups] scale matrix.
__global__ void __launch_bounds__(ROWS)
pack_scales_kernel(const uint8_t* __restrict__ s, uint8_t* __restrict__ out, int rows,
                   int groups, int ksteps) {
    grid_dependents_launch();  // the product that follows may set itself up meanwhile
    const int rb = blockIdx.x;
    pack_block(s + (long long)rb * ROWS * groups, min(ROWS, rows - rb * ROWS),
               out + (long long)rb * ksteps * 512, groups, ksteps, blockIdx.y);
}

// Grouped form: the rows of group g are [row_start[g], row_start[g+1]) and its
// packed blocks start at block block_start[g] (= the sum of ceil(rows/128)
// over the groups before it), so every group begins on a 128-row block.
constexpr int MAX_GROUPS = 256;
struct GroupedPack {
    int groups_n;                      // number of groups
    int row_start[MAX_GROUPS + 1];
    int block_start[MAX_GROUPS + 1];
};

// The map comes from the kernel parameters, or, when gp_dev is not null, from
// device memory (written by the grouped schedule kernel); then the grid is an
// upper bound and CTAs past the last block return.
__global__ void __launch_bounds__(ROWS)
pack_scales_grouped_kernel(const uint8_t* __restrict__ s, uint8_t* __restrict__ out,
                           const __grid_constant__ GroupedPack gp_param,
                           const GroupedPack* __restrict__ gp_dev, int groups, int ksteps) {
    grid_dependents_launch();  // the product that follows may set itself up meanwhile
    const GroupedPack& gp = gp_dev ? *gp_dev : gp_param;
    const int b = blockIdx.x;
    if (b >= gp.block_start[gp.groups_n]) return;
    int lo = 0, hi = gp.groups_n;  // block_start[lo] <= b < block_start[hi]
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (gp.block_start[mid] <= b) lo = mid; else hi = mid;
    }
    const int r0 = gp.row_start[lo] + (b - gp.block_start[lo]) * ROWS;
    pack_block(s + (long long)r0 * groups, min(ROWS, gp.row_start[lo + 1] - r0),
               out + (long long)b * ksteps * 512, groups, ksteps, blockIdx.y);
}

}  // namespace pack
}  // namespace nvfp4
