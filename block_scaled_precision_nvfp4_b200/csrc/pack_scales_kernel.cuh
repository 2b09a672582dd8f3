// pack_scales_kernel.cuh -- plain E4M3 group scales -> the block-scaled MMA's
// scale layout, so the matmul can move them with plain TMA tile loads.
//
// Plain layout: s[rows][K/16], one byte per (row, 16-group).
// Packed layout (per 128-row block rb and K = 64 step ks, a 512-byte atom):
//     packed[rb][ks][i][j][t] = s[rb*128 + 32*j + i][4*ks + t]
// for i < 32, j < 4, t < 4: atom line i holds rows i, i+32, i+64, i+96, four
// scale bytes each.  Rows past `rows` are zero.  This is the layout in which
// one tcgen05.cp 32x128b.warpx4 puts a K = 64 step's scales for 128 rows into
// TMEM.  The rearrangement is pure data movement (HBM-bound).
#pragma once
#include <cstdint>

namespace nvfp4 {
namespace pack {

constexpr int ROWS = 128;  // one row block per CTA
constexpr int KCHUNK = 8;  // K = 64 steps per CTA (32 scale bytes of each row)

// CTA (rb, kc): reads the 32-byte segment of each of its 128 rows (one row
// per thread, whole sectors), transposes through shared memory, and writes
// the KCHUNK consecutive 512-byte atoms [rb][8*kc .. 8*kc+7] as one contiguous
// 4 KB run.
__global__ void __launch_bounds__(ROWS)
pack_scales_kernel(const uint8_t* __restrict__ s, uint8_t* __restrict__ out, int rows,
                   int groups, int ksteps) {
    __shared__ uint32_t tile[ROWS][KCHUNK + 1];  // +1 word: conflict-free column reads
    const int rb = blockIdx.x, kc = blockIdx.y, t = threadIdx.x;
    const int r = rb * ROWS + t;
    const int ks0 = kc * KCHUNK;
    const int nks = min(KCHUNK, ksteps - ks0);
    const uint8_t* src = s + (long long)r * groups + 4 * ks0;
    if (r < rows && (groups % 16) == 0 && nks == KCHUNK) {
        const uint4 a = *reinterpret_cast<const uint4*>(src);
        const uint4 b = *reinterpret_cast<const uint4*>(src + 16);
        tile[t][0] = a.x; tile[t][1] = a.y; tile[t][2] = a.z; tile[t][3] = a.w;
        tile[t][4] = b.x; tile[t][5] = b.y; tile[t][6] = b.z; tile[t][7] = b.w;
    } else {
#pragma unroll
        for (int w = 0; w < KCHUNK; ++w)
            tile[t][w] = (r < rows && w < nks) ? *reinterpret_cast<const uint32_t*>(src + 4 * w) : 0u;
    }
    __syncthreads();
    uint4* dst = reinterpret_cast<uint4*>(out + ((long long)rb * ksteps + ks0) * 512);
    for (int line = t; line < nks * 32; line += ROWS) {
        const int ksl = line >> 5, i = line & 31;
        dst[line] = make_uint4(tile[i][ksl], tile[i + 32][ksl], tile[i + 64][ksl], tile[i + 96][ksl]);
    }
}

}  // namespace pack
}  // namespace nvfp4
