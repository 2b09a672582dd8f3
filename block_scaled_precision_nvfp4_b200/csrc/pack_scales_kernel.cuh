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

// One thread per 16-byte atom line (i, rb, ks): four 4-byte row slices in,
// 16 bytes out.  Consecutive threads write consecutive lines.
__global__ void pack_scales_kernel(const uint8_t* __restrict__ s, uint8_t* __restrict__ out,
                                   int rows, int groups, int ksteps, long long lines) {
    const long long line = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (line >= lines) return;
    const int i = (int)(line % 32);
    const long long atom = line / 32;
    const int ks = (int)(atom % ksteps);
    const long long rb = atom / ksteps;
    uint32_t w[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const long long r = rb * 128 + 32 * j + i;
        uint32_t v = 0u;
        if (r < rows) {
            const uint8_t* p = s + r * (long long)groups + 4 * ks;
            if ((reinterpret_cast<uintptr_t>(p) & 3u) == 0)
                v = *reinterpret_cast<const uint32_t*>(p);
            else
                v = (uint32_t)p[0] | ((uint32_t)p[1] << 8) | ((uint32_t)p[2] << 16) |
                    ((uint32_t)p[3] << 24);
        }
        w[j] = v;
    }
    reinterpret_cast<uint4*>(out)[line] = make_uint4(w[0], w[1], w[2], w[3]);
}

}  // namespace pack
}  // namespace nvfp4
