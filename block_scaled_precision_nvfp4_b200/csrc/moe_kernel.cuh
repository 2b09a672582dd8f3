// moe_kernel.cuh -- the MoE steps around the grouped product (page 2, the
// MegaMoE swap-AB kernel's dispatch and combine around its grouped GEMM):
//
//  * route: (token, slot) pairs with expert ids -> expert offsets and, for
//    every pair, its row in the expert-grouped order.  The order is stable:
//    inside an expert, pairs keep their order p = t*k + j.  Three launches
//    (per-chunk histograms, one scan, per-chunk ranks), deterministic: no
//    atomic touches the outputs.
//  * permute: grouped row r <- token row of the pair that lands on r (a gather
//    of whole rows, one warp per row, 16-byte copies).
//  * combine: Y[t] = BF16( sum_j w[t,j] * Yg[row of (t,j)] ), FP32 in the
//    order j = 0..k-1.
#pragma once
#include <cuda_bf16.h>
#include <cstdint>

#include "ptx.cuh"

namespace nvfp4 {
namespace moe {

constexpr int MAX_EXPERTS = 256;
constexpr int ROUTE_THREADS = 1024;          // one sub-chunk of pairs per pass
constexpr int ROUTE_WARPS = ROUTE_THREADS / 32;
constexpr int MAX_CHUNKS = 128;              // route chunks (one CTA each) at most
constexpr int BAD_EXPERT_ID = 0x10000;       // device error word bit: an id outside [0, E)

// wcnt[w][x] (pairs of warp w for expert x in this sub-chunk) -> run[x] plus the
// pairs of expert x in warps before w; run[x] advances by the sub-chunk's total.
// Warp v takes experts v, v + 32, ...; its lanes scan the 32 warps' counts.
__device__ __forceinline__ void prefix_over_warps(int32_t (&wcnt)[ROUTE_WARPS][MAX_EXPERTS],
                                                  int32_t* run, int E) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int x = warp; x < E; x += ROUTE_WARPS) {
        const int32_t c = wcnt[lane][x];
        int32_t incl = c;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int32_t v = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += v;
        }
        const int32_t base = run[x];
        wcnt[lane][x] = base + incl - c;
        __syncwarp();
        if (lane == 31) run[x] = base + incl;
    }
}

// Pass 1: counts[c][e] = pairs of chunk c routed to expert e.  Chunk c is
// pairs [c*chunk, min((c+1)*chunk, P)).  An id outside [0, E) is left out of
// every expert and recorded in the device error word.
__global__ void __launch_bounds__(ROUTE_THREADS)
route_count_kernel(const int32_t* __restrict__ ids, int P, int E, int chunk,
                   int32_t* __restrict__ counts) {
    __shared__ int32_t h[MAX_EXPERTS];
    for (int e = threadIdx.x; e < E; e += ROUTE_THREADS) h[e] = 0;
    __syncthreads();
    const int p0 = blockIdx.x * chunk, p1 = min(P, p0 + chunk);
    for (int p = p0 + threadIdx.x; p < p1; p += ROUTE_THREADS) {
        const int e = ids[p];
        if (e < 0 || e >= E) {
            atomicOr(&g_device_error, BAD_EXPERT_ID);
        } else {
            atomicAdd(&h[e], 1);
        }
    }
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += ROUTE_THREADS) counts[(size_t)blockIdx.x * E + e] = h[e];
}

// Pass 2 (one CTA): offsets[e] = pairs of experts < e; base[c][e] = offsets[e]
// + pairs of expert e in chunks < c.
__global__ void __launch_bounds__(MAX_EXPERTS)
route_scan_kernel(const int32_t* __restrict__ counts, int C, int E, int32_t* __restrict__ base,
                  int32_t* __restrict__ offsets) {
    __shared__ int32_t tot[MAX_EXPERTS];
    const int e = threadIdx.x;
    int32_t s = 0;
    if (e < E)
        for (int c = 0; c < C; ++c) s += counts[(size_t)c * E + e];
    tot[e] = e < E ? s : 0;
    __syncthreads();
    // exclusive scan over experts (E <= 256, sequential per thread for clarity of order)
    if (e == 0) {
        int32_t run = 0;
        for (int i = 0; i < E; ++i) {
            const int32_t t = tot[i];
            tot[i] = run;
            run += t;
        }
        offsets[E] = run;
    }
    __syncthreads();
    if (e < E) {
        offsets[e] = tot[e];
        int32_t run = tot[e];
        for (int c = 0; c < C; ++c) {
            base[(size_t)c * E + e] = run;
            run += counts[(size_t)c * E + e];
        }
    }
}

// Pass 3: dest[p] = base[c][e] + rank of p among the pairs of chunk c with
// expert e that precede it; src[dest[p]] = p.  A chunk is walked in
// sub-chunks of 1024 pairs; inside one, pairs are ranked by warp, then by lane.
__global__ void __launch_bounds__(ROUTE_THREADS)
route_rank_kernel(const int32_t* __restrict__ ids, int P, int E, int chunk,
                  const int32_t* __restrict__ base, int32_t* __restrict__ dest,
                  int32_t* __restrict__ src) {
    __shared__ int32_t run[MAX_EXPERTS];                    // pairs of e placed so far in this chunk
    __shared__ int32_t wcnt[ROUTE_WARPS][MAX_EXPERTS];      // per warp, per expert, this sub-chunk
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int e = threadIdx.x; e < E; e += ROUTE_THREADS) run[e] = base[(size_t)blockIdx.x * E + e];
    const int p0 = blockIdx.x * chunk, p1 = min(P, p0 + chunk);
    for (int s0 = p0; s0 < p1; s0 += ROUTE_THREADS) {
        for (int i = threadIdx.x; i < ROUTE_WARPS * E; i += ROUTE_THREADS) wcnt[i / E][i % E] = 0;
        __syncthreads();
        const int p = s0 + threadIdx.x;
        const bool live = p < p1;
        int e = live ? ids[p] : -1;
        if (e < 0 || e >= E) e = -1;  // counted as bad in pass 1; not placed
        // lanes of this warp with the same expert, and this lane's rank among them
        const unsigned peers = __match_any_sync(0xffffffffu, e);
        const int lrank = __popc(peers & ((1u << lane) - 1u));
        if (e >= 0 && lrank == 0) wcnt[warp][e] = __popc(peers);
        __syncthreads();
        // exclusive prefix over warps, per expert; then advance the running counts
        prefix_over_warps(wcnt, run, E);
        __syncthreads();
        if (e >= 0) {
            const int32_t d = wcnt[warp][e] + lrank;
            dest[p] = d;
            src[d] = p;
        }
        __syncthreads();
    }
}

// The three passes in one CTA, for up to SMALL_PAIRS pairs (one launch, no memsets):
// histogram, scan, then ranks by sub-chunks of 1024 pairs in order.  Pairs with an
// out-of-range id get dest = -1; grouped rows past the last placed one get src = -1.
constexpr int SMALL_PAIRS = 65536;

__global__ void __launch_bounds__(ROUTE_THREADS)
route_small_kernel(const int32_t* __restrict__ ids, int P, int E, int32_t* __restrict__ offsets,
                   int32_t* __restrict__ dest, int32_t* __restrict__ src) {
    __shared__ int32_t run[MAX_EXPERTS];
    __shared__ int32_t wcnt[ROUTE_WARPS][MAX_EXPERTS];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int e = threadIdx.x; e < E; e += ROUTE_THREADS) run[e] = 0;
    __syncthreads();
    for (int p0 = 0; p0 < P; p0 += ROUTE_THREADS) {  // whole warps: the match needs all lanes
        const int p = p0 + threadIdx.x;
        int e = p < P ? ids[p] : -1;
        if (p < P && (e < 0 || e >= E)) {
            atomicOr(&g_device_error, BAD_EXPERT_ID);
            dest[p] = -1;
        }
        if (e < 0 || e >= E) e = -1;
        const unsigned peers = __match_any_sync(0xffffffffu, e);  // one atomic per expert per warp
        if (e >= 0 && (peers & ((1u << lane) - 1u)) == 0) atomicAdd(&run[e], __popc(peers));
    }
    __syncthreads();
    if (threadIdx.x == 0) {  // exclusive scan over experts, in expert order
        int32_t acc = 0;
        for (int e = 0; e < E; ++e) {
            const int32_t c = run[e];
            run[e] = acc;
            offsets[e] = acc;
            acc += c;
        }
        offsets[E] = acc;
        wcnt[0][0] = acc;  // placed pairs, read below before the first sub-chunk reset
    }
    __syncthreads();
    const int placed = wcnt[0][0];
    for (int r = placed + threadIdx.x; r < P; r += ROUTE_THREADS) src[r] = -1;
    for (int s0 = 0; s0 < P; s0 += ROUTE_THREADS) {
        __syncthreads();
        for (int i = threadIdx.x; i < ROUTE_WARPS * E; i += ROUTE_THREADS) wcnt[i / E][i % E] = 0;
        __syncthreads();
        const int p = s0 + threadIdx.x;
        int e = p < P ? ids[p] : -1;
        if (e < 0 || e >= E) e = -1;
        const unsigned peers = __match_any_sync(0xffffffffu, e);
        const int lrank = __popc(peers & ((1u << lane) - 1u));
        if (e >= 0 && lrank == 0) wcnt[warp][e] = __popc(peers);
        __syncthreads();
        prefix_over_warps(wcnt, run, E);
        __syncthreads();
        if (e >= 0) {
            const int32_t d = wcnt[warp][e] + lrank;
            dest[p] = d;
            src[d] = p;
        }
    }
}

// Grouped row r <- row src[r] / k of `in` (row_bytes bytes, a multiple of 16).
// One warp per row.  A source outside [0, in_rows) (a pair whose id was out of
// range, so nothing was placed on r) leaves the row untouched.
__global__ void __launch_bounds__(256)
permute_rows_kernel(const uint8_t* __restrict__ in, size_t row_bytes, int in_rows, int rows, int k,
                    const int32_t* __restrict__ src, uint8_t* __restrict__ out) {
    const int r = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
    if (r >= rows) return;
    const int sp = src[r];
    if (sp < 0 || sp / k >= in_rows) return;
    const uint4* s = reinterpret_cast<const uint4*>(in + (size_t)(sp / k) * row_bytes);
    uint4* d = reinterpret_cast<uint4*>(out + (size_t)r * row_bytes);
    const size_t n = row_bytes / 16;
    for (size_t i = lane; i < n; i += 32) d[i] = __ldg(s + i);
}

// Y[t][n] = BF16( sum_j w[t][j] * Yg[dest[t*k+j]][n] ) with FP32 FMAs in j order
// (w == nullptr: weight 1).  Eight columns per thread; N % 8 == 0.  A row index
// outside [0, rows) contributes nothing.
__global__ void __launch_bounds__(256)
combine_kernel(const __nv_bfloat16* __restrict__ Yg, int rows, const int32_t* __restrict__ dest,
               const float* __restrict__ w, int T, int k, int N, __nv_bfloat16* __restrict__ Y) {
    const int c8 = blockIdx.x * 256 + threadIdx.x;  // group of 8 columns
    if (c8 * 8 >= N) return;
    for (int t = blockIdx.y; t < T; t += gridDim.y) {
        float acc[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[i] = 0.f;
        for (int j = 0; j < k; ++j) {
            const int r = dest[(size_t)t * k + j];
            if (r < 0 || r >= rows) continue;
            const float wj = w ? w[(size_t)t * k + j] : 1.0f;
            const uint4 v = __ldg(reinterpret_cast<const uint4*>(Yg + (size_t)r * N) + c8);
            const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                acc[2 * i] = fmaf(wj, __uint_as_float(u[i] << 16), acc[2 * i]);
                acc[2 * i + 1] = fmaf(wj, __uint_as_float(u[i] & 0xFFFF0000u), acc[2 * i + 1]);
            }
        }
        uint32_t o[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            __nv_bfloat162 h = __floats2bfloat162_rn(acc[2 * i], acc[2 * i + 1]);
            o[i] = *reinterpret_cast<uint32_t*>(&h);
        }
        reinterpret_cast<uint4*>(Y + (size_t)t * N)[c8] = make_uint4(o[0], o[1], o[2], o[3]);
    }
}

}  // namespace moe
}  // namespace nvfp4
