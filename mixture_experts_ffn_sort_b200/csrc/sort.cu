// sort.cu -- stable sort of the routes by expert (moe_sort).
//
// The step of the Nemotron-H sorted prefill path that orders tokens by expert
// (spark_model/layers/nemotron_moe.rs, `prefill` step 5), the NKI Permute
// Routed Tokens kernel, and the sort with an inverse route map that the aiter
// gfx950 prefill PR reuses.  A counting sort in three passes:
//   1. each chunk of routes builds an expert histogram;
//   2. an exclusive scan in (expert, chunk) order gives every chunk the first
//      sorted position of each of its experts, and the per-expert offsets;
//   3. each chunk walks its routes in order and scatters them, ranking equal
//      experts within a 32-route step with __match_any_sync.
// Order within an expert is therefore route order: the result is unique and
// deterministic.  Small inputs run all three passes in one thread block;
// larger ones give each tile of kSortChunk routes a thread block (8 warps of
// 256 routes) and scan per expert over the tiles.
#include <algorithm>

#include "device_common.cuh"
#include "launch.h"

namespace moe {

namespace {

__device__ __forceinline__ uint32_t lanemask_lt() {
    uint32_t m;
    asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
    return m;
}

// Scatter the 32 routes r0 .. r0 + 31 of a warp (lane's route r0 + lane, its
// expert e, `in` false past the chunk's end) given the chunk's start
// positions `cursor[e * stride]` (shared memory, advanced in place): equal
// experts are ranked by lane with __match_any_sync.
__device__ __forceinline__ void scatter32(long r0, bool in, int e, int E, int32_t* cursor,
                                          int32_t* __restrict__ sorted_route, int32_t* __restrict__ inv_route,
                                          int stride) {
    const int lane = threadIdx.x & 31;
    const uint32_t lt = lanemask_lt();
    const long r = r0 + lane;
    const bool ok = in && e >= 0 && e < E;
    const uint32_t peers = __match_any_sync(0xffffffffu, ok ? e : (E + lane));
    int32_t pos = 0;
    if (ok) pos = cursor[e * stride] + __popc(peers & lt);
    __syncwarp();
    // The highest lane of each group of equal experts advances the cursor.
    if (ok && (peers >> lane) == 1u) cursor[e * stride] += __popc(peers);
    __syncwarp();
    if (ok) {
        sorted_route[pos] = static_cast<int32_t>(r);
        inv_route[r] = pos;
    } else if (in) {
        inv_route[r] = -1;
    }
}

// Scatter one warp-chunk [r_begin, r_end) given the chunk's start positions
// `cursor[e * stride]` (shared memory, advanced in place).
__device__ __forceinline__ void scatter_chunk(const int32_t* __restrict__ ids, long r_begin,
                                              long r_end, int E, int32_t* cursor,
                                              int32_t* __restrict__ sorted_route,
                                              int32_t* __restrict__ inv_route, int stride = 1) {
    const int lane = threadIdx.x & 31;
    for (long r0 = r_begin; r0 < r_end; r0 += 32) {
        const long r = r0 + lane;
        const bool in = r < r_end;
        scatter32(r0, in, in ? ids[r] : -1, E, cursor, sorted_route, inv_route, stride);
    }
}

// Count one warp-chunk into hist[e * stride] (shared memory, zeroed by the
// caller).  Returns true if an id outside [0, E) was seen.
__device__ __forceinline__ bool count_chunk(const int32_t* __restrict__ ids, long r_begin,
                                            long r_end, int E, int32_t* hist, int stride = 1) {
    const int lane = threadIdx.x & 31;
    bool bad = false;
    for (long r = r_begin + lane; r < r_end; r += 32) {
        const int e = ids[r];
        if (e >= 0 && e < E)
            atomicAdd(&hist[e * stride], 1);
        else
            bad = true;
    }
    return __any_sync(0xffffffffu, bad);
}

// Block-wide exclusive scan of one int per thread; returns the prefix and
// writes the block total to *total.  blockDim.x is a multiple of 32, <= 1024.
__device__ int block_exclusive_scan(int v, int* scratch /*[32]*/, int* total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int nw = blockDim.x >> 5;
    int x = v;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, x, off);
        if (lane >= off) x += y;
    }
    if (lane == 31) scratch[warp] = x;
    __syncthreads();
    if (warp == 0) {
        int s = lane < nw ? scratch[lane] : 0;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, s, off);
            if (lane >= off) s += y;
        }
        scratch[lane] = s;  // inclusive warp totals
    }
    __syncthreads();
    const int warp_prefix = warp ? scratch[warp - 1] : 0;
    *total = scratch[nw - 1];
    __syncthreads();
    return warp_prefix + x - v;
}

// ---------------------------------------------------------------- small: one block

// smem: hist[E][NW] ints (expert-major, so the scan in (expert, warp) order
// reads it contiguously), then 32 ints of scan scratch.  PER > 0: each lane
// keeps its PER ids of the warp's chunk (routes rb + lane + 32 i) in registers
// from one round of loads, for the count and the scatter alike (a warp's chunk
// is at most 32 PER routes); PER = 0 reads them from global memory twice.
template <int PER>
__global__ void __launch_bounds__(1024) sort_small_kernel(const int32_t* __restrict__ ids, long R,
                                                          int E, int32_t* __restrict__ offsets,
                                                          int32_t* __restrict__ sorted_route,
                                                          int32_t* __restrict__ inv_route,
                                                          int32_t* status) {
    extern __shared__ int32_t sm[];
    const int NW = blockDim.x >> 5;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    int32_t* hist = sm;                      // [E][NW]
    int32_t* scratch = sm + NW * E;          // [32]
    const long chunk = ((R + NW - 1) / NW + 31) / 32 * 32;
    const long rb = min(R, warp * chunk), re = min(R, rb + chunk);
    int myid[PER > 0 ? PER : 1];
    if constexpr (PER > 0) {
#pragma unroll
        for (int i = 0; i < PER; ++i) {
            const long r = rb + lane + 32 * i;
            myid[i] = r < re ? __ldg(ids + r) : -1;
        }
    }
    for (int i = threadIdx.x; i < NW * E; i += blockDim.x) hist[i] = 0;
    __syncthreads();

    bool bad;
    if constexpr (PER > 0) {
        bool b = false;
#pragma unroll
        for (int i = 0; i < PER; ++i) {
            if (rb + lane + 32 * i >= re) continue;
            const int e = myid[i];
            if (e >= 0 && e < E)
                atomicAdd(&hist[e * NW + warp], 1);
            else
                b = true;
        }
        bad = __any_sync(0xffffffffu, b);
    } else {
        bad = count_chunk(ids, rb, re, E, hist + warp, NW);
    }
    if (bad && lane == 0) report_status(status, MOE_STATUS_BAD_ID);
    __syncthreads();

    // Exclusive scan over (expert, warp) order; each thread owns a contiguous
    // run of that order.
    const int N = NW * E;
    const int per = (N + blockDim.x - 1) / blockDim.x;
    const int i0 = min(N, static_cast<int>(threadIdx.x) * per), i1 = min(N, i0 + per);
    int s = 0;
    for (int i = i0; i < i1; ++i) s += hist[i];
    int total;
    int prefix = block_exclusive_scan(s, scratch, &total);
    for (int i = i0; i < i1; ++i) {
        const int c = hist[i];
        if (i % NW == 0) offsets[i / NW] = prefix;
        hist[i] = prefix;
        prefix += c;
    }
    if (threadIdx.x == 0) offsets[E] = total;
    for (long p = total + threadIdx.x; p < R; p += blockDim.x) sorted_route[p] = -1;
    __syncthreads();

    if constexpr (PER > 0) {
#pragma unroll
        for (int i = 0; i < PER; ++i) {
            const long r0 = rb + 32 * i;
            if (r0 >= re) break;  // warp-uniform
            scatter32(r0, r0 + lane < re, myid[i], E, hist + warp, sorted_route, inv_route, NW);
        }
    } else {
        scatter_chunk(ids, rb, re, E, hist + warp, sorted_route, inv_route, NW);
    }
}

// ---------------------------------------------------------------- large: three kernels
//
// Tiles of kSortChunk routes, one thread block each; the block's 8 warps take
// 256 consecutive routes apiece.  The workspace holds one counter per
// (tile, expert), tile-major.

constexpr int kSortWarpsPerBlock = 8;
constexpr int kSortWarpRoutes = kSortChunk / kSortWarpsPerBlock;

// Per-warp expert histograms of tile b into hist[warp][E] (shared memory).
// Returns (in every thread of the warp) whether an id outside [0, E) was seen.
__device__ __forceinline__ bool count_tile(const int32_t* __restrict__ ids, long R, int E, int32_t* hist) {
    const int warp = threadIdx.x >> 5;
    for (int i = threadIdx.x; i < kSortWarpsPerBlock * E; i += blockDim.x) hist[i] = 0;
    __syncthreads();
    const long rb = static_cast<long>(blockIdx.x) * kSortChunk + static_cast<long>(warp) * kSortWarpRoutes;
    const bool bad = count_chunk(ids, min(R, rb), min(R, rb + kSortWarpRoutes), E, hist + warp * E);
    __syncthreads();
    return bad;
}

// counts[b * E + e] = routes of tile b with expert e.
__global__ void __launch_bounds__(kSortWarpsPerBlock * 32)
    sort_count_kernel(const int32_t* __restrict__ ids, long R, int E, int32_t* __restrict__ counts,
                      int32_t* status) {
    extern __shared__ int32_t sm[];
    if (count_tile(ids, R, E, sm) && (threadIdx.x & 31) == 0) report_status(status, MOE_STATUS_BAD_ID);
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        int c = 0;
#pragma unroll
        for (int w = 0; w < kSortWarpsPerBlock; ++w) c += sm[w * E + e];
        counts[static_cast<size_t>(blockIdx.x) * E + e] = c;
    }
}

// One thread per expert (E <= blockDim.x): the expert's total over the tiles,
// offsets = exclusive scan of the totals, and counts[b * E + e] replaced by
// tile b's first sorted position of expert e.
__global__ void __launch_bounds__(1024)
    sort_scan_kernel(int32_t* __restrict__ counts, int E, int ntiles, long R, int32_t* __restrict__ offsets,
                     int32_t* __restrict__ sorted_route) {
    __shared__ int scratch[32];
    const int e = threadIdx.x;
    int tot = 0;
    if (e < E) {
        int part[8] = {0, 0, 0, 0, 0, 0, 0, 0};
        int b = 0;
        for (; b + 8 <= ntiles; b += 8)
#pragma unroll
            for (int k = 0; k < 8; ++k) part[k] += counts[static_cast<size_t>(b + k) * E + e];
        for (; b < ntiles; ++b) part[0] += counts[static_cast<size_t>(b) * E + e];
#pragma unroll
        for (int k = 0; k < 8; ++k) tot += part[k];
    }
    int total;
    int run = block_exclusive_scan(tot, scratch, &total);
    if (e < E) {
        offsets[e] = run;
        for (int b = 0; b < ntiles; ++b) {
            const size_t i = static_cast<size_t>(b) * E + e;
            const int c = counts[i];
            counts[i] = run;
            run += c;
        }
    }
    if (threadIdx.x == 0) offsets[E] = total;
    for (long p = total + threadIdx.x; p < R; p += blockDim.x) sorted_route[p] = -1;
}

// Tile b: recount per warp, turn the counts into per-warp cursors starting at
// the tile's base positions, and scatter each warp's routes in order.
__global__ void __launch_bounds__(kSortWarpsPerBlock * 32)
    sort_scatter_kernel(const int32_t* __restrict__ ids, long R, int E, const int32_t* __restrict__ base,
                        int32_t* __restrict__ sorted_route, int32_t* __restrict__ inv_route) {
    extern __shared__ int32_t sm[];
    count_tile(ids, R, E, sm);
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        int run = base[static_cast<size_t>(blockIdx.x) * E + e];
#pragma unroll
        for (int w = 0; w < kSortWarpsPerBlock; ++w) {
            const int c = sm[w * E + e];
            sm[w * E + e] = run;
            run += c;
        }
    }
    __syncthreads();
    const int warp = threadIdx.x >> 5;
    const long rb = static_cast<long>(blockIdx.x) * kSortChunk + static_cast<long>(warp) * kSortWarpRoutes;
    scatter_chunk(ids, min(R, rb), min(R, rb + kSortWarpRoutes), E, sm + warp * E, sorted_route, inv_route);
}

int small_sort_warps(int E) {
    int nw = 32;
    while (nw > 1 && (static_cast<long>(nw) * E + 32) * 4 > 48 * 1024) nw >>= 1;
    return nw;
}

}  // namespace

size_t sort_workspace_bytes(long R, int E) {
    if (R <= kSortSmallMaxRoutes) return 0;
    const long nchunks = (R + kSortChunk - 1) / kSortChunk;
    return static_cast<size_t>(nchunks) * E * sizeof(int32_t);
}

cudaError_t launch_sort(const int32_t* ids, long R, int E, int32_t* offsets, int32_t* sorted_route,
                        int32_t* inv_route, void* ws, int32_t* status, cudaStream_t stream) {
    if (R <= kSortSmallMaxRoutes) {
        // A warp per 128 routes (at least four warps, and no more than 32-route
        // slices), up to what shared memory holds: the per-warp histograms and
        // their scan grow with the warps, so fewer, fuller warps win until the
        // block is too narrow to hide its load latency.
        const long want = std::min<long>((R + 31) / 32, std::max<long>(4, (R + 127) / 128));
        const int nw = static_cast<int>(std::min<long>(small_sort_warps(E), std::max<long>(1, want)));
        const size_t smem = (static_cast<size_t>(nw) * E + 32) * sizeof(int32_t);
        const long per = ((R + nw - 1) / nw + 31) / 32;  // ids per lane of a warp's chunk
#define MOE_SORT_SMALL(P) \
    sort_small_kernel<P><<<1, nw * 32, smem, stream>>>(ids, R, E, offsets, sorted_route, inv_route, status)
        if (per <= 1)
            MOE_SORT_SMALL(1);
        else if (per <= 2)
            MOE_SORT_SMALL(2);
        else if (per <= 4)
            MOE_SORT_SMALL(4);
        else if (per <= 8)
            MOE_SORT_SMALL(8);
        else if (per <= 16)
            MOE_SORT_SMALL(16);
        else
            MOE_SORT_SMALL(0);
#undef MOE_SORT_SMALL
        return cudaGetLastError();
    }
    const int ntiles = static_cast<int>((R + kSortChunk - 1) / kSortChunk);
    int32_t* counts = static_cast<int32_t*>(ws);
    const size_t smem = static_cast<size_t>(kSortWarpsPerBlock) * E * sizeof(int32_t);
    sort_count_kernel<<<ntiles, kSortWarpsPerBlock * 32, smem, stream>>>(ids, R, E, counts, status);
    sort_scan_kernel<<<1, 1024, 0, stream>>>(counts, E, ntiles, R, offsets, sorted_route);
    sort_scatter_kernel<<<ntiles, kSortWarpsPerBlock * 32, smem, stream>>>(ids, R, E, counts, sorted_route,
                                                                          inv_route);
    return cudaGetLastError();
}

}  // namespace moe
