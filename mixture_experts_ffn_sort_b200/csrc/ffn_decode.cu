// ffn_decode.cu -- expert FFN for the memory-bound regime (moe_expert_ffn,
// MOE_MODE_DECODE).
//
// The computation of the FP8 W8A16 MoE decode kernel
// (dstair/gated-deltanet-nki-trainium, "FP8 MoE decode kernel"): gate/up GEMM
// -> SwiGLU -> down GEMM -> affinity scale, with E4M3FN weights and one fp32
// scale per 128x128 block decoded to BF16 tile by tile; the row order is the
// expert-sorted order of the Nemotron-H sorted path, read from device-side
// offsets (no host sync).
//
// Design (B200):
//  * One CTA owns a slice of ONE expert's weights: 32 intermediate features
//    (gate and up rows) in the gate/up kernel, 64 output features in the down
//    kernel.  CTAs whose expert received no route exit at once, so only the
//    touched experts' weights are read, each exactly once per token group.
//  * A producer warp streams the slice from HBM with TMA in stages of 128
//    reduction columns (one scale block), 128-byte swizzled, through a
//    6-deep shared-memory ring (mbarrier full/empty pairs, bounded waits).
//  * Eight consumer warps load the FP8 bytes with ldmatrix, decode them to
//    BF16 in registers (exact), and run mma.sync m16n8k16 against the
//    expert's token rows staged in shared memory.  The reduction columns are
//    permuted identically on both operands so that one ldmatrix register (4
//    codes of one row) feeds one A-fragment pair.  Each 128-wide fp32 partial
//    sum is multiplied by its block scale.
//  * In the gate/up tile the 16 MMA rows are 8 gate + 8 up rows of the same
//    features, so SwiGLU is thread-local in the epilogue.
//  * Two warps share each 16-row tile, each taking half of every stage's
//    columns; their sums meet in shared memory for a coalesced epilogue.
#include <algorithm>

#include "device_common.cuh"
#include "launch.h"

namespace moe {

namespace {

constexpr int kStages = 6;
constexpr int kConsumerWarps = 8;
constexpr int kThreads = (kConsumerWarps + 1) * 32;
constexpr int kStageBytes = 8192;  // 64 rows x 128 bytes
constexpr int kGateUpRows = 32;    // intermediate features per gate/up CTA
constexpr int kDownRows = 64;      // output features per down CTA
constexpr int kRedGU = 36;         // padded token stride (floats) of the gate/up reduction tile
constexpr int kRedDn = 68;         // same for the down tile

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
    return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

__device__ __forceinline__ uint2 lds64(uint32_t addr) {
    uint2 v;
    asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(addr));
    return v;
}

__device__ __forceinline__ uint4 ldg_nc_v4(const void* p) {
    uint4 v;
    asm volatile("ld.global.nc.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

// Row range [p0, p0 + n) of expert e.  Returns false (BAD_MAP) for corrupt offsets.
__device__ __forceinline__ bool expert_rows(const FfnArgs& a, int e, long& p0, long& n) {
    if (a.identity) {
        p0 = 0;
        n = a.T;
        return true;
    }
    const long R = static_cast<long>(a.T) * a.K;
    const long b = a.offsets[e], f = a.offsets[e + 1];
    if (b < 0 || f < b || f > R) return false;
    p0 = b;
    n = f - b;
    return true;
}

// Token of sorted row p, -1 if the route map entry is out of range.
__device__ __forceinline__ int row_token(const FfnArgs& a, long p) {
    if (a.identity) return static_cast<int>(p);
    const int r = a.sorted_route[p];
    const long R = static_cast<long>(a.T) * a.K;
    if (r < 0 || r >= R) return -1;
    return r / a.K;
}

// Producer: stream `total` stages (cycling the slice's KB column blocks) into the ring.
__device__ __forceinline__ void produce(const CUtensorMap* m0, const CUtensorMap* m1, int row,
                                        int KB, long total, uint8_t* ring, uint64_t* full,
                                        uint64_t* empty, uint32_t bytes_each, volatile int* abort_flag,
                                        int32_t* status) {
    tma_prefetch_desc(m0);
    if (m1) tma_prefetch_desc(m1);
    for (long it = 0; it < total; ++it) {
        const int s = static_cast<int>(it % kStages);
        if (it >= kStages &&
            !mbar_wait_or_abort(&empty[s], static_cast<uint32_t>((it / kStages - 1) & 1), abort_flag, status))
            return;
        mbar_arrive_expect_tx(&full[s], m1 ? 2 * bytes_each : bytes_each);
        const int kb = static_cast<int>(it % KB);
        uint8_t* dst = ring + static_cast<size_t>(s) * kStageBytes;
        tma_load_2d(dst, m0, &full[s], kb * 128, row);
        if (m1) tma_load_2d(dst + bytes_each, m1, &full[s], kb * 128, row);
    }
}

// One stage of one warp: 16 rows (two 8-row halves r_lo / r_hi from the
// ldmatrix register pairs) x 64 columns (chunks j0..j0+3) against NT token tiles.
template <int NT>
__device__ __forceinline__ void stage_mma(uint32_t stage_base, uint32_t lm_off0, uint32_t lm_off1,
                                          uint32_t b_base, int xstride, int b_col_bytes,
                                          float (&part)[NT][4]) {
#pragma unroll
    for (int q = 0; q < 2; ++q) {
        uint32_t r0, r1, r2, r3;
        ldmatrix_x4(stage_base + (q ? lm_off1 : lm_off0), r0, r1, r2, r3);
        uint32_t lo0, hi0, lo1, hi1;
        e4m3x4_to_bf16(r0, lo0, hi0);
        e4m3x4_to_bf16(r1, lo1, hi1);
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            const uint2 b = lds64(b_base + nt * 8 * xstride + b_col_bytes + (2 * q) * 32);
            mma_bf16_16816(part[nt], lo0, lo1, hi0, hi1, b.x, b.y);
        }
        e4m3x4_to_bf16(r2, lo0, hi0);
        e4m3x4_to_bf16(r3, lo1, hi1);
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            const uint2 b = lds64(b_base + nt * 8 * xstride + b_col_bytes + (2 * q + 1) * 32);
            mma_bf16_16816(part[nt], lo0, lo1, hi0, hi1, b.x, b.y);
        }
    }
}

// ------------------------------------------------------------------ gate/up + SwiGLU

template <int NT>
__global__ void __launch_bounds__(kThreads, 1)
    gateup_decode_kernel(const __grid_constant__ CUtensorMap tm_gate,
                         const __grid_constant__ CUtensorMap tm_up, const FfnArgs a) {
    constexpr int NG = 8 * NT;  // tokens per group
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = align1024(smem_raw);
    const int e = blockIdx.y;
    const int H = a.H, I = a.ex.inter;
    const int i0 = blockIdx.x * kGateUpRows;
    long p0, n;
    if (!expert_rows(a, e, p0, n)) {
        if (threadIdx.x == 0) report_status(a.status, MOE_STATUS_BAD_MAP);
        return;
    }
    if (n == 0) return;
    const int KB = H / 128;
    const int groups = static_cast<int>((n + NG - 1) / NG);
    const int xstride = 2 * H + 32;

    uint8_t* ring = smem;
    uint8_t* xs = ring + kStages * kStageBytes;
    float* red = reinterpret_cast<float*>(xs + NG * xstride);  // [2 halves][gate, up][NG][kRedGU]
    int* tok = reinterpret_cast<int*>(red + 4 * NG * kRedGU);
    uint64_t* full = reinterpret_cast<uint64_t*>(tok + NG + (NG & 1));
    uint64_t* empty = full + kStages;
    volatile int* abort_flag = reinterpret_cast<volatile int*>(empty + kStages);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kConsumerWarps);
        }
        *abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();

    if (warp == kConsumerWarps) {
        if (lane == 0)
            produce(&tm_gate, &tm_up, e * I + i0, KB, static_cast<long>(groups) * KB, ring, full,
                    empty, kStageBytes / 2, abort_flag, a.status);
        return;
    }

    const int u = warp & 3, hh = warp >> 2;  // 16-row tile (8 gate + 8 up), column half
    const int g = lane >> 2, c = lane & 3;
    const int mi = lane >> 3, rr = lane & 7;
    const uint32_t lm_tile = (mi & 1) ? kStageBytes / 2 : 0;  // gate / up sub-tile
    const uint32_t lm_off0 = lm_tile + sw128_offset(8 * u + rr, 4 * hh + (mi >> 1));
    const uint32_t lm_off1 = lm_tile + sw128_offset(8 * u + rr, 4 * hh + 2 + (mi >> 1));
    const uint32_t ring_u32 = smem_u32(ring);
    const uint32_t b_base = smem_u32(xs) + g * xstride + 4 * c * 2 + 4 * hh * 32;
    const size_t sblk = (static_cast<size_t>(e) * (I / 128) + i0 / 128) * KB;
    const float* sg = a.ex.s_gate + sblk;
    const float* su = a.ex.s_up + sblk;

    long it = 0;
    for (int grp = 0; grp < groups; ++grp) {
        const long gp0 = p0 + static_cast<long>(grp) * NG;
        const int gn = static_cast<int>(min(static_cast<long>(NG), n - static_cast<long>(grp) * NG));
        if (threadIdx.x < NG) {
            int t = -1;
            if (static_cast<int>(threadIdx.x) < gn) {
                t = row_token(a, gp0 + threadIdx.x);
                if (t < 0) report_status(a.status, MOE_STATUS_BAD_MAP);
            }
            tok[threadIdx.x] = t;
        }
        named_barrier_sync(1, kConsumerWarps * 32);
        const int vpr = H / 8;  // 16-byte vectors per row
        for (int v = threadIdx.x; v < NG * vpr; v += kConsumerWarps * 32) {
            const int q = v / vpr, col = v - q * vpr;
            const int t = tok[q];
            uint4 val = make_uint4(0, 0, 0, 0);
            if (t >= 0) val = ldg_nc_v4(a.x + static_cast<size_t>(t) * H + col * 8);
            *reinterpret_cast<uint4*>(xs + q * xstride + col * 16) = val;
        }
        named_barrier_sync(1, kConsumerWarps * 32);

        float acc[NT][4];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.f;
        for (int kb = 0; kb < KB; ++kb, ++it) {
            const int s = static_cast<int>(it % kStages);
            float part[NT][4];
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) part[nt][0] = part[nt][1] = part[nt][2] = part[nt][3] = 0.f;
            if (mbar_wait_or_abort(&full[s], static_cast<uint32_t>((it / kStages) & 1), abort_flag, a.status)) {
                stage_mma<NT>(ring_u32 + s * kStageBytes, lm_off0, lm_off1, b_base, xstride, kb * 256, part);
                __syncwarp();
                if (lane == 0) mbar_arrive(&empty[s]);
            }
            const float gs = __ldg(sg + kb), us = __ldg(su + kb);
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                acc[nt][0] = fmaf(part[nt][0], gs, acc[nt][0]);
                acc[nt][1] = fmaf(part[nt][1], gs, acc[nt][1]);
                acc[nt][2] = fmaf(part[nt][2], us, acc[nt][2]);
                acc[nt][3] = fmaf(part[nt][3], us, acc[nt][3]);
            }
        }
        // Partial sums of this column half -> shared memory.
        float* rg = red + (hh * 2 + 0) * NG * kRedGU;
        float* ru = red + (hh * 2 + 1) * NG * kRedGU;
        const int il = 8 * u + g;
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            const int t0 = nt * 8 + 2 * c;
            rg[t0 * kRedGU + il] = acc[nt][0];
            rg[(t0 + 1) * kRedGU + il] = acc[nt][1];
            ru[t0 * kRedGU + il] = acc[nt][2];
            ru[(t0 + 1) * kRedGU + il] = acc[nt][3];
        }
        named_barrier_sync(1, kConsumerWarps * 32);
        // SwiGLU and a coalesced bf16 store of h[row, i0 .. i0+31].
        for (int v = threadIdx.x; v < NG * 4; v += kConsumerWarps * 32) {
            const int q = v >> 2, ch = v & 3;
            if (q < gn && tok[q] >= 0) {
                const float* g0 = red + (0 * NG + q) * kRedGU + ch * 8;
                const float* u0 = red + (1 * NG + q) * kRedGU + ch * 8;
                const float* g1 = red + (2 * NG + q) * kRedGU + ch * 8;
                const float* u1 = red + (3 * NG + q) * kRedGU + ch * 8;
                uint32_t pk[4];
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const float ga = g0[2 * k] + g1[2 * k], gb = g0[2 * k + 1] + g1[2 * k + 1];
                    const float ua = u0[2 * k] + u1[2 * k], ub = u0[2 * k + 1] + u1[2 * k + 1];
                    pk[k] = pack_bf16x2(silu_f32(ga) * ua, silu_f32(gb) * ub);
                }
                *reinterpret_cast<uint4*>(a.h + static_cast<size_t>(gp0 + q) * I + i0 + ch * 8) =
                    make_uint4(pk[0], pk[1], pk[2], pk[3]);
            }
        }
        named_barrier_sync(1, kConsumerWarps * 32);
    }
}

// ------------------------------------------------------------------ down + affinity

template <int NT>
__global__ void __launch_bounds__(kThreads, 1)
    down_decode_kernel(const __grid_constant__ CUtensorMap tm_down, const FfnArgs a) {
    constexpr int NG = 8 * NT;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = align1024(smem_raw);
    const int e = blockIdx.y;
    const int H = a.H, I = a.ex.inter;
    const int n0 = blockIdx.x * kDownRows;
    long p0, n;
    if (!expert_rows(a, e, p0, n)) {
        if (threadIdx.x == 0) report_status(a.status, MOE_STATUS_BAD_MAP);
        return;
    }
    if (n == 0) return;
    const int KB = I / 128;
    const int groups = static_cast<int>((n + NG - 1) / NG);
    const int hstride = 2 * I + 32;

    uint8_t* ring = smem;
    uint8_t* hs = ring + kStages * kStageBytes;
    float* red = reinterpret_cast<float*>(hs + NG * hstride);  // [2 halves][NG][kRedDn]
    float* wr = red + 2 * NG * kRedDn;                         // [NG] route weights
    int* tok = reinterpret_cast<int*>(wr + NG);
    uint64_t* full = reinterpret_cast<uint64_t*>(tok + NG + (NG & 1));
    uint64_t* empty = full + kStages;
    volatile int* abort_flag = reinterpret_cast<volatile int*>(empty + kStages);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kConsumerWarps);
        }
        *abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();

    if (warp == kConsumerWarps) {
        if (lane == 0)
            produce(&tm_down, nullptr, e * H + n0, KB, static_cast<long>(groups) * KB, ring, full,
                    empty, kStageBytes, abort_flag, a.status);
        return;
    }

    const int mt = warp & 3, hh = warp >> 2;
    const int g = lane >> 2, c = lane & 3;
    const int mi = lane >> 3, rr = lane & 7;
    const int lm_row = 16 * mt + ((mi & 1) ? 8 : 0) + rr;
    const uint32_t lm_off0 = sw128_offset(lm_row, 4 * hh + (mi >> 1));
    const uint32_t lm_off1 = sw128_offset(lm_row, 4 * hh + 2 + (mi >> 1));
    const uint32_t ring_u32 = smem_u32(ring);
    const uint32_t b_base = smem_u32(hs) + g * hstride + 4 * c * 2 + 4 * hh * 32;
    const float* sd = a.ex.s_down + (static_cast<size_t>(e) * (H / 128) + n0 / 128) * KB;

    long it = 0;
    for (int grp = 0; grp < groups; ++grp) {
        const long gp0 = p0 + static_cast<long>(grp) * NG;
        const int gn = static_cast<int>(min(static_cast<long>(NG), n - static_cast<long>(grp) * NG));
        if (threadIdx.x < NG) {
            int t = -1;
            float wv = 0.f;
            if (static_cast<int>(threadIdx.x) < gn) {
                const long p = gp0 + threadIdx.x;
                if (a.identity) {
                    t = static_cast<int>(p);
                    wv = 1.f;
                } else {
                    const int r = a.sorted_route[p];
                    if (r >= 0 && r < static_cast<long>(a.T) * a.K) {
                        t = r / a.K;
                        wv = a.topk_w[r];
                    } else {
                        report_status(a.status, MOE_STATUS_BAD_MAP);
                    }
                }
            }
            tok[threadIdx.x] = t;
            wr[threadIdx.x] = wv;
        }
        // h rows of this group are contiguous: rows gp0 .. gp0 + gn - 1.
        const int vpr = I / 8;
        for (int v = threadIdx.x; v < NG * vpr; v += kConsumerWarps * 32) {
            const int q = v / vpr, col = v - q * vpr;
            uint4 val = make_uint4(0, 0, 0, 0);
            if (q < gn) val = *reinterpret_cast<const uint4*>(a.h + static_cast<size_t>(gp0 + q) * I + col * 8);
            *reinterpret_cast<uint4*>(hs + q * hstride + col * 16) = val;
        }
        named_barrier_sync(1, kConsumerWarps * 32);

        float acc[NT][4];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.f;
        for (int kb = 0; kb < KB; ++kb, ++it) {
            const int s = static_cast<int>(it % kStages);
            float part[NT][4];
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) part[nt][0] = part[nt][1] = part[nt][2] = part[nt][3] = 0.f;
            if (mbar_wait_or_abort(&full[s], static_cast<uint32_t>((it / kStages) & 1), abort_flag, a.status)) {
                stage_mma<NT>(ring_u32 + s * kStageBytes, lm_off0, lm_off1, b_base, hstride, kb * 256, part);
                __syncwarp();
                if (lane == 0) mbar_arrive(&empty[s]);
            }
            const float ds = __ldg(sd + kb);
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int k = 0; k < 4; ++k) acc[nt][k] = fmaf(part[nt][k], ds, acc[nt][k]);
        }
        float* rh = red + hh * NG * kRedDn;
        const int rl = 16 * mt + g;
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            const int t0 = nt * 8 + 2 * c;
            rh[t0 * kRedDn + rl] = acc[nt][0];
            rh[(t0 + 1) * kRedDn + rl] = acc[nt][1];
            rh[t0 * kRedDn + rl + 8] = acc[nt][2];
            rh[(t0 + 1) * kRedDn + rl + 8] = acc[nt][3];
        }
        named_barrier_sync(1, kConsumerWarps * 32);
        // y[row, n0 .. n0+63] = bf16(w * (sum of both halves)), 16-byte stores.
        for (int v = threadIdx.x; v < NG * 8; v += kConsumerWarps * 32) {
            const int q = v >> 3, ch = v & 7;
            if (q < gn && tok[q] >= 0) {
                const float* y0 = red + q * kRedDn + ch * 8;
                const float* y1 = red + (NG + q) * kRedDn + ch * 8;
                const float wv = wr[q];
                uint32_t pk[4];
#pragma unroll
                for (int k = 0; k < 4; ++k)
                    pk[k] = pack_bf16x2(wv * (y0[2 * k] + y1[2 * k]), wv * (y0[2 * k + 1] + y1[2 * k + 1]));
                *reinterpret_cast<uint4*>(a.y + static_cast<size_t>(gp0 + q) * H + n0 + ch * 8) =
                    make_uint4(pk[0], pk[1], pk[2], pk[3]);
            }
        }
        named_barrier_sync(1, kConsumerWarps * 32);
    }
}

size_t gateup_smem(int NT, int H) {
    const int NG = 8 * NT;
    return 1024 + kStages * kStageBytes + static_cast<size_t>(NG) * (2 * H + 32) +
           4 * NG * kRedGU * sizeof(float) + (NG + 2) * sizeof(int) + 2 * kStages * sizeof(uint64_t) + 16;
}

size_t down_smem(int NT, int I) {
    const int NG = 8 * NT;
    return 1024 + kStages * kStageBytes + static_cast<size_t>(NG) * (2 * I + 32) +
           2 * NG * kRedDn * sizeof(float) + NG * sizeof(float) + (NG + 2) * sizeof(int) +
           2 * kStages * sizeof(uint64_t) + 16;
}

constexpr size_t kSmemLimit = 227 * 1024;

template <int NT>
cudaError_t launch_nt(const FfnArgs& a, const CUtensorMap& tg, const CUtensorMap& tu,
                      const CUtensorMap& td, cudaStream_t stream) {
    const size_t s1 = gateup_smem(NT, a.H), s2 = down_smem(NT, a.ex.inter);
    cudaError_t err = cudaFuncSetAttribute(gateup_decode_kernel<NT>,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(s1));
    if (err != cudaSuccess) return err;
    err = cudaFuncSetAttribute(down_decode_kernel<NT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(s2));
    if (err != cudaSuccess) return err;
    const int E = a.ex.n;
    gateup_decode_kernel<NT><<<dim3(a.ex.inter / kGateUpRows, E), kThreads, s1, stream>>>(tg, tu, a);
    err = cudaGetLastError();
    if (err != cudaSuccess) return err;
    down_decode_kernel<NT><<<dim3(a.H / kDownRows, E), kThreads, s2, stream>>>(td, a);
    return cudaGetLastError();
}

}  // namespace

bool ffn_decode_supported(int H, int I) {
    return gateup_smem(1, H) <= kSmemLimit && down_smem(1, I) <= kSmemLimit;
}

cudaError_t launch_ffn_decode(const FfnArgs& a, cudaStream_t stream) {
    CUtensorMap tg, tu, td;
    const uint64_t E = static_cast<uint64_t>(a.ex.n), I = a.ex.inter, H = a.H;
    cudaError_t err = make_tmap_u8_2d(&tg, a.ex.w_gate, E * I, H, 128, kGateUpRows);
    if (err == cudaSuccess) err = make_tmap_u8_2d(&tu, a.ex.w_up, E * I, H, 128, kGateUpRows);
    if (err == cudaSuccess) err = make_tmap_u8_2d(&td, a.ex.w_down, E * H, I, 128, kDownRows);
    if (err != cudaSuccess) return err;
    // Token tile: the host only knows the average rows per expert.
    int NT = a.avg_rows > 12 ? 4 : (a.avg_rows > 6 ? 2 : 1);
    while (NT > 1 && (gateup_smem(NT, a.H) > kSmemLimit || down_smem(NT, a.ex.inter) > kSmemLimit))
        NT >>= 1;
    switch (NT) {
        case 4: return launch_nt<4>(a, tg, tu, td, stream);
        case 2: return launch_nt<2>(a, tg, tu, td, stream);
        default: return launch_nt<1>(a, tg, tu, td, stream);
    }
}

}  // namespace moe
