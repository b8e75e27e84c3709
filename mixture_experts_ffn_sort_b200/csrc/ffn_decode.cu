// ffn_decode.cu -- expert FFN for the memory-bound regime (moe_expert_ffn,
// MOE_MODE_DECODE).
//
// The computation of the FP8 W8A16 MoE decode kernel
// (dstair/gated-deltanet-nki-trainium, "FP8 MoE decode kernel"): gate/up GEMM
// -> SwiGLU -> down GEMM -> affinity scale, with E4M3FN weights and one fp32
// scale per 128x128 block decoded tile by tile into 16-bit MMA operands; the
// row order is the expert-sorted order of the Nemotron-H sorted path, read from
// device-side offsets (no host sync).
//
// Design (B200):
//  * Persistent kernels (as many CTAs as the GPU holds at once).  Each CTA
//    lists the experts that received rows (from the device-side offsets, no
//    host sync) and takes a contiguous, equal share of the items (touched
//    expert, token group, slice of weight rows): 64 intermediate features
//    (their gate and up rows) in the gate/up kernel, 128 output features in
//    the down kernel.  Every item streams the same weight bytes, so skewed
//    expert loads stay balanced, and only the touched experts' weights are
//    read, once per token group.  Consecutive items of a CTA share their token
//    group, which is staged once.
//  * A producer warp streams the slices from HBM with TMA (evict-first L2
//    policy) in 16 KB stages of 128 reduction columns (one scale block),
//    128-byte swizzled, through a 4-deep shared-memory ring (mbarrier
//    full/empty pairs with bounded waits) that runs on across items.
//  * Eight consumer warps each own 16 MMA rows.  They read the FP8 bytes with
//    ldmatrix (conflict-free on the swizzled tile) and convert them with the
//    one-instruction E4M3x2 -> f16x2 conversion, which is exact: the decoded
//    weight is the E4M3 value itself.  Its 128x128 block scale multiplies each
//    128-column fp32 partial sum.  mma.sync m16n8k16 (f16 x f16 -> fp32) runs
//    against the expert's token rows staged in shared memory.  The reduction
//    columns are permuted identically on both operands so that one ldmatrix
//    register (4 codes of one row) feeds one A-fragment pair.
//  * Activations reach the MMA as f16: each bf16 row is multiplied by a power
//    of two 2^k that puts its largest magnitude in [2^14, 2^15), which makes
//    the bf16 -> f16 conversion exact (f16 holds 11 significant bits to bf16's
//    8); the epilogue multiplies by 2^-k in fp32.
//  * In the gate/up tile the 16 MMA rows are 8 gate + 8 up rows of the same
//    features, so SwiGLU is thread-local in the epilogue; outputs go through a
//    shared-memory tile to coalesced 16-byte stores.
//  * The down kernel is a programmatic dependent launch: its producer starts
//    streaming weights while the gate/up grid drains, and its consumers wait
//    (griddepcontrol.wait) before reading h.
//  * W8A8 (moe_expert_ffn_w8a8, template flag Q): the activations become
//    E4M3FN codes in blocks with power-of-two scales -- x per 128 columns as
//    it is staged, h per 64 features in the gate/up epilogue -- and both GEMMs
//    run as m16n8k32 E4M3FN MMAs whose A fragment is one ldmatrix of the
//    weight codes (no conversion); the weight and activation block scales
//    multiply each fp32 partial.
#include <algorithm>

#include "device_common.cuh"
#include "launch.h"

namespace moe {

namespace {

constexpr int kStages = 4;
constexpr int kConsumerWarps = 8;
constexpr int kConsumers = kConsumerWarps * 32;
constexpr int kThreads = kConsumers + 32;
constexpr int kStageBytes = 16384;  // 128 rows x 128 bytes
constexpr int kGateUpFeat = 64;     // intermediate features per gate/up CTA (8 per warp)
constexpr int kDownRows = 128;      // output features per down CTA (16 per warp)
constexpr int kGuTile = kGateUpFeat + 8;  // bf16 stride of the gate/up output tile
constexpr int kDnTile = kDownRows + 8;    // bf16 stride of the down output tile

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
    return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

__device__ __forceinline__ uint2 lds64(uint32_t addr) {
    uint2 v;
    asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(addr));
    return v;
}

__device__ __forceinline__ uint4 ldg_v4(const void* p) {
    uint4 v;
    asm volatile("ld.global.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

// Row range [p0, p0 + n) of expert e.  Returns false for corrupt offsets.
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

// Producer: stream `count` stages (cycling the slice's KB column blocks) into
// the ring; `it` is the CTA's running stage counter.  Returns false once a
// wait has expired.
__device__ __forceinline__ bool produce(const CUtensorMap* m0, const CUtensorMap* m1, int row, int KB,
                                        long count, long& it, uint8_t* ring, uint64_t* full, uint64_t* empty,
                                        uint64_t policy, volatile int* abort_flag, int32_t* status) {
    for (long j = 0; j < count; ++j, ++it) {
        const int s = static_cast<int>(it % kStages);
        if (it >= kStages &&
            !mbar_wait_or_abort(&empty[s], static_cast<uint32_t>((it / kStages - 1) & 1), abort_flag, status))
            return false;
        mbar_arrive_expect_tx(&full[s], kStageBytes);
        const int kb = static_cast<int>(j % KB);
        uint8_t* dst = ring + static_cast<size_t>(s) * kStageBytes;
        if (m1) {
            tma_load_2d_hint(dst, m0, &full[s], kb * 128, row, policy);
            tma_load_2d_hint(dst + kStageBytes / 2, m1, &full[s], kb * 128, row, policy);
        } else {
            tma_load_2d_hint(dst, m0, &full[s], kb * 128, row, policy);
        }
    }
    return true;
}

// Largest |x| bit pattern (sign cleared) among the 8 bf16 of a 16-byte vector.
__device__ __forceinline__ uint32_t absmax_bf16x8(const uint4& v) {
    uint32_t m = __vmaxu2(__vmaxu2(v.x & 0x7FFF7FFFu, v.y & 0x7FFF7FFFu),
                          __vmaxu2(v.z & 0x7FFF7FFFu, v.w & 0x7FFF7FFFu));
    return max(m & 0xFFFFu, m >> 16);
}

__device__ __forceinline__ uint32_t bf16x2_to_f16x2_scaled(uint32_t w, float up) {
    const float a = __uint_as_float(w << 16) * up;
    const float b = __uint_as_float(w & 0xFFFF0000u) * up;
    __half2 h = __floats2half2_rn(a, b);
    return *reinterpret_cast<uint32_t*>(&h);
}

// Stage NG rows of W bf16 values into shared memory (row stride `stride`
// bytes) as f16 times 2^k, k chosen per row so that its largest magnitude
// lies in [2^14, 2^15); inv_scale[q] = 2^-k.  row_ptr(q) gives the source row
// or nullptr for a padding row (zeros).  Warp w handles rows w, w + 8, ...
template <int NG, class RowPtr>
__device__ __forceinline__ void stage_rows_f16(RowPtr row_ptr, int W, uint8_t* dst, int stride,
                                               float* inv_scale) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int vpr = W / 8;
    for (int q = warp; q < NG; q += kConsumerWarps) {
        const uint16_t* src = row_ptr(q);
        uint8_t* d = dst + q * stride;
        uint32_t amax = 0;
        for (int v = lane; v < vpr; v += 32) {
            const uint4 val = src ? ldg_v4(src + v * 8) : make_uint4(0, 0, 0, 0);
            *reinterpret_cast<uint4*>(d + v * 16) = val;
            amax = max(amax, absmax_bf16x8(val));
        }
        amax = __reduce_max_sync(0xffffffffu, amax);
        // |x|max = 2^e * m with e = (bits >> 7) - 127; k = 14 - e, at most 64.
        const int k = amax ? min(64, 14 - (static_cast<int>(amax >> 7) - 127)) : 0;
        const float up = __uint_as_float(static_cast<uint32_t>(k + 127) << 23);
        if (lane == 0) inv_scale[q] = __uint_as_float(static_cast<uint32_t>(127 - k) << 23);
        __syncwarp();
        for (int v = lane; v < vpr; v += 32) {
            uint4 val = *reinterpret_cast<const uint4*>(d + v * 16);
            val.x = bf16x2_to_f16x2_scaled(val.x, up);
            val.y = bf16x2_to_f16x2_scaled(val.y, up);
            val.z = bf16x2_to_f16x2_scaled(val.z, up);
            val.w = bf16x2_to_f16x2_scaled(val.w, up);
            *reinterpret_cast<uint4*>(d + v * 16) = val;
        }
    }
}

// W8A8 form.  Activation rows in shared memory are E4M3FN codes laid out per
// 32-byte slab (32 reduction columns) so that one 8-byte load gives the two
// registers of an m16n8k32 B fragment: unit u (bytes 8u .. 8u+7) holds the
// codes of columns 4u .. 4u+3 and then 16+4u .. 16+4u+3 of the slab.
__device__ __forceinline__ uint32_t slab_offset(int col) {  // byte of column col (multiple of 4) in its row
    const int q = col & 31;
    return static_cast<uint32_t>((col & ~31) + 8 * ((q & 15) >> 2) + 4 * (q >> 4));
}

// Stage NG rows of W bf16 values as E4M3FN codes: each 128-column block of a
// row is multiplied by its own power of two 2^k (act_scale_exp of the block's
// largest magnitude; exact) and rounded to nearest even;
// qs[q * nqb + b] = 2^-k.  row_ptr(q) gives the source row or nullptr for a
// padding row (zeros).  Warp w handles rows w, w + 8, ...; each half-warp
// covers one block of 16 vectors.
template <int NG, class RowPtr>
__device__ __forceinline__ void stage_rows_e4m3(RowPtr row_ptr, int W, uint8_t* dst, int stride, float* qs,
                                                int nqb) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int vpr = W / 8;  // a multiple of 16: half-warps stay whole
    for (int q = warp; q < NG; q += kConsumerWarps) {
        const uint16_t* src = row_ptr(q);
        uint8_t* d = dst + q * stride;
        for (int v0 = 0; v0 < vpr; v0 += 32) {
            const int v = v0 + lane;
            const bool in = v < vpr;
            const uint4 val = (src && in) ? ldg_v4(src + v * 8) : make_uint4(0, 0, 0, 0);
            uint32_t m = absmax_bf16x8(val);
#pragma unroll
            for (int o = 1; o < 16; o <<= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, o));
            const int k = act_scale_exp(m << 16);
            if (!in) continue;
            if ((lane & 15) == 0) qs[q * nqb + v / 16] = pow2_f32(-k);
            const float up = pow2_f32(k);
            const uint32_t w[4] = {val.x, val.y, val.z, val.w};
            float f[8];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                f[2 * i] = __uint_as_float(w[i] << 16) * up;
                f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u) * up;
            }
            *reinterpret_cast<uint32_t*>(d + slab_offset(8 * v)) = f32x4_to_e4m3x4(f[0], f[1], f[2], f[3]);
            *reinterpret_cast<uint32_t*>(d + slab_offset(8 * v + 4)) = f32x4_to_e4m3x4(f[4], f[5], f[6], f[7]);
        }
    }
}

// Stage NG rows of W E4M3FN codes (already quantised, 16-byte vectors) into
// the slab layout, and their nqb block scales.  row(q) gives the source row
// index or -1 for a padding row (zeros).
template <int NG, class RowIdx>
__device__ __forceinline__ void stage_codes(RowIdx row, const uint8_t* codes, const float* scales, int W,
                                            uint8_t* dst, int stride, float* qs, int nqb) {
    const int vpr = W / 16;
    for (int v = threadIdx.x; v < NG * vpr; v += kConsumers) {
        const int q = v / vpr, c = v - q * vpr;
        const long r = row(q);
        const uint4 val = r >= 0 ? ldg_v4(codes + static_cast<size_t>(r) * W + c * 16) : make_uint4(0, 0, 0, 0);
        uint8_t* d = dst + q * stride;
        *reinterpret_cast<uint32_t*>(d + slab_offset(16 * c)) = val.x;
        *reinterpret_cast<uint32_t*>(d + slab_offset(16 * c + 4)) = val.y;
        *reinterpret_cast<uint32_t*>(d + slab_offset(16 * c + 8)) = val.z;
        *reinterpret_cast<uint32_t*>(d + slab_offset(16 * c + 12)) = val.w;
    }
    for (int i = threadIdx.x; i < NG * nqb; i += kConsumers) {
        const int q = i / nqb, b = i - q * nqb;
        const long r = row(q);
        qs[i] = r >= 0 ? __ldg(scales + static_cast<size_t>(r) * nqb + b) : 0.f;
    }
}

// W8A8: one 128-column stage of one warp with FP8 activations: per 32-column
// slab p, one ldmatrix_x4 of the weight codes is exactly the A fragment of an
// m16n8k32 E4M3FN MMA (matrices 0/1: the 16 rows in chunk 2p, 2/3: in chunk
// 2p+1).  SPLIT: slabs 0-1 accumulate into part[0] and slabs 2-3 into
// part[1] (two 64-column activation scale blocks per stage).
template <int NT, bool SPLIT>
__device__ __forceinline__ void stage_mma_q(uint32_t tile0, uint32_t tile1, uint32_t row, uint32_t chunk_sel,
                                            uint32_t b_addr, int stride, float (&part)[2][NT][4]) {
#pragma unroll
    for (int p = 0; p < 4; ++p) {
        const uint32_t chunk = 2 * p + (chunk_sel & 1);
        uint32_t r0, r1, r2, r3;
        ldmatrix_x4((chunk_sel & 2 ? tile1 : tile0) + sw128_offset(row, chunk & 7), r0, r1, r2, r3);
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            const uint2 b = lds64(b_addr + nt * 8 * stride + p * 32);
            mma_e4m3_16832(part[SPLIT && p >= 2 ? 1 : 0][nt], r0, r1, r2, r3, b.x, b.y);
        }
    }
}

// One 128-column stage of one warp: 16 rows x 128 columns against NT token
// tiles.  This lane's ldmatrix row is `row` of sub-tile tile0 (chunk_sel bit 1
// clear) or tile1 (set), in chunk j (bit 0 clear) or j+1 (set) of each chunk
// pair; b_addr is this lane's B address for chunk 0 of the stage.
template <int NT>
__device__ __forceinline__ void stage_mma(uint32_t tile0, uint32_t tile1, uint32_t row,
                                          uint32_t chunk_sel, uint32_t b_addr, int xstride,
                                          float (&part)[NT][4]) {
#pragma unroll
    for (int p = 0; p < 4; ++p) {
        const uint32_t chunk = 2 * p + (chunk_sel & 1);
        uint32_t r0, r1, r2, r3;
        ldmatrix_x4((chunk_sel & 2 ? tile1 : tile0) + sw128_offset(row, chunk & 7), r0, r1, r2, r3);
        uint32_t lo0, hi0, lo1, hi1;
        e4m3x4_to_f16(r0, lo0, hi0);
        e4m3x4_to_f16(r1, lo1, hi1);
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            const uint2 b = lds64(b_addr + nt * 8 * xstride + (2 * p) * 32);
            mma_f16_16816(part[nt], lo0, lo1, hi0, hi1, b.x, b.y);
        }
        e4m3x4_to_f16(r2, lo0, hi0);
        e4m3x4_to_f16(r3, lo1, hi1);
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            const uint2 b = lds64(b_addr + nt * 8 * xstride + (2 * p + 1) * 32);
            mma_f16_16816(part[nt], lo0, lo1, hi0, hi1, b.x, b.y);
        }
    }
}

template <int NT>
__device__ __forceinline__ void zero_acc(float (&a)[NT][4]) {
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) a[nt][0] = a[nt][1] = a[nt][2] = a[nt][3] = 0.f;
}

// Shared-memory carve-up common to both kernels.
struct Smem {
    float* qs;        // W8A8: activation block scales [NG][nqb]
    uint8_t* ring;
    uint8_t* rows;    // staged activation rows (f16)
    uint16_t* otile;  // output tile (bf16)
    int* tok;
    float* wr;
    float* inv;
    uint64_t* full;
    uint64_t* empty;
    volatile int* abort_flag;
    int* touched;  // [E]: experts with at least one row
    int* gpre;     // [E + 1]: exclusive prefix of their token groups
};

__host__ __device__ constexpr size_t smem_bytes(int NG, int row_stride, int otile_stride, int E, int nqb = 0) {
    return 1024 + static_cast<size_t>(kStages) * kStageBytes + static_cast<size_t>(NG) * row_stride +
           static_cast<size_t>(NG) * otile_stride * 2 + 3 * NG * 4 + 2 * kStages * 8 + 16 +
           static_cast<size_t>(2 * E + 1) * 4 + static_cast<size_t>(NG) * nqb * 4;
}

__device__ __forceinline__ Smem carve(uint8_t* raw, int NG, int row_stride, int otile_stride, int E, int nqb = 0) {
    Smem s;
    uint8_t* p = align1024(raw);
    s.ring = p;
    p += kStages * kStageBytes;
    s.rows = p;
    p += NG * row_stride;
    s.otile = reinterpret_cast<uint16_t*>(p);
    p += NG * otile_stride * 2;
    s.tok = reinterpret_cast<int*>(p);
    s.wr = reinterpret_cast<float*>(s.tok + NG);
    s.inv = s.wr + NG;
    p = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(s.inv + NG) + 7) & ~uintptr_t(7));
    s.full = reinterpret_cast<uint64_t*>(p);
    s.empty = s.full + kStages;
    s.abort_flag = reinterpret_cast<volatile int*>(s.empty + kStages);
    s.touched = reinterpret_cast<int*>(s.empty + kStages) + 4;
    s.gpre = s.touched + E;
    s.qs = nqb ? reinterpret_cast<float*>(s.gpre + E + 1) : nullptr;
    return s;
}

// The experts of this call with at least one row (and at most a.row_split
// rows when a.row_split > 0), in increasing order, into
// touched[0 .. count), and the exclusive prefix of their token groups (of NG
// rows) into gpre[0 .. count]; returns the total number of groups.  Experts
// whose offsets are corrupt are left out (and flagged); *ntouched = count.
// Contains __syncthreads.
__device__ long build_touched(const FfnArgs& a, int NG, int* touched, int* gpre, int* ntouched) {
    const int E = a.identity ? 1 : a.ex.n;
    __shared__ int warp_sums[32][2];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
    const int per = (E + blockDim.x - 1) / blockDim.x;
    const int e0 = min(E, static_cast<int>(threadIdx.x) * per), e1 = min(E, e0 + per);
    int cnt = 0, grp = 0;
    for (int e = e0; e < e1; ++e) {
        long p0, n;
        if (!expert_rows(a, e, p0, n)) {
            report_status(a.status, MOE_STATUS_BAD_MAP);
            continue;
        }
        if (a.row_split > 0 && n > a.row_split) continue;  // left to the prefill form
        cnt += n > 0;
        grp += static_cast<int>((n + NG - 1) / NG);
    }
    int xc = cnt, xg = grp;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int yc = __shfl_up_sync(0xffffffffu, xc, off), yg = __shfl_up_sync(0xffffffffu, xg, off);
        if (lane >= off) xc += yc, xg += yg;
    }
    if (lane == 31) warp_sums[warp][0] = xc, warp_sums[warp][1] = xg;
    __syncthreads();
    if (warp == 0) {
        int vc = lane < nw ? warp_sums[lane][0] : 0, vg = lane < nw ? warp_sums[lane][1] : 0;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int yc = __shfl_up_sync(0xffffffffu, vc, off), yg = __shfl_up_sync(0xffffffffu, vg, off);
            if (lane >= off) vc += yc, vg += yg;
        }
        warp_sums[lane][0] = vc, warp_sums[lane][1] = vg;
    }
    __syncthreads();
    int pc = (warp ? warp_sums[warp - 1][0] : 0) + xc - cnt;
    int pg = (warp ? warp_sums[warp - 1][1] : 0) + xg - grp;
    for (int e = e0; e < e1; ++e) {
        long p0, n;
        if (expert_rows(a, e, p0, n) && n > 0 && (a.row_split <= 0 || n <= a.row_split)) {
            touched[pc] = e;
            gpre[pc] = pg;
            ++pc;
            pg += static_cast<int>((n + NG - 1) / NG);
        }
    }
    const int count = warp_sums[nw - 1][0], total = warp_sums[nw - 1][1];
    if (threadIdx.x == 0) gpre[count] = total;
    *ntouched = count;
    __syncthreads();
    return total;
}

// Walks a contiguous range of the balanced item list: (touched expert j,
// token group of that expert, block of its weight rows), blocks fastest.
// Every item streams the same weight bytes.  One search finds the start;
// next() then advances without searching.
struct ItemWalk {
    long item, end;
    int j, grp, blk;
    int e;       // expert touched[j]
    int ngrp;    // token groups of expert j
    const Smem* s;
    int bpe;

    __device__ ItemWalk(const Smem& sm, long first, long last, int bpe_, int ntouched)
        : item(first), end(last), s(&sm), bpe(bpe_) {
        const int gi = static_cast<int>(first / bpe);
        int lo = 0, hi = max(ntouched - 1, 0);  // last j with gpre[j] <= gi
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (sm.gpre[mid] <= gi)
                lo = mid;
            else
                hi = mid - 1;
        }
        j = lo;
        grp = gi - sm.gpre[lo];
        blk = static_cast<int>(first % bpe);
        load();
    }
    __device__ void load() {
        e = s->touched[j];
        ngrp = s->gpre[j + 1] - s->gpre[j];
    }
    __device__ bool valid() const { return item < end; }
    __device__ void next() {
        ++item;
        if (++blk < bpe) return;
        blk = 0;
        if (++grp < ngrp) return;
        grp = 0;
        ++j;
        if (item < end) load();
    }
};

__device__ __forceinline__ void init_barriers(const Smem& s) {
    if (threadIdx.x == 0) {
        for (int i = 0; i < kStages; ++i) {
            mbar_init(&s.full[i], 1);
            mbar_init(&s.empty[i], kConsumerWarps);
        }
        *s.abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();
}

// ------------------------------------------------------------------ gate/up + SwiGLU

// Q: the W8A8 form (FP8 activations, m16n8k32 E4M3FN MMAs, h quantised in the epilogue).
template <int NT, bool Q>
__global__ void __launch_bounds__(kThreads, 2)
    gateup_decode_kernel(const __grid_constant__ CUtensorMap tm_gate,
                         const __grid_constant__ CUtensorMap tm_up, const FfnArgs a) {
    constexpr int NG = 8 * NT;  // tokens per group
    if (threadIdx.x == 0) grid_dependency_launch();  // the down kernel may start streaming
    extern __shared__ uint8_t smem_raw[];
    const int H = a.H, I = a.ex.inter;
    const int KB = H / 128;
    const int xstride = Q ? H + 32 : 2 * H + 32;
    const int E = a.identity ? 1 : a.ex.n;
    const Smem s = carve(smem_raw, NG, xstride, kGuTile, E, Q ? KB : 0);
    init_barriers(s);
    // Items: (touched expert, token group, block of kGateUpFeat features); each
    // CTA of the persistent grid takes a contiguous, equal share.
    const int bpe = I / kGateUpFeat;
    int ntouched = 0;
    const long items = build_touched(a, NG, s.touched, s.gpre, &ntouched) * bpe;


    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (warp == kConsumerWarps) {
        if (lane == 0) {
            tma_prefetch_desc(&tm_gate);
            tma_prefetch_desc(&tm_up);
            const uint64_t policy = l2_evict_first_policy();
            long it = 0;
            for (ItemWalk w(s, items * blockIdx.x / gridDim.x, items * (blockIdx.x + 1) / gridDim.x, bpe, ntouched);
                 w.valid(); w.next())
                if (!produce(&tm_gate, &tm_up, w.e * I + w.blk * kGateUpFeat, KB, KB, it, s.ring, s.full, s.empty,
                             policy, s.abort_flag, a.status))
                    break;
        }
        return;
    }

    const int g = lane >> 2, c = lane & 3;
    const int mi = lane >> 3, rr = lane & 7;
    // ldmatrix: matrices 0/2 read gate rows 8w+rr, 1/3 the up rows; 0/1 chunk j, 2/3 chunk j+1.
    const uint32_t lm_row = 8 * warp + rr;
    const uint32_t chunk_sel = (mi >> 1) | ((mi & 1) << 1);  // bit 0: chunk j+1, bit 1: up tile
    const uint32_t ring_u32 = smem_u32(s.ring);
    const uint32_t b_lane = smem_u32(s.rows) + g * xstride + 8 * c;
    const long R = static_cast<long>(a.T) * a.K;

    long it = 0;
    long staged = -1;  // token group (of the item list) staged in s.rows
    for (ItemWalk w(s, items * blockIdx.x / gridDim.x, items * (blockIdx.x + 1) / gridDim.x, bpe, ntouched);
         w.valid(); w.next()) {
        const int e = w.e, i0 = w.blk * kGateUpFeat;
        long p0, n;
        expert_rows(a, e, p0, n);
        const size_t sblk = (static_cast<size_t>(e) * (I / 128) + i0 / 128) * KB;
        const float* sg = a.ex.s_gate + sblk;
        const float* su = a.ex.s_up + sblk;
        const long gp0 = p0 + static_cast<long>(w.grp) * NG;
        const int gn = static_cast<int>(min(static_cast<long>(NG), n - static_cast<long>(w.grp) * NG));
        // Consecutive items of a CTA share a token group for bpe items: its
        // rows are staged once.
        const bool restage = staged != w.item / bpe;
        staged = w.item / bpe;
        if (restage) {
            if (threadIdx.x < NG) {
                int t = -1;
                if (static_cast<int>(threadIdx.x) < gn) {
                    if (a.identity) {
                        t = static_cast<int>(gp0 + threadIdx.x);
                    } else {
                        const int r = a.sorted_route[gp0 + threadIdx.x];
                        if (r >= 0 && r < R)
                            t = r / a.K;
                        else
                            report_status(a.status, MOE_STATUS_BAD_MAP);
                    }
                }
                s.tok[threadIdx.x] = t;
            }
            named_barrier_sync(1, kConsumers);
            auto x_row = [&](int q) -> const uint16_t* {
                const int t = s.tok[q];
                return t >= 0 ? a.x + static_cast<size_t>(t) * H : nullptr;
            };
            if constexpr (Q)
                stage_rows_e4m3<NG>(x_row, H, s.rows, xstride, s.qs, KB);
            else
                stage_rows_f16<NG>(x_row, H, s.rows, xstride, s.inv);
            named_barrier_sync(1, kConsumers);
        }

        float acc[NT][4];
        zero_acc<NT>(acc);
        for (int kb = 0; kb < KB; ++kb, ++it) {
            const int st = static_cast<int>(it % kStages);
            float part[2][NT][4];
            zero_acc<NT>(part[0]);
            if (mbar_wait_or_abort(&s.full[st], static_cast<uint32_t>((it / kStages) & 1), s.abort_flag,
                                   a.status)) {
                const uint32_t tile = ring_u32 + st * kStageBytes;
                // chunk_sel bit 1 selects the up sub-tile (second half of the stage).
                if constexpr (Q)
                    stage_mma_q<NT, false>(tile, tile + kStageBytes / 2, lm_row, chunk_sel, b_lane + kb * 128,
                                           xstride, part);
                else
                    stage_mma<NT>(tile, tile + kStageBytes / 2, lm_row, chunk_sel, b_lane + kb * 256, xstride,
                                  part[0]);
                __syncwarp();
                if (lane == 0) mbar_arrive(&s.empty[st]);
            }
            const float gs = __ldg(sg + kb), us = __ldg(su + kb);
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                // W8A8: the activation block scales of this thread's two token columns.
                float x0 = 1.f, x1 = 1.f;
                if constexpr (Q) {
                    x0 = s.qs[(nt * 8 + 2 * c) * KB + kb];
                    x1 = s.qs[(nt * 8 + 2 * c + 1) * KB + kb];
                }
                acc[nt][0] = fmaf(part[0][nt][0], gs * x0, acc[nt][0]);
                acc[nt][1] = fmaf(part[0][nt][1], gs * x1, acc[nt][1]);
                acc[nt][2] = fmaf(part[0][nt][2], us * x0, acc[nt][2]);
                acc[nt][3] = fmaf(part[0][nt][3], us * x1, acc[nt][3]);
            }
        }
        const int il = 8 * warp + g;
        if constexpr (!Q) {
            // SwiGLU on the true sums (undo the activation scale first).
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                const int t0 = nt * 8 + 2 * c;
                const float s0 = s.inv[t0], s1 = s.inv[t0 + 1];
                const float h0 = silu_f32(acc[nt][0] * s0) * (acc[nt][2] * s0);
                const float h1 = silu_f32(acc[nt][1] * s1) * (acc[nt][3] * s1);
                s.otile[t0 * kGuTile + il] = __bfloat16_as_ushort(__float2bfloat16_rn(h0));
                s.otile[(t0 + 1) * kGuTile + il] = __bfloat16_as_ushort(__float2bfloat16_rn(h1));
            }
            named_barrier_sync(1, kConsumers);
            for (int v = threadIdx.x; v < NG * (kGateUpFeat / 8); v += kConsumers) {
                const int q = v / (kGateUpFeat / 8), ch = v % (kGateUpFeat / 8);
                if (q < gn && s.tok[q] >= 0)
                    *reinterpret_cast<uint4*>(a.h + static_cast<size_t>(gp0 + q) * I + i0 + ch * 8) =
                        *reinterpret_cast<const uint4*>(s.otile + q * kGuTile + ch * 8);
            }
            named_barrier_sync(1, kConsumers);
        } else {
            // SwiGLU, then h quantised in registers: the item's 64 features are
            // one scale block, so each token's scale comes from the largest |h|
            // over the eight warps (8 features each: shuffles over g, then the
            // warps' maxima through shared memory).  Codes go through a byte
            // tile (rows of kQRow bytes) to 16-byte stores.
            constexpr int kQRow = kGateUpFeat + 16;
            uint8_t* qtile = reinterpret_cast<uint8_t*>(s.otile);
            float* wmax = reinterpret_cast<float*>(qtile + NG * kQRow);  // [NG][kConsumerWarps]
            float hv[NT][2];
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                hv[nt][0] = silu_f32(acc[nt][0]) * acc[nt][2];
                hv[nt][1] = silu_f32(acc[nt][1]) * acc[nt][3];
#pragma unroll
                for (int j = 0; j < 2; ++j) {
                    float m = fabsf(hv[nt][j]);
#pragma unroll
                    for (int o = 4; o < 32; o <<= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
                    if (g == 0) wmax[(nt * 8 + 2 * c + j) * kConsumerWarps + warp] = m;
                }
            }
            named_barrier_sync(1, kConsumers);
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int j = 0; j < 2; ++j) {
                    const int t = nt * 8 + 2 * c + j;
                    float m = 0.f;
#pragma unroll
                    for (int w2 = 0; w2 < kConsumerWarps; ++w2) m = fmaxf(m, wmax[t * kConsumerWarps + w2]);
                    const float up = pow2_f32(act_scale_exp(__float_as_uint(m)));
                    qtile[t * kQRow + il] = static_cast<uint8_t>(
                        __nv_cvt_float_to_fp8(hv[nt][j] * up, __NV_SATFINITE, __NV_E4M3));
                }
            named_barrier_sync(1, kConsumers);
            uint8_t* hq = reinterpret_cast<uint8_t*>(a.h);
            for (int v = threadIdx.x; v < NG * (kGateUpFeat / 16); v += kConsumers) {
                const int q = v / (kGateUpFeat / 16), ch = v % (kGateUpFeat / 16);
                if (q < gn && s.tok[q] >= 0)
                    *reinterpret_cast<uint4*>(hq + static_cast<size_t>(gp0 + q) * I + i0 + ch * 16) =
                        *reinterpret_cast<const uint4*>(qtile + q * kQRow + ch * 16);
            }
            if (threadIdx.x < NG && static_cast<int>(threadIdx.x) < gn && s.tok[threadIdx.x] >= 0) {
                const int q = threadIdx.x;
                float m = 0.f;
#pragma unroll
                for (int w2 = 0; w2 < kConsumerWarps; ++w2) m = fmaxf(m, wmax[q * kConsumerWarps + w2]);
                a.hscale[static_cast<size_t>(gp0 + q) * (I / kGateUpFeat) + i0 / kGateUpFeat] =
                    pow2_f32(-act_scale_exp(__float_as_uint(m)));
            }
            named_barrier_sync(1, kConsumers);
        }
    }
}

// ------------------------------------------------------------------ down + affinity

template <int NT, bool Q>
__global__ void __launch_bounds__(kThreads, 2)
    down_decode_kernel(const __grid_constant__ CUtensorMap tm_down, const FfnArgs a) {
    constexpr int NG = 8 * NT;
    // A following programmatic-dependent launch (a tensor-core gate/up grid
    // chained after this one) may start on the SMs this grid leaves idle.
    if (threadIdx.x == 0) grid_dependency_launch();
    extern __shared__ uint8_t smem_raw[];
    const int H = a.H, I = a.ex.inter;
    const int KB = I / 128;
    const int hstride = Q ? I + 32 : 2 * I + 32;
    const int E = a.identity ? 1 : a.ex.n;
    const int nqb = I / kGateUpFeat;  // W8A8: h scale blocks per row
    const Smem s = carve(smem_raw, NG, hstride, kDnTile, E, Q ? nqb : 0);
    init_barriers(s);
    // Items: (touched expert, token group, block of kDownRows output rows); each
    // CTA of the persistent grid takes a contiguous, equal share.  Offsets come
    // from the sort, which finished before the gate/up grid began.
    const int bpe = H / kDownRows;
    int ntouched = 0;
    const long items = build_touched(a, NG, s.touched, s.gpre, &ntouched) * bpe;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (warp == kConsumerWarps) {
        if (lane == 0) {
            tma_prefetch_desc(&tm_down);
            const uint64_t policy = l2_evict_first_policy();
            long it = 0;
            for (ItemWalk w(s, items * blockIdx.x / gridDim.x, items * (blockIdx.x + 1) / gridDim.x, bpe, ntouched);
                 w.valid(); w.next())
                if (!produce(&tm_down, nullptr, w.e * H + w.blk * kDownRows, KB, KB, it, s.ring, s.full, s.empty,
                             policy, s.abort_flag, a.status))
                    break;
        }
        return;
    }
    grid_dependency_wait();  // h is written by the gate/up grid

    const int g = lane >> 2, c = lane & 3;
    const int mi = lane >> 3, rr = lane & 7;
    // ldmatrix: matrices 0/2 rows 16w+rr, 1/3 rows 16w+8+rr; 0/1 chunk j, 2/3 chunk j+1.
    const uint32_t lm_row = 16 * warp + ((mi & 1) << 3) + rr;
    const uint32_t chunk_sel = mi >> 1;
    const uint32_t ring_u32 = smem_u32(s.ring);
    const uint32_t b_lane = smem_u32(s.rows) + g * hstride + 8 * c;
    const long R = static_cast<long>(a.T) * a.K;

    long it = 0;
    long staged = -1;  // token group (of the item list) staged in s.rows
    for (ItemWalk w(s, items * blockIdx.x / gridDim.x, items * (blockIdx.x + 1) / gridDim.x, bpe, ntouched);
         w.valid(); w.next()) {
        const int e = w.e, n0 = w.blk * kDownRows;
        long p0, n;
        expert_rows(a, e, p0, n);
        const float* sd = a.ex.s_down + (static_cast<size_t>(e) * (H / 128) + n0 / 128) * KB;
        const long gp0 = p0 + static_cast<long>(w.grp) * NG;
        const int gn = static_cast<int>(min(static_cast<long>(NG), n - static_cast<long>(w.grp) * NG));
        const bool restage = staged != w.item / bpe;
        staged = w.item / bpe;
        if (restage) {
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
                        if (r >= 0 && r < R) {
                            t = r / a.K;
                            wv = a.topk_w[r];
                        } else {
                            report_status(a.status, MOE_STATUS_BAD_MAP);
                        }
                    }
                }
                s.tok[threadIdx.x] = t;
                s.wr[threadIdx.x] = wv;
            }
            named_barrier_sync(1, kConsumers);
            if constexpr (Q)
                stage_codes<NG>(
                    [&](int q) -> long { return (q < gn && s.tok[q] >= 0) ? gp0 + q : -1; },
                    reinterpret_cast<const uint8_t*>(a.h), a.hscale, I, s.rows, hstride, s.qs, nqb);
            else
                stage_rows_f16<NG>(
                    [&](int q) -> const uint16_t* {
                        return (q < gn && s.tok[q] >= 0) ? a.h + static_cast<size_t>(gp0 + q) * I : nullptr;
                    },
                    I, s.rows, hstride, s.inv);
            named_barrier_sync(1, kConsumers);
        }

        float acc[NT][4];
        zero_acc<NT>(acc);
        for (int kb = 0; kb < KB; ++kb, ++it) {
            const int st = static_cast<int>(it % kStages);
            float part[2][NT][4];
            zero_acc<NT>(part[0]);
            if constexpr (Q) zero_acc<NT>(part[1]);
            if (mbar_wait_or_abort(&s.full[st], static_cast<uint32_t>((it / kStages) & 1), s.abort_flag,
                                   a.status)) {
                const uint32_t tile = ring_u32 + st * kStageBytes;
                if constexpr (Q)
                    stage_mma_q<NT, true>(tile, tile, lm_row, chunk_sel, b_lane + kb * 128, hstride, part);
                else
                    stage_mma<NT>(tile, tile, lm_row, chunk_sel, b_lane + kb * 256, hstride, part[0]);
                __syncwarp();
                if (lane == 0) mbar_arrive(&s.empty[st]);
            }
            const float ds = __ldg(sd + kb);
            if constexpr (Q) {
                // Two 64-feature scale blocks of h per 128-column stage.
#pragma unroll
                for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        const int t = nt * 8 + 2 * c + (k & 1);
                        const float lo = s.qs[t * nqb + 2 * kb], hi = s.qs[t * nqb + 2 * kb + 1];
                        acc[nt][k] = fmaf(fmaf(part[0][nt][k], lo, part[1][nt][k] * hi), ds, acc[nt][k]);
                    }
            } else {
#pragma unroll
                for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                    for (int k = 0; k < 4; ++k) acc[nt][k] = fmaf(part[0][nt][k], ds, acc[nt][k]);
            }
        }
        const int rl = 16 * warp + g;
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            const int t0 = nt * 8 + 2 * c;
            // The f16 form still carries each row's power-of-two scale; the W8A8
            // form applied its block scales per stage.
            const float f0 = (Q ? 1.f : s.inv[t0]) * s.wr[t0], f1 = (Q ? 1.f : s.inv[t0 + 1]) * s.wr[t0 + 1];
            s.otile[t0 * kDnTile + rl] = __bfloat16_as_ushort(__float2bfloat16_rn(acc[nt][0] * f0));
            s.otile[(t0 + 1) * kDnTile + rl] = __bfloat16_as_ushort(__float2bfloat16_rn(acc[nt][1] * f1));
            s.otile[t0 * kDnTile + rl + 8] = __bfloat16_as_ushort(__float2bfloat16_rn(acc[nt][2] * f0));
            s.otile[(t0 + 1) * kDnTile + rl + 8] = __bfloat16_as_ushort(__float2bfloat16_rn(acc[nt][3] * f1));
        }
        named_barrier_sync(1, kConsumers);
        for (int v = threadIdx.x; v < NG * (kDownRows / 8); v += kConsumers) {
            const int q = v / (kDownRows / 8), ch = v % (kDownRows / 8);
            if (q < gn && s.tok[q] >= 0)
                *reinterpret_cast<uint4*>(a.y + static_cast<size_t>(gp0 + q) * H + n0 + ch * 8) =
                    *reinterpret_cast<const uint4*>(s.otile + q * kDnTile + ch * 8);
        }
        named_barrier_sync(1, kConsumers);
    }
}

size_t gateup_smem(int NT, int H, int E, bool q = false) {
    return q ? smem_bytes(8 * NT, H + 32, kGuTile, E, H / 128) : smem_bytes(8 * NT, 2 * H + 32, kGuTile, E);
}
size_t down_smem(int NT, int I, int E, bool q = false) {
    return q ? smem_bytes(8 * NT, I + 32, kDnTile, E, I / kGateUpFeat) : smem_bytes(8 * NT, 2 * I + 32, kDnTile, E);
}

int sm_count() {
    static int sms = 0;
    if (!sms) {
        int dev = 0;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        if (sms <= 0) sms = 148;
    }
    return sms;
}

// Persistent grid: every CTA the GPU holds at once, but no more than the items
// of the call could use.
template <class K>
int persistent_grid(K kernel, size_t smem, long max_items, int sm_limit) {
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, kThreads, smem) != cudaSuccess || per_sm < 1)
        per_sm = 1;
    const int sms = sm_limit > 0 ? std::min(sm_limit, sm_count()) : sm_count();
    return static_cast<int>(std::max(1L, std::min(static_cast<long>(per_sm) * sms, max_items)));
}

constexpr size_t kSmemLimit = 227 * 1024;

template <int NT, bool Q>
cudaError_t launch_nt(const FfnArgs& a, const CUtensorMap& tg, const CUtensorMap& tu,
                      const CUtensorMap& td, cudaStream_t stream) {
    const int E = a.ex.n;
    const size_t s1 = gateup_smem(NT, a.H, E, Q), s2 = down_smem(NT, a.ex.inter, E, Q);
    cudaError_t err = cudaFuncSetAttribute(gateup_decode_kernel<NT, Q>,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(s1));
    if (err != cudaSuccess) return err;
    err = cudaFuncSetAttribute(down_decode_kernel<NT, Q>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(s2));
    if (err != cudaSuccess) return err;
    const int g1 =
        persistent_grid(gateup_decode_kernel<NT, Q>, s1, static_cast<long>(E) * (a.ex.inter / kGateUpFeat), a.sm_limit);
    const int g2 =
        persistent_grid(down_decode_kernel<NT, Q>, s2, static_cast<long>(E) * (a.H / kDownRows), a.sm_limit);
    gateup_decode_kernel<NT, Q><<<g1, kThreads, s1, stream>>>(tg, tu, a);
    err = cudaGetLastError();
    if (err != cudaSuccess) return err;

    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(g2);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = s2;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, down_decode_kernel<NT, Q>, td, a);
}

}  // namespace

bool ffn_decode_supported(int H, int I) {
    return H % kDownRows == 0 && I % kGateUpFeat == 0 && gateup_smem(1, H, MOE_MAX_E) <= kSmemLimit &&
           down_smem(1, I, MOE_MAX_E) <= kSmemLimit;
}

cudaError_t launch_ffn_decode(const FfnArgs& a, cudaStream_t stream) {
    CUtensorMap tg, tu, td;
    const uint64_t E = static_cast<uint64_t>(a.ex.n), I = a.ex.inter, H = a.H;
    cudaError_t err = make_tmap_u8_2d(&tg, a.ex.w_gate, E * I, H, 128, kGateUpFeat);
    if (err == cudaSuccess) err = make_tmap_u8_2d(&tu, a.ex.w_up, E * I, H, 128, kGateUpFeat);
    if (err == cudaSuccess) err = make_tmap_u8_2d(&td, a.ex.w_down, E * H, I, 128, kDownRows);
    if (err != cudaSuccess) return err;
    // Token tile: the host only knows the average rows per expert.
    int NT = a.avg_rows > 12 ? 4 : (a.avg_rows > 6 ? 2 : 1);
    while (NT > 1 && (gateup_smem(NT, a.H, a.ex.n, a.w8a8) > kSmemLimit ||
                      down_smem(NT, a.ex.inter, a.ex.n, a.w8a8) > kSmemLimit))
        NT >>= 1;
    if (a.w8a8) {
        switch (NT) {
            case 4: return launch_nt<4, true>(a, tg, tu, td, stream);
            case 2: return launch_nt<2, true>(a, tg, tu, td, stream);
            default: return launch_nt<1, true>(a, tg, tu, td, stream);
        }
    }
    switch (NT) {
        case 4: return launch_nt<4, false>(a, tg, tu, td, stream);
        case 2: return launch_nt<2, false>(a, tg, tu, td, stream);
        default: return launch_nt<1, false>(a, tg, tu, td, stream);
    }
}

}  // namespace moe
