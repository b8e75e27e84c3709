// combine.cu -- top-K reduce back to token order (moe_combine).
//
// The unpermute-reduce of the Nemotron-H sorted path
// (spark_model/layers/nemotron_moe.rs, `moe_unpermute_reduce_indexed`), the
// FP32 route reduction of the aiter gfx950 prefill PR and the NKI Top-K Reduce
// kernel: out[t] = sum_j y_sorted[inv_route[t*K + j]] (+ y_shared[t]), summed
// in fp32 in slot order, rounded once.  Each thread owns 8 consecutive
// columns of one token and reads them with 16-byte loads.  A position outside
// [0, T*K) other than -1 is a corrupt map: that term is skipped (never read
// out of bounds) and MOE_STATUS_BAD_MAP is OR-ed into the status word.
#include "device_common.cuh"
#include "launch.h"

namespace moe {

namespace {

__device__ __forceinline__ void add_bf16x8(float (&acc)[8], const uint4& v) {
    const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        acc[2 * i] += __uint_as_float(u[i] << 16);
        acc[2 * i + 1] += __uint_as_float(u[i] & 0xFFFF0000u);
    }
}

template <bool OUT_F32>
__global__ void __launch_bounds__(256) combine_kernel(const uint16_t* __restrict__ y_sorted,
                                                      const int32_t* __restrict__ inv_route,
                                                      const uint16_t* __restrict__ y_shared,
                                                      int T, int K, int H, void* __restrict__ out,
                                                      int32_t* __restrict__ status) {
    const int chunks = H >> 3;
    const long total = static_cast<long>(T) * chunks;
    const long R = static_cast<long>(T) * K;
    bool bad = false;
    for (long idx = static_cast<long>(blockIdx.x) * blockDim.x + threadIdx.x; idx < total;
         idx += static_cast<long>(gridDim.x) * blockDim.x) {
        const int t = static_cast<int>(idx / chunks);
        const int c = static_cast<int>(idx - static_cast<long>(t) * chunks);
        float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        // Slots in batches of 8: all positions, then all rows, then the sums
        // in slot order (independent loads overlap; the order of the fp32
        // additions is unchanged).
        for (int j0 = 0; j0 < K; j0 += 8) {
            int32_t p[8];
#pragma unroll
            for (int jj = 0; jj < 8; ++jj) {
                p[jj] = j0 + jj < K ? __ldg(inv_route + static_cast<size_t>(t) * K + j0 + jj) : -1;
                if (p[jj] >= R || p[jj] < -1) {
                    bad = true;
                    p[jj] = -1;
                }
            }
            uint4 v[8];
#pragma unroll
            for (int jj = 0; jj < 8; ++jj)
                v[jj] = p[jj] >= 0
                            ? __ldg(reinterpret_cast<const uint4*>(y_sorted + static_cast<size_t>(p[jj]) * H) + c)
                            : make_uint4(0, 0, 0, 0);
#pragma unroll
            for (int jj = 0; jj < 8; ++jj)
                if (p[jj] >= 0) add_bf16x8(acc, v[jj]);
        }
        if (y_shared) {
            const uint4 v = __ldg(reinterpret_cast<const uint4*>(y_shared + static_cast<size_t>(t) * H) + c);
            add_bf16x8(acc, v);
        }
        if (OUT_F32) {
            float4* o = reinterpret_cast<float4*>(static_cast<float*>(out) + static_cast<size_t>(t) * H) + 2 * c;
            o[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
            o[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
        } else {
            uint4 r;
            r.x = pack_bf16x2(acc[0], acc[1]);
            r.y = pack_bf16x2(acc[2], acc[3]);
            r.z = pack_bf16x2(acc[4], acc[5]);
            r.w = pack_bf16x2(acc[6], acc[7]);
            reinterpret_cast<uint4*>(static_cast<uint16_t*>(out) + static_cast<size_t>(t) * H)[c] = r;
        }
    }
    if (bad) report_status(status, MOE_STATUS_BAD_MAP);
}

}  // namespace

cudaError_t launch_combine(const uint16_t* y_sorted, const int32_t* inv_route,
                           const uint16_t* y_shared, int T, int K, int H, void* out, int out_f32,
                           int32_t* status, cudaStream_t stream) {
    const long total = static_cast<long>(T) * (H >> 3);
    const int threads = 256;
    long blocks = (total + threads - 1) / threads;
    if (blocks > 148L * 64) blocks = 148L * 64;
    if (out_f32)
        combine_kernel<true><<<static_cast<int>(blocks), threads, 0, stream>>>(y_sorted, inv_route,
                                                                                y_shared, T, K, H, out, status);
    else
        combine_kernel<false><<<static_cast<int>(blocks), threads, 0, stream>>>(y_sorted, inv_route,
                                                                                 y_shared, T, K, H, out, status);
    return cudaGetLastError();
}

}  // namespace moe
