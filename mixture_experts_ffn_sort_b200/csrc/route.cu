// route.cu -- softmax top-K routing with renormalisation (moe_route).
//
// Router of the FP8 MoE decode kernel page's serving contract ("softmax ->
// top-8 -> norm", dstair/gated-deltanet-nki-trainium) and the NKI Router Top-K
// kernel.  One warp per token: each lane holds ceil(E/32) logits in registers;
// K rounds of a warp-wide arg-max (larger logit first, lower expert id on ties;
// two redux.sync reductions on an order-preserving key) pick the experts in
// descending order.  Softmax is strictly increasing in the
// logit, so this is the top-K of the probabilities; the weights are
// exp(l_j - l_max) / sum_j' exp(l_j' - l_max), the full-softmax normaliser
// cancelling in the renormalisation.
#include <math.h>

#include "device_common.cuh"
#include "launch.h"

namespace moe {

template <int EPL>
__global__ void __launch_bounds__(256) route_kernel(const float* __restrict__ logits, int T, int E,
                                                    int K, const uint8_t* __restrict__ zero_mask,
                                                    int32_t* __restrict__ ids,
                                                    float* __restrict__ w) {
    const int lane = threadIdx.x & 31;
    const int t = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    if (t >= T) return;
    const float* l = logits + static_cast<size_t>(t) * E;

    float v[EPL];
    uint32_t taken = 0;  // bit i: element lane + 32 i already chosen (or padding)
#pragma unroll
    for (int i = 0; i < EPL; ++i) {
        const int e = lane + 32 * i;
        if (e < E) {
            v[i] = __ldg(l + e);
        } else {
            v[i] = -INFINITY;
            taken |= 1u << i;
        }
    }

    float lmax = 0.f, sum = 0.f, my_ex = 0.f;
    int my_id = 0;
    for (int j = 0; j < K; ++j) {
        float bv = -INFINITY;
        int bi = 0x7fffffff;
#pragma unroll
        for (int i = 0; i < EPL; ++i) {
            const int e = lane + 32 * i;
            const bool free_ = !((taken >> i) & 1u);
            if (free_ && (v[i] > bv || (v[i] == bv && e < bi))) {
                bv = v[i];
                bi = e;
            }
        }
        // Warp arg-max: the largest value, then the lowest expert id holding it,
        // as two warp reductions on an order-preserving integer key.
        const float bz = bv == 0.f ? 0.f : bv;  // -0 and +0 are the same logit
        const uint32_t u = __float_as_uint(bz);
        const uint32_t key = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
        const uint32_t kmax = __reduce_max_sync(0xffffffffu, key);
        bi = static_cast<int>(__reduce_min_sync(0xffffffffu, key == kmax ? static_cast<uint32_t>(bi) : 0xffffffffu));
        bv = __uint_as_float((kmax & 0x80000000u) ? (kmax & 0x7fffffffu) : ~kmax);
        if (bi >= E) bi = E - 1;  // only reachable with NaN logits (unspecified ids)
        if ((bi & 31) == lane) taken |= 1u << (bi >> 5);
        if (j == 0) lmax = bv;
        const float ex = expf(bv - lmax);
        sum += ex;
        if (lane == j) {
            my_id = bi;
            my_ex = ex;
        }
    }
    if (lane < K) {
        const size_t o = static_cast<size_t>(t) * K + lane;
        float wv = my_ex / sum;
        if (zero_mask && zero_mask[o]) wv = 0.f;
        ids[o] = my_id;
        w[o] = wv;
    }
}

cudaError_t launch_route(const float* logits, int T, int E, int K, const uint8_t* zero_mask,
                         int32_t* ids, float* w, cudaStream_t stream) {
    const int threads = 256;
    const int blocks = (T + 7) / 8;
#define MOE_ROUTE_CASE(EPL)                                                                    \
    route_kernel<EPL><<<blocks, threads, 0, stream>>>(logits, T, E, K, zero_mask, ids, w); \
    break;
    switch ((E + 31) / 32) {
        case 1: MOE_ROUTE_CASE(1)
        case 2: MOE_ROUTE_CASE(2)
        case 3:
        case 4: MOE_ROUTE_CASE(4)
        case 5: case 6: case 7:
        case 8: MOE_ROUTE_CASE(8)
        case 9: case 10: case 11: case 12: case 13: case 14: case 15:
        case 16: MOE_ROUTE_CASE(16)
        default: MOE_ROUTE_CASE(32)
    }
#undef MOE_ROUTE_CASE
    return cudaGetLastError();
}

}  // namespace moe
