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

// Order-preserving integer key of a float (larger float -> larger key; -0 and
// +0 share a key) and its inverse.
__device__ __forceinline__ uint32_t order_key(float v) {
    const uint32_t u = __float_as_uint(v == 0.f ? 0.f : v);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float key_value(uint32_t k) {
    return __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k);
}

// Routing variants (moe_route_ex).  One warp per token, as route_kernel:
// lane `lane` holds experts lane + 32 i.  Scores s (softmax or sigmoid, fp32),
// selection keys c = s + bias (or the logit itself when there is neither a
// bias nor a group limit), then, with groups, each group's score (sum of its
// two largest c, found by two warp arg-max passes) lands on lane g and
// topk_group warp arg-max passes over the lanes keep the best groups; the
// experts of the other groups are marked taken.  K warp arg-max rounds pick
// the experts; the chosen expert's s is read from its owner lane.
template <int EPL>
__global__ void __launch_bounds__(256) route_ex_kernel(const float* __restrict__ logits, int T, int E, int K,
                                                       const RouteCfg cfg, const uint8_t* __restrict__ zero_mask,
                                                       int32_t* __restrict__ ids, float* __restrict__ w) {
    const int lane = threadIdx.x & 31;
    const int t = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    if (t >= T) return;
    const float* l = logits + static_cast<size_t>(t) * E;
    const uint32_t full = 0xffffffffu;

    float s[EPL], c[EPL];
    uint32_t taken = 0;  // bit i: expert lane + 32 i chosen, ineligible or padding
    float lmax = -INFINITY;
#pragma unroll
    for (int i = 0; i < EPL; ++i) {
        const int e = lane + 32 * i;
        if (e < E) {
            c[i] = __ldg(l + e);
            lmax = fmaxf(lmax, c[i]);
        } else {
            c[i] = -INFINITY;
            taken |= 1u << i;
        }
    }
    if (cfg.score == MOE_SCORE_SOFTMAX) {
        lmax = key_value(__reduce_max_sync(full, order_key(lmax)));
        float z = 0.f;
#pragma unroll
        for (int i = 0; i < EPL; ++i) {
            s[i] = (taken >> i) & 1u ? 0.f : expf(c[i] - lmax);
            z += s[i];
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) z += __shfl_xor_sync(full, z, off);
#pragma unroll
        for (int i = 0; i < EPL; ++i) s[i] = s[i] / z;
    } else {
#pragma unroll
        for (int i = 0; i < EPL; ++i) s[i] = (taken >> i) & 1u ? 0.f : 1.f / (1.f + expf(-c[i]));
    }
    // Selection keys: the logit itself (exact) unless a bias or groups need s.
    if (cfg.bias || cfg.n_group > 1) {
#pragma unroll
        for (int i = 0; i < EPL; ++i) {
            const int e = lane + 32 * i;
            if (!((taken >> i) & 1u)) c[i] = s[i] + (cfg.bias ? __ldg(cfg.bias + e) : 0.f);
        }
    }

    if (cfg.n_group > 1) {
        const int G = E / cfg.n_group;
        int grp[EPL];
#pragma unroll
        for (int i = 0; i < EPL; ++i) grp[i] = (lane + 32 * i) / G;
        float gs = 0.f;  // lane g: score of group g
        for (int g = 0; g < cfg.n_group; ++g) {
            float top = 0.f;
            int skip = -1;  // the group's largest, excluded from the second pass
            for (int pass = 0; pass < (G > 1 ? 2 : 1); ++pass) {
                uint32_t key = 0;
                int bi = 0x7fffffff;
#pragma unroll
                for (int i = 0; i < EPL; ++i) {
                    const int e = lane + 32 * i;
                    if (e < E && grp[i] == g && e != skip) {
                        const uint32_t k = order_key(c[i]);
                        if (k > key) {
                            key = k;
                            bi = e;
                        }
                    }
                }
                const uint32_t kmax = __reduce_max_sync(full, key);
                skip = static_cast<int>(__reduce_min_sync(full, key == kmax ? static_cast<uint32_t>(bi) : 0xffffffffu));
                top += key_value(kmax);
            }
            if (lane == g) gs = top;
        }
        uint32_t keep = 0;
        for (int r = 0; r < cfg.topk_group; ++r) {
            const bool cand = lane < cfg.n_group && !((keep >> lane) & 1u);
            const uint32_t key = cand ? order_key(gs) : 0u;
            const uint32_t kmax = __reduce_max_sync(full, key);
            const uint32_t gsel = __reduce_min_sync(full, cand && key == kmax ? static_cast<uint32_t>(lane) : 31u);
            keep |= 1u << gsel;
        }
#pragma unroll
        for (int i = 0; i < EPL; ++i)
            if (grp[i] >= 32 || !((keep >> grp[i]) & 1u)) taken |= 1u << i;  // padding: grp may pass 31
    }

    float sum = 0.f, my_s = 0.f;
    int my_id = 0;
    for (int j = 0; j < K; ++j) {
        uint32_t key = 0;
        int bi = 0x7fffffff;
#pragma unroll
        for (int i = 0; i < EPL; ++i) {
            if ((taken >> i) & 1u) continue;
            const uint32_t k = order_key(c[i]);
            if (k > key) {  // ascending i: the first of equal keys keeps the lower id
                key = k;
                bi = lane + 32 * i;
            }
        }
        const uint32_t kmax = __reduce_max_sync(full, key);
        bi = static_cast<int>(__reduce_min_sync(full, key == kmax ? static_cast<uint32_t>(bi) : 0xffffffffu));
        if (bi >= E) bi = E - 1;  // only reachable with NaN logits (unspecified ids)
        float sv = 0.f;
#pragma unroll
        for (int i = 0; i < EPL; ++i)
            if (i == (bi >> 5)) sv = s[i];
        sv = __shfl_sync(full, sv, bi & 31);
        if ((bi & 31) == lane) taken |= 1u << (bi >> 5);
        sum += sv;
        if (lane == j) {
            my_id = bi;
            my_s = sv;
        }
    }
    if (lane < K) {
        const size_t o = static_cast<size_t>(t) * K + lane;
        float wv = (cfg.renormalize ? my_s / sum : my_s) * cfg.scaling;
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

cudaError_t launch_route_ex(const float* logits, int T, int E, int K, const RouteCfg& cfg,
                            const uint8_t* zero_mask, int32_t* ids, float* w, cudaStream_t stream) {
    const int threads = 256;
    const int blocks = (T + 7) / 8;
#define MOE_ROUTE_EX_CASE(EPL)                                                                        \
    route_ex_kernel<EPL><<<blocks, threads, 0, stream>>>(logits, T, E, K, cfg, zero_mask, ids, w); \
    break;
    switch ((E + 31) / 32) {
        case 1: MOE_ROUTE_EX_CASE(1)
        case 2: MOE_ROUTE_EX_CASE(2)
        case 3:
        case 4: MOE_ROUTE_EX_CASE(4)
        case 5: case 6: case 7:
        case 8: MOE_ROUTE_EX_CASE(8)
        case 9: case 10: case 11: case 12: case 13: case 14: case 15:
        case 16: MOE_ROUTE_EX_CASE(16)
        default: MOE_ROUTE_EX_CASE(32)
    }
#undef MOE_ROUTE_EX_CASE
    return cudaGetLastError();
}

}  // namespace moe
