// route_device.cuh -- per-token top-K routing, shared by the routing kernel
// (logits read from global memory) and the fused router (logits staged in
// shared memory by the gate GEMM's epilogue).
//
// One warp per token.  Lane `lane` holds experts lane + 32 i as
// order-preserving integer keys (larger key = larger value, -0 == +0; 0 marks
// an expert that cannot be chosen).  The key is the fp32 logit itself when
// there is neither a bias nor a group limit -- both scores are strictly
// increasing in the logit, so ranking logits is exact -- and the fp32
// selection score s + bias otherwise.  With groups, each group's score (the
// sum of its two largest keys' values) comes from lane-local top-two lists
// (groups of a multiple of 32 experts) or from two warp arg-max passes, and
// topk_group arg-max passes over the lanes keep the best groups.  K rounds of
// a warp arg-max (two redux.sync: largest key, then lowest expert id holding
// it) pick the experts in descending order, over the few candidate keys a
// threshold leaves when it can (see the selection below).  The chosen experts' scores are
// then recomputed from their logits, lane j taking choice j: softmax weights
// are exp(l_j - l_max) over their sum (renormalised; the full-softmax
// normaliser cancels) or over the full normaliser, sigmoid weights
// 1 / (1 + exp(-l_j)); the sum is a warp butterfly.
#pragma once

#include <math.h>

#include "device_common.cuh"
#include "launch.h"

namespace moe {

// Order-preserving integer key of a float (larger float -> larger key; -0 and
// +0 share a key; every key is nonzero) and its inverse.
__device__ __forceinline__ uint32_t order_key(float v) {
    const uint32_t u = __float_as_uint(v == 0.f ? 0.f : v);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float key_value(uint32_t k) {
    return __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k);
}

__device__ __forceinline__ float sigmoid(float x) { return __frcp_rn(1.f + expf(-x)); }

// Logit loads: through the read-only path from global memory, or plain (shared memory).
struct LoadGlobal {
    __device__ __forceinline__ float operator()(const float* p) const { return __ldg(p); }
};
struct LoadPlain {
    __device__ __forceinline__ float operator()(const float* p) const { return *p; }
};

// Route token t from its E logits `lg` (one warp, all lanes; see above).
// COMPUTED: rank by s (+ bias) -- a bias or a group limit is present.
// logits_out (optional): row t of a [T, E] f32 copy of the logits.
template <int EPL, bool COMPUTED, class Load>
__device__ __forceinline__ void route_token(const float* lg, int t, int E, int K, const RouteCfg& cfg,
                                            const uint8_t* __restrict__ zero_mask, int32_t* __restrict__ ids,
                                            float* __restrict__ w, float* __restrict__ logits_out) {
    const Load ld;
    const int lane = threadIdx.x & 31;
    const uint32_t full = 0xffffffffu;
    const bool softmax = cfg.score == MOE_SCORE_SOFTMAX;

    float l[EPL];
    float lmax = -INFINITY;
#pragma unroll
    for (int i = 0; i < EPL; ++i) {
        const int e = lane + 32 * i;
        l[i] = e < E ? ld(lg + e) : -INFINITY;
        lmax = fmaxf(lmax, l[i]);
    }
    if (logits_out) {
        float* o = logits_out + static_cast<size_t>(t) * E;
#pragma unroll
        for (int i = 0; i < EPL; ++i)
            if (lane + 32 * i < E) o[lane + 32 * i] = l[i];
    }
    float z = 1.f;  // softmax normaliser (sum of exp(l - l_max))
    if (softmax) {
        lmax = key_value(__reduce_max_sync(full, order_key(lmax)));
        if (COMPUTED || !cfg.renormalize) {
            z = 0.f;
#pragma unroll
            for (int i = 0; i < EPL; ++i) z += lane + 32 * i < E ? expf(l[i] - lmax) : 0.f;
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) z += __shfl_xor_sync(full, z, off);
        }
    }
    uint32_t key[EPL];
#pragma unroll
    for (int i = 0; i < EPL; ++i) {
        const int e = lane + 32 * i;
        float c = l[i];
        if (COMPUTED && e < E) {
            c = softmax ? expf(l[i] - lmax) / z : sigmoid(l[i]);
            if (cfg.bias) c += __ldg(cfg.bias + e);
        }
        key[i] = e < E ? order_key(c) : 0u;
    }

    if (COMPUTED && cfg.n_group > 1) {
        const int G = E / cfg.n_group;
        float gs = 0.f;  // lane g: score of group g
        if (G % 32 == 0) {
            // Group of register i: i / (G / 32).  Lane-local top two of each
            // group, then the group's best (largest lane top) and second best
            // (the winner lane's second or another lane's top).
            const int rpg = G / 32;
            for (int g = 0; g < cfg.n_group; ++g) {
                uint32_t a = 0, b = 0;
#pragma unroll
                for (int i = 0; i < EPL; ++i) {
                    if (i / rpg != g) continue;
                    const uint32_t k = key[i];
                    if (k > a) {
                        b = a;
                        a = k;
                    } else if (k > b) {
                        b = k;
                    }
                }
                const uint32_t k1 = __reduce_max_sync(full, a);
                const uint32_t win = __reduce_min_sync(full, a == k1 ? static_cast<uint32_t>(lane) : 32u);
                const uint32_t k2 = __reduce_max_sync(full, lane == static_cast<int>(win) ? b : a);
                if (lane == g) gs = key_value(k1) + key_value(k2);
            }
        } else {
            // Any group size: two warp arg-max passes per group.
            for (int g = 0; g < cfg.n_group; ++g) {
                float top = 0.f;
                int skip = -1;  // the group's best expert, excluded from the second pass
                for (int pass = 0; pass < (G > 1 ? 2 : 1); ++pass) {
                    uint32_t best = 0;
                    int bi = 0x7fffffff;
#pragma unroll
                    for (int i = 0; i < EPL; ++i) {
                        const int e = lane + 32 * i;
                        if (e / G == g && e != skip && key[i] > best) {
                            best = key[i];
                            bi = e;
                        }
                    }
                    const uint32_t kmax = __reduce_max_sync(full, best);
                    skip = static_cast<int>(
                        __reduce_min_sync(full, best == kmax ? static_cast<uint32_t>(bi) : 0xffffffffu));
                    top += key_value(kmax);
                }
                if (lane == g) gs = top;
            }
        }
        uint32_t keep = 0;
        for (int r = 0; r < cfg.topk_group; ++r) {
            const bool cand = lane < cfg.n_group && !((keep >> lane) & 1u);
            const uint32_t k = cand ? order_key(gs) : 0u;
            const uint32_t kmax = __reduce_max_sync(full, k);
            keep |= 1u << __reduce_min_sync(full, cand && k == kmax ? static_cast<uint32_t>(lane) : 31u);
        }
#pragma unroll
        for (int i = 0; i < EPL; ++i) {
            const int g = (lane + 32 * i) / G;  // >= 32 only for padding, whose key is already 0
            if (g >= 32 || !((keep >> g) & 1u)) key[i] = 0u;
        }
    }

    // Lane j keeps the j-th choice's id and logit; the scores are computed
    // after the K rounds, one per lane, and summed across the warp.
    float my_l = 0.f;
    int my_id = 0;
    // theta = the K-th largest of the lanes' largest keys.  At least K keys
    // are >= theta, so every chosen key is: the candidates (nonzero keys >=
    // theta) are few.  Each lane keeps its four best candidates in order
    // (key descending, then expert id ascending); when no lane has more than
    // four, the K rounds take the best lane head and advance that lane,
    // otherwise they scan every key.
    uint32_t theta = 0;
    {
        uint32_t m = 0;
#pragma unroll
        for (int i = 0; i < EPL; ++i) m = key[i] > m ? key[i] : m;
        for (int j = 0; j < K; ++j) {
            theta = __reduce_max_sync(full, m);
            const uint32_t win = __reduce_min_sync(full, m == theta ? static_cast<uint32_t>(lane) : 32u);
            if (lane == static_cast<int>(win)) m = 0;
        }
    }
    uint32_t h0 = 0, h1 = 0, h2 = 0, h3 = 0;
    int i0 = 0, i1 = 0, i2 = 0, i3 = 0, cnt = 0;
#pragma unroll
    for (int i = 0; i < EPL; ++i) {
        const uint32_t k = key[i];
        if (k != 0u && k >= theta) {
            ++cnt;
            if (k > h3) {  // a key equal to one held goes after it (larger expert id)
                if (k > h2) {
                    h3 = h2; i3 = i2;
                    if (k > h1) {
                        h2 = h1; i2 = i1;
                        if (k > h0) {
                            h1 = h0; i1 = i0; h0 = k; i0 = i;
                        } else {
                            h1 = k; i1 = i;
                        }
                    } else {
                        h2 = k; i2 = i;
                    }
                } else {
                    h3 = k; i3 = i;
                }
            }
        }
    }
    if (__all_sync(full, cnt <= 4)) {
        for (int j = 0; j < K; ++j) {
            const uint32_t kmax = __reduce_max_sync(full, h0);
            int e = static_cast<int>(
                __reduce_min_sync(full, h0 == kmax && kmax ? static_cast<uint32_t>(lane + 32 * i0) : 0xffffffffu));
            // With no candidate left (kmax == 0) the min's sentinel casts to -1.
            // That needs fewer than K nonzero keys, i.e. NaN logits whose key is 0
            // (sign bit set); such a token's ids are unspecified but stay in [0, E).
            if (e < 0 || e >= E) e = E - 1;
            if (lane == (e & 31)) {
                h0 = h1; i0 = i1; h1 = h2; i1 = i2; h2 = h3; i2 = i3; h3 = 0u;
            }
            if (lane == j) {
                my_id = e;
                // The chosen logit: the key itself when ranking by logit, else reloaded.
                my_l = COMPUTED ? ld(lg + e) : key_value(kmax);
            }
        }
    } else {
        for (int j = 0; j < K; ++j) {
            uint32_t best = 0;
            int bi = 0;
#pragma unroll
            for (int i = 0; i < EPL; ++i) {
                if (key[i] > best) {  // ascending i: equal keys keep the lower expert id
                    best = key[i];
                    bi = i;
                }
            }
            const uint32_t kmax = __reduce_max_sync(full, best);
            int e = static_cast<int>(
                __reduce_min_sync(full, best == kmax && best ? static_cast<uint32_t>(lane + 32 * bi) : 0xffffffffu));
            if (e < 0 || e >= E) e = E - 1;
            const int slot = e >> 5;
            if (lane == (e & 31)) {
#pragma unroll
                for (int i = 0; i < EPL; ++i)
                    if (i == slot) key[i] = 0u;
            }
            if (lane == j) {
                my_id = e;
                my_l = COMPUTED ? ld(lg + e) : key_value(kmax);
            }
        }
    }
    const float mine = lane < K ? (softmax ? expf(my_l - lmax) : sigmoid(my_l)) : 0.f;
    float sum = mine;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(full, sum, off);
    if (lane < K) {
        const size_t o = static_cast<size_t>(t) * K + lane;
        float wv = cfg.renormalize ? mine / sum : mine / z;  // z = 1 for sigmoid scores
        wv *= cfg.scaling;
        if (zero_mask && zero_mask[o]) wv = 0.f;
        ids[o] = my_id;
        w[o] = wv;
    }
}

}  // namespace moe
