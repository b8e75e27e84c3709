// route.cu -- top-K routing (moe_route, moe_route_ex).
//
// moe_route is the router of the FP8 MoE decode kernel page's serving
// contract (softmax, top-8, renormalise; dstair/gated-deltanet-nki-trainium)
// and the NKI Router Top-K kernel; moe_route_ex adds the variants the pages
// name (the Nemotron-H layer's sigmoid top-K with a routed scaling factor,
// spark_model/layers/nemotron_moe.rs; the NKI library's DeepSeek-V3
// group-limited router) in the published DeepSeek-V3 form: a selection-only
// bias, groups scored by the sum of their two best experts, a kept-group
// limit, optional renormalisation and a scaling factor.
//
// One warp per token (route_token, route_device.cuh).
#include "route_device.cuh"

namespace moe {

namespace {

template <int EPL, bool COMPUTED>
__global__ void __launch_bounds__(256) route_kernel(const float* __restrict__ logits, int T, int E, int K,
                                                    const RouteCfg cfg, const uint8_t* __restrict__ zero_mask,
                                                    int32_t* __restrict__ ids, float* __restrict__ w) {
    const int t = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    if (t >= T) return;
    route_token<EPL, COMPUTED, LoadGlobal>(logits + static_cast<size_t>(t) * E, t, E, K, cfg, zero_mask, ids, w,
                                          nullptr);
}

}  // namespace

cudaError_t launch_route_ex(const float* logits, int T, int E, int K, const RouteCfg& cfg,
                            const uint8_t* zero_mask, int32_t* ids, float* w, cudaStream_t stream) {
    const int threads = 256;
    const int blocks = (T + 7) / 8;
    const bool computed = cfg.bias != nullptr || cfg.n_group > 1;
#define MOE_ROUTE_CASE(EPL)                                                                                  \
    if (computed)                                                                                            \
        route_kernel<EPL, true><<<blocks, threads, 0, stream>>>(logits, T, E, K, cfg, zero_mask, ids, w);   \
    else                                                                                                     \
        route_kernel<EPL, false><<<blocks, threads, 0, stream>>>(logits, T, E, K, cfg, zero_mask, ids, w);  \
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

cudaError_t launch_route(const float* logits, int T, int E, int K, const uint8_t* zero_mask, int32_t* ids,
                         float* w, cudaStream_t stream) {
    const RouteCfg plain{MOE_SCORE_SOFTMAX, nullptr, 1, 1, 1, 1.f};
    return launch_route_ex(logits, T, E, K, plain, zero_mask, ids, w, stream);
}

}  // namespace moe
