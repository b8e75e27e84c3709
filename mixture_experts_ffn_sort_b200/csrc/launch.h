// launch.h -- internal host-side launchers of the library's kernels (C++ only;
// the public boundary is include/moe_ffn.h).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace moe {

// ---------------------------------------------------------------- route
cudaError_t launch_route(const float* logits, int T, int E, int K, const uint8_t* zero_mask,
                         int32_t* ids, float* w, cudaStream_t stream);
// Routing variants (moe_route_ex); the fields as in moe_route_config.
struct RouteCfg {
    int score;
    const float* bias;
    int n_group;
    int topk_group;
    int renormalize;
    float scaling;
};
cudaError_t launch_route_ex(const float* logits, int T, int E, int K, const RouteCfg& cfg,
                            const uint8_t* zero_mask, int32_t* ids, float* w, cudaStream_t stream);

// ---------------------------------------------------------------- sort
// Routes per tile (one thread block) of the multi-kernel sort, and the largest route count
// handled by the single-block sort.
constexpr int kSortChunk = 2048;
constexpr long kSortSmallMaxRoutes = 16384;
size_t sort_workspace_bytes(long R, int E);
cudaError_t launch_sort(const int32_t* ids, long R, int E, int32_t* offsets, int32_t* sorted_route,
                        int32_t* inv_route, void* ws, int32_t* status, cudaStream_t stream);

// ---------------------------------------------------------------- combine
cudaError_t launch_combine(const uint16_t* y_sorted, const int32_t* inv_route,
                           const uint16_t* y_shared, int T, int K, int H, void* out, int out_f32,
                           int32_t* status, cudaStream_t stream);

// ---------------------------------------------------------------- expert FFN (decode)
// One projection set of experts as the kernels see it.
struct ExpertsView {
    const uint8_t* w_gate;
    const uint8_t* w_up;
    const uint8_t* w_down;
    const float* s_gate;
    const float* s_up;
    const float* s_down;
    int n;      // experts
    int inter;  // I
};

struct FfnArgs {
    const uint16_t* x;  // [T, H]
    int T, H, K;
    ExpertsView ex;
    // Rows of this call: either routed (offsets / sorted_route / topk_w) or
    // the identity group of all T tokens with weight 1 (shared expert).
    bool identity;
    const int32_t* offsets;
    const int32_t* sorted_route;
    const float* topk_w;
    uint16_t* h;  // [rows, I] bf16 scratch
    uint16_t* y;  // [rows, H] bf16 output
    int32_t* status;
    int avg_rows;  // host-known rows per expert (sizes the token tile)
    // Prefill form only: an always-on expert run in the same launches as the
    // routed rows (its rows are the T tokens in order, route weight 1).
    ExpertsView sh;  // sh.n == 0: none
    uint16_t* h_sh;  // [T, sh.inter] bf16 scratch
    uint16_t* y_sh;  // [T, H] bf16 output
    // Split of the routed experts between the two forms (MOE_MODE_HYBRID):
    // when > 0, the decode form takes the experts with 1..row_split rows and
    // the prefill form those with more; 0 = every expert.
    int row_split;
    // Prefill form only: scratch for the f16 copy of x ([T, H], each row
    // scaled by a power of two, see launch_ffn_prefill) and the inverse row
    // scales ([T] f32).
    uint16_t* x16;
    float* xinv;
    // Prefill form only: when not null, the down epilogue adds each row's
    // bf16 result (route weight applied) into out_acc[token] ([T, H] f32, zeroed
    // by the caller) with fp32 reductions instead of storing y / y_sh.
    float* out_acc;
    // Decode form only, W8A8: the activations of both GEMMs as E4M3FN codes in
    // blocks with power-of-two scales (x: 128 columns, quantised as it is
    // staged; h: 64 features, quantised in the gate/up epilogue).  h then holds
    // [rows, I] E4M3FN bytes and hscale [rows, I / 64] the inverse scales 2^-k.
    bool w8a8;
    float* hscale;
    // > 0: the persistent grids use at most this many SMs (MOE_MODE_HYBRID runs
    // the two forms side by side on disjoint SMs).
    int sm_limit;
};

// W8A8 form: the workspace region of h holds the codes and, after them, the scales.
inline size_t ffn_hq_codes_bytes(long rows, int I) { return (static_cast<size_t>(rows) * I + 255) & ~size_t(255); }

// Bytes of the prefill form's f16 activation copy and its row scales (256-byte aligned).
inline size_t ffn_x16_bytes(long T, int H) { return (static_cast<size_t>(T) * H * 2 + 255) & ~size_t(255); }
inline size_t ffn_xinv_bytes(long T) { return (static_cast<size_t>(T) * 4 + 255) & ~size_t(255); }

cudaError_t launch_ffn_decode(const FfnArgs& a, cudaStream_t stream);

// ---------------------------------------------------------------- TMA descriptors
// 2-D row-major uint8 matrix [rows, cols] (cols contiguous), box
// {box_cols, box_rows}, 128-byte (default) or 64-byte swizzle.
cudaError_t make_tmap_u8_2d(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols,
                            uint32_t box_cols, uint32_t box_rows, int swizzle_bytes = 128);
// 2-D row-major bf16 matrix [rows, cols], box {box_cols, box_rows}, 128-byte swizzle.
cudaError_t make_tmap_bf16_2d(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols,
                              uint32_t box_cols, uint32_t box_rows);

// ---------------------------------------------------------------- expert FFN (prefill, tcgen05)
// Routed rows (a.identity must be false) plus the optional shared expert a.sh.
// x16_done: the f16 copy of x (launch_x16) was already launched on the stream.
// gateup_after_decode: the preceding launch is the weight-streaming down
// kernel of the same call, which gate/up overlaps (programmatic dependent
// launch); the hybrid form runs the forms on two streams and does not use it.
cudaError_t launch_ffn_prefill(const FfnArgs& a, cudaStream_t stream, bool x16_done = false,
                               bool gateup_after_decode = false);
// The f16 copy of x and its row scales (a.x16, a.xinv) for the tensor-core kernels.
cudaError_t launch_x16(const FfnArgs& a, cudaStream_t stream);
bool ffn_prefill_supported(int H, int I);
// out[T, H] = bf16(acc[T, H]) (the last step of the fused down + combine).
cudaError_t launch_acc_to_bf16(const float* acc, long n, uint16_t* out, cudaStream_t stream);

}  // namespace moe
