// router.h -- internal host-side interface of the fused router (moe_router).
#pragma once

#include "launch.h"

namespace moe {

// ---------------------------------------------------------------- fused router
// Launch shape of the fused router for T tokens and E experts: `tiles` tiles
// of 128 tokens, `cn` CTAs per tile (a cluster), `ne` experts per CTA.
struct RouterPlan {
    int tiles, cn, ne, stages, tmem_cols, S, xrows, kch;
    size_t smem;
};
// kch: 64-column chunks per K stage (1, 2 or 4; H / 64 a multiple of it).
RouterPlan plan_router(int T, int H, int E, int kch_max);
// Name of the first plan field that breaks the kernel's indexing invariants, or nullptr.
const char* router_plan_violation(const RouterPlan& p, int H, int E);
// x [rows, cols] bf16 viewed as (64 columns, rows, cols / 64 chunks), box
// 64 x box_rows x box_chunks, 128-byte swizzle (cols a multiple of 64).
cudaError_t make_tmap_bf16_kchunks(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols,
                                   uint32_t box_rows, uint32_t box_chunks);
// tx: x [T, H] bf16, tw: w_router [E, H] bf16; boxes of 64 columns x plan.xrows (x) or
// plan.ne (w_router) rows: 2-D maps (make_tmap_bf16_2d) when plan.kch == 1, else 3-D maps of
// plan.kch chunks (make_tmap_bf16_kchunks).
cudaError_t launch_router(const RouterPlan& plan, const CUtensorMap& tx, const CUtensorMap& tw, int T, int H, int E,
                          int K,
                          const RouteCfg& cfg, const uint8_t* zero_mask, int32_t* ids, float* w, float* logits,
                          int32_t* status, cudaStream_t stream);

}  // namespace moe
