// router.h -- internal host-side interface of the fused router (moe_router).
#pragma once

#include "launch.h"

namespace moe {

// ---------------------------------------------------------------- fused router
// Launch shape of the fused router for T tokens and E experts: `tiles` tiles
// of 128 tokens, `cn` CTAs per tile (a cluster), `ne` experts per CTA.
struct RouterPlan {
    int tiles, cn, ne, stages, tmem_cols, S, xrows;
    size_t smem;
};
RouterPlan plan_router(int T, int E);
// tx: x [T, H] bf16, box 64 x plan.xrows; tw: w_router [E, H] bf16, box 64 x plan.ne.
cudaError_t launch_router(const CUtensorMap& tx, const CUtensorMap& tw, int T, int H, int E, int K,
                          const RouteCfg& cfg, const uint8_t* zero_mask, int32_t* ids, float* w, float* logits,
                          int32_t* status, cudaStream_t stream);

}  // namespace moe
