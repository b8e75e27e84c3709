// router.cu -- fused router (moe_router): the gate GEMM logits = x . W_r^T on
// the tensor cores, then top-K routing of each token, in one kernel.
//
// The Nemotron-H layer computes the router as a dense gate GEMM [N, H] x
// [H, E]^T -> [N, E] followed by a top-K kernel
// (spark_model/layers/nemotron_moe.rs, `prefill`, steps 2 and 5), and the NKI
// library ships the two fused (Router Top-K).  Here the logits never reach
// HBM unless the caller asks for a copy.
//
// A tile is 128 tokens (the 128 TMEM lanes).  A cluster of CN CTAs shares a
// tile: CTA c computes the logits of experts [c NE, (c+1) NE) (NE a multiple
// of 16, at most 256: the MMA's N) for all 128 tokens, so small batches still
// spread over CN SMs.  Per CTA:
//   warp 0      TMA: K stages of kch 64-column chunks of the x tile (128
//               rows, or the batch's rows when T < 128, x 128 B per chunk)
//               and of the expert slice of W_r (NE x 128 B per chunk), each
//               chunk a 128-byte-swizzled tile, into a ring of `stages`
//               stages.  kch = 1 loads one chunk per 2-D box; small batches
//               load up to four per 3-D box (64 columns x rows x chunks),
//               because the producer issues boxes at a fixed rate whatever
//               their size;
//   warp 1      TMEM allocation and the MMA issuer: tcgen05.mma kind::f16,
//               A = x chunk, B = W_r chunk (both from shared memory), fp32
//               accumulators in TMEM columns 0..NE-1, four K=16 steps per
//               chunk and a commit that frees the stage;
//   all warps   (16) once every MMA has completed: the accumulators go from
//               TMEM to the shared memory of the CTA that routes each token
//               (token rows split evenly over the cluster, written through
//               distributed shared memory as 16-byte vectors), then each warp
//               routes its tokens with route_token, which also writes the
//               optional logit copy.
// The ring is reused as the staging rows after a cluster barrier (every CTA's
// MMAs have read their stages by then).  Waits on mbarriers are bounded; an
// expired wait records MOE_STATUS_TIMEOUT and the kernel runs to its end.
#include "route_device.cuh"
#include "router.h"
#include "router_common.cuh"

namespace moe {

namespace {

static_assert(kStatusTimeout == MOE_STATUS_TIMEOUT, "timeout status bit of the bounded waits");

constexpr int kRouterThreads = 512;
constexpr int kTileM = 128;             // tokens per tile (TMEM lanes)
constexpr int kKStage = 64;             // bf16 columns per stage: one 128-byte swizzle row
constexpr int kXStageBytes = kTileM * 128;
constexpr int kMaxStages = 16;

struct RouterArgs {
    int T, H, E, K;
    int CN;         // CTAs per tile (cluster size)
    int NE;         // experts per CTA (MMA N): multiple of 16, 16..256
    int stages;     // K stages in the ring
    int tmem_cols;  // allocated TMEM columns (power of two >= max(32, NE))
    int S;          // row stride (floats) of the staging rows
    int xrows;      // token rows a stage loads (128, or T rounded up to 8 when T < 128)
    int kch;        // 64-column chunks per stage
    RouteCfg cfg;
    const uint8_t* zero_mask;
    int32_t* ids;
    float* w;
    float* logits;  // optional [T, E] copy
    int32_t* status;
};

struct RouterBars {
    uint64_t full[kMaxStages], empty[kMaxStages], done;
    uint32_t tmem_base;
    int abort_flag;
};

template <int EPL, bool COMPUTED>
__global__ void __launch_bounds__(kRouterThreads, 1)
    router_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_w,
                  const RouterArgs a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    RouterBars* B = reinterpret_cast<RouterBars*>(smem);
    uint8_t* ring = smem + 1024;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // A stage: kch chunks of the x rows (xrows x 128 B each), then kch chunks
    // of the expert slice (NE x 128 B each), every chunk a 64-column K slice.
    const int xc_bytes = a.xrows * 128, wc_bytes = a.NE * 128;
    const int x_bytes = a.kch * xc_bytes;
    const int stage_bytes = a.kch * (xc_bytes + wc_bytes);
    const uint32_t tx_bytes = static_cast<uint32_t>(stage_bytes);
    const uint32_t rank = cluster_ctarank();
    const int m0 = static_cast<int>(blockIdx.x / a.CN) * kTileM;
    const int e0 = static_cast<int>(rank) * a.NE;
    const int nk = a.H / (kKStage * a.kch);

    if (threadIdx.x == 0) {
        for (int s = 0; s < a.stages; ++s) {
            mbar_init(&B->full[s], 1);
            mbar_init(&B->empty[s], 1);
        }
        mbar_init(&B->done, 1);
        B->abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 1) tmem_alloc(&B->tmem_base, static_cast<uint32_t>(a.tmem_cols));
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = B->tmem_base;
    volatile int* abort_flag = &B->abort_flag;

    if (warp == 0) {
        // ------------------------------------------------ TMA producer
        if (lane == 0) {
            tma_prefetch_desc(&tm_x);
            tma_prefetch_desc(&tm_w);
            for (int k = 0; k < nk; ++k) {
                const int s = k % a.stages;
                if (k >= a.stages)
                    mbar_wait_or_abort(&B->empty[s], static_cast<uint32_t>((k / a.stages - 1) & 1), abort_flag,
                                       a.status);
                uint8_t* st = ring + s * stage_bytes;
                mbar_arrive_expect_tx(&B->full[s], tx_bytes);
                if (a.kch == 1) {  // 2-D maps: box 64 columns x rows
                    tma_load_2d(st, &tm_x, &B->full[s], k * kKStage, m0);
                    tma_load_2d(st + x_bytes, &tm_w, &B->full[s], k * kKStage, e0);
                } else {  // 3-D maps: box 64 columns x rows x kch chunks
                    tma_load_3d(st, &tm_x, &B->full[s], 0, m0, k * a.kch);
                    tma_load_3d(st + x_bytes, &tm_w, &B->full[s], 0, e0, k * a.kch);
                }
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer (whole warp, one elected lane issues)
        const uint32_t idesc = umma_idesc_bf16(kTileM, a.NE);
        const uint32_t ring_u32 = smem_u32(ring);
        for (int k = 0; k < nk; ++k) {
            const int s = k % a.stages;
            mbar_wait_or_abort(&B->full[s], static_cast<uint32_t>((k / a.stages) & 1), abort_flag, a.status);
            tc_fence_after();
            const uint32_t st = ring_u32 + static_cast<uint32_t>(s * stage_bytes);
            for (int j = 0; j < a.kch - 1; ++j)
                umma_ss_f16_x4_elect(tmem, umma_desc_sw128(st + j * xc_bytes),
                                     umma_desc_sw128(st + x_bytes + j * wc_bytes), idesc, k > 0 || j > 0 ? 1u : 0u);
            const int j = a.kch - 1;
            umma_ss_f16_x4_commit_elect(tmem, umma_desc_sw128(st + j * xc_bytes),
                                        umma_desc_sw128(st + x_bytes + j * wc_bytes), idesc,
                                        k > 0 || j > 0 ? 1u : 0u, &B->empty[s]);
        }
        umma_commit_elect(&B->done);
    }

    // ---------------------------------------------------- epilogue (all warps)
    mbar_wait_or_abort(&B->done, 0u, abort_flag, a.status);
    tc_fence_after();
    // Every CTA of the cluster has finished with its ring: it becomes the
    // staging rows, which other CTAs write into.
    cluster_sync_all();

    const int TPC = kTileM / a.CN;  // tokens routed by each CTA of the cluster
    float* stage = reinterpret_cast<float*>(ring);
    {
        // The four warps w with w % 4 == q read TMEM lane quarter q (tile rows
        // 32 q .. 32 q + 31), each a quarter of the 16-column chunks, and store
        // them as 16-byte vectors into the row of the token's routing CTA
        // (row stride S = 4 mod 8 words: the eight rows of a store phase fall
        // in distinct bank groups).
        const int q = warp & 3, part = warp >> 2;
        const int row = 32 * q + lane;
        const uint32_t dst = static_cast<uint32_t>(row / TPC);
        const uint32_t remote =
            cluster_map_shared(smem_u32(stage + static_cast<size_t>(row % TPC) * a.S + e0), dst);
        const int nch = a.NE / 16;
        const int c0 = part * nch / 4, c1 = (part + 1) * nch / 4;
        for (int c = c0; c < c1 && e0 + 16 * c < a.E; ++c) {
            uint32_t v[16];
            tmem_ld32x32b_x16(tmem + (static_cast<uint32_t>(32 * q) << 16) + static_cast<uint32_t>(16 * c), v);
            tmem_ld_wait();
#pragma unroll
            for (int k = 0; k < 4; ++k)
                st_cluster_v4(remote + static_cast<uint32_t>(4 * (16 * c + 4 * k)), v[4 * k], v[4 * k + 1],
                              v[4 * k + 2], v[4 * k + 3]);
        }
    }
    tc_fence_before();
    cluster_sync_all();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem, static_cast<uint32_t>(a.tmem_cols));

    // Route this CTA's tokens: tile rows rank * TPC .. rank * TPC + TPC - 1.
    for (int i = warp; i < TPC; i += kRouterThreads / 32) {
        const int t = m0 + static_cast<int>(rank) * TPC + i;
        if (t >= a.T) break;
        route_token<EPL, COMPUTED, LoadPlain>(stage + static_cast<size_t>(i) * a.S, t, a.E, a.K, a.cfg,
                                              a.zero_mask, a.ids, a.w, a.logits);
    }
}

template <int EPL, bool COMPUTED>
cudaError_t launch_router_t(const CUtensorMap& tx, const CUtensorMap& tw, const RouterArgs& a, int grid,
                            size_t smem, cudaStream_t stream) {
    auto kern = router_kernel<EPL, COMPUTED>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(grid));
    cfg.blockDim = dim3(kRouterThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = static_cast<unsigned>(a.CN);
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, tx, tw, a);
}

}  // namespace

RouterPlan plan_router(int T, int H, int E, int kch_max) {
    RouterPlan p{};
    const int tiles = (T + kTileM - 1) / kTileM;
    int cn = E > 256 ? 2 : 1;
    // Spread a tile over more SMs while the grid still fits one wave and each
    // CTA keeps at least 16 real experts.
    while (cn < 8 && static_cast<long>(tiles) * cn * 2 <= 148 && (E + 2 * cn - 1) / (2 * cn) >= 16) cn *= 2;
    p.cn = cn;
    p.ne = ((E + cn - 1) / cn + 15) / 16 * 16;
    p.tiles = tiles;
    // A batch smaller than a tile loads only its rows (the MMA's other rows
    // read whatever shared memory follows and produce accumulator rows nobody
    // reads; the allocation keeps a full x tile of slack after the ring).
    p.xrows = T < kTileM ? (T + 7) / 8 * 8 : kTileM;
    // Chunks per stage: as many (up to kch_max) as keep a stage within 48 KB,
    // so that at least four stages fit; fewer, larger TMA boxes per stage.
    p.kch = 1;
    while (p.kch * 2 <= kch_max && (H / 64) % (p.kch * 2) == 0 && p.kch * 2 * (p.xrows + p.ne) * 128 <= 48 * 1024)
        p.kch *= 2;
    const int stage_bytes = p.kch * (p.xrows + p.ne) * 128;
    p.stages = 200 * 1024 / stage_bytes;
    if (p.stages > kMaxStages) p.stages = kMaxStages;
    p.tmem_cols = 32;
    while (p.tmem_cols < p.ne) p.tmem_cols *= 2;
    p.S = (E + 15) / 16 * 16 + 4;
    const size_t ring = static_cast<size_t>(p.stages) * stage_bytes + kXStageBytes;
    const size_t staging = static_cast<size_t>(kTileM / cn) * p.S * sizeof(float);
    p.smem = 2048 + (ring > staging ? ring : staging);
    return p;
}

// The plan's invariants, which the kernel's indexing relies on: a cluster of
// at most 8 CTAs splitting 128 tokens evenly, an MMA N of 16..256 in steps of
// 16 within the TMEM allocation that covers the cluster's share of E, at
// least two stages, chunks that divide H, x rows a multiple of 8 within a
// tile, and shared memory within one CTA's limit.  Returns the name of the
// first field that breaks one, or nullptr.
const char* router_plan_violation(const RouterPlan& p, int H, int E) {
    if (p.cn < 1 || p.cn > 8 || kTileM % p.cn) return "cn";
    if (p.ne < 16 || p.ne > 256 || p.ne % 16 || static_cast<long>(p.ne) * p.cn < E) return "ne";
    if (p.tmem_cols < 32 || p.tmem_cols > 512 || (p.tmem_cols & (p.tmem_cols - 1)) || p.ne > p.tmem_cols)
        return "tmem_cols";
    if (p.stages < 2 || p.stages > kMaxStages) return "stages";
    if (p.kch < 1 || (H / kKStage) % p.kch) return "kch";
    if (p.xrows < 8 || p.xrows > kTileM || p.xrows % 8) return "xrows";
    if (p.S < E + 4 || p.S % 4) return "S";
    if (p.smem > 227 * 1024) return "smem";
    return nullptr;
}

cudaError_t launch_router(const RouterPlan& p, const CUtensorMap& tx, const CUtensorMap& tw, int T, int H, int E,
                          int K, const RouteCfg& cfg, const uint8_t* zero_mask, int32_t* ids, float* w,
                          float* logits, int32_t* status, cudaStream_t stream) {
    RouterArgs a{};
    a.T = T;
    a.H = H;
    a.E = E;
    a.K = K;
    a.CN = p.cn;
    a.NE = p.ne;
    a.stages = p.stages;
    a.tmem_cols = p.tmem_cols;
    a.S = p.S;
    a.xrows = p.xrows;
    a.kch = p.kch;
    a.cfg = cfg;
    a.zero_mask = zero_mask;
    a.ids = ids;
    a.w = w;
    a.logits = logits;
    a.status = status;
    if (router_plan_violation(p, H, E)) return cudaErrorInvalidConfiguration;
    const int grid = p.tiles * p.cn;
    const bool computed = cfg.bias != nullptr || cfg.n_group > 1;
#define MOE_ROUTER_CASE(EPL)                                                                    \
    return computed ? launch_router_t<EPL, true>(tx, tw, a, grid, p.smem, stream)               \
                    : launch_router_t<EPL, false>(tx, tw, a, grid, p.smem, stream);
    switch ((E + 31) / 32) {
        case 1: MOE_ROUTER_CASE(1)
        case 2: MOE_ROUTER_CASE(2)
        case 3:
        case 4: MOE_ROUTER_CASE(4)
        case 5: case 6: case 7:
        case 8: MOE_ROUTER_CASE(8)
        default: MOE_ROUTER_CASE(16)
    }
#undef MOE_ROUTER_CASE
}

}  // namespace moe
