// moe_api.cu -- the extern "C" boundary (include/moe_ffn.h): argument and
// tensor-contract validation on the host, workspace carving, kernel launch,
// and the thread-local error message.  Like the C-ABI entry points of the
// aiter gfx950 prefill PR, the launcher checks the tensor contracts; like the
// Nemotron-H layer's constructor, an out-of-range top_k is reported with a
// message naming the bound.
#include <math.h>
#include <stdarg.h>
#include <stdio.h>

#include <mutex>
#include <string>

#include "../../include/moe_ffn.h"
#include "launch.h"
#include "router.h"

namespace moe {
bool ffn_decode_supported(int H, int I);
}

namespace {

thread_local std::string g_err;

int fail(int code, const char* fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof buf, fmt, ap);
    va_end(ap);
    g_err = buf;
    return code;
}

int cuda_fail(cudaError_t e, const char* what) {
    return fail(MOE_ERR_CUDA, "%s: %s (%s)", what, cudaGetErrorString(e), cudaGetErrorName(e));
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

size_t round256(size_t n) { return (n + 255) & ~size_t(255); }

int check_topk(int T, int E, int K) {
    if (T < 0 || T > MOE_MAX_T) return fail(MOE_ERR_INVALID_ARG, "T=%d must be in 0..=%d", T, MOE_MAX_T);
    if (E < 1 || E > MOE_MAX_E)
        return fail(MOE_ERR_UNSUPPORTED_SHAPE, "num_experts=%d must be in 1..=%d", E, MOE_MAX_E);
    if (K < 1 || K > E || K > MOE_MAX_K)
        return fail(MOE_ERR_INVALID_ARG,
                    "top_k=%d must be in 1..=%d and within the routing kernels' bounds "
                    "(top_k max %d, num_experts=%d max %d)",
                    K, E, MOE_MAX_K, E, MOE_MAX_E);
    return MOE_OK;
}

// Sizes of the calls after routing: they need no K <= E (any ids sort).
int check_sizes(int T, int E, int K) {
    if (T < 0 || T > MOE_MAX_T) return fail(MOE_ERR_INVALID_ARG, "T=%d must be in 0..=%d", T, MOE_MAX_T);
    if (E < 1 || E > MOE_MAX_E)
        return fail(MOE_ERR_UNSUPPORTED_SHAPE, "num_experts=%d must be in 1..=%d", E, MOE_MAX_E);
    if (K < 1 || K > MOE_MAX_K) return fail(MOE_ERR_INVALID_ARG, "top_k=%d must be in 1..=%d", K, MOE_MAX_K);
    return MOE_OK;
}

int check_experts(const moe_fp8_experts* ex, int H, const char* which) {
    if (!ex->w_gate || !ex->w_up || !ex->w_down || !ex->s_gate || !ex->s_up || !ex->s_down)
        return fail(MOE_ERR_INVALID_ARG, "%s experts: NULL weight or scale pointer", which);
    if (!aligned16(ex->w_gate) || !aligned16(ex->w_up) || !aligned16(ex->w_down) ||
        !aligned16(ex->s_gate) || !aligned16(ex->s_up) || !aligned16(ex->s_down))
        return fail(MOE_ERR_MISALIGNED, "%s experts: weight and scale bases must be 16-byte aligned", which);
    const int I = ex->inter;
    if (I < 128 || I > 4096 || I % MOE_BLOCK)
        return fail(MOE_ERR_UNSUPPORTED_SHAPE, "%s experts: inter=%d must be a multiple of 128 in 128..=4096",
                    which, I);
    if (!moe::ffn_decode_supported(H, I))
        return fail(MOE_ERR_UNSUPPORTED_SHAPE, "%s experts: H=%d, inter=%d exceed the shared-memory tiles",
                    which, H, I);
    return MOE_OK;
}

size_t ffn_h_bytes(long R, int I) { return round256(static_cast<size_t>(R) * I * 2); }

// The hybrid form's second stream and its fork/join events, one set per
// device, created by the first hybrid call on that device (host set-up, like
// the kernels' attributes).  `mu` serialises the enqueue of a fork ... join
// sequence, so that calls from several host threads never interleave their
// event records.
struct SideStream {
    int device = -1;
    cudaStream_t stream = nullptr;
    cudaEvent_t fork = nullptr, join = nullptr;
    std::mutex* mu = nullptr;
};

cudaError_t side_stream(SideStream* out) {
    static std::mutex mu;
    static SideStream table[64];
    static std::mutex enqueue_mu[64];
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(mu);
    SideStream& t = table[dev];
    if (t.device != dev) {
        e = cudaStreamCreateWithFlags(&t.stream, cudaStreamNonBlocking);
        if (e == cudaSuccess) e = cudaEventCreateWithFlags(&t.fork, cudaEventDisableTiming);
        if (e == cudaSuccess) e = cudaEventCreateWithFlags(&t.join, cudaEventDisableTiming);
        if (e != cudaSuccess) return e;
        t.mu = &enqueue_mu[dev];
        t.device = dev;
    }
    *out = t;
    return cudaSuccess;
}

int device_sms() {
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        sms <= 0)
        sms = 148;
    return sms;
}

}  // namespace

namespace moe {
// Records an error message for moe_last_error() from another translation unit.
int api_error(int code, const char* msg) {
    g_err = msg;
    return code;
}
void api_clear_error() { g_err.clear(); }
}  // namespace moe

namespace moe {
// selftest.cu
cudaError_t launch_bounded_wait_probe(int32_t* status, unsigned long long* elapsed_ns, cudaStream_t stream);
}  // namespace moe

extern "C" {

const char* moe_last_error(void) { return g_err.c_str(); }

int moe_abi_version(void) { return MOE_ABI_VERSION; }

int moe_route(const float* logits, int T, int E, int K, const uint8_t* zero_mask, int32_t* topk_ids,
              float* topk_w, moe_stream_t stream) {
    g_err.clear();
    int rc = check_topk(T, E, K);
    if (rc) return rc;
    if (T == 0) return MOE_OK;
    if (!logits || !topk_ids || !topk_w)
        return fail(MOE_ERR_INVALID_ARG, "moe_route: logits, topk_ids and topk_w must not be NULL");
    if (!aligned16(logits) || !aligned16(topk_ids) || !aligned16(topk_w))
        return fail(MOE_ERR_MISALIGNED, "moe_route: tensor bases must be 16-byte aligned");
    cudaError_t e = moe::launch_route(logits, T, E, K, zero_mask, topk_ids, topk_w, stream);
    return e == cudaSuccess ? MOE_OK : cuda_fail(e, "moe_route launch");
}

namespace {

// Range checks of a moe_route_config (messages prefixed with the caller's name).
int check_route_cfg(const char* fn, const moe_route_config* cfg, int E, int K) {
    if (cfg->score != MOE_SCORE_SOFTMAX && cfg->score != MOE_SCORE_SIGMOID)
        return fail(MOE_ERR_INVALID_ARG, "%s: unknown score function %d", fn, cfg->score);
    if (cfg->n_group < 1 || cfg->n_group > MOE_MAX_GROUPS || E % cfg->n_group)
        return fail(MOE_ERR_INVALID_ARG, "%s: n_group=%d must be in 1..%d and divide E=%d", fn, cfg->n_group,
                    MOE_MAX_GROUPS, E);
    if (cfg->topk_group < 1 || cfg->topk_group > cfg->n_group ||
        static_cast<long>(cfg->topk_group) * (E / cfg->n_group) < K)
        return fail(MOE_ERR_INVALID_ARG, "%s: topk_group=%d must be in 1..n_group and keep >= K=%d experts", fn,
                    cfg->topk_group, K);
    if (cfg->renormalize != 0 && cfg->renormalize != 1)
        return fail(MOE_ERR_INVALID_ARG, "%s: renormalize must be 0 or 1", fn);
    if (!(cfg->scaling > 0.f) || !isfinite(cfg->scaling))
        return fail(MOE_ERR_INVALID_ARG, "%s: scaling must be finite and > 0", fn);
    if (reinterpret_cast<uintptr_t>(cfg->sel_bias) % 4)
        return fail(MOE_ERR_MISALIGNED, "%s: sel_bias must be 4-byte aligned", fn);
    return MOE_OK;
}

}  // namespace

int moe_route_ex(const float* logits, int T, int E, int K, const moe_route_config* cfg, const uint8_t* zero_mask,
                 int32_t* topk_ids, float* topk_w, moe_stream_t stream) {
    g_err.clear();
    int rc = check_topk(T, E, K);
    if (rc) return rc;
    if (!cfg) return fail(MOE_ERR_INVALID_ARG, "moe_route_ex: cfg must not be NULL");
    rc = check_route_cfg("moe_route_ex", cfg, E, K);
    if (rc && rc != MOE_ERR_MISALIGNED) return rc;
    if (T == 0) return MOE_OK;
    if (!logits || !topk_ids || !topk_w)
        return fail(MOE_ERR_INVALID_ARG, "moe_route_ex: logits, topk_ids and topk_w must not be NULL");
    if (!aligned16(logits) || !aligned16(topk_ids) || !aligned16(topk_w))
        return fail(MOE_ERR_MISALIGNED, "moe_route_ex: tensor bases must be 16-byte aligned");
    if (rc) return rc;
    const moe::RouteCfg rc_dev{cfg->score, cfg->sel_bias, cfg->n_group, cfg->topk_group, cfg->renormalize,
                               cfg->scaling};
    cudaError_t e = moe::launch_route_ex(logits, T, E, K, rc_dev, zero_mask, topk_ids, topk_w, stream);
    return e == cudaSuccess ? MOE_OK : cuda_fail(e, "moe_route_ex launch");
}

int moe_selftest_bounded_wait(int32_t* status, uint64_t* elapsed_ns, moe_stream_t stream) {
    g_err.clear();
    if (!status || !elapsed_ns)
        return fail(MOE_ERR_INVALID_ARG, "moe_selftest_bounded_wait: status and elapsed_ns must not be NULL");
    if ((reinterpret_cast<uintptr_t>(status) & 3) || (reinterpret_cast<uintptr_t>(elapsed_ns) & 7))
        return fail(MOE_ERR_MISALIGNED, "moe_selftest_bounded_wait: misaligned pointer");
    cudaError_t e = moe::launch_bounded_wait_probe(status, reinterpret_cast<unsigned long long*>(elapsed_ns), stream);
    return e == cudaSuccess ? MOE_OK : cuda_fail(e, "moe_selftest_bounded_wait launch");
}

int moe_router(const uint16_t* x, int T, int H, const uint16_t* w_router, int E, int K, const moe_route_config* cfg,
               const uint8_t* zero_mask, int32_t* topk_ids, float* topk_w, float* logits, int32_t* status,
               moe_stream_t stream) {
    g_err.clear();
    int rc = check_topk(T, E, K);
    if (rc) return rc;
    if (E > MOE_ROUTER_MAX_E)
        return fail(MOE_ERR_UNSUPPORTED_SHAPE, "moe_router: num_experts=%d must be in 1..=%d", E, MOE_ROUTER_MAX_E);
    if (H < 64 || H > MOE_ROUTER_MAX_H || H % 64)
        return fail(MOE_ERR_UNSUPPORTED_SHAPE, "moe_router: H=%d must be a multiple of 64 in 64..=%d", H,
                    MOE_ROUTER_MAX_H);
    if (cfg) {
        rc = check_route_cfg("moe_router", cfg, E, K);
        if (rc) return rc;
    }
    if (T == 0) return MOE_OK;
    if (!x || !w_router || !topk_ids || !topk_w)
        return fail(MOE_ERR_INVALID_ARG, "moe_router: x, w_router, topk_ids and topk_w must not be NULL");
    if (!aligned16(x) || !aligned16(w_router) || !aligned16(topk_ids) || !aligned16(topk_w) || !aligned16(logits) ||
        (status && (reinterpret_cast<uintptr_t>(status) & 3)))
        return fail(MOE_ERR_MISALIGNED, "moe_router: tensor bases must be 16-byte aligned and status 4-byte aligned");
    const moe::RouteCfg rc_dev = cfg ? moe::RouteCfg{cfg->score, cfg->sel_bias, cfg->n_group, cfg->topk_group,
                                                     cfg->renormalize, cfg->scaling}
                                     : moe::RouteCfg{MOE_SCORE_SOFTMAX, nullptr, 1, 1, 1, 1.f};
    // Stages of several 64-column chunks (3-D boxes); one chunk if the
    // driver declines the 3-D view.
    moe::RouterPlan plan = moe::plan_router(T, H, E, 4);
    if (const char* field = moe::router_plan_violation(plan, H, E))
        return fail(MOE_ERR_UNSUPPORTED_SHAPE,
                    "moe_router: the launch plan for T=%d, H=%d, E=%d breaks the kernel's invariant on '%s'", T, H,
                    E, field);
    CUtensorMap tx, tw;
    cudaError_t e = cudaSuccess;
    for (int attempt = 0; attempt < 2; ++attempt) {
        if (plan.kch == 1) {
            e = moe::make_tmap_bf16_2d(&tx, x, static_cast<uint64_t>(T), static_cast<uint64_t>(H), 64,
                                       static_cast<uint32_t>(plan.xrows));
            if (e == cudaSuccess)
                e = moe::make_tmap_bf16_2d(&tw, w_router, static_cast<uint64_t>(E), static_cast<uint64_t>(H), 64,
                                           static_cast<uint32_t>(plan.ne));
        } else {
            e = moe::make_tmap_bf16_kchunks(&tx, x, static_cast<uint64_t>(T), static_cast<uint64_t>(H),
                                            static_cast<uint32_t>(plan.xrows), static_cast<uint32_t>(plan.kch));
            if (e == cudaSuccess)
                e = moe::make_tmap_bf16_kchunks(&tw, w_router, static_cast<uint64_t>(E), static_cast<uint64_t>(H),
                                                static_cast<uint32_t>(plan.ne), static_cast<uint32_t>(plan.kch));
        }
        if (e == cudaSuccess || plan.kch == 1) break;
        plan = moe::plan_router(T, H, E, 1);
        if (const char* field = moe::router_plan_violation(plan, H, E))
            return fail(MOE_ERR_UNSUPPORTED_SHAPE,
                        "moe_router: the launch plan for T=%d, H=%d, E=%d breaks the kernel's invariant on '%s'", T,
                        H, E, field);
    }
    if (e != cudaSuccess) return cuda_fail(e, "moe_router tensor maps");
    e = moe::launch_router(plan, tx, tw, T, H, E, K, rc_dev, zero_mask, topk_ids, topk_w, logits, status, stream);
    return e == cudaSuccess ? MOE_OK : cuda_fail(e, "moe_router launch");
}

int moe_router_plan_check(int T, int H, int E, int kch_max, int32_t* fields) {
    g_err.clear();
    if (T < 1 || H < 64 || H % 64 || E < 1 || E > MOE_ROUTER_MAX_E || (kch_max != 1 && kch_max != 2 && kch_max != 4))
        return fail(MOE_ERR_INVALID_ARG, "moe_router_plan_check: T=%d, H=%d, E=%d, kch_max=%d out of range", T, H, E,
                    kch_max);
    const moe::RouterPlan p = moe::plan_router(T, H, E, kch_max);
    if (fields) {
        const int32_t v[9] = {p.tiles, p.cn, p.ne, p.stages, p.tmem_cols, p.S, p.xrows, p.kch,
                              static_cast<int32_t>(p.smem)};
        for (int i = 0; i < 9; ++i) fields[i] = v[i];
    }
    if (const char* field = moe::router_plan_violation(p, H, E))
        return fail(MOE_ERR_UNSUPPORTED_SHAPE, "moe_router_plan_check: T=%d, H=%d, E=%d: invariant on '%s' broken", T,
                    H, E, field);
    return MOE_OK;
}

size_t moe_sort_workspace_bytes(int T, int K, int E) {
    if (T < 0 || K < 1 || E < 1) return 0;
    return moe::sort_workspace_bytes(static_cast<long>(T) * K, E);
}

int moe_sort(const int32_t* topk_ids, int T, int K, int E, int32_t* expert_offsets,
             int32_t* sorted_route, int32_t* inv_route, void* workspace, size_t workspace_bytes,
             int32_t* status, moe_stream_t stream) {
    g_err.clear();
    int rc = check_sizes(T, E, K);
    if (rc) return rc;
    if (!expert_offsets) return fail(MOE_ERR_INVALID_ARG, "moe_sort: expert_offsets must not be NULL");
    if (T > 0 && (!topk_ids || !sorted_route || !inv_route))
        return fail(MOE_ERR_INVALID_ARG, "moe_sort: topk_ids, sorted_route and inv_route must not be NULL");
    if (!aligned16(topk_ids) || !aligned16(expert_offsets) || !aligned16(sorted_route) ||
        !aligned16(inv_route) || !aligned16(workspace) || (status && (reinterpret_cast<uintptr_t>(status) & 3)))
        return fail(MOE_ERR_MISALIGNED, "moe_sort: tensor bases must be 16-byte aligned and status 4-byte aligned");
    const long R = static_cast<long>(T) * K;
    const size_t need = moe::sort_workspace_bytes(R, E);
    if (workspace_bytes < need || (need && !workspace))
        return fail(MOE_ERR_WORKSPACE_TOO_SMALL, "moe_sort: workspace of %zu bytes, need %zu",
                    workspace_bytes, need);
    if (T == 0) {
        // No routes: all offsets are 0.
        cudaError_t e = cudaMemsetAsync(expert_offsets, 0, sizeof(int32_t) * (E + 1), stream);
        return e == cudaSuccess ? MOE_OK : cuda_fail(e, "moe_sort memset");
    }
    cudaError_t e = moe::launch_sort(topk_ids, R, E, expert_offsets, sorted_route, inv_route, workspace,
                                     status, stream);
    return e == cudaSuccess ? MOE_OK : cuda_fail(e, "moe_sort launch");
}

int moe_ffn_resolve_mode(int T, int K, int E, int mode) {
    g_err.clear();
    if (T < 0 || K < 1 || E < 1)
        return fail(MOE_ERR_INVALID_ARG, "moe_ffn_resolve_mode: T=%d, K=%d, E=%d out of range", T, K, E);
    if (mode == MOE_MODE_DECODE || mode == MOE_MODE_PREFILL || mode == MOE_MODE_HYBRID) return mode;
    if (mode != MOE_MODE_AUTO)
        return fail(MOE_ERR_INVALID_ARG, "moe_ffn_resolve_mode: mode=%d is not AUTO/DECODE/PREFILL/HYBRID", mode);
    const long R = static_cast<long>(T) * K;
    if (R <= MOE_DECODE_MAX_ROUTES && R <= static_cast<long>(MOE_DECODE_MAX_ROWS_PER_EXPERT) * E)
        return MOE_MODE_DECODE;
    return R <= static_cast<long>(MOE_HYBRID_MAX_ROWS_PER_EXPERT) * E ? MOE_MODE_HYBRID : MOE_MODE_PREFILL;
}

size_t moe_ffn_workspace_bytes(int T, int K, int H, int E, int I, int I_shared, int mode) {
    if (T < 0 || K < 1 || I < 0 || I_shared < 0 || H < 0) return 0;
    const long R = static_cast<long>(T) * K;
    size_t b = ffn_h_bytes(R, I) + ffn_h_bytes(T, I_shared);
    // The tensor-core form also keeps an f16 copy of x and its row scales.
    const std::string saved = g_err;
    const int form = moe_ffn_resolve_mode(T, K, E < 1 ? 1 : E, mode);
    g_err = saved;
    if (form != MOE_MODE_DECODE) b += moe::ffn_x16_bytes(T, H) + moe::ffn_xinv_bytes(T);
    return b;
}

int moe_expert_ffn(const uint16_t* x, int T, int H, int K, const moe_fp8_experts* routed,
                   const moe_fp8_experts* shared, const int32_t* expert_offsets,
                   const int32_t* sorted_route, const float* topk_w, uint16_t* y_sorted,
                   uint16_t* y_shared, int mode, void* workspace, size_t workspace_bytes,
                   int32_t* status, moe_stream_t stream) {
    g_err.clear();
    if (!routed) return fail(MOE_ERR_INVALID_ARG, "moe_expert_ffn: routed must not be NULL");
    const int E = routed->n_experts, I = routed->inter;
    int rc = check_sizes(T, E, K);
    if (rc) return rc;
    if (mode != MOE_MODE_AUTO && mode != MOE_MODE_DECODE && mode != MOE_MODE_PREFILL && mode != MOE_MODE_HYBRID)
        return fail(MOE_ERR_INVALID_ARG, "moe_expert_ffn: mode=%d is not AUTO/DECODE/PREFILL/HYBRID", mode);
    if (H < 128 || H % MOE_BLOCK || H > 8192)
        return fail(MOE_ERR_UNSUPPORTED_SHAPE, "moe_expert_ffn: H=%d must be a multiple of 128 in 128..=8192", H);
    if ((rc = check_experts(routed, H, "routed"))) return rc;
    if (shared) {
        if (shared->n_experts != 1)
            return fail(MOE_ERR_INVALID_ARG, "moe_expert_ffn: shared->n_experts=%d must be 1", shared->n_experts);
        if ((rc = check_experts(shared, H, "shared"))) return rc;
    }
    if (T == 0) return MOE_OK;
    if (!x || !expert_offsets || !sorted_route || !topk_w || !y_sorted || (shared && !y_shared))
        return fail(MOE_ERR_INVALID_ARG, "moe_expert_ffn: NULL tensor pointer");
    if (!aligned16(x) || !aligned16(expert_offsets) || !aligned16(sorted_route) || !aligned16(topk_w) ||
        !aligned16(y_sorted) || (shared && !aligned16(y_shared)) || !aligned16(workspace) ||
        (status && (reinterpret_cast<uintptr_t>(status) & 3)))
        return fail(MOE_ERR_MISALIGNED,
                    "moe_expert_ffn: tensor bases must be 16-byte aligned and status 4-byte aligned");
    const long R = static_cast<long>(T) * K;
    const int Is = shared ? shared->inter : 0;
    const size_t need = moe_ffn_workspace_bytes(T, K, H, E, I, Is, mode);
    if (workspace_bytes < need || !workspace)
        return fail(MOE_ERR_WORKSPACE_TOO_SMALL, "moe_expert_ffn: workspace of %zu bytes, need %zu",
                    workspace_bytes, need);
    const int form = moe_ffn_resolve_mode(T, K, E, mode);
    const bool prefill = form == MOE_MODE_PREFILL || form == MOE_MODE_HYBRID;
    if (prefill && !moe::ffn_prefill_supported(H, I))
        return fail(MOE_ERR_UNSUPPORTED_SHAPE, "moe_expert_ffn: H=%d, inter=%d not supported by the PREFILL kernels", H, I);

    uint8_t* ws = static_cast<uint8_t*>(workspace);
    moe::FfnArgs a{};
    a.x = x;
    a.T = T;
    a.H = H;
    a.K = K;
    a.ex = {routed->w_gate, routed->w_up, routed->w_down, routed->s_gate, routed->s_up, routed->s_down, E, I};
    a.identity = false;
    a.offsets = expert_offsets;
    a.sorted_route = sorted_route;
    a.topk_w = topk_w;
    a.h = reinterpret_cast<uint16_t*>(ws);
    a.y = y_sorted;
    a.status = status;
    a.avg_rows = static_cast<int>((R + E - 1) / E);
    if (prefill) {
        // The shared expert runs in the same two launches as the routed rows.
        if (shared) {
            a.sh = {shared->w_gate, shared->w_up, shared->w_down, shared->s_gate, shared->s_up, shared->s_down, 1, Is};
            a.h_sh = reinterpret_cast<uint16_t*>(ws + ffn_h_bytes(R, I));
            a.y_sh = y_shared;
        }
        a.x16 = reinterpret_cast<uint16_t*>(ws + ffn_h_bytes(R, I) + ffn_h_bytes(T, Is));
        a.xinv = reinterpret_cast<float*>(ws + ffn_h_bytes(R, I) + ffn_h_bytes(T, Is) + moe::ffn_x16_bytes(T, H));
        if (form == MOE_MODE_PREFILL) {
            const cudaError_t e = moe::launch_ffn_prefill(a, stream);
            return e == cudaSuccess ? MOE_OK : cuda_fail(e, "moe_expert_ffn launch");
        }
        // HYBRID: the experts with at most MOE_HYBRID_ROW_SPLIT rows in the
        // weight-streaming kernels (token groups of 8 rows), the others and the
        // shared expert in the tensor-core kernels.  The two forms run at the
        // same time on disjoint SMs: the tensor-core grids (one CTA per SM,
        // launched first) on 7/10 of them, the weight-streaming grids (two CTAs
        // per SM) on the rest, from a second stream forked from and joined back
        // to `stream` with events.  Each form skips the experts of the other.
        // (The share is a measured optimum on a skewed 512-token batch: 1/2,
        // 3/5, 13/20, 7/10, 3/4, 4/5 and 17/20 of the SMs gave 164, 135, 131,
        // 125-127, 133, 141 and 137 us against 129-131 us for the two forms
        // one after the other.)
        SideStream side;
        cudaError_t e = side_stream(&side);
        if (e != cudaSuccess) return cuda_fail(e, "moe_expert_ffn side stream");
        std::lock_guard<std::mutex> enqueue(*side.mu);
        e = moe::launch_x16(a, stream);
        if (e == cudaSuccess) e = cudaEventRecord(side.fork, stream);
        if (e == cudaSuccess) e = cudaStreamWaitEvent(side.stream, side.fork, 0);
        if (e != cudaSuccess) return cuda_fail(e, "moe_expert_ffn launch");
        const int sms = device_sms(), tc_sms = (7 * sms + 9) / 10;
        a.row_split = MOE_HYBRID_ROW_SPLIT;
        a.sm_limit = tc_sms;
        e = moe::launch_ffn_prefill(a, stream, /*x16_done=*/true);
        if (e != cudaSuccess) return cuda_fail(e, "moe_expert_ffn launch");
        moe::FfnArgs d = a;
        d.avg_rows = MOE_HYBRID_ROW_SPLIT / 2;
        d.sh = {};
        d.sm_limit = sms - tc_sms;
        e = moe::launch_ffn_decode(d, side.stream);
        if (e == cudaSuccess) e = cudaEventRecord(side.join, side.stream);
        if (e == cudaSuccess) e = cudaStreamWaitEvent(stream, side.join, 0);
        return e == cudaSuccess ? MOE_OK : cuda_fail(e, "moe_expert_ffn routed launch");
    }
    cudaError_t e = moe::launch_ffn_decode(a, stream);
    if (e != cudaSuccess) return cuda_fail(e, "moe_expert_ffn routed launch");
    if (shared && form == MOE_MODE_DECODE) {
        moe::FfnArgs s = a;
        s.ex = {shared->w_gate, shared->w_up, shared->w_down, shared->s_gate, shared->s_up, shared->s_down, 1, Is};
        s.identity = true;
        s.offsets = nullptr;
        s.sorted_route = nullptr;
        s.topk_w = nullptr;
        s.h = reinterpret_cast<uint16_t*>(ws + ffn_h_bytes(R, I));
        s.y = y_shared;
        s.avg_rows = T;
        e = moe::launch_ffn_decode(s, stream);
        if (e != cudaSuccess) return cuda_fail(e, "moe_expert_ffn shared launch");
    }
    return MOE_OK;
}

namespace {
// W8A8 workspace: E4M3FN codes of h and their 64-feature block scales, routed then shared.
size_t w8a8_part_bytes(long rows, int I) {
    return round256(static_cast<size_t>(rows) * I) + round256(static_cast<size_t>(rows) * (I / 64) * 4);
}
}  // namespace

size_t moe_ffn_w8a8_workspace_bytes(int T, int K, int I, int I_shared) {
    if (T < 0 || K < 1 || I < 0 || I_shared < 0) return 0;
    return w8a8_part_bytes(static_cast<long>(T) * K, I) + w8a8_part_bytes(T, I_shared);
}

int moe_expert_ffn_w8a8(const uint16_t* x, int T, int H, int K, const moe_fp8_experts* routed,
                        const moe_fp8_experts* shared, const int32_t* expert_offsets, const int32_t* sorted_route,
                        const float* topk_w, uint16_t* y_sorted, uint16_t* y_shared, void* workspace,
                        size_t workspace_bytes, int32_t* status, moe_stream_t stream) {
    g_err.clear();
    if (!routed) return fail(MOE_ERR_INVALID_ARG, "moe_expert_ffn_w8a8: routed must not be NULL");
    const int E = routed->n_experts, I = routed->inter;
    int rc = check_sizes(T, E, K);
    if (rc) return rc;
    if (H < 128 || H % MOE_BLOCK || H > 8192)
        return fail(MOE_ERR_UNSUPPORTED_SHAPE, "moe_expert_ffn_w8a8: H=%d must be a multiple of 128 in 128..=8192",
                    H);
    if ((rc = check_experts(routed, H, "routed"))) return rc;
    if (shared) {
        if (shared->n_experts != 1)
            return fail(MOE_ERR_INVALID_ARG, "moe_expert_ffn_w8a8: shared->n_experts=%d must be 1", shared->n_experts);
        if ((rc = check_experts(shared, H, "shared"))) return rc;
    }
    if (T == 0) return MOE_OK;
    if (!x || !expert_offsets || !sorted_route || !topk_w || !y_sorted || (shared && !y_shared))
        return fail(MOE_ERR_INVALID_ARG, "moe_expert_ffn_w8a8: NULL tensor pointer");
    if (!aligned16(x) || !aligned16(expert_offsets) || !aligned16(sorted_route) || !aligned16(topk_w) ||
        !aligned16(y_sorted) || (shared && !aligned16(y_shared)) || !aligned16(workspace) ||
        (status && (reinterpret_cast<uintptr_t>(status) & 3)))
        return fail(MOE_ERR_MISALIGNED,
                    "moe_expert_ffn_w8a8: tensor bases must be 16-byte aligned and status 4-byte aligned");
    const long R = static_cast<long>(T) * K;
    const int Is = shared ? shared->inter : 0;
    const size_t need = moe_ffn_w8a8_workspace_bytes(T, K, I, Is);
    if (workspace_bytes < need || !workspace)
        return fail(MOE_ERR_WORKSPACE_TOO_SMALL, "moe_expert_ffn_w8a8: workspace of %zu bytes, need %zu",
                    workspace_bytes, need);

    uint8_t* ws = static_cast<uint8_t*>(workspace);
    moe::FfnArgs a{};
    a.x = x;
    a.T = T;
    a.H = H;
    a.K = K;
    a.ex = {routed->w_gate, routed->w_up, routed->w_down, routed->s_gate, routed->s_up, routed->s_down, E, I};
    a.offsets = expert_offsets;
    a.sorted_route = sorted_route;
    a.topk_w = topk_w;
    a.h = reinterpret_cast<uint16_t*>(ws);
    a.hscale = reinterpret_cast<float*>(ws + round256(static_cast<size_t>(R) * I));
    a.y = y_sorted;
    a.status = status;
    a.avg_rows = static_cast<int>((R + E - 1) / E);
    a.w8a8 = true;
    cudaError_t e = moe::launch_ffn_decode(a, stream);
    if (e != cudaSuccess) return cuda_fail(e, "moe_expert_ffn_w8a8 routed launch");
    if (shared) {
        moe::FfnArgs sa = a;
        sa.ex = {shared->w_gate, shared->w_up, shared->w_down, shared->s_gate, shared->s_up, shared->s_down, 1, Is};
        sa.identity = true;
        sa.offsets = nullptr;
        sa.sorted_route = nullptr;
        sa.topk_w = nullptr;
        uint8_t* sh_ws = ws + w8a8_part_bytes(R, I);
        sa.h = reinterpret_cast<uint16_t*>(sh_ws);
        sa.hscale = reinterpret_cast<float*>(sh_ws + round256(static_cast<size_t>(T) * Is));
        sa.y = y_shared;
        sa.avg_rows = T;
        e = moe::launch_ffn_decode(sa, stream);
        if (e != cudaSuccess) return cuda_fail(e, "moe_expert_ffn_w8a8 shared launch");
    }
    return MOE_OK;
}

size_t moe_ffn_combine_workspace_bytes(int T, int K, int H, int E, int I, int I_shared, int out_dtype) {
    (void)E;
    if (T < 0 || K < 1 || I < 0 || I_shared < 0 || H < 0) return 0;
    const long R = static_cast<long>(T) * K;
    size_t b = ffn_h_bytes(R, I) + ffn_h_bytes(T, I_shared) + moe::ffn_x16_bytes(T, H) + moe::ffn_xinv_bytes(T);
    if (out_dtype != MOE_OUT_F32) b += round256(static_cast<size_t>(T) * H * 4);  // the fp32 accumulator
    return b;
}

int moe_expert_ffn_combine(const uint16_t* x, int T, int H, int K, const moe_fp8_experts* routed,
                           const moe_fp8_experts* shared, const int32_t* expert_offsets, const int32_t* sorted_route,
                           const float* topk_w, void* out, int out_dtype, void* workspace, size_t workspace_bytes,
                           int32_t* status, moe_stream_t stream) {
    g_err.clear();
    if (!routed) return fail(MOE_ERR_INVALID_ARG, "moe_expert_ffn_combine: routed must not be NULL");
    const int E = routed->n_experts, I = routed->inter;
    int rc = check_sizes(T, E, K);
    if (rc) return rc;
    if (out_dtype != MOE_OUT_BF16 && out_dtype != MOE_OUT_F32)
        return fail(MOE_ERR_INVALID_ARG, "moe_expert_ffn_combine: out_dtype=%d is not BF16/F32", out_dtype);
    if (H < 128 || H % MOE_BLOCK || H > 8192)
        return fail(MOE_ERR_UNSUPPORTED_SHAPE, "moe_expert_ffn_combine: H=%d must be a multiple of 128 in 128..=8192",
                    H);
    if ((rc = check_experts(routed, H, "routed"))) return rc;
    if (shared) {
        if (shared->n_experts != 1)
            return fail(MOE_ERR_INVALID_ARG, "moe_expert_ffn_combine: shared->n_experts=%d must be 1",
                        shared->n_experts);
        if ((rc = check_experts(shared, H, "shared"))) return rc;
    }
    if (!moe::ffn_prefill_supported(H, I))
        return fail(MOE_ERR_UNSUPPORTED_SHAPE, "moe_expert_ffn_combine: H=%d, inter=%d not supported", H, I);
    if (T == 0) return MOE_OK;
    if (!x || !expert_offsets || !sorted_route || !topk_w || !out)
        return fail(MOE_ERR_INVALID_ARG, "moe_expert_ffn_combine: NULL tensor pointer");
    if (!aligned16(x) || !aligned16(expert_offsets) || !aligned16(sorted_route) || !aligned16(topk_w) ||
        !aligned16(out) || !aligned16(workspace) || (reinterpret_cast<uintptr_t>(status) & 3))
        return fail(MOE_ERR_MISALIGNED,
                    "moe_expert_ffn_combine: tensor bases must be 16-byte aligned and status 4-byte aligned");
    const long R = static_cast<long>(T) * K;
    const int Is = shared ? shared->inter : 0;
    const size_t need = moe_ffn_combine_workspace_bytes(T, K, H, E, I, Is, out_dtype);
    if (workspace_bytes < need || !workspace)
        return fail(MOE_ERR_WORKSPACE_TOO_SMALL, "moe_expert_ffn_combine: workspace of %zu bytes, need %zu",
                    workspace_bytes, need);
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    const size_t off_x16 = ffn_h_bytes(R, I) + ffn_h_bytes(T, Is);
    const size_t off_acc = off_x16 + moe::ffn_x16_bytes(T, H) + moe::ffn_xinv_bytes(T);
    float* acc = out_dtype == MOE_OUT_F32 ? static_cast<float*>(out) : reinterpret_cast<float*>(ws + off_acc);
    cudaError_t e = cudaMemsetAsync(acc, 0, static_cast<size_t>(T) * H * 4, stream);
    if (e != cudaSuccess) return cuda_fail(e, "moe_expert_ffn_combine memset");
    moe::FfnArgs a{};
    a.x = x;
    a.T = T;
    a.H = H;
    a.K = K;
    a.ex = {routed->w_gate, routed->w_up, routed->w_down, routed->s_gate, routed->s_up, routed->s_down, E, I};
    a.offsets = expert_offsets;
    a.sorted_route = sorted_route;
    a.topk_w = topk_w;
    a.h = reinterpret_cast<uint16_t*>(ws);
    a.status = status;
    a.avg_rows = static_cast<int>((R + E - 1) / E);
    if (shared) {
        a.sh = {shared->w_gate, shared->w_up, shared->w_down, shared->s_gate, shared->s_up, shared->s_down, 1, Is};
        a.h_sh = reinterpret_cast<uint16_t*>(ws + ffn_h_bytes(R, I));
    }
    a.x16 = reinterpret_cast<uint16_t*>(ws + off_x16);
    a.xinv = reinterpret_cast<float*>(ws + off_x16 + moe::ffn_x16_bytes(T, H));
    a.out_acc = acc;
    e = moe::launch_ffn_prefill(a, stream);
    if (e != cudaSuccess) return cuda_fail(e, "moe_expert_ffn_combine launch");
    if (out_dtype == MOE_OUT_BF16) {
        e = moe::launch_acc_to_bf16(acc, static_cast<long>(T) * H, static_cast<uint16_t*>(out), stream);
        if (e != cudaSuccess) return cuda_fail(e, "moe_expert_ffn_combine convert");
    }
    return MOE_OK;
}

int moe_combine(const uint16_t* y_sorted, const int32_t* inv_route, const uint16_t* y_shared, int T,
                int K, int H, void* out, int out_dtype, int32_t* status, moe_stream_t stream) {
    g_err.clear();
    if (T < 0 || T > MOE_MAX_T) return fail(MOE_ERR_INVALID_ARG, "moe_combine: T=%d out of range", T);
    if (K < 1 || K > MOE_MAX_K) return fail(MOE_ERR_INVALID_ARG, "moe_combine: K=%d must be in 1..=%d", K, MOE_MAX_K);
    if (H < 8 || H % 8) return fail(MOE_ERR_UNSUPPORTED_SHAPE, "moe_combine: H=%d must be a positive multiple of 8", H);
    if (out_dtype != MOE_OUT_BF16 && out_dtype != MOE_OUT_F32)
        return fail(MOE_ERR_INVALID_ARG, "moe_combine: out_dtype=%d is not BF16/F32", out_dtype);
    if (T == 0) return MOE_OK;
    if (!y_sorted || !inv_route || !out)
        return fail(MOE_ERR_INVALID_ARG, "moe_combine: y_sorted, inv_route and out must not be NULL");
    if (!aligned16(y_sorted) || !aligned16(inv_route) || !aligned16(y_shared) || !aligned16(out) ||
        (reinterpret_cast<uintptr_t>(status) & 3))
        return fail(MOE_ERR_MISALIGNED,
                    "moe_combine: tensor bases must be 16-byte aligned and status 4-byte aligned");
    cudaError_t e = moe::launch_combine(y_sorted, inv_route, y_shared, T, K, H, out,
                                        out_dtype == MOE_OUT_F32, status, stream);
    return e == cudaSuccess ? MOE_OK : cuda_fail(e, "moe_combine launch");
}

}  // extern "C"
