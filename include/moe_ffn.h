/*
 * moe_ffn.h -- C ABI of the routed Mixture-of-Experts FFN library for NVIDIA
 * B200 (sm_100a).
 *
 * The four calls run the routed MoE FFN hot path:
 *
 *   moe_route      router logits -> top-K expert ids and renormalised weights
 *   moe_sort       ids -> expert-contiguous route order, per-expert offsets,
 *                  inverse route map (all on the device, no host sync)
 *   moe_expert_ffn grouped gate/up GEMM over block-scaled E4M3FN weights
 *                  decoded to BF16, fused SwiGLU, down GEMM with the routing
 *                  weight fused in; optional always-on shared expert
 *   moe_combine    top-K reduce back to token order (+ shared expert)
 *
 * plus the routing variants (moe_route_ex), the fused router that computes the
 * logits from the token rows and routes in one kernel (moe_router), a sort
 * with library-owned scratch (moe_sort_static_ws) and a diagnostic of the
 * kernels' bounded waits (moe_selftest_bounded_wait).
 *
 * Sources (page title, section):
 *  - dstair/gated-deltanet-nki-trainium, "FP8 MoE decode kernel
 *    (moe_fused_w8_35b)": the fused chain gate/up GEMM -> SwiGLU -> down GEMM
 *    -> affinity scale -> expert-sum, official E4M3FN weights with 128x128
 *    block scales decoded to BF16 tile by tile; "Interface" (hidden, gate_up,
 *    down, scales, affinities -> [B, H] f32); "Serving contract" (softmax ->
 *    top-8 -> norm router; the shared expert is added after the routed sum).
 *  - spark_model/layers/nemotron_moe.rs: module doc (expert dispatch stays on the
 *    device, with no device-to-host synchronisation), `new` (top_k bounds checked with an error
 *    message), `prefill` step 2 (the router's dense gate GEMM) and step 5 (sort
 *    by expert, grouped GEMM, unpermute-reduce, ids and weights as [N, top_k]
 *    4-byte arrays).
 *  - ROCm/aiter PR #5988: ctypes C-ABI entry point whose launcher validates the
 *    tensor contracts; reuse of a sort with an inverse route map; FP32 route
 *    reduction; zero routing weights and caller-provided output buffers.
 *  - NKI Library kernel reference, MoE kernels: Router Top-K, Permute Routed
 *    Tokens, Top-K Reduce, MoE TKG (decode) / MoE CTE (prefill).
 *
 * Conventions for every call:
 *  - All tensor pointers are DEVICE pointers owned by the caller.  The library
 *    allocates no device memory in any call; scratch is caller-provided through
 *    the `workspace` arguments, sized by the *_workspace_bytes queries.
 *  - Every call is asynchronous on `stream` (a cudaStream_t; NULL = the legacy
 *    default stream), never synchronises the host, and reads no device value
 *    back.  The first call of a process also does one-time host set-up (kernel
 *    attributes, driver entry points); make one call before capturing a CUDA
 *    graph, after which moe_route, moe_route_ex, moe_router, moe_sort,
 *    moe_expert_ffn, moe_expert_ffn_w8a8, moe_expert_ffn_combine and
 *    moe_combine may be captured.
 *  - Return value: MOE_OK (0) or a negative moe_status.  On error nothing has
 *    been launched and moe_last_error() holds a message (thread-local, valid
 *    until the next call on the same thread).  MOE_ERR_CUDA reports a launch
 *    error, with the CUDA error string in the message.
 *  - T = 0 (no tokens) is valid: nothing is launched and MOE_OK is returned.
 *  - Tensor base addresses must be 16-byte aligned (MOE_ERR_MISALIGNED).
 *  - Layouts are row-major with the last index contiguous.  Route r = t*K + j
 *    is token t's j-th choice (descending weight).
 *  - bf16 tensors are passed as uint16_t bit patterns.
 */
#ifndef MOE_FFN_H
#define MOE_FFN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Exported symbols of the shared library (everything else is hidden). */
#if defined(__GNUC__)
#define MOE_API __attribute__((visibility("default")))
#else
#define MOE_API
#endif

/* A cudaStream_t (the runtime's stream handle type is `struct CUstream_st*`). */
typedef struct CUstream_st* moe_stream_t;

typedef enum moe_status {
    MOE_OK = 0,
    MOE_ERR_INVALID_ARG = -1,          /* NULL pointer, negative size, bad enum, K > E */
    MOE_ERR_UNSUPPORTED_SHAPE = -2,    /* H or I not a multiple of 128, E > MOE_MAX_E, ... */
    MOE_ERR_MISALIGNED = -3,           /* a tensor base not 16-byte aligned */
    MOE_ERR_WORKSPACE_TOO_SMALL = -4,  /* workspace_bytes below the query's answer */
    MOE_ERR_CUDA = -5                  /* the CUDA runtime reported an error */
} moe_status;

#define MOE_MAX_E 1024      /* experts per call */
#define MOE_MAX_K 32        /* top-K */
#define MOE_BLOCK 128       /* FP8 scale block edge: one fp32 scale per 128 x 128 */
#define MOE_MAX_T (1 << 24) /* tokens per call */

/* Bits OR-ed into the optional device status word (int32) by the kernels. */
#define MOE_STATUS_BAD_ID 1      /* an expert id outside [0, E) was skipped */
#define MOE_STATUS_BAD_MAP 2     /* offsets / route map out of range: rows skipped */
#define MOE_STATUS_TIMEOUT 4     /* a bounded wait inside a kernel expired (a copy or MMA that never
                                    completed; never expected): that call's outputs are invalid */

/* moe_expert_ffn `mode`. */
#define MOE_MODE_AUTO 0     /* see moe_ffn_resolve_mode */
#define MOE_MODE_DECODE 1   /* weight-streaming kernels (memory-bound regime) */
#define MOE_MODE_PREFILL 2  /* tcgen05 / TMEM grouped GEMM kernels (compute-bound regime) */
#define MOE_MODE_HYBRID 3   /* experts with <= MOE_HYBRID_ROW_SPLIT rows in the DECODE kernels, the rest
                               (and the shared expert) in the PREFILL kernels */
#define MOE_HYBRID_ROW_SPLIT 8
#define MOE_HYBRID_MAX_ROWS_PER_EXPERT 32
#define MOE_DECODE_MAX_ROUTES 8192
#define MOE_DECODE_MAX_ROWS_PER_EXPERT 8

/* moe_combine `out_dtype`. */
#define MOE_OUT_BF16 0
#define MOE_OUT_F32 1

/* Thread-local message describing the last error on this thread ("" if none). */
MOE_API const char* moe_last_error(void);

/* ABI version of this header (incremented on incompatible changes; 2: moe_combine
 * takes a status word). */
#define MOE_ABI_VERSION 2
MOE_API int moe_abi_version(void);

/* ---------------------------------------------------------------------------
 * moe_route -- softmax top-K routing with renormalisation.
 *
 * Defined by the decode kernel page's serving contract (router "softmax ->
 * top-8 -> norm") and the NKI Router Top-K kernel.  Per token t:
 *   p = softmax(logits[t, :]);  topk_ids[t, 0..K-1] = the K largest p in
 *   descending order, equal logits going to the lower expert id;
 *   topk_w[t, j] = p[topk_ids[t, j]] / sum_j' p[topk_ids[t, j']].
 * The kernel ranks by the fp32 logit (softmax is strictly increasing, so the
 * order is the same) and computes the weights in fp32 as
 * exp(l_j - l_max) / sum_j' exp(l_j' - l_max).
 *
 *   logits    [T, E] f32 (read)
 *   zero_mask [T, K] u8 or NULL (read): a nonzero entry sets topk_w[t, j] = 0
 *             after the renormalisation, with no second renormalisation (the
 *             zero-routing-weight case of the aiter prefill PR)
 *   topk_ids  [T, K] i32 (written)
 *   topk_w    [T, K] f32 (written)
 * Limits: 1 <= K <= min(E, MOE_MAX_K), 1 <= E <= MOE_MAX_E, 0 <= T <= MOE_MAX_T.
 * Logits must be finite; a NaN logit gives unspecified ids for that token.
 * ------------------------------------------------------------------------- */
MOE_API int moe_route(const float* logits, int T, int E, int K, const uint8_t* zero_mask,
              int32_t* topk_ids, float* topk_w, moe_stream_t stream);

/* ---------------------------------------------------------------------------
 * moe_route_ex -- routing variants: score function, selection-only bias,
 * group-limited choice, optional renormalisation, routed scaling factor.
 *
 * The pages name these routers without giving their formulas: the Nemotron-H
 * layer's sigmoid top-K routing scaled by `routed_scaling_factor`
 * (spark_model/layers/nemotron_moe.rs, module doc and `prefill`) and the NKI
 * library's DeepSeek-V3 group-limited `noaux_tc` router (NKI Library kernel
 * reference, MoE kernels).  Both are taken in the published DeepSeek-V3
 * router's form.  Per token t, with l = logits[t, :]:
 *   s_e = softmax(l)_e            (cfg->score == MOE_SCORE_SOFTMAX)
 *       = 1 / (1 + exp(-l_e))     (cfg->score == MOE_SCORE_SIGMOID)
 *   c_e = s_e + sel_bias[e]       (selection score; sel_bias NULL -> c = s)
 *   n_group > 1: expert e is in group e / (E / n_group); a group's score is
 *     the sum of its two largest c (its only c for one-expert groups); the
 *     topk_group groups of largest score are kept, equal scores going to the
 *     lower group index, and only their experts can be chosen;
 *   topk_ids[t, :] = the K eligible experts of largest c, descending, equal c
 *     going to the lower expert id;
 *   topk_w[t, j]   = scaling * s_{ids[t,j]} / (renormalize ? sum_j' s_{ids[t,j']} : 1).
 * The bias changes which experts are chosen, never their weights.  With
 * MOE_SCORE_SOFTMAX, no bias, n_group = 1, renormalize = 1 and scaling = 1
 * this is moe_route.
 * Precision: with no bias and n_group = 1 experts are ranked by the fp32 logit
 * (both scores are strictly increasing in it), exactly as moe_route; otherwise
 * by the kernel's fp32 c (expf-based), so experts whose c differ by a few fp32
 * ulps may be ranked either way.  Weights are computed in fp32.
 *
 *   cfg       host pointer (read during the call): score, sel_bias ([E] f32
 *             device pointer or NULL), n_group (1..MOE_MAX_GROUPS, divides E),
 *             topk_group (1..n_group, topk_group * (E / n_group) >= K),
 *             renormalize (0 or 1), scaling (finite, > 0)
 *   other arguments and limits as moe_route.
 * Errors: MOE_ERR_INVALID_ARG for a NULL cfg or a field outside its range.
 * ------------------------------------------------------------------------- */
#define MOE_SCORE_SOFTMAX 0
#define MOE_SCORE_SIGMOID 1
#define MOE_MAX_GROUPS 32

typedef struct moe_route_config {
    int score;             /* MOE_SCORE_SOFTMAX or MOE_SCORE_SIGMOID */
    const float* sel_bias; /* [E] f32 selection-only bias (device), or NULL */
    int n_group;           /* expert groups; 1 = no group limit */
    int topk_group;        /* groups kept per token (== n_group when n_group == 1) */
    int renormalize;       /* 1: divide the K weights by their sum */
    float scaling;         /* routed scaling factor applied to every weight */
} moe_route_config;

MOE_API int moe_route_ex(const float* logits, int T, int E, int K, const moe_route_config* cfg,
                         const uint8_t* zero_mask, int32_t* topk_ids, float* topk_w, moe_stream_t stream);

/* ---------------------------------------------------------------------------
 * moe_router -- fused router: gate GEMM and top-K routing in one kernel.
 *
 * The Nemotron-H layer's router is a dense gate GEMM, [N, H] x [H, E]^T ->
 * [N, E] logits (spark_model/layers/nemotron_moe.rs, `prefill`, step 2),
 * followed by the top-K kernel; the NKI library fuses the two (NKI Library
 * kernel reference, Router Top-K).  Per token t:
 *   logits[t, e] = sum_h x[t, h] * w_router[e, h]   (bf16 inputs, fp32 result)
 * then exactly what moe_route_ex computes from those fp32 logits (moe_route
 * when cfg is NULL).  The products are summed by the tensor cores in fp32, so
 * a logit differs from the exact sum by fp32 rounding; experts whose logits
 * (or selection scores) lie that close may be ranked either way.
 *
 *   x         [T, H] bf16 (read)
 *   w_router  [E, H] bf16 (read): row e = the gate vector of expert e
 *   cfg       host pointer or NULL (NULL = softmax, no bias, no groups,
 *             renormalised, scaling 1); fields and checks as moe_route_ex
 *   zero_mask, topk_ids, topk_w   as moe_route
 *   logits    [T, E] f32 (written) or NULL: a copy of the fp32 logits
 *   status    optional device int32: MOE_STATUS_TIMEOUT is OR-ed in if a
 *             bounded wait expired (never expected)
 * Limits: H % 64 == 0, 64 <= H <= MOE_ROUTER_MAX_H, 1 <= E <= MOE_ROUTER_MAX_E,
 *   1 <= K <= min(E, MOE_MAX_K), 0 <= T <= MOE_MAX_T; x and w_router 16-byte
 *   aligned (MOE_ERR_UNSUPPORTED_SHAPE / MOE_ERR_INVALID_ARG /
 *   MOE_ERR_MISALIGNED otherwise).  Allocates nothing; graph capturable.
 * ------------------------------------------------------------------------- */
#define MOE_ROUTER_MAX_E 512
#define MOE_ROUTER_MAX_H 16384
MOE_API int moe_router(const uint16_t* x, int T, int H, const uint16_t* w_router, int E, int K,
                       const moe_route_config* cfg, const uint8_t* zero_mask, int32_t* topk_ids, float* topk_w,
                       float* logits, int32_t* status, moe_stream_t stream);

/* ---------------------------------------------------------------------------
 * moe_router_plan_check -- a host-only diagnostic with no counterpart in the
 * pages: the launch plan moe_router would use for T tokens, width H and E
 * experts (with at most kch_max 64-column chunks per pipeline stage), checked
 * against the invariants the router kernel's indexing relies on.  Launches
 * nothing and touches no GPU.
 *   fields  host int32[9] or NULL: tiles, CTAs per cluster, experts per CTA,
 *           stages, TMEM columns, staging row stride (floats), x rows per
 *           tile, chunks per stage, dynamic shared memory bytes
 * Returns MOE_OK, MOE_ERR_INVALID_ARG for arguments outside moe_router's
 * limits (kch_max must be 1, 2 or 4), or MOE_ERR_UNSUPPORTED_SHAPE when the
 * plan breaks an invariant (moe_last_error names the field); moe_router
 * refuses such a plan the same way before launching.
 * ------------------------------------------------------------------------- */
MOE_API int moe_router_plan_check(int T, int H, int E, int kch_max, int32_t* fields);

/* ---------------------------------------------------------------------------
 * moe_selftest_bounded_wait -- a diagnostic with no counterpart in the pages:
 * it makes the kernels' bounded wait run out on purpose, without a fault.
 *
 * One CTA of the library's wait mechanism: two threads wait on mbarriers that
 * nothing completes.  Each wait gives up after the library's wait limit (2 s
 * of the GPU's global timer), ORs MOE_STATUS_TIMEOUT into *status and returns;
 * the kernel ends normally and the context stays usable.  Takes about 2 s.
 *   status      device int32 (required; the caller clears it)
 *   elapsed_ns  device uint64[2] (required): how long each wait took
 * Errors: MOE_ERR_INVALID_ARG for a NULL pointer, MOE_ERR_MISALIGNED for a
 * misaligned one.
 * ------------------------------------------------------------------------- */
MOE_API int moe_selftest_bounded_wait(int32_t* status, uint64_t* elapsed_ns, moe_stream_t stream);

/* ---------------------------------------------------------------------------
 * moe_sort -- stable sort of the R = T*K routes by expert.
 *
 * The step of the Nemotron prefill path that sorts the tokens by expert, the NKI
 * Permute Routed Tokens kernel, and the aiter pipeline's sort with inverse
 * route map.  A counting sort: per-chunk expert histograms, an expert-major
 * exclusive scan, and an in-order scatter, so the result is deterministic.
 *   expert_offsets[e]   = number of valid routes with id < e;
 *                         expert_offsets[E] = number of valid routes   [E+1] i32
 *   sorted_route[p]     = route r at sorted position p, routes of one expert in
 *                         increasing r; -1 for p >= expert_offsets[E]  [R] i32
 *   inv_route[r]        = sorted position of route r, -1 if skipped    [R] i32
 * Ids outside [0, E) are skipped (never written out of bounds) and set
 * MOE_STATUS_BAD_ID in *status (optional device int32, may be NULL; the
 * library only ORs bits into it, the caller clears it).
 *   workspace: device scratch of moe_sort_workspace_bytes(T, K, E) bytes, any
 *   contents; overwritten.
 * Limits: 1 <= K <= MOE_MAX_K, 1 <= E <= MOE_MAX_E (K > E is allowed: ids
 * need not be distinct within a token).
 * ------------------------------------------------------------------------- */
MOE_API size_t moe_sort_workspace_bytes(int T, int K, int E);
MOE_API int moe_sort(const int32_t* topk_ids, int T, int K, int E, int32_t* expert_offsets,
             int32_t* sorted_route, int32_t* inv_route, void* workspace,
             size_t workspace_bytes, int32_t* status, moe_stream_t stream);

/* ---------------------------------------------------------------------------
 * moe_sort_static_ws -- moe_sort for callers that cannot allocate device memory.
 *
 * The source paper has no counterpart of this call.  It exists for callers
 * that may not call cudaMalloc or any allocating routine: plugins whose host
 * framework owns every device allocation and hands out no scratch, and
 * processes held to a fixed device-memory budget.  It computes exactly what
 * moe_sort computes (same arguments, same outputs, bit for bit) but takes no
 * workspace: the scratch its multi-kernel path needs (one int32 counter per
 * expert per 2048-route chunk) lives in a statically allocated device array of
 * MOE_SORT_STATIC_WS_BYTES bytes inside the library, which every GPU that
 * loads the library holds until the process exits.  The call itself allocates
 * nothing (no cudaMalloc, cudaFree or allocating library routine).
 *  - Sizes whose scratch would exceed the array (E * ceil(T*K / 2048) * 4 >
 *    MOE_SORT_STATIC_WS_BYTES) are rejected with MOE_ERR_UNSUPPORTED_SHAPE and a
 *    message naming both byte counts; use moe_sort with a workspace for them.
 *  - The first call on a device looks up the array's device address (a host
 *    set-up step, with that device current); so does the first call after the
 *    device's context changed (a cudaDeviceReset, another context made
 *    current).  Make that first call before any stream capture.
 *  - Every call shares the one array and leaves its contents behind.  Nothing
 *    in it needs to start at zero: each call overwrites every counter it reads.
 *    Calls that overlap on the GPU (on different streams without ordering, or
 *    from several host threads) race on the array and give undefined results;
 *    order them on one stream.
 * ------------------------------------------------------------------------- */
#define MOE_SORT_STATIC_WS_BYTES (1u << 20)
MOE_API int moe_sort_static_ws(const int32_t* topk_ids, int T, int K, int E, int32_t* expert_offsets,
                               int32_t* sorted_route, int32_t* inv_route, int32_t* status,
                               moe_stream_t stream);

/* Block-scaled FP8 expert weights, expert-major (the caller owns the memory).
 * Rows are output features and the reduction index is contiguous:
 *   w_gate, w_up  [n_experts, inter, H] u8 E4M3FN codes
 *   w_down        [n_experts, H, inter] u8 E4M3FN codes
 *   s_gate, s_up  [n_experts, inter/128, H/128] f32 block scales
 *   s_down        [n_experts, H/128, inter/128] f32 block scales
 * Weight value W[n, k] = e4m3fn(code[n, k]) * s[n/128, k/128] (the exact
 * 128x128 block mapping of the decode kernel page's block_pow2 variant).
 * E4M3FN: bias 7, 3 mantissa bits, subnormals, S.1111.111 = NaN, no inf. */
typedef struct moe_fp8_experts {
    const uint8_t* w_gate;
    const uint8_t* w_up;
    const uint8_t* w_down;
    const float* s_gate;
    const float* s_up;
    const float* s_down;
    int n_experts;
    int inter;
} moe_fp8_experts;

/* ---------------------------------------------------------------------------
 * moe_ffn_resolve_mode -- the FFN form moe_expert_ffn runs for a given mode.
 *
 * No counterpart on the pages (they pick a kernel per serving phase: the NKI
 * library's MoE TKG for decode and MoE CTE for prefill).  Host-only, launches
 * nothing.  DECODE, PREFILL and HYBRID resolve to themselves; AUTO resolves
 * from host-known sizes alone (never from the device-side expert counts) to
 *   MOE_MODE_DECODE   when T*K <= MOE_DECODE_MAX_ROUTES and
 *                     T*K <= MOE_DECODE_MAX_ROWS_PER_EXPERT * E
 *                     (few rows per expert: streaming the touched weights
 *                     bounds the time),
 *   MOE_MODE_HYBRID   otherwise when T*K <= MOE_HYBRID_MAX_ROWS_PER_EXPERT * E
 *                     (a few tens of rows per expert on average: under a
 *                     skewed load many experts have a few rows and a few have
 *                     many, and each form takes the experts it is fast on; the
 *                     split is made on the device from the expert offsets),
 *   MOE_MODE_PREFILL  otherwise (enough rows per expert for the tensor-core
 *                     grouped GEMM to win).
 * Returns the resolved mode, or MOE_ERR_INVALID_ARG for an unknown mode or
 * T < 0, K < 1, E < 1.
 * ------------------------------------------------------------------------- */
MOE_API int moe_ffn_resolve_mode(int T, int K, int E, int mode);

/* ---------------------------------------------------------------------------
 * moe_expert_ffn -- grouped expert FFN over the sorted routes.
 *
 * For every expert e and sorted position p in [expert_offsets[e],
 * expert_offsets[e+1]), with route r = sorted_route[p] and token t = r / K:
 *   h        = silu(Wg_e x[t]) * (Wu_e x[t])          (SwiGLU, `_silu_mul`)
 *   y_sorted[p, :] = bf16( topk_w[r] * (Wd_e h) )     (affinity in the epilogue)
 * and, when `shared` is not NULL, for every token t:
 *   y_shared[t, :] = bf16( Wd_s (silu(Wg_s x[t]) * (Wu_s x[t])) )
 * This is the decode kernel page's fused chain (gate/up -> SwiGLU -> down ->
 * affinity scale) over the Nemotron page's sorted grouped-GEMM order; the
 * shared expert is the single always-on expert of the aiter PR, weight 1.
 * Numerics: bf16 x bf16 products accumulated in fp32; weights decoded from
 * E4M3FN to BF16 (DECODE mode: the exact E4M3 value, its block scale applied to
 * each 128-wide fp32 partial sum; PREFILL mode: bf16(e4m3 * scale));
 * h is rounded to bf16 between the two GEMMs.
 *
 *   x              [T, H] bf16 (read)
 *   routed         routed experts; routed->n_experts = E, routed->inter = I
 *   shared         NULL or one always-on expert (n_experts = 1, inter = I_s)
 *   expert_offsets [E+1] i32, sorted_route [T*K] i32 (as moe_sort writes them)
 *   topk_w         [T, K] f32 (read; route r's weight is topk_w[r])
 *   y_sorted       [T*K, H] bf16 (written for rows p < expert_offsets[E])
 *   y_shared       [T, H] bf16 (written) when shared != NULL, else ignored
 *   mode           MOE_MODE_AUTO | MOE_MODE_DECODE | MOE_MODE_PREFILL |
 *                  MOE_MODE_HYBRID (AUTO as moe_ffn_resolve_mode resolves it;
 *                  HYBRID launches both forms, each skipping the experts the
 *                  other takes, so every row is written exactly once; they
 *                  run side by side on disjoint SMs, the weight-streaming pair
 *                  on a library-owned second stream (created by the first
 *                  HYBRID call on a device) forked from `stream` and joined
 *                  back to it with events, so the call stays ordered on
 *                  `stream` and can be captured like the other forms)
 *   workspace      moe_ffn_workspace_bytes(...) bytes of device scratch
 *   status         optional device int32: MOE_STATUS_BAD_MAP is OR-ed in when
 *                  offsets or route ids are out of range (those rows skipped)
 * Limits: H % 128 == 0, I % 128 == 0, I_s % 128 == 0, 128 <= H <= 8192,
 *   128 <= I, I_s <= 4096, 1 <= E <= MOE_MAX_E, 1 <= K <= MOE_MAX_K
 *   (MOE_ERR_UNSUPPORTED_SHAPE / MOE_ERR_INVALID_ARG otherwise).
 * Zero-weight routes produce rows equal to +0 or -0 (a zero contribution) as
 * long as Wd_e h is finite.
 * ------------------------------------------------------------------------- */
MOE_API size_t moe_ffn_workspace_bytes(int T, int K, int H, int E, int I, int I_shared, int mode);
MOE_API int moe_expert_ffn(const uint16_t* x, int T, int H, int K, const moe_fp8_experts* routed,
                   const moe_fp8_experts* shared, const int32_t* expert_offsets,
                   const int32_t* sorted_route, const float* topk_w, uint16_t* y_sorted,
                   uint16_t* y_shared, int mode, void* workspace, size_t workspace_bytes,
                   int32_t* status, moe_stream_t stream);

/* ---------------------------------------------------------------------------
 * moe_expert_ffn_w8a8 -- moe_expert_ffn with FP8 activations (opt-in W8A8 form).
 *
 * The activation quantisation the pages describe for their low-precision
 * pipelines -- the NKI Library's Blockwise MM Forward MXFP8 kernel (FP8
 * activations against FP8 weights) and the aiter gfx950 PR's in-register
 * quantisation of the hidden activation -- applied to this library's FP8
 * E4M3FN weights with their 128x128 fp32 block scales:
 *   xq = quant(x) in blocks of 128 columns;  h = silu(Wg xq) * (Wu xq);
 *   hq = quant(h) in blocks of 64 features;  y_sorted[p] = w[r] * (Wd hq),
 * where quant(v) on a block is e4m3fn(v * 2^k) * 2^-k, with k the exponent
 * that puts the block's largest |v| in (224, 448] (k in [-126, 126], 0 for an
 * all-zero block), e4m3fn rounding to nearest even.  x is quantised from its
 * bf16 values as it is staged; h from its fp32 value in the gate/up epilogue
 * (it never exists as bf16).  Both GEMMs run as E4M3FN x E4M3FN tensor-core
 * MMAs with fp32 accumulation, the weight block scale and the activation
 * block scale applied to each 128-column (gate/up) or 64-column (down)
 * partial sum.  The weight-streaming (decode) kernels run for every T; the
 * result differs from moe_expert_ffn by the activation rounding (about 2 %
 * relative in the library's tests; see its parity tests for the bound).
 *   Arguments, layouts, limits and errors: those of moe_expert_ffn without
 *   `mode`.  workspace: moe_ffn_w8a8_workspace_bytes(T, K, I, I_shared)
 *   bytes (h as E4M3FN bytes and its block scales), any contents.
 * ------------------------------------------------------------------------- */
MOE_API size_t moe_ffn_w8a8_workspace_bytes(int T, int K, int I, int I_shared);
MOE_API int moe_expert_ffn_w8a8(const uint16_t* x, int T, int H, int K, const moe_fp8_experts* routed,
                   const moe_fp8_experts* shared, const int32_t* expert_offsets,
                   const int32_t* sorted_route, const float* topk_w, uint16_t* y_sorted,
                   uint16_t* y_shared, void* workspace, size_t workspace_bytes,
                   int32_t* status, moe_stream_t stream);

/* ---------------------------------------------------------------------------
 * moe_expert_ffn_combine -- the expert FFN and the combine in one call
 * (tensor-core form), without the sorted rows.
 *
 * out[t, :] = sum_j topk_w[t*K+j] * FFN_{e(t,j)}(x[t])  (+ FFN_shared(x[t]))
 * -- what moe_expert_ffn followed by moe_combine computes, the reduction of
 * the aiter PR's fused producer and the Nemotron-H page's unpermute-reduce
 * (spark_model/layers/nemotron_moe.rs, `prefill` step 5) -- with the down
 * GEMM's epilogue adding each sorted row (bf16, route weight applied, as the
 * row moe_expert_ffn would store) into its token's fp32 output row with vector
 * fp32 reductions at L2, instead of writing y_sorted for moe_combine to read
 * back.  The order of the fp32 additions is not fixed: results may differ
 * from run to run by fp32 rounding (moe_expert_ffn + moe_combine is the
 * deterministic form).  Always runs the PREFILL kernels.
 *   x, routed, shared, expert_offsets, sorted_route, topk_w   as moe_expert_ffn
 *   out        [T, H], bf16 (out_dtype MOE_OUT_BF16) or f32 (MOE_OUT_F32)
 *   workspace  moe_ffn_combine_workspace_bytes(...) bytes (bf16 output: it
 *              also holds the [T, H] f32 accumulator)
 *   status     optional device int32, as moe_expert_ffn
 * Limits and errors as moe_expert_ffn.
 * ------------------------------------------------------------------------- */
MOE_API size_t moe_ffn_combine_workspace_bytes(int T, int K, int H, int E, int I, int I_shared, int out_dtype);
MOE_API int moe_expert_ffn_combine(const uint16_t* x, int T, int H, int K, const moe_fp8_experts* routed,
                                   const moe_fp8_experts* shared, const int32_t* expert_offsets,
                                   const int32_t* sorted_route, const float* topk_w, void* out, int out_dtype,
                                   void* workspace, size_t workspace_bytes, int32_t* status, moe_stream_t stream);

/* ---------------------------------------------------------------------------
 * moe_combine -- top-K reduce back to token order.
 *
 * The Nemotron unpermute-reduce, the aiter FP32 route reduction and the NKI
 * Top-K Reduce:  out[t, :] = sum_{j=0..K-1} y_sorted[inv_route[t*K + j], :]
 *                            (+ y_shared[t, :] if y_shared != NULL),
 * summed in fp32 in slot order j = 0..K-1 (then the shared term), one rounding
 * at the end.  Routes with inv_route = -1 add nothing.
 *   y_sorted  [T*K, H] bf16; inv_route [T*K] i32; y_shared [T, H] bf16 or NULL
 *   out       [T, H], bf16 (out_dtype MOE_OUT_BF16) or f32 (MOE_OUT_F32)
 *   status    optional device int32 (4-byte aligned, may be NULL): an
 *             inv_route entry outside [0, T*K) other than -1 is skipped (never
 *             read out of bounds) and sets MOE_STATUS_BAD_MAP
 * Limits: H % 8 == 0, 1 <= K <= MOE_MAX_K.
 * ------------------------------------------------------------------------- */
MOE_API int moe_combine(const uint16_t* y_sorted, const int32_t* inv_route, const uint16_t* y_shared,
                int T, int K, int H, void* out, int out_dtype, int32_t* status, moe_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* MOE_FFN_H */
