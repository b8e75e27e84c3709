/*
 * moe_oracle.c -- plain, slow fp64 CPU oracle of the routed MoE FFN.
 *
 * TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and
 * bench.py's cpu_baseline / reference leg may load this library.  It shares no
 * code, header, table or constant with the CUDA library (it includes nothing
 * but the C standard library) and the CUDA library never calls it.
 *
 * What it computes, for every token t (x[t] in R^H, logits[t] in R^E):
 *
 *   p          = softmax(logits[t])                                  (route)
 *   ids[t, :]  = the K experts of largest p, descending, ties -> lower id
 *   w[t, j]    = p[ids[t,j]] / sum_j' p[ids[t,j']]                   (renormalise)
 *   W[n, k]    = e4m3fn(q[n, k]) * s[n/128, k/128]                    (block-scaled FP8)
 *   FFN_e(x)   = Wd_e (silu(Wg_e x) * (Wu_e x)),  silu(z) = z / (1 + e^-z)
 *   out[t]     = sum_j w[t,j] FFN_{ids[t,j]}(x[t]) + FFN_shared(x[t])
 *   logits[t]  = W_r x[t]   (the router's gate GEMM, when the logits are not given)
 *
 * Sources (page title, section):
 *  - dstair/gated-deltanet-nki-trainium, "FP8 MoE decode kernel
 *    (moe_fused_w8_35b)": the fused expert chain gate/up GEMM -> SwiGLU ->
 *    down GEMM -> affinity scale -> expert-sum with E4M3FN weights and 128x128
 *    block scales; "Serving contract": router softmax -> top-8 -> norm, shared
 *    expert added after the routed sum.
 *  - nemo_automodel ... qwen3_5.layers, `_silu_mul`: SwiGLU is silu(gate) * up.
 *  - spark_model/layers/nemotron_moe.rs, module doc and `prefill` step 5: sort
 *    tokens by expert, grouped GEMM over each expert's rows, unpermute-reduce.
 *  - ROCm/aiter PR #5988 description: the sorted pipeline with an inverse
 *    route map and an FP32 route reduction; ten routed experts and one shared
 *    expert per token.
 *  - spark_model/layers/nemotron_moe.rs, `prefill` step 2: the router's dense
 *    gate GEMM [N, H] x [H, E]^T -> [N, E] logits.
 *  - NKI Library kernel reference, MoE kernels: Router Top-K, Permute Routed
 *    Tokens (sort by expert), Top-K Reduce.
 *
 * Precision: fp64 throughout (exp, silu, every product and sum).  Inputs are
 * bf16 / fp32 / E4M3FN bit patterns and are widened exactly.  The one place
 * where floating point decides an integer is the top-K choice; it compares the
 * fp32 logits themselves.  Softmax is strictly increasing in the logit, so the
 * K largest logits are the K largest probabilities; comparing the fp32 inputs
 * takes that decision exactly, in the same precision as the kernel.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_BLOCK 128

/* ---------------------------------------------------------------- threads */

static int g_threads = 1;

int oracle_set_threads(int n) {
#ifdef _OPENMP
    if (n < 1) n = 1;
    g_threads = n;
    return n;
#else
    (void)n;
    g_threads = 1;
    return 1;
#endif
}

int oracle_get_threads(void) { return g_threads; }

/* ---------------------------------------------------------------- formats */

/* OCP FP8 E4M3FN (the weight format the decode kernel page names):
 * 1 sign bit, 4 exponent bits with bias 7, 3 mantissa bits.
 * exponent 0: subnormal, value (m/8) * 2^-6.  exponent 1..15: (1 + m/8) * 2^(e-7).
 * S.1111.111 is NaN; there is no infinity (so S.1111.110 = 448 is the maximum). */
double oracle_e4m3fn_value(uint8_t code) {
    int sign = (code >> 7) & 1;
    int e = (code >> 3) & 0xF;
    int m = code & 0x7;
    double v;
    if (e == 0xF && m == 0x7) return NAN;
    if (e == 0)
        v = ldexp((double)m / 8.0, -6);
    else
        v = ldexp(1.0 + (double)m / 8.0, e - 7);
    return sign ? -v : v;
}

/* bfloat16: the upper 16 bits of an IEEE binary32. */
double oracle_bf16_value(uint16_t bits) {
    uint32_t u = (uint32_t)bits << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* oracle_e4m3fn_value of every code, filled once before any parallel region. */
static double g_e4m3[256];
static int g_e4m3_ready = 0;

static void init_tables(void) {
    if (g_e4m3_ready) return;
    for (int c = 0; c < 256; ++c) g_e4m3[c] = oracle_e4m3fn_value((uint8_t)c);
    g_e4m3_ready = 1;
}

/* One weight element of a block-scaled FP8 matrix [rows, cols] (cols contiguous):
 * W[n, k] = e4m3fn(q[n, k]) * s[n / 128, k / 128]. */
static double weight(const uint8_t* q, const float* s, int cols, int n, int k) {
    int ncb = cols / ORACLE_BLOCK;
    return g_e4m3[q[(size_t)n * cols + k]] *
           (double)s[(size_t)(n / ORACLE_BLOCK) * ncb + (k / ORACLE_BLOCK)];
}

/* ---------------------------------------------------------------- route */

/* Router of the decode kernel page's serving contract: softmax over the E
 * logits, the top-K experts, then their probabilities renormalised to sum 1.
 * Slot j holds the j-th largest; equal logits go to the lower expert id.
 * zero_mask (nullable, [T, K]): a nonzero entry forces w[t, j] = 0 after the
 * renormalisation, with no second renormalisation (the "zero routing weights"
 * replay case of the aiter prefill PR). */
void oracle_route(const float* logits, int T, int E, int K, const uint8_t* zero_mask,
                  int32_t* ids, double* w) {
#pragma omp parallel for num_threads(g_threads) schedule(static)
    for (int t = 0; t < T; ++t) {
        const float* l = logits + (size_t)t * E;
        double* p = (double*)malloc(sizeof(double) * (size_t)E);
        unsigned char* taken = (unsigned char*)calloc((size_t)E, 1);
        double lmax = -INFINITY, z = 0.0;
        for (int e = 0; e < E; ++e)
            if ((double)l[e] > lmax) lmax = (double)l[e];
        for (int e = 0; e < E; ++e) {
            p[e] = exp((double)l[e] - lmax);
            z += p[e];
        }
        for (int e = 0; e < E; ++e) p[e] /= z;

        double sel = 0.0;
        for (int j = 0; j < K; ++j) {
            int best = -1;
            for (int e = 0; e < E; ++e) {
                if (taken[e]) continue;
                if (best < 0 || l[e] > l[best]) best = e; /* strict >: ties keep the lower id */
            }
            taken[best] = 1;
            ids[(size_t)t * K + j] = best;
            sel += p[best];
        }
        for (int j = 0; j < K; ++j) {
            double v = p[ids[(size_t)t * K + j]] / sel;
            if (zero_mask && zero_mask[(size_t)t * K + j]) v = 0.0;
            w[(size_t)t * K + j] = v;
        }
        free(p);
        free(taken);
    }
}

/* Routing variants named by the pages without a formula -- the Nemotron-H
 * layer's sigmoid top-K routing scaled by `routed_scaling_factor`
 * (spark_model/layers/nemotron_moe.rs, module doc and `prefill`) and the NKI
 * library's "DeepSeek-V3 group-limited noaux_tc routing" (NKI Library kernel
 * reference, MoE kernels) -- taken in the published DeepSeek-V3 router's form:
 *   s_e  = softmax(l)_e (score 0) or 1 / (1 + e^-l_e) (score 1)
 *   c_e  = s_e + bias[e]                 (selection only; bias NULL -> 0)
 *   with n_group > 1, expert e is in group e / (E / n_group); a group scores
 *   the sum of its two largest c (its one c if it has one expert); the
 *   topk_group best groups are kept (equal scores -> lower group index) and
 *   only their experts may be chosen
 *   ids  = the K eligible experts of largest c, descending, ties -> lower id
 *   w_j  = scaling * s_{ids_j} / (renormalize ? sum_j' s_{ids_j'} : 1)
 * With no bias and one group the ranking compares the fp32 logits themselves
 * (both scores are strictly increasing in the logit); otherwise it compares
 * the fp64 c.  zero_mask as in oracle_route. */
static void route_scores(const float* l, int E, int score, double* s) {
    if (score == 0) {
        double lmax = -INFINITY, z = 0.0;
        for (int e = 0; e < E; ++e)
            if ((double)l[e] > lmax) lmax = (double)l[e];
        for (int e = 0; e < E; ++e) {
            s[e] = exp((double)l[e] - lmax);
            z += s[e];
        }
        for (int e = 0; e < E; ++e) s[e] /= z;
    } else {
        for (int e = 0; e < E; ++e) s[e] = 1.0 / (1.0 + exp(-(double)l[e]));
    }
}

void oracle_route_ex(const float* logits, int T, int E, int K, int score, const float* bias,
                     int n_group, int topk_group, int renormalize, double scaling,
                     const uint8_t* zero_mask, int32_t* ids, double* w) {
    const int by_logit = bias == NULL && n_group <= 1;
    const int G = n_group > 1 ? E / n_group : E;
#pragma omp parallel for num_threads(g_threads) schedule(static)
    for (int t = 0; t < T; ++t) {
        const float* l = logits + (size_t)t * E;
        double* s = (double*)malloc(sizeof(double) * (size_t)E);
        double* c = (double*)malloc(sizeof(double) * (size_t)E);
        unsigned char* ok = (unsigned char*)malloc((size_t)E);
        route_scores(l, E, score, s);
        for (int e = 0; e < E; ++e) {
            c[e] = by_logit ? (double)l[e] : s[e] + (bias ? (double)bias[e] : 0.0);
            ok[e] = 1;
        }
        if (n_group > 1) {
            double gs[64];
            unsigned char keep[64];
            for (int g = 0; g < n_group; ++g) {
                double a = -INFINITY, b = -INFINITY; /* two largest c of the group */
                for (int e = g * G; e < (g + 1) * G; ++e) {
                    if (c[e] > a) {
                        b = a;
                        a = c[e];
                    } else if (c[e] > b) {
                        b = c[e];
                    }
                }
                gs[g] = G > 1 ? a + b : a;
                keep[g] = 0;
            }
            for (int r = 0; r < topk_group; ++r) {
                int best = -1;
                for (int g = 0; g < n_group; ++g)
                    if (!keep[g] && (best < 0 || gs[g] > gs[best])) best = g;
                keep[best] = 1;
            }
            for (int e = 0; e < E; ++e) ok[e] = keep[e / G];
        }
        double sum = 0.0;
        for (int j = 0; j < K; ++j) {
            int best = -1;
            for (int e = 0; e < E; ++e) {
                if (!ok[e]) continue;
                if (best < 0 || c[e] > c[best]) best = e; /* strict >: ties keep the lower id */
            }
            ok[best] = 0;
            ids[(size_t)t * K + j] = best;
            sum += s[best];
        }
        for (int j = 0; j < K; ++j) {
            double v = scaling * s[ids[(size_t)t * K + j]] / (renormalize ? sum : 1.0);
            if (zero_mask && zero_mask[(size_t)t * K + j]) v = 0.0;
            w[(size_t)t * K + j] = v;
        }
        free(s);
        free(c);
        free(ok);
    }
}

/* The weights the routing variants give a chosen set of experts: w[t, j] as in
 * oracle_route_ex for ids[t, :] supplied by the caller (used to score a choice
 * that differs from the oracle's only between experts whose selection scores
 * tie to fp32 rounding). */
void oracle_route_weights(const float* logits, int T, int E, int K, int score, int renormalize,
                          double scaling, const int32_t* ids, double* w) {
    double* s = (double*)malloc(sizeof(double) * (size_t)E);
    for (int t = 0; t < T; ++t) {
        route_scores(logits + (size_t)t * E, E, score, s);
        double sum = 0.0;
        for (int j = 0; j < K; ++j) sum += s[ids[(size_t)t * K + j]];
        for (int j = 0; j < K; ++j)
            w[(size_t)t * K + j] = scaling * s[ids[(size_t)t * K + j]] / (renormalize ? sum : 1.0);
    }
    free(s);
}

/* The selection score c of every expert (fp64), as oracle_route_ex ranks them
 * when a bias or groups are present. */
void oracle_route_select_scores(const float* logits, int T, int E, int score, const float* bias,
                                double* c) {
    for (int t = 0; t < T; ++t) {
        double* ct = c + (size_t)t * E;
        route_scores(logits + (size_t)t * E, E, score, ct);
        if (bias)
            for (int e = 0; e < E; ++e) ct[e] += (double)bias[e];
    }
}

/* ---------------------------------------------------------------- router GEMM */

/* The router's gate GEMM (spark_model/layers/nemotron_moe.rs, `prefill`, step
 * 2: [N, H] x [H, E]^T -> [N, E] gate logits): for every token t and expert e,
 *   logits[t, e] = sum_h x[t, h] * w_router[e, h],
 * the bf16 inputs widened exactly, every product and the sum in fp64, h in
 * increasing order.  The route step takes fp32 logits; the caller rounds. */
void oracle_router_logits(const uint16_t* x, const uint16_t* w_router, int T, int H, int E, double* logits) {
#pragma omp parallel for num_threads(g_threads) schedule(static)
    for (int t = 0; t < T; ++t) {
        for (int e = 0; e < E; ++e) {
            double acc = 0.0;
            for (int h = 0; h < H; ++h)
                acc += oracle_bf16_value(x[(size_t)t * H + h]) * oracle_bf16_value(w_router[(size_t)e * H + h]);
            logits[(size_t)t * E + e] = acc;
        }
    }
}

/* ---------------------------------------------------------------- sort */

/* Sort the R = T*K routes (route r = t*K + j carries expert ids[r]) by expert,
 * keeping route order within an expert (a stable counting sort: count, exclusive
 * scan, scatter in route order).  This is the step that sorts the tokens by expert in the
 * Nemotron prefill path and the NKI "Permute Routed Tokens" kernel.
 *   offsets[e]       = number of valid routes with id < e; offsets[E] = valid routes
 *   sorted_route[p]  = the route at sorted position p (p < offsets[E]); -1 after
 *   inv_route[r]     = the sorted position of route r; -1 for an id outside [0, E)
 * Returns the number of routes whose id is outside [0, E) (they are skipped). */
int oracle_sort(const int32_t* ids, int T, int K, int E, int32_t* offsets,
                int32_t* sorted_route, int32_t* inv_route) {
    long R = (long)T * K;
    int bad = 0;
    int32_t* count = (int32_t*)calloc((size_t)E + 1, sizeof(int32_t));
    for (long r = 0; r < R; ++r) {
        int e = ids[r];
        if (e < 0 || e >= E) { bad++; continue; }
        count[e]++;
    }
    offsets[0] = 0;
    for (int e = 0; e < E; ++e) offsets[e + 1] = offsets[e] + count[e];
    int32_t* cursor = count;
    for (int e = 0; e < E; ++e) cursor[e] = offsets[e];
    for (long p = 0; p < R; ++p) sorted_route[p] = -1;
    for (long r = 0; r < R; ++r) {
        int e = ids[r];
        if (e < 0 || e >= E) { inv_route[r] = -1; continue; }
        int32_t pos = cursor[e]++;
        sorted_route[pos] = (int32_t)r;
        inv_route[r] = pos;
    }
    free(count);
    return bad;
}

/* ---------------------------------------------------------------- expert FFN */

/* One expert applied to one row: y = Wd (silu(Wg x) * (Wu x)).
 * Wg, Wu: [I, H] codes with [I/128, H/128] scales; Wd: [H, I] with [H/128, I/128].
 * SwiGLU as `_silu_mul` of the qwen3_5.layers page: silu(gate) * up. */
static void expert_row(const double* x, int H, int I,
                       const uint8_t* wg, const float* sg, const uint8_t* wu, const float* su,
                       const uint8_t* wd, const float* sd, double* h, double* y) {
    for (int i = 0; i < I; ++i) {
        double g = 0.0, u = 0.0;
        for (int k = 0; k < H; ++k) {
            g += weight(wg, sg, H, i, k) * x[k];
            u += weight(wu, su, H, i, k) * x[k];
        }
        h[i] = (g / (1.0 + exp(-g))) * u;
    }
    for (int n = 0; n < H; ++n) {
        double acc = 0.0;
        for (int i = 0; i < I; ++i) acc += weight(wd, sd, I, n, i) * h[i];
        y[n] = acc;
    }
}

/* Expert tensors, expert-major as the CUDA library also takes them. */
typedef struct {
    const uint8_t* w_gate; const float* s_gate;
    const uint8_t* w_up;   const float* s_up;
    const uint8_t* w_down; const float* s_down;
    int n_experts; int inter;
} oracle_experts;

static void expert_ptrs(const oracle_experts* ex, int e, int H,
                        const uint8_t** wg, const float** sg, const uint8_t** wu,
                        const float** su, const uint8_t** wd, const float** sd) {
    size_t I = (size_t)ex->inter;
    size_t nw = I * (size_t)H, ns = (I / ORACLE_BLOCK) * ((size_t)H / ORACLE_BLOCK);
    *wg = ex->w_gate + (size_t)e * nw; *sg = ex->s_gate + (size_t)e * ns;
    *wu = ex->w_up + (size_t)e * nw;   *su = ex->s_up + (size_t)e * ns;
    *wd = ex->w_down + (size_t)e * nw; *sd = ex->s_down + (size_t)e * ns;
}

static void load_row(const uint16_t* x, int H, int t, double* xr) {
    for (int k = 0; k < H; ++k) xr[k] = oracle_bf16_value(x[(size_t)t * H + k]);
}

/* Grouped expert FFN over the sorted routes (the grouped GEMM over expert-sorted rows of the
 * Nemotron prefill path): for each expert e and each sorted position p in
 * [offsets[e], offsets[e+1]), route r = sorted_route[p], token t = r / K:
 *     y_sorted[p] = w[r] * FFN_e(x[t])
 * (the affinity scale of the decode kernel page's chain, applied per route). */
void oracle_ffn_sorted(const uint16_t* x, int T, int H, int K, const oracle_experts* ex,
                       const int32_t* offsets, const int32_t* sorted_route, const double* w,
                       double* y_sorted) {
    init_tables();
    (void)T;
    int E = ex->n_experts, I = ex->inter;
    for (int e = 0; e < E; ++e) {
        const uint8_t *wg, *wu, *wd; const float *sg, *su, *sd;
        expert_ptrs(ex, e, H, &wg, &sg, &wu, &su, &wd, &sd);
        int p0 = offsets[e], p1 = offsets[e + 1];
#pragma omp parallel for num_threads(g_threads) schedule(dynamic, 1)
        for (int p = p0; p < p1; ++p) {
            double* xr = (double*)malloc(sizeof(double) * (size_t)H);
            double* h = (double*)malloc(sizeof(double) * (size_t)I);
            int r = sorted_route[p];
            load_row(x, H, r / K, xr);
            double* y = y_sorted + (size_t)p * H;
            expert_row(xr, H, I, wg, sg, wu, su, wd, sd, h, y);
            for (int n = 0; n < H; ++n) y[n] *= w[r];
            free(xr);
            free(h);
        }
    }
}

/* The always-on shared expert (weight 1, every token): y_shared[t] = FFN_s(x[t]). */
void oracle_ffn_shared(const uint16_t* x, int T, int H, const oracle_experts* sh,
                       double* y_shared) {
    init_tables();
    const uint8_t *wg, *wu, *wd; const float *sg, *su, *sd;
    expert_ptrs(sh, 0, H, &wg, &sg, &wu, &su, &wd, &sd);
    int I = sh->inter;
#pragma omp parallel for num_threads(g_threads) schedule(dynamic, 1)
    for (int t = 0; t < T; ++t) {
        double* xr = (double*)malloc(sizeof(double) * (size_t)H);
        double* h = (double*)malloc(sizeof(double) * (size_t)I);
        load_row(x, H, t, xr);
        expert_row(xr, H, I, wg, sg, wu, su, wd, sd, h, y_shared + (size_t)t * H);
        free(xr);
        free(h);
    }
}

/* Top-K reduce through the inverse route map (Nemotron's unpermute-reduce, the
 * aiter FP32 route reduction, NKI Top-K Reduce): out[t] = sum over slots j of
 * y_sorted[inv_route[t*K + j]] (+ y_shared[t]); routes with inv_route -1 add 0. */
void oracle_combine(const double* y_sorted, const int32_t* inv_route, const double* y_shared,
                    int T, int K, int H, double* out) {
#pragma omp parallel for num_threads(g_threads) schedule(static)
    for (int t = 0; t < T; ++t) {
        double* o = out + (size_t)t * H;
        for (int n = 0; n < H; ++n) o[n] = y_shared ? y_shared[(size_t)t * H + n] : 0.0;
        for (int j = 0; j < K; ++j) {
            int32_t p = inv_route[(size_t)t * K + j];
            if (p < 0) continue;
            const double* y = y_sorted + (size_t)p * H;
            for (int n = 0; n < H; ++n) o[n] += y[n];
        }
    }
}

/* The same reduction over bf16 operands (for checking the combine step alone). */
void oracle_combine_bf16(const uint16_t* y_sorted, const int32_t* inv_route,
                         const uint16_t* y_shared, int T, int K, int H, double* out) {
#pragma omp parallel for num_threads(g_threads) schedule(static)
    for (int t = 0; t < T; ++t) {
        double* o = out + (size_t)t * H;
        for (int n = 0; n < H; ++n)
            o[n] = y_shared ? oracle_bf16_value(y_shared[(size_t)t * H + n]) : 0.0;
        for (int j = 0; j < K; ++j) {
            int32_t p = inv_route[(size_t)t * K + j];
            if (p < 0) continue;
            for (int n = 0; n < H; ++n) o[n] += oracle_bf16_value(y_sorted[(size_t)p * H + n]);
        }
    }
}

/* ---------------------------------------------------------------- whole path */

/* Structured form: route -> sort -> grouped FFN -> shared -> combine, returning
 * every intermediate.  y_sorted is [T*K, H]; y_shared may be NULL when sh is NULL. */
int oracle_moe(const uint16_t* x, const float* logits, int T, int H, int E, int K,
               const uint8_t* zero_mask, const oracle_experts* routed, const oracle_experts* sh,
               int32_t* ids, double* w, int32_t* offsets, int32_t* sorted_route,
               int32_t* inv_route, double* y_sorted, double* y_shared, double* out) {
    oracle_route(logits, T, E, K, zero_mask, ids, w);
    int bad = oracle_sort(ids, T, K, E, offsets, sorted_route, inv_route);
    oracle_ffn_sorted(x, T, H, K, routed, offsets, sorted_route, w, y_sorted);
    if (sh) oracle_ffn_shared(x, T, H, sh, y_shared);
    oracle_combine(y_sorted, inv_route, sh ? y_shared : NULL, T, K, H, out);
    return bad;
}

/* Brute-force form, straight from the per-token definition, for a list of tokens
 * (tokens == NULL: all T in order): out[i] = sum_j w[t,j] FFN_{ids[t,j]}(x[t]) + FFN_s(x[t])
 * with t = tokens[i].  No sort, no inverse map. */
void oracle_moe_tokens(const uint16_t* x, const float* logits, int T, int H, int E, int K,
                       const uint8_t* zero_mask, const oracle_experts* routed,
                       const oracle_experts* sh, const int32_t* tokens, int n_tokens,
                       double* out) {
    init_tables();
    (void)T;
    int I = routed->inter;
    int Is = sh ? sh->inter : 0;
    int Imax = I > Is ? I : Is;
#pragma omp parallel for num_threads(g_threads) schedule(dynamic, 1)
    for (int i = 0; i < n_tokens; ++i) {
        int t = tokens ? tokens[i] : i;
        double* xr = (double*)malloc(sizeof(double) * (size_t)H);
        double* h = (double*)malloc(sizeof(double) * (size_t)Imax);
        double* y = (double*)malloc(sizeof(double) * (size_t)H);
        int32_t* tid = (int32_t*)malloc(sizeof(int32_t) * (size_t)K);
        double* tw = (double*)malloc(sizeof(double) * (size_t)K);
        double* o = out + (size_t)i * H;
        load_row(x, H, t, xr);
        oracle_route(logits + (size_t)t * E, 1, E, K, zero_mask ? zero_mask + (size_t)t * K : NULL,
                     tid, tw);
        for (int n = 0; n < H; ++n) o[n] = 0.0;
        for (int j = 0; j < K; ++j) {
            const uint8_t *wg, *wu, *wd; const float *sg, *su, *sd;
            expert_ptrs(routed, tid[j], H, &wg, &sg, &wu, &su, &wd, &sd);
            expert_row(xr, H, I, wg, sg, wu, su, wd, sd, h, y);
            for (int n = 0; n < H; ++n) o[n] += tw[j] * y[n];
        }
        if (sh) {
            const uint8_t *wg, *wu, *wd; const float *sg, *su, *sd;
            expert_ptrs(sh, 0, H, &wg, &sg, &wu, &su, &wd, &sd);
            expert_row(xr, H, Is, wg, sg, wu, su, wd, sd, h, y);
            for (int n = 0; n < H; ++n) o[n] += y[n];
        }
        free(xr); free(h); free(y); free(tid); free(tw);
    }
}

/* oracle_moe_tokens with the routing given: row i of ids / w ([n_tokens, K])
 * holds the experts and weights of token tokens[i] (any router's choice). */
void oracle_moe_tokens_routed(const uint16_t* x, int H, int K, const int32_t* ids, const double* w,
                              const oracle_experts* routed, const oracle_experts* sh,
                              const int32_t* tokens, int n_tokens, double* out) {
    init_tables();
    int I = routed->inter;
    int Is = sh ? sh->inter : 0;
    int Imax = I > Is ? I : Is;
#pragma omp parallel for num_threads(g_threads) schedule(dynamic, 1)
    for (int i = 0; i < n_tokens; ++i) {
        int t = tokens ? tokens[i] : i;
        double* xr = (double*)malloc(sizeof(double) * (size_t)H);
        double* h = (double*)malloc(sizeof(double) * (size_t)Imax);
        double* y = (double*)malloc(sizeof(double) * (size_t)H);
        double* o = out + (size_t)i * H;
        load_row(x, H, t, xr);
        for (int n = 0; n < H; ++n) o[n] = 0.0;
        for (int j = 0; j < K; ++j) {
            const uint8_t *wg, *wu, *wd; const float *sg, *su, *sd;
            expert_ptrs(routed, ids[(size_t)i * K + j], H, &wg, &sg, &wu, &su, &wd, &sd);
            expert_row(xr, H, I, wg, sg, wu, su, wd, sd, h, y);
            for (int n = 0; n < H; ++n) o[n] += w[(size_t)i * K + j] * y[n];
        }
        if (sh) {
            const uint8_t *wg, *wu, *wd; const float *sg, *su, *sd;
            expert_ptrs(sh, 0, H, &wg, &sg, &wu, &su, &wd, &sd);
            expert_row(xr, H, Is, wg, sg, wu, su, wd, sd, h, y);
            for (int n = 0; n < H; ++n) o[n] += y[n];
        }
        free(xr); free(h); free(y);
    }
}

/* One expert FFN on explicit rows (no routing): y[i] = FFN_e(x[rows[i]]). */
void oracle_expert_rows(const uint16_t* x, int H, const oracle_experts* ex, int e,
                        const int32_t* rows, int n_rows, double* y) {
    init_tables();
    const uint8_t *wg, *wu, *wd; const float *sg, *su, *sd;
    expert_ptrs(ex, e, H, &wg, &sg, &wu, &su, &wd, &sd);
    int I = ex->inter;
#pragma omp parallel for num_threads(g_threads) schedule(dynamic, 1)
    for (int i = 0; i < n_rows; ++i) {
        double* xr = (double*)malloc(sizeof(double) * (size_t)H);
        double* h = (double*)malloc(sizeof(double) * (size_t)I);
        load_row(x, H, rows[i], xr);
        expert_row(xr, H, I, wg, sg, wu, su, wd, sd, h, y + (size_t)i * H);
        free(xr);
        free(h);
    }
}

/* SwiGLU alone, for pinning: h[i] = silu(g[i]) * u[i]. */
void oracle_swiglu(const double* g, const double* u, int n, double* h) {
    for (int i = 0; i < n; ++i) h[i] = (g[i] / (1.0 + exp(-g[i]))) * u[i];
}

/* ---------------------------------------------------------------- FP8 activations (W8A8) */

/* The opt-in W8A8 form: the activations of both GEMMs also become E4M3FN
 * values, in blocks with one power-of-two scale each (the FP8 activation
 * quantisation of the NKI Library's Blockwise MM Forward MXFP8 kernel and the
 * in-register quantisation of the hidden activation of the aiter gfx950 PR,
 * there with MX formats; here E4M3FN with a power-of-two scale per block, the
 * plainest reading that keeps the weights' own format).  Blocks: 128 columns
 * of x (one weight scale block), 64 features of h. */
#define ORACLE_XQ_BLOCK 128
#define ORACLE_HQ_BLOCK 64

/* Nearest E4M3FN value to v, ties to the even mantissa (round to nearest
 * even), magnitudes at or above the largest finite value 448 giving 448
 * (saturating conversion).  Subnormals are the multiples of 2^-9 below 2^-6;
 * in the binade [2^e, 2^(e+1)) the values are the multiples of 2^(e-3). */
double oracle_e4m3fn_round(double v) {
    if (v != v) return NAN;
    double a = fabs(v), q;
    if (a >= 448.0) {
        q = 448.0;
    } else if (a < ldexp(1.0, -6)) {
        q = nearbyint(ldexp(a, 9)) * ldexp(1.0, -9);
    } else {
        int e;
        frexp(a, &e); /* a = f * 2^e, f in [0.5, 1): the binade is [2^(e-1), 2^e) */
        q = ldexp(nearbyint(ldexp(a, 4 - e)), e - 4);
    }
    return v < 0 ? -q : q;
}

void oracle_e4m3fn_round_array(const double* v, int n, double* out) {
    for (int i = 0; i < n; ++i) out[i] = oracle_e4m3fn_round(v[i]);
}

/* Scale exponent k of an activation block whose largest magnitude is amax:
 * amax * 2^k lies in (224, 448] (the top binade of E4M3FN up to its largest
 * value), k limited to [-126, 126]; 0 for an all-zero block. */
int oracle_act_scale_exp(double amax) {
    if (!(amax > 0.0)) return 0;
    int e;
    double f = frexp(amax, &e); /* amax = (2f) * 2^(e-1), 2f in [1, 2) */
    int k = (2.0 * f <= 1.75 ? 8 : 7) - (e - 1);
    if (k > 126) k = 126;
    if (k < -126) k = -126;
    return k;
}

/* v[0..n) in blocks of `block`: each block becomes e4m3fn(v * 2^k) * 2^-k
 * with k = oracle_act_scale_exp(largest |v| of the block). */
void oracle_act_quantize(const double* v, int n, int block, double* out) {
    for (int b0 = 0; b0 < n; b0 += block) {
        int b1 = b0 + block < n ? b0 + block : n;
        double amax = 0.0;
        for (int i = b0; i < b1; ++i) amax = fabs(v[i]) > amax ? fabs(v[i]) : amax;
        int k = oracle_act_scale_exp(amax);
        for (int i = b0; i < b1; ++i) out[i] = ldexp(oracle_e4m3fn_round(ldexp(v[i], k)), -k);
    }
}

/* One expert on one row in the W8A8 form: xq = quantised x (blocks of 128
 * columns); h = silu(Wg xq) * (Wu xq); hq = quantised h (blocks of 64
 * features); y = Wd hq.  Every product and sum in fp64. */
static void expert_row_w8a8(const double* x, int H, int I,
                            const uint8_t* wg, const float* sg, const uint8_t* wu, const float* su,
                            const uint8_t* wd, const float* sd, double* xq, double* h, double* y) {
    oracle_act_quantize(x, H, ORACLE_XQ_BLOCK, xq);
    for (int i = 0; i < I; ++i) {
        double g = 0.0, u = 0.0;
        for (int k = 0; k < H; ++k) {
            g += weight(wg, sg, H, i, k) * xq[k];
            u += weight(wu, su, H, i, k) * xq[k];
        }
        h[i] = (g / (1.0 + exp(-g))) * u;
    }
    oracle_act_quantize(h, I, ORACLE_HQ_BLOCK, h);
    for (int n = 0; n < H; ++n) {
        double acc = 0.0;
        for (int i = 0; i < I; ++i) acc += weight(wd, sd, I, n, i) * h[i];
        y[n] = acc;
    }
}

/* oracle_ffn_sorted in the W8A8 form: y_sorted[p] = w[r] * FFN_e^{W8A8}(x[t]). */
void oracle_ffn_sorted_w8a8(const uint16_t* x, int T, int H, int K, const oracle_experts* ex,
                            const int32_t* offsets, const int32_t* sorted_route, const double* w,
                            double* y_sorted) {
    init_tables();
    (void)T;
    int E = ex->n_experts, I = ex->inter;
    for (int e = 0; e < E; ++e) {
        const uint8_t *wg, *wu, *wd; const float *sg, *su, *sd;
        expert_ptrs(ex, e, H, &wg, &sg, &wu, &su, &wd, &sd);
        int p0 = offsets[e], p1 = offsets[e + 1];
#pragma omp parallel for num_threads(g_threads) schedule(dynamic, 1)
        for (int p = p0; p < p1; ++p) {
            double* xr = (double*)malloc(sizeof(double) * (size_t)H);
            double* xq = (double*)malloc(sizeof(double) * (size_t)H);
            double* h = (double*)malloc(sizeof(double) * (size_t)I);
            int r = sorted_route[p];
            load_row(x, H, r / K, xr);
            double* y = y_sorted + (size_t)p * H;
            expert_row_w8a8(xr, H, I, wg, sg, wu, su, wd, sd, xq, h, y);
            for (int n = 0; n < H; ++n) y[n] *= w[r];
            free(xr);
            free(xq);
            free(h);
        }
    }
}

/* The shared expert in the W8A8 form: y_shared[t] = FFN_s^{W8A8}(x[t]). */
void oracle_ffn_shared_w8a8(const uint16_t* x, int T, int H, const oracle_experts* sh, double* y_shared) {
    init_tables();
    const uint8_t *wg, *wu, *wd; const float *sg, *su, *sd;
    expert_ptrs(sh, 0, H, &wg, &sg, &wu, &su, &wd, &sd);
    int I = sh->inter;
#pragma omp parallel for num_threads(g_threads) schedule(dynamic, 1)
    for (int t = 0; t < T; ++t) {
        double* xr = (double*)malloc(sizeof(double) * (size_t)H);
        double* xq = (double*)malloc(sizeof(double) * (size_t)H);
        double* h = (double*)malloc(sizeof(double) * (size_t)I);
        load_row(x, H, t, xr);
        expert_row_w8a8(xr, H, I, wg, sg, wu, su, wd, sd, xq, h, y_shared + (size_t)t * H);
        free(xr);
        free(xq);
        free(h);
    }
}
