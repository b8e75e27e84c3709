// ffn_prefill.cu -- expert FFN for the compute-bound regime (moe_expert_ffn,
// MOE_MODE_PREFILL): grouped GEMMs on the 5th-generation tensor cores.
//
// Computes what the decode path computes -- gate/up GEMM -> SwiGLU -> down
// GEMM -> affinity scale over the expert-sorted rows -- in the shape of the
// sorted grouped-GEMM prefill of the Nemotron-H layer
// (spark_model/layers/nemotron_moe.rs, `prefill` step 5) and the fused
// prefill producer of the aiter gfx950 PR (gate/up, SiLU, down and the
// routing-weight multiply in one pipeline), with the block-scaled E4M3FN
// weights of the FP8 MoE decode kernel page decoded to BF16 tile by tile.
//
// One persistent kernel per GEMM (gate/up, then down); each CTA owns one SM
// and walks a list of output tiles built on the device from the expert
// offsets (no host sync).  A tile is 128 weight rows x up to 256 token rows:
//  * swap-AB: the weights are the M=128 operand A, the tokens the N operand B,
//    so the FP8 decode writes tensor memory, not shared memory;
//  * loader warps 0-3: the weight tile's FP8 bytes by TMA (64-byte swizzle)
//    and the token rows by cp.async into the 128-byte-swizzled K-major layout
//    the MMA reads (token rows are gathered through sorted_route for gate/up,
//    contiguous rows of h for down);
//  * transform warps 4-7: each thread owns one TMEM lane (one weight row),
//    decodes its 64 FP8 codes per stage to bf16(e4m3 * block scale) and
//    stores them to TMEM with tcgen05.st (A operand, two bf16 per column);
//  * warp 12: one thread issues tcgen05.mma (kind::f16, A in TMEM, B in
//    shared memory, fp32 accumulator D in TMEM) and commits to mbarriers;
//  * epilogue warps 8-11: tcgen05.ld of D; gate/up rows are interleaved
//    (row 2j = gate of feature j, row 2j+1 = up of feature j), so a lane pair
//    holds gate and up of one feature and SwiGLU needs one shuffle; the down
//    epilogue multiplies by the route weight.  bf16 results go to global.
// Every mbarrier wait is bounded; an expired wait sets a CTA-wide abort flag
// and every role runs to the end without waiting, so the CTA always reaches
// the TMEM de-allocation.
#include "device_common.cuh"
#include "launch.h"

namespace moe {

namespace {

constexpr int kS = 4;                       // pipeline stages of 64 reduction columns
constexpr int kNMax = 256;                  // token rows per tile (MMA N)
constexpr int kWStage = 128 * 64;           // FP8 weight rows x 64 codes (64-byte swizzle)
constexpr int kBStage = kNMax * 128;        // token rows x 64 bf16 (128-byte swizzle)
constexpr int kWarpXform = 4, kWarpEpi = 8, kWarpMma = 12;
constexpr int kThreads = 13 * 32;
constexpr int kLoaders = 128;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kDCol = 0;    // D: columns [0, 256)
constexpr uint32_t kACol = 256;  // A stages: 32 columns each
constexpr int kLag = 2;          // cp.async stages kept in flight before a stage is published

enum Mode { kGateUp = 0, kDown = 1 };

struct Barriers {
    uint64_t w_full[kS], w_empty[kS], b_full[kS], a_full[kS], done[kS];
    uint64_t d_full, d_empty, final_bar;
    uint32_t tmem_base;
    int abort_flag;
};

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
    return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

struct Tile {
    int e;
    long p0;
    int n;
    int fb;
};

// Tile list: expert e contributes ceil(n_e / 256) token tiles x FB feature blocks,
// pre[] holds the exclusive prefix over experts.  Returns the total.
__device__ int build_tiles(const FfnArgs& a, int FB, int* pre) {
    const int E = a.identity ? 1 : a.ex.n;
    const long R = static_cast<long>(a.T) * a.K;
    const int per = (E + blockDim.x - 1) / blockDim.x;
    const int e0 = min(E, static_cast<int>(threadIdx.x) * per), e1 = min(E, e0 + per);
    int local = 0;
    for (int e = e0; e < e1; ++e) {
        long n;
        if (a.identity) {
            n = a.T;
        } else {
            const long b = a.offsets[e], f = a.offsets[e + 1];
            n = (b < 0 || f < b || f > R) ? 0 : f - b;
            if (n == 0 && (b < 0 || f < b || f > R)) report_status(a.status, MOE_STATUS_BAD_MAP);
        }
        local += static_cast<int>((n + kNMax - 1) / kNMax) * FB;
    }
    // Block exclusive scan of `local`.
    __shared__ int warp_sums[32];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
    int x = local;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, x, off);
        if (lane >= off) x += y;
    }
    if (lane == 31) warp_sums[warp] = x;
    __syncthreads();
    if (warp == 0) {
        int s = lane < nw ? warp_sums[lane] : 0;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, s, off);
            if (lane >= off) s += y;
        }
        warp_sums[lane] = s;
    }
    __syncthreads();
    int run = (warp ? warp_sums[warp - 1] : 0) + x - local;
    for (int e = e0; e < e1; ++e) {
        pre[e] = run;
        long n;
        if (a.identity) {
            n = a.T;
        } else {
            const long b = a.offsets[e], f = a.offsets[e + 1];
            n = (b < 0 || f < b || f > R) ? 0 : f - b;
        }
        run += static_cast<int>((n + kNMax - 1) / kNMax) * FB;
    }
    const int total = warp_sums[nw - 1];
    if (threadIdx.x == 0) pre[E] = total;
    __syncthreads();
    return total;
}

__device__ __forceinline__ Tile tile_of(const FfnArgs& a, const int* pre, int FB, int item) {
    const int E = a.identity ? 1 : a.ex.n;
    int lo = 0, hi = E - 1;  // last e with pre[e] <= item
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (pre[mid] <= item)
            lo = mid;
        else
            hi = mid - 1;
    }
    Tile t;
    t.e = lo;
    const int local = item - pre[lo];
    const int tt = local / FB;
    t.fb = local - tt * FB;
    const long base = a.identity ? 0 : a.offsets[lo];
    const long n_e = a.identity ? a.T : a.offsets[lo + 1] - base;
    t.p0 = base + static_cast<long>(tt) * kNMax;
    t.n = static_cast<int>(min(static_cast<long>(kNMax), n_e - static_cast<long>(tt) * kNMax));
    return t;
}

__device__ __forceinline__ bool wait_bar(uint64_t* bar, uint32_t parity, Barriers* B, int32_t* status) {
    return mbar_wait_or_abort(bar, parity, &B->abort_flag, status);
}

// bf16(e4m3 * s) for two codes.
__device__ __forceinline__ uint32_t decode_scaled(uint16_t codes, float s) {
    const uint32_t h = e4m3x2_to_f16x2(codes);
    const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&h));
    return pack_bf16x2(f.x * s, f.y * s);
}

template <int MODE>
__global__ void __launch_bounds__(kThreads, 1)
    prefill_kernel(const __grid_constant__ CUtensorMap tm_w0, const __grid_constant__ CUtensorMap tm_w1,
                   const FfnArgs a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = align1024(smem_raw);
    uint8_t* w_ring = sm;                          // kS x 8 KB
    uint8_t* b_ring = w_ring + kS * kWStage;       // kS x 32 KB
    Barriers* B = reinterpret_cast<Barriers*>(b_ring + kS * kBStage);
    int* row_tok = reinterpret_cast<int*>(B + 1);  // [kNMax] token row offsets of the loaders' tile
    int* pre = row_tok + kNMax;                    // [E + 1]

    const int H = a.H, I = a.ex.inter;
    const int Kred = MODE == kGateUp ? H : I;       // reduction length
    const int KB = Kred / 64;                       // stages per tile
    const int FB = MODE == kGateUp ? I / 64 : H / 128;
    const int rowstride = MODE == kGateUp ? H : I;  // elements between activation rows
    const uint16_t* act = MODE == kGateUp ? a.x : a.h;
    const long R = static_cast<long>(a.T) * a.K;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kS; ++s) {
            mbar_init(&B->w_full[s], 1);
            mbar_init(&B->w_empty[s], 4);
            mbar_init(&B->b_full[s], kLoaders);
            mbar_init(&B->a_full[s], 4);
            mbar_init(&B->done[s], 1);
        }
        mbar_init(&B->d_full, 1);
        mbar_init(&B->d_empty, 4);
        mbar_init(&B->final_bar, 1);
        B->abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == kWarpMma) {
        tmem_alloc(&B->tmem_base, kTmemCols);
        tc_fence_before();
    }
    const int total = build_tiles(a, FB, pre);  // contains __syncthreads
    tc_fence_after();
    const uint32_t tmem = B->tmem_base;
    if (MODE == kGateUp && threadIdx.x == 0) grid_dependency_launch();

    if (warp < 4) {
        // ------------------------------------------------ loaders
        const int lt = threadIdx.x;
        if (MODE == kDown) grid_dependency_wait();  // h comes from the gate/up grid
        if (lt == 0) {
            tma_prefetch_desc(&tm_w0);
            if (MODE == kGateUp) tma_prefetch_desc(&tm_w1);
        }
        long g = 0;
        long published = 0;  // stages whose b_full has been signalled
        for (int item = blockIdx.x; item < total; item += gridDim.x) {
            const Tile t = tile_of(a, pre, FB, item);
            const int N = (t.n + 15) & ~15;
            named_barrier_sync(2, kLoaders);
            for (int r = lt; r < kNMax; r += kLoaders) {
                int off = -1;
                if (r < t.n) {
                    const long p = t.p0 + r;
                    if (MODE == kDown || a.identity) {
                        off = static_cast<int>(p);
                    } else {
                        const int rt = a.sorted_route[p];
                        off = (rt >= 0 && rt < R) ? rt / a.K : -1;
                    }
                }
                row_tok[r] = off;
            }
            named_barrier_sync(2, kLoaders);
            for (int kb = 0; kb < KB; ++kb, ++g) {
                const int s = static_cast<int>(g % kS);
                if (g >= kS) wait_bar(&B->done[s], static_cast<uint32_t>((g / kS - 1) & 1), B, a.status);
                if (lt == 0) {
                    if (g >= kS) wait_bar(&B->w_empty[s], static_cast<uint32_t>((g / kS - 1) & 1), B, a.status);
                    uint8_t* dst = w_ring + s * kWStage;
                    mbar_arrive_expect_tx(&B->w_full[s], kWStage);
                    if (MODE == kGateUp) {
                        const int row = t.e * I + t.fb * 64;  // 64 gate rows, 64 up rows
                        tma_load_2d(dst, &tm_w0, &B->w_full[s], kb * 64, row);
                        tma_load_2d(dst + kWStage / 2, &tm_w1, &B->w_full[s], kb * 64, row);
                    } else {
                        tma_load_2d(dst, &tm_w0, &B->w_full[s], kb * 64, t.e * H + t.fb * 128);
                    }
                }
                const uint32_t bdst = smem_u32(b_ring + s * kBStage);
                for (int ci = lt; ci < N * 8; ci += kLoaders) {
                    const int r = ci >> 3, ch = ci & 7;
                    const int off = row_tok[r];
                    const uint16_t* src = off >= 0 ? act + static_cast<size_t>(off) * rowstride + kb * 64 + ch * 8 : act;
                    cp_async16(bdst + r * 128 + ((ch ^ (r & 7)) << 4), src, off >= 0 ? 16u : 0u);
                }
                cp_async_commit();
                if (g - published >= kLag) {
                    cp_async_wait<kLag>();
                    fence_proxy_async_smem();
                    mbar_arrive(&B->b_full[published % kS]);
                    ++published;
                }
            }
        }
        cp_async_wait<0>();
        fence_proxy_async_smem();
        while (published < g) {
            mbar_arrive(&B->b_full[published % kS]);
            ++published;
        }
    } else if (warp < kWarpEpi) {
        // ------------------------------------------------ transform: FP8 -> bf16 -> TMEM (A)
        const int q = warp - kWarpXform;
        const int row = 32 * q + lane;  // TMEM lane = weight row of the tile
        long g = 0;
        for (int item = blockIdx.x; item < total; item += gridDim.x) {
            const Tile t = tile_of(a, pre, FB, item);
            int srow, sub;
            const float* sp;
            if (MODE == kGateUp) {
                const int j = row >> 1, feat = t.fb * 64 + j;
                sub = (row & 1) ? kWStage / 2 : 0;
                srow = j;
                sp = ((row & 1) ? a.ex.s_up : a.ex.s_gate) +
                     (static_cast<size_t>(t.e) * (I / 128) + feat / 128) * (H / 128);
            } else {
                const int feat = t.fb * 128 + row;
                sub = 0;
                srow = row;
                sp = a.ex.s_down + (static_cast<size_t>(t.e) * (H / 128) + feat / 128) * (I / 128);
            }
            for (int kb = 0; kb < KB; ++kb, ++g) {
                const int s = static_cast<int>(g % kS);
                const bool ok1 = wait_bar(&B->w_full[s], static_cast<uint32_t>((g / kS) & 1), B, a.status);
                bool ok2 = true;
                if (g >= kS) ok2 = wait_bar(&B->done[s], static_cast<uint32_t>((g / kS - 1) & 1), B, a.status);
                uint32_t v[32];
                if (ok1 && ok2) {
                    const float sc = __ldg(sp + (kb >> 1));
                    const uint8_t* base = w_ring + s * kWStage + sub + srow * 64;
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        const uint4 w = *reinterpret_cast<const uint4*>(base + ((c ^ ((srow >> 1) & 3)) << 4));
                        const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                        for (int k = 0; k < 4; ++k) {
                            v[c * 8 + 2 * k] = decode_scaled(static_cast<uint16_t>(ws[k] & 0xFFFFu), sc);
                            v[c * 8 + 2 * k + 1] = decode_scaled(static_cast<uint16_t>(ws[k] >> 16), sc);
                        }
                    }
                } else {
#pragma unroll
                    for (int k = 0; k < 32; ++k) v[k] = 0;
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&B->w_empty[s]);
                tmem_st32(tmem + (static_cast<uint32_t>(32 * q) << 16) + kACol + s * 32, v);
                tmem_st_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&B->a_full[s]);
            }
        }
    } else if (warp < kWarpMma) {
        // ------------------------------------------------ epilogue
        const int q = warp - kWarpEpi;
        int tc = 0;
        for (int item = blockIdx.x; item < total; item += gridDim.x, ++tc) {
            const Tile t = tile_of(a, pre, FB, item);
            const bool ok = wait_bar(&B->d_full, static_cast<uint32_t>(tc & 1), B, a.status);
            tc_fence_after();
            for (int c0 = 0; c0 < t.n; c0 += 32) {
                uint32_t v[32];
                tmem_ld32(tmem + (static_cast<uint32_t>(32 * q) << 16) + kDCol + c0, v);
                tmem_ld_wait();
                if (!ok) continue;
                if (MODE == kGateUp) {
                    // Lane 2j: gate of feature j; lane 2j+1: up of feature j.  Even lanes
                    // write column c, odd lanes column c+1.
                    const int feat = t.fb * 64 + 16 * q + (lane >> 1);
                    const bool odd = lane & 1;
#pragma unroll
                    for (int c = 0; c < 32; c += 2) {
                        const float x0 = __uint_as_float(v[c]), x1 = __uint_as_float(v[c + 1]);
                        const float y0 = __shfl_xor_sync(0xffffffffu, x0, 1);
                        const float y1 = __shfl_xor_sync(0xffffffffu, x1, 1);
                        const float gte = odd ? y1 : x0, up = odd ? x1 : y0;
                        const int col = c0 + c + (odd ? 1 : 0);
                        if (col < t.n)
                            a.h[static_cast<size_t>(t.p0 + col) * I + feat] =
                                __bfloat16_as_ushort(__float2bfloat16_rn(silu_f32(gte) * up));
                    }
                } else {
                    const int feat = t.fb * 128 + 32 * q + lane;
                    float wl = 0.f;
                    if (c0 + lane < t.n) {
                        const long p = t.p0 + c0 + lane;
                        if (a.identity) {
                            wl = 1.f;
                        } else {
                            const int rt = a.sorted_route[p];
                            wl = (rt >= 0 && rt < R) ? a.topk_w[rt] : 0.f;
                        }
                    }
#pragma unroll
                    for (int c = 0; c < 32; ++c) {
                        const float wv = __shfl_sync(0xffffffffu, wl, c);
                        if (c0 + c < t.n)
                            a.y[static_cast<size_t>(t.p0 + c0 + c) * H + feat] =
                                __bfloat16_as_ushort(__float2bfloat16_rn(__uint_as_float(v[c]) * wv));
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&B->d_empty);
        }
    } else {
        // ------------------------------------------------ MMA issuer
        if (lane == 0) {
            long g = 0;
            int tc = 0;
            for (int item = blockIdx.x; item < total; item += gridDim.x, ++tc) {
                const Tile t = tile_of(a, pre, FB, item);
                const int N = (t.n + 15) & ~15;
                const uint32_t idesc = umma_idesc_bf16(128, N);
                if (tc >= 1) wait_bar(&B->d_empty, static_cast<uint32_t>((tc - 1) & 1), B, a.status);
                tc_fence_after();
                for (int kb = 0; kb < KB; ++kb, ++g) {
                    const int s = static_cast<int>(g % kS);
                    const uint32_t ph = static_cast<uint32_t>((g / kS) & 1);
                    const bool ok = wait_bar(&B->a_full[s], ph, B, a.status) & wait_bar(&B->b_full[s], ph, B, a.status);
                    tc_fence_after();
                    if (ok) {
                        const uint32_t bbase = smem_u32(b_ring + s * kBStage);
#pragma unroll
                        for (int k = 0; k < 4; ++k)
                            umma_ts_f16(tmem + kDCol, tmem + kACol + s * 32 + k * 8, umma_desc_sw128(bbase + k * 32),
                                        idesc, (kb > 0 || k > 0) ? 1u : 0u);
                    }
                    umma_commit(&B->done[s]);
                }
                umma_commit(&B->d_full);
            }
            // Every MMA has completed once this barrier flips.
            umma_commit(&B->final_bar);
            mbar_wait(&B->final_bar, 0, a.status);
        }
        __syncwarp();
    }
    __syncthreads();
    if (warp == kWarpMma) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

size_t prefill_smem(int E) {
    return 1024 + kS * (kWStage + kBStage) + sizeof(Barriers) + kNMax * 4 + (E + 1) * 4 + 64;
}

int num_sms() {
    static int sms = 0;
    if (!sms) {
        int dev = 0;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        if (sms <= 0) sms = 148;
    }
    return sms;
}

}  // namespace

bool ffn_prefill_supported(int H, int I) { return H % 128 == 0 && I % 64 == 0 && prefill_smem(MOE_MAX_E) <= 227 * 1024; }

cudaError_t launch_ffn_prefill(const FfnArgs& a, cudaStream_t stream) {
    const uint64_t E = static_cast<uint64_t>(a.ex.n), I = a.ex.inter, H = a.H;
    CUtensorMap tg, tu, td;
    cudaError_t err = make_tmap_u8_2d(&tg, a.ex.w_gate, E * I, H, 64, 64, 64);
    if (err == cudaSuccess) err = make_tmap_u8_2d(&tu, a.ex.w_up, E * I, H, 64, 64, 64);
    if (err == cudaSuccess) err = make_tmap_u8_2d(&td, a.ex.w_down, E * H, I, 64, 128, 64);
    if (err != cudaSuccess) return err;
    const size_t smem = prefill_smem(a.identity ? 1 : a.ex.n);
    err = cudaFuncSetAttribute(prefill_kernel<kGateUp>, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (err == cudaSuccess)
        err = cudaFuncSetAttribute(prefill_kernel<kDown>, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (err != cudaSuccess) return err;
    const int grid = num_sms();
    prefill_kernel<kGateUp><<<grid, kThreads, smem, stream>>>(tg, tu, a);
    err = cudaGetLastError();
    if (err != cudaSuccess) return err;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, prefill_kernel<kDown>, td, td, a);
}

}  // namespace moe
