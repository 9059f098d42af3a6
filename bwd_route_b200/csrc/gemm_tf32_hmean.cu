// gemm_tf32_hmean.cu -- the forward through the horizon mean on tcgen05 TF32
// tensor cores ("Single source of truth for the attention path", MHA
// additions: the gate's output [B, N_H, H] is averaged over the horizon axis
// into ctx_mean [B, H]), in a translation unit of its own.
#include <cstdint>

#include "common.cuh"
#include "hmean.h"
#include "internal.h"

namespace moe {
namespace {

constexpr int kMaxStages = 8;
constexpr int kGEpiWarps = 8;  // epilogue warps 0-7: warp w drains TMEM lane quadrant w % 4

// Hint: bring the 128-byte line at p into L2 (p always points into a live
// buffer here; no data is returned).
__device__ __forceinline__ void prefetch_l2(const void* p) {
    asm volatile("prefetch.global.L2 [%0];" ::"l"(p));
}

// ------------------------------------------------------------------ forward through the horizon mean
// ctx_mean[b] = (1/N_H) sum_h (W[e_bh] x[b,h] + bias[e_bh]) ("Single source of
// truth for the attention path", MHA additions: the gate's output is averaged
// over the horizon axis). The horizon tokens of row b that chose expert e are
// summed first, X_be = sum_{h : e_bh = e} x[b,h] (ascending h, fp32), so
//   ctx_mean[b] = (1/N_H) (sum_e W[e] X_be + sum_e n_be bias[e]),
// one dense GEMM per tile of 128 batch rows with K = E*H, accumulated in TMEM
// over the experts in a fixed order: no sum crosses a CTA and no [T, H] array
// is written. Warps 8-15 build X_be (K-major, 128-byte swizzle) in a 4-deep
// ring from the rows of x: each thread owns 4 rows and loads up to 4 tokens of
// each before adding any, so a stage costs about one memory latency; warp 17
// streams W[e] by TMA exactly as the forward does; one thread of warp 16
// issues the MMAs into one of two accumulators; warps 0-7 add the bias terms,
// scale by 1/N_H and store the rows.
constexpr int kThreadsHmean = 576;
constexpr int kHProducer0 = 256;   // warps 8-15
constexpr int kHProducers = 256;
constexpr int kHMmaWarp = 16;
constexpr int kHBLoadWarp = 17;
constexpr int kHMaxHorizon = 32;   // horizon tokens per row (one bit each in a 32-bit mask)
constexpr int kHTokAhead = 4;      // tokens of a row loaded before the first add

struct __align__(8) HCtl {
    uint64_t afull[kMaxStages];
    uint64_t aempty[kMaxStages];
    uint64_t bfull[kMaxStages];
    uint64_t bempty[kMaxStages];
    uint64_t tfull[2];
    uint64_t tempty[2];
    uint32_t tmem_base;
    int abort;
};

template <int H>
struct HCfg {
    static constexpr int BM = 128;
    static constexpr int KCH = H / 32;
    static constexpr int A_BYTES = BM * 128;                  // 16 KiB
    static constexpr int B_BYTES = H * 128;                   // 16 / 32 KiB
    static constexpr int A_STAGES = 4;
    static constexpr int B_STAGES = (H == 256) ? 3 : 4;
    static constexpr int RING_BYTES = A_STAGES * A_BYTES + B_STAGES * B_BYTES;
    static constexpr int BIAS_BYTES = 32 * H * 4;             // bias of up to 32 experts
    static constexpr int IDX_BYTES = 8 * 16 * kHMaxHorizon;   // producer warp w: experts of its 16 rows
    static constexpr int CNT_BYTES = kGEpiWarps * 32 * 32;    // epilogue lane: tokens per expert of its row
    static constexpr int TMEM_COLS = 2 * H;
    static constexpr int SMEM_BYTES =
        1024 + RING_BYTES + BIAS_BYTES + IDX_BYTES + CNT_BYTES + static_cast<int>(sizeof(HCtl));
    static_assert(A_STAGES <= kMaxStages && B_STAGES <= kMaxStages, "stages");
    static_assert(SMEM_BYTES <= 227 * 1024, "shared memory");
};

template <int H>
__global__ void __launch_bounds__(kThreadsHmean, 1)
hmean_fwd_tf32_kernel(const float* __restrict__ x, const __grid_constant__ CUtensorMap tm_b,
                      const float* __restrict__ bias, const int32_t* __restrict__ expert_idx, int B, int N_H, int E,
                      float inv_nh, float* __restrict__ out, uint32_t* __restrict__ dev_flags) {
    using C = HCfg<H>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* aring = smem;
    uint8_t* bring = smem + C::A_STAGES * C::A_BYTES;
    float* bias_s = reinterpret_cast<float*>(smem + C::RING_BYTES);
    uint8_t* idx_s = smem + C::RING_BYTES + C::BIAS_BYTES;
    uint8_t* cnt_s = idx_s + C::IDX_BYTES;
    HCtl* ctl = reinterpret_cast<HCtl*>(cnt_s + C::CNT_BYTES);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < C::A_STAGES; ++s) {
            mbar_init(&ctl->afull[s], kHProducers);  // every producer thread
            mbar_init(&ctl->aempty[s], 1);           // tcgen05.commit
        }
        for (int s = 0; s < C::B_STAGES; ++s) {
            mbar_init(&ctl->bfull[s], 1);    // arrive.expect_tx + TMA bytes
            mbar_init(&ctl->bempty[s], 1);   // tcgen05.commit
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&ctl->tfull[b], 1);
            mbar_init(&ctl->tempty[b], kGEpiWarps);
        }
        ctl->abort = 0;
        fence_mbar_init();
    }
    if (warp == kHBLoadWarp && lane == 0) tma_prefetch_desc(&tm_b);
    if (warp == kHMmaWarp) {
        tmem_alloc(&ctl->tmem_base, C::TMEM_COLS);
        tmem_relinquish();
    }
    griddep_wait();  // the prologue above overlaps the previous kernel; global memory from here on
    for (int k = threadIdx.x; k < E * H / 4; k += blockDim.x)
        reinterpret_cast<float4*>(bias_s)[k] = __ldg(reinterpret_cast<const float4*>(bias) + k);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = ctl->tmem_base;
    const int ntiles = (B + C::BM - 1) / C::BM;
    volatile int* abort = &ctl->abort;

    if (warp >= kHProducer0 / 32 && warp < (kHProducer0 + kHProducers) / 32) {
        // ---------------- producers: X_be for 128 rows x one 32-column k-chunk per stage.
        // Thread (prow, pg) owns rows r = it * 32 + prow (it = 0..3) and the 16-byte
        // granule pg of each; warp pw's rows are the prow values 4 pw .. 4 pw + 3, and
        // it keeps their experts in its own block of idx_s (warp-local row rl = 4 it + lane / 8).
        const int pw = warp - kHProducer0 / 32;
        const int ptid = threadIdx.x - kHProducer0;
        const int prow = ptid >> 3, pg = ptid & 7;
        uint8_t* sidx = idx_s + pw * 16 * kHMaxHorizon;
        int sa = 0;
        uint32_t pa = 0;
        bool ok = true;
        for (int tile = blockIdx.x; tile < ntiles && ok; tile += gridDim.x) {
            const int b0 = tile * C::BM;
            __syncwarp();
#pragma unroll 4
            for (int k = lane; k < 16 * N_H; k += 32) {
                const int rl = k / N_H, h = k - rl * N_H;
                const int b = b0 + (rl >> 2) * 32 + pw * 4 + (rl & 3);
                const int e = (b < B) ? expert_idx[static_cast<int64_t>(b) * N_H + h] : -1;
                sidx[rl * kHMaxHorizon + h] = (e >= 0 && e < E) ? static_cast<uint8_t>(e) : uint8_t{0xFF};
            }
            __syncwarp();
            for (int e = 0; e < E && ok; ++e) {
                uint32_t mask[4];  // bit h: horizon token h of the row chose expert e
#pragma unroll
                for (int it = 0; it < 4; ++it) {
                    const uint8_t* row = sidx + (it * 4 + (lane >> 3)) * kHMaxHorizon;
                    uint32_t m = 0;
                    for (int h = 0; h < N_H; ++h) m |= static_cast<uint32_t>(row[h] == e) << h;
                    mask[it] = m;
                }
                // the k-chunks of a token row are consumed one stage apart: fetch each
                // matching row whole into L2 now (the row's 8 granule threads take one
                // 128-byte chunk each), so that stages kc >= 1 read it from L2
                if (pg < C::KCH) {
#pragma unroll
                    for (int it = 0; it < 4; ++it) {
                        const int64_t t0 = static_cast<int64_t>(b0 + it * 32 + prow) * N_H;
                        for (uint32_t m = mask[it]; m; m &= m - 1)
                            prefetch_l2(x + (t0 + __ffs(m) - 1) * H + pg * 32);
                    }
                }
                for (int kc = 0; kc < C::KCH; ++kc) {
                    ok = mbar_wait(&ctl->aempty[sa], pa ^ 1, abort, dev_flags);
                    if (!(ok = __all_sync(0xffffffffu, ok))) break;
                    const float* xk = x + kc * 32 + pg * 4;
                    float4 v[4][kHTokAhead];
#pragma unroll
                    for (int it = 0; it < 4; ++it) {
                        const int64_t t0 = static_cast<int64_t>(b0 + it * 32 + prow) * N_H;
                        uint32_t m = mask[it];
#pragma unroll
                        for (int j = 0; j < kHTokAhead; ++j) {
                            v[it][j] = make_float4(0.f, 0.f, 0.f, 0.f);
                            if (m) {
                                v[it][j] = __ldcs(reinterpret_cast<const float4*>(xk + (t0 + __ffs(m) - 1) * H));
                                m &= m - 1;
                            }
                        }
                    }
                    const uint32_t a_u32 = smem_u32(aring + sa * C::A_BYTES);
#pragma unroll
                    for (int it = 0; it < 4; ++it) {
                        const int r = it * 32 + prow;
                        const int n = __popc(mask[it]);
                        float4 acc = v[it][0];
#pragma unroll
                        for (int j = 1; j < kHTokAhead; ++j) {
                            if (j < n) {
                                acc.x += v[it][j].x;
                                acc.y += v[it][j].y;
                                acc.z += v[it][j].z;
                                acc.w += v[it][j].w;
                            }
                        }
                        if (n > kHTokAhead) {  // rare: more tokens of this expert than were loaded ahead
                            uint32_t m = mask[it];
                            for (int j = 0; j < kHTokAhead; ++j) m &= m - 1;
                            const int64_t t0 = static_cast<int64_t>(b0 + r) * N_H;
                            for (; m; m &= m - 1) {
                                const float4 u = __ldcs(reinterpret_cast<const float4*>(xk + (t0 + __ffs(m) - 1) * H));
                                acc.x += u.x;
                                acc.y += u.y;
                                acc.z += u.z;
                                acc.w += u.w;
                            }
                        }
                        st_shared_v4(a_u32 + r * 128 + ((pg ^ (r & 7)) << 4), acc.x, acc.y, acc.z, acc.w);
                    }
                    fence_proxy_async_smem();  // the MMA reads these stores through the async proxy
                    mbar_arrive(&ctl->afull[sa]);
                    if (++sa == C::A_STAGES) {
                        sa = 0;
                        pa ^= 1;
                    }
                }
            }
        }
    } else if (warp == kHBLoadWarp) {
        // ---------------- W[e] k-chunks by TMA, in the producers' (e, kc) order
        if (lane == 0) {
            int sb = 0;
            uint32_t pb = 0;
            bool ok = true;
            for (int tile = blockIdx.x; tile < ntiles && ok; tile += gridDim.x) {
                for (int e = 0; e < E && ok; ++e) {
                    for (int kc = 0; kc < C::KCH; ++kc) {
                        if (!(ok = mbar_wait(&ctl->bempty[sb], pb ^ 1, abort, dev_flags))) break;
                        mbar_arrive_expect_tx(&ctl->bfull[sb], C::B_BYTES);
                        tma_load_2d(bring + sb * C::B_BYTES, &tm_b, kc * 32, e * H, &ctl->bfull[sb]);
                        if (++sb == C::B_STAGES) {
                            sb = 0;
                            pb ^= 1;
                        }
                    }
                }
            }
        }
        __syncwarp();
    } else if (warp == kHMmaWarp) {
        // ---------------- MMA issuer (one thread): D = sum over (e, kc) of X_be W[e]^T
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_tf32(128, H, 0, 0);
            int sa = 0, sb = 0;
            uint32_t pa = 0, pb = 0;
            int acc = 0;
            uint32_t acc_phase = 0;
            bool ok = true;
            for (int tile = blockIdx.x; tile < ntiles && ok; tile += gridDim.x) {
                if (!(ok = mbar_wait(&ctl->tempty[acc], acc_phase ^ 1, abort, dev_flags))) break;
                tc_fence_after();
                const uint32_t d = tmem + static_cast<uint32_t>(acc * H);
                uint32_t accumulate = 0;
                for (int e = 0; e < E && ok; ++e) {
                    for (int kc = 0; kc < C::KCH; ++kc) {
                        if (!(ok = mbar_wait(&ctl->afull[sa], pa, abort, dev_flags))) break;
                        if (!(ok = mbar_wait(&ctl->bfull[sb], pb, abort, dev_flags))) break;
                        fence_proxy_async_smem();
                        tc_fence_after();
                        const uint32_t a_addr = smem_u32(aring + sa * C::A_BYTES);
                        const uint32_t b_addr = smem_u32(bring + sb * C::B_BYTES);
#pragma unroll
                        for (int ks = 0; ks < 4; ++ks) {
                            mma_tf32(d, sw128_desc(a_addr + ks * 32, 16, 1024), sw128_desc(b_addr + ks * 32, 16, 1024),
                                     idesc, accumulate);
                            accumulate = 1u;
                        }
                        mma_commit(&ctl->aempty[sa]);
                        mma_commit(&ctl->bempty[sb]);
                        if (++sa == C::A_STAGES) {
                            sa = 0;
                            pa ^= 1;
                        }
                        if (++sb == C::B_STAGES) {
                            sb = 0;
                            pb ^= 1;
                        }
                    }
                }
                if (!ok) break;
                mma_commit(&ctl->tfull[acc]);
                acc ^= 1;
                if (acc == 0) acc_phase ^= 1;
            }
        }
        __syncwarp();
    } else if (warp < kGEpiWarps) {
        // ---------------- epilogue: row b = lane of TMEM quadrant q; column half c0.
        // (acc + sum_e n_be bias[e]) / N_H, n_be counted from the row's experts.
        constexpr int HALF = H / 2;
        const int q = warp & 3;
        const int c0 = (warp >> 2) * HALF;
        uint8_t* cnt = cnt_s + (warp * 32 + lane) * 32;
        int acc = 0;
        uint32_t acc_phase = 0;
        for (int tile = blockIdx.x; tile < ntiles; tile += gridDim.x) {
            const int b = tile * C::BM + 32 * q + lane;
#pragma unroll
            for (int k = 0; k < 8; ++k) reinterpret_cast<uint32_t*>(cnt)[k] = 0u;
            if (b < B) {
#pragma unroll 4
                for (int h = 0; h < N_H; ++h) {
                    const int e = expert_idx[static_cast<int64_t>(b) * N_H + h];
                    if (e >= 0 && e < E) cnt[e] += 1;
                }
            }
            bool ok = mbar_wait(&ctl->tfull[acc], acc_phase, abort, dev_flags);
            if (!__all_sync(0xffffffffu, ok)) break;
            tc_fence_after();
#pragma unroll 1
            for (int cc = 0; cc < HALF / 32; ++cc) {
                float v[32];
                tmem_ld_32x32b_x32(tmem + (static_cast<uint32_t>(32 * q) << 16) +
                                       static_cast<uint32_t>(acc * H + c0 + cc * 32), v);
                for (int e = 0; e < E; ++e) {
                    const float n = static_cast<float>(cnt[e]);
                    if (!__any_sync(0xffffffffu, n != 0.0f)) continue;
                    const float4* bs = reinterpret_cast<const float4*>(bias_s + e * H + c0 + cc * 32);
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        const float4 bb = bs[j];
                        v[4 * j] = fmaf(n, bb.x, v[4 * j]);
                        v[4 * j + 1] = fmaf(n, bb.y, v[4 * j + 1]);
                        v[4 * j + 2] = fmaf(n, bb.z, v[4 * j + 2]);
                        v[4 * j + 3] = fmaf(n, bb.w, v[4 * j + 3]);
                    }
                }
                if (b < B) {
                    float4* dst = reinterpret_cast<float4*>(out + static_cast<int64_t>(b) * H + c0 + cc * 32);
#pragma unroll
                    for (int j = 0; j < 8; ++j)
                        __stcs(dst + j, make_float4(v[4 * j] * inv_nh, v[4 * j + 1] * inv_nh, v[4 * j + 2] * inv_nh,
                                                    v[4 * j + 3] * inv_nh));
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&ctl->tempty[acc]);
            acc ^= 1;
            if (acc == 0) acc_phase ^= 1;
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == kHMmaWarp) {
        tc_fence_after();
        tmem_dealloc(tmem, C::TMEM_COLS);
    }
}

// ------------------------------------------------------------------ the same mean, raw rows staged by TMA (E <= 8, N_H <= 16)
// Same result definition and the same arithmetic as hmean_fwd_tf32_kernel (X_be
// summed in fp32 in ascending h; the MMA products of (e, k) added into TMEM;
// then sum_e n_be bias[e] and the 1/N_H scale), organised so that memory
// latency is never exposed: x is streamed into shared memory by TMA in raw
// stages of 8 batch rows x N_H tokens x 16 columns (the tile's rows are one
// contiguous block of x), and reducer warps build X_be for all experts of one
// 16-column k-chunk from them. Every CTA owns a contiguous range of batch rows
// (B / grid each), walked in tiles of 128 rows, so no wave of tiles is left
// half-empty. The reducers write X_be into one shared-memory staging buffer
// (64-byte swizzle, K-major); the MMA thread copies it into one of two
// tensor-memory A buffers (tcgen05.cp) and releases the staging buffer as soon
// as the copy is done, so the reducers build k-chunk kc + 1 while the MMAs of
// k-chunk kc run from tensor memory.
//   warps 0-3   epilogue: TMEM lane quadrant = warp, all H columns; they also
//               build each tile's token lists (tokens of a row sorted by expert)
//               one tile ahead, into two list buffers
//   warps 4-11  reducers: raw stage q (launch-wide index) goes to warp q % 8
//   warp 12     MMA issuer: per k-chunk, the copy of X_be into tensor memory,
//               then for each expert 2 MMAs of K = 8 on X_be (A in tensor
//               memory) and the W[e] k-chunk (shared memory)
//   warp 13     raw x stages by TMA (rows of 16 floats, 64-byte swizzle, so that
//               the eight rows a reducer warp reads at once fall in different banks)
//   warp 14     W[e] k-chunks by TMA (64-byte swizzle)
constexpr int kSThreads = 480;
constexpr int kSEpiWarps = 4;
constexpr int kSRed0 = 4;
constexpr int kSReducers = 8;
constexpr int kSMmaWarp = 12;
constexpr int kSRawWarp = 13;
constexpr int kSWWarp = 14;
constexpr int kSMaxE = 8;
constexpr int kSRowsPerStage = 8;
constexpr int kSMaxHorizon = 16;  // tokens per batch row on this path
constexpr int kSRawMaxStages = 16;
static_assert(kSRawMaxStages % 8 == 0, "raw slots come in multiples of the reducer warps");
constexpr int kSBStages = 5;

struct __align__(8) SCtl {
    uint64_t raw_full[kSRawMaxStages];
    uint64_t raw_empty[kSRawMaxStages];
    uint64_t a_full, a_empty;
    uint64_t b_full[kSBStages];
    uint64_t b_empty[kSBStages];
    uint64_t t_full[2];
    uint64_t t_empty[2];
    uint64_t ord_full[2], ord_empty[2];  // the two token-list buffers
    uint32_t tmem_base;
    int abort;
};

template <int H>
struct SCfg {
    static constexpr int BM = 128;
    static constexpr int KC = H / 16;                           // 16-column k-chunks
    static constexpr int A_BYTES = BM * 64;                     // X_be of one expert and k-chunk: 8 KiB
    static constexpr int A_REGION = kSMaxE * A_BYTES;           // 64 KiB
    static constexpr int B_BYTES = H * 64;                      // W[e] k-chunk
    static constexpr int RAW_BUDGET = 64 * 1024;
    static constexpr int ORDER_BYTES = 2 * BM * kSMaxHorizon * 2;  // two lists of uint16 (h | e << 8)
    static constexpr int BIAS_BYTES = kSMaxE * H * 4;
    // tensor memory: D_BUFS accumulators of H columns, then two A buffers of
    // kSMaxE x 16 columns (X_be of one k-chunk for every expert)
    static constexpr int D_BUFS = H == 256 ? 1 : 2;
    static constexpr int A_TCOLS = kSMaxE * 16;
    static constexpr int A_TCOL0 = D_BUFS * H;
    static constexpr int TMEM_COLS = 512;
    static_assert(A_TCOL0 + 2 * A_TCOLS <= TMEM_COLS, "tensor memory");
    static constexpr int SMEM_BYTES = 1024 + A_REGION + kSBStages * B_BYTES + RAW_BUDGET + ORDER_BYTES + BIAS_BYTES +
                                      static_cast<int>(sizeof(SCtl));
    static_assert(SMEM_BYTES <= 227 * 1024, "shared memory");
};

__device__ __forceinline__ void advance_stage(int& s, uint32_t& ph, int n) {
    if (++s == n) {
        s = 0;
        ph ^= 1;
    }
}

template <int H>
__global__ void __launch_bounds__(kSThreads, 1)
hmean_fwd_tf32_sum_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_w,
                          const float* __restrict__ bias, const int32_t* __restrict__ expert_idx, int B, int N_H,
                          int E, float inv_nh, int raw_stages, float* __restrict__ out,
                          uint32_t* __restrict__ dev_flags) {
    using C = SCfg<H>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* aregion = smem;
    uint8_t* bring = aregion + C::A_REGION;
    uint8_t* rawring = bring + kSBStages * C::B_BYTES;
    uint16_t* order = reinterpret_cast<uint16_t*>(rawring + C::RAW_BUDGET);
    float* bias_s = reinterpret_cast<float*>(rawring + C::RAW_BUDGET + C::ORDER_BYTES);
    SCtl* ctl = reinterpret_cast<SCtl*>(rawring + C::RAW_BUDGET + C::ORDER_BYTES + C::BIAS_BYTES);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int raw_bytes = kSRowsPerStage * N_H * 64;
    const int64_t b_lo = static_cast<int64_t>(B) * blockIdx.x / gridDim.x;
    const int64_t b_hi = static_cast<int64_t>(B) * (blockIdx.x + 1) / gridDim.x;
    const int ntiles = static_cast<int>((b_hi - b_lo + C::BM - 1) / C::BM);
    if (threadIdx.x == 0) {
        for (int s = 0; s < raw_stages; ++s) {
            mbar_init(&ctl->raw_full[s], 1);   // arrive.expect_tx + TMA bytes
            mbar_init(&ctl->raw_empty[s], 1);  // the reducer warp that read it
        }
        mbar_init(&ctl->a_full, kSReducers);   // one arrival per reducer warp and k-chunk
        mbar_init(&ctl->a_empty, 1);           // tcgen05.commit
        for (int s = 0; s < kSBStages; ++s) {
            mbar_init(&ctl->b_full[s], 1);
            mbar_init(&ctl->b_empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&ctl->t_full[b], 1);
            mbar_init(&ctl->t_empty[b], kSEpiWarps);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&ctl->ord_full[b], kSEpiWarps);
            mbar_init(&ctl->ord_empty[b], kSReducers);
        }
        ctl->abort = 0;
        fence_mbar_init();
    }
    if (warp == kSRawWarp && lane == 0) tma_prefetch_desc(&tm_x);
    if (warp == kSWWarp && lane == 0) tma_prefetch_desc(&tm_w);
    if (warp == kSMmaWarp) {
        tmem_alloc(&ctl->tmem_base, C::TMEM_COLS);
        tmem_relinquish();
    }
    griddep_wait();  // the prologue above overlaps the previous kernel; global memory from here on
    for (int k = threadIdx.x; k < E * H / 4; k += blockDim.x)
        reinterpret_cast<float4*>(bias_s)[k] = __ldg(reinterpret_cast<const float4*>(bias) + k);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = ctl->tmem_base;
    volatile int* abort = &ctl->abort;

    if (warp == kSRawWarp) {
        // ---------------- raw stages: rows (b0 + 8 g) * N_H .. + 8 N_H - 1 of x, columns 16 kc .. + 15
        if (lane == 0) {
            int slot = 0;
            uint32_t ph = 0;
            int issued[kSRawMaxStages];
            for (int s = 0; s < kSRawMaxStages; ++s) issued[s] = 0;
            bool ok = true;
            for (int tile = 0; tile < ntiles && ok; ++tile) {
                const int64_t b0 = b_lo + static_cast<int64_t>(tile) * C::BM;
                const int nrows = static_cast<int>(b_hi - b0 < C::BM ? b_hi - b0 : C::BM);
                const int ngroups = (nrows + kSRowsPerStage - 1) / kSRowsPerStage;
                for (int kc = 0; kc < C::KC && ok; ++kc) {
                    for (int g = 0; g < ngroups; ++g) {
                        if (!(ok = mbar_wait(&ctl->raw_empty[slot], ph ^ 1, abort, dev_flags))) break;
                        mbar_arrive_expect_tx(&ctl->raw_full[slot], raw_bytes);
                        tma_load_2d(rawring + slot * raw_bytes, &tm_x, kc * 16,
                                    static_cast<int32_t>((b0 + kSRowsPerStage * g) * N_H), &ctl->raw_full[slot]);
                        issued[slot] = static_cast<int>(ph) + 1;
                        advance_stage(slot, ph, raw_stages);
                    }
                }
            }
            for (int s = 0; s < raw_stages; ++s)
                if (issued[s]) mbar_wait_drain(&ctl->raw_full[s], static_cast<uint32_t>(issued[s] - 1), kWaitLimitCycles);
        }
        __syncwarp();
    } else if (warp == kSWWarp) {
        // ---------------- W[e] k-chunks, in the MMA's (kc, e) order
        if (lane == 0) {
            int sb = 0;
            uint32_t pb = 0;
            int issued[kSBStages];
            for (int k = 0; k < kSBStages; ++k) issued[k] = 0;
            bool ok = true;
            for (int tile = 0; tile < ntiles && ok; ++tile) {
                for (int kc = 0; kc < C::KC && ok; ++kc) {
                    for (int e = 0; e < E; ++e) {
                        if (!(ok = mbar_wait(&ctl->b_empty[sb], pb ^ 1, abort, dev_flags))) break;
                        mbar_arrive_expect_tx(&ctl->b_full[sb], C::B_BYTES);
                        tma_load_2d(bring + sb * C::B_BYTES, &tm_w, kc * 16, e * H, &ctl->b_full[sb]);
                        issued[sb] = static_cast<int>(pb) + 1;
                        advance_stage(sb, pb, kSBStages);
                    }
                }
            }
            for (int s = 0; s < kSBStages; ++s)
                if (issued[s]) mbar_wait_drain(&ctl->b_full[s], static_cast<uint32_t>(issued[s] - 1), kWaitLimitCycles);
        }
        __syncwarp();
    } else if (warp >= kSRed0 && warp < kSRed0 + kSReducers) {
        // ---------------- reducers
        const int rw = warp - kSRed0;
        const int r = lane >> 2, q4 = lane & 3;
        const uint32_t a_u32 = smem_u32(aregion);
        const uint32_t raw_u32 = smem_u32(rawring);
        int64_t qtile = 0;  // raw stages issued before this tile
        uint32_t pa = 0;
        bool ok = true;
        for (int tile = 0; tile < ntiles && ok; ++tile) {
            const int64_t b0 = b_lo + static_cast<int64_t>(tile) * C::BM;
            const int nrows = static_cast<int>(b_hi - b0 < C::BM ? b_hi - b0 : C::BM);
            const int ngroups = (nrows + kSRowsPerStage - 1) / kSRowsPerStage;
            // the tile's token lists (built by the epilogue warps a tile ahead)
            if (!(ok = mbar_wait(&ctl->ord_full[tile & 1], static_cast<uint32_t>((tile >> 1) & 1), abort, dev_flags)))
                break;
            const uint32_t obuf = smem_u32(order + (tile & 1) * (C::BM * kSMaxHorizon));
            for (int kc = 0; kc < C::KC && ok; ++kc) {
                // the previous k-chunk's X_be has been copied out of the staging buffer
                if (!(ok = mbar_wait(&ctl->a_empty, pa ^ 1, abort, dev_flags))) break;
                // raw stage q (launch-wide index) is reduced by warp q % 8, and the ring has
                // a multiple of 8 slots: every use of a slot has the same reducer warp, which
                // waits for its uses in order, so its parity waits cannot alias a stage two
                // uses back (as they could if a slot's uses went to different warps)
                const int64_t qbase = qtile + static_cast<int64_t>(kc) * ngroups;
                const int g0 = static_cast<int>((rw - qbase % kSReducers + kSReducers) % kSReducers);
#pragma unroll 1
                for (int g = g0; g < ngroups; g += kSReducers) {
                    const int64_t q = qbase + g;
                    const int slot = static_cast<int>(q % raw_stages);
                    const int m = g * kSRowsPerStage + r;
                    // the row's list: 16 entries (h | e << 8), sorted by expert, ascending h
                    // within one; entries of no expert (e = 0xFF) come last
                    const uint4 oa = ld_shared_u4(obuf + m * (kSMaxHorizon * 2));
                    const uint4 ob = ld_shared_u4(obuf + m * (kSMaxHorizon * 2) + 16);
                    const uint32_t o[16] = {oa.x & 0xFFFFu, oa.x >> 16, oa.y & 0xFFFFu, oa.y >> 16,
                                            oa.z & 0xFFFFu, oa.z >> 16, oa.w & 0xFFFFu, oa.w >> 16,
                                            ob.x & 0xFFFFu, ob.x >> 16, ob.y & 0xFFFFu, ob.y >> 16,
                                            ob.z & 0xFFFFu, ob.z >> 16, ob.w & 0xFFFFu, ob.w >> 16};
                    if (!(ok = mbar_wait(&ctl->raw_full[slot], static_cast<uint32_t>((q / raw_stages) & 1), abort,
                                         dev_flags)))
                        break;
                    // token row rr = r N_H + h of the stage holds 16 floats, stored with the
                    // 64-byte swizzle: 16-byte granule q4 sits at granule q4 ^ ((rr >> 1) & 3)
                    const uint32_t sbase = raw_u32 + slot * raw_bytes;
                    float4 vv[16];  // every listed row is requested before the first add
#pragma unroll
                    for (int u = 0; u < 16; ++u) {
                        const int rr = r * N_H + static_cast<int>(o[u] & 0xFFu);
                        vv[u] = ld_shared_v4_if(sbase + rr * 64 + ((q4 ^ ((rr >> 1) & 3)) << 4),
                                                static_cast<int>(o[u] >> 8) < E);
                    }
                    const uint32_t arow = a_u32 + m * 64 + ((q4 ^ ((m >> 1) & 3)) << 4);
                    // the list is sorted by expert, so each expert's tokens are one run: the sum
                    // restarts at a run's first token and is stored after its last (no branches;
                    // the same additions in the same order as a token-by-token walk). Entries of no
                    // expert (e >= E) come last and are never stored.
                    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
                    uint32_t present = 0;
#pragma unroll
                    for (int u = 0; u < 16; ++u) {
                        const int e = static_cast<int>(o[u] >> 8);
                        const bool first = (u == 0) || static_cast<int>(o[u - 1] >> 8) != e;
                        const bool last = e < E && (u == 15 || static_cast<int>(o[u + 1] >> 8) != e);
                        acc.x = first ? vv[u].x : acc.x + vv[u].x;
                        acc.y = first ? vv[u].y : acc.y + vv[u].y;
                        acc.z = first ? vv[u].z : acc.z + vv[u].z;
                        acc.w = first ? vv[u].w : acc.w + vv[u].w;
                        st_shared_v4_if(arow + (e < E ? e : 0) * C::A_BYTES, acc, last);
                        present |= (e < E) ? (1u << e) : 0u;
                    }
#pragma unroll
                    for (int e = 0; e < kSMaxE; ++e)  // experts with no token of this row: zeros
                        st_shared_v4_if(arow + e * C::A_BYTES, make_float4(0.f, 0.f, 0.f, 0.f),
                                        e < E && !((present >> e) & 1u));
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&ctl->raw_empty[slot]);
                }
                fence_proxy_async_smem();  // the copy to tensor memory reads these stores through the async proxy
                __syncwarp();
                if (lane == 0) mbar_arrive(&ctl->a_full);  // once per warp and k-chunk
                pa ^= 1;
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&ctl->ord_empty[tile & 1]);
            qtile += static_cast<int64_t>(C::KC) * ngroups;
        }
    } else if (warp == kSMmaWarp) {
        // ---------------- MMA issuer (one thread)
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_tf32(128, H, 0, 0);
            const uint32_t a_u32 = smem_u32(aregion);
            int sb = 0;
            uint32_t pb = 0, pa = 0;
            int acc = 0;
            uint32_t acc_phase = 0;
            int abuf = 0;  // tensor-memory A buffer of the next k-chunk
            bool ok = true;
            for (int tile = 0; tile < ntiles && ok; ++tile) {
                const uint32_t d = tmem + static_cast<uint32_t>(acc * H);
                uint32_t accumulate = 0;
                for (int kc = 0; kc < C::KC && ok; ++kc) {
                    if (!(ok = mbar_wait(&ctl->a_full, pa, abort, dev_flags))) break;
                    fence_proxy_async_smem();
                    tc_fence_after();
                    // X_be of this k-chunk -> A buffer abuf. The buffer was last read by the
                    // MMAs of k-chunk kc - 2, which completed before the staging buffer was
                    // released for k-chunk kc (the commit below covers every earlier op).
                    const uint32_t a_t = tmem + static_cast<uint32_t>(C::A_TCOL0 + abuf * C::A_TCOLS);
                    for (int e = 0; e < E; ++e)
#pragma unroll
                        for (int ks = 0; ks < 2; ++ks)
                            tmem_cp_128x256b(a_t + static_cast<uint32_t>(e * 16 + ks * 8),
                                             sw64_desc(a_u32 + e * C::A_BYTES + ks * 32, 512));
                    mma_commit(&ctl->a_empty);  // the staging buffer is free once the copies are done
                    pa ^= 1;
                    if (kc == 0) {
                        // the accumulator must have been read out by the epilogue
                        if (!(ok = mbar_wait(&ctl->t_empty[acc], acc_phase ^ 1, abort, dev_flags))) break;
                        tc_fence_after();
                    }
                    for (int e = 0; e < E; ++e) {
                        if (!(ok = mbar_wait(&ctl->b_full[sb], pb, abort, dev_flags))) break;
                        tc_fence_after();
                        const uint32_t b_addr = smem_u32(bring + sb * C::B_BYTES);
#pragma unroll
                        for (int ks = 0; ks < 2; ++ks) {
                            mma_tf32_ts(d, a_t + static_cast<uint32_t>(e * 16 + ks * 8), sw64_desc(b_addr + ks * 32, 512),
                                        idesc, accumulate);
                            accumulate = 1u;
                        }
                        mma_commit(&ctl->b_empty[sb]);
                        advance_stage(sb, pb, kSBStages);
                    }
                    abuf ^= 1;
                }
                if (!ok) break;
                mma_commit(&ctl->t_full[acc]);
                if (C::D_BUFS > 1) acc ^= 1;
                if (acc == 0) acc_phase ^= 1;
            }
        }
        __syncwarp();
    } else if (warp < kSEpiWarps) {
        // ---------------- epilogue: row m = 32 q + lane of the tile, all H columns;
        // (acc + sum_e n_be bias[e]) / N_H with n_be counted from the row's experts.
        // These warps also build the reducers' token lists, one tile ahead.
        const int q = warp;
        const int m = 32 * q + lane;  // this thread's row of every tile
        // Tile t's list for row m into order buffer t & 1: 16 entries (h | e << 8)
        // sorted by expert, ascending h within one, entries of no expert (past N_H,
        // or an index outside [0, E)) last; and the row's token count per expert.
        auto build = [&](int t, int (&cnt)[kSMaxE]) -> bool {
            const bool ok = mbar_wait(&ctl->ord_empty[t & 1], static_cast<uint32_t>(((t >> 1) & 1) ^ 1), abort,
                                      dev_flags);
            if (!__all_sync(0xffffffffu, ok)) return false;
            const int64_t b = b_lo + static_cast<int64_t>(t) * C::BM + m;
            const bool valid = b < b_hi;
            int ek[kSMaxHorizon];  // requested together, then sorted
#pragma unroll
            for (int h = 0; h < kSMaxHorizon; ++h) {
                const int e = (valid && h < N_H) ? expert_idx[b * N_H + h] : -1;
                ek[h] = (e >= 0 && e < E) ? e : kSMaxE;
            }
            int pos[kSMaxE + 1];
#pragma unroll
            for (int f = 0; f <= kSMaxE; ++f) pos[f] = 0;
#pragma unroll
            for (int h = 0; h < kSMaxHorizon; ++h)
#pragma unroll
                for (int f = 0; f <= kSMaxE; ++f) pos[f] += (f == ek[h]) ? 1 : 0;
#pragma unroll
            for (int f = 0; f < kSMaxE; ++f) cnt[f] = pos[f];
            int run = 0;
#pragma unroll
            for (int f = 0; f <= kSMaxE; ++f) {
                const int c = pos[f];
                pos[f] = run;
                run += c;
            }
            uint16_t* ord = order + (t & 1) * (C::BM * kSMaxHorizon) + m * kSMaxHorizon;
#pragma unroll
            for (int h = 0; h < kSMaxHorizon; ++h) {
                int p = 0;
#pragma unroll
                for (int f = 0; f <= kSMaxE; ++f)
                    if (f == ek[h]) p = pos[f]++;
                ord[p] = static_cast<uint16_t>(h | ((ek[h] == kSMaxE ? 0xFF : ek[h]) << 8));
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&ctl->ord_full[t & 1]);
            return true;
        };
        int acc = 0;
        uint32_t acc_phase = 0;
        int cnt[kSMaxE], cnt_next[kSMaxE];
        bool eok = build(0, cnt);
        for (int tile = 0; tile < ntiles && eok; ++tile) {
            if (tile + 1 < ntiles && !(eok = build(tile + 1, cnt_next))) break;
            const int64_t b = b_lo + static_cast<int64_t>(tile) * C::BM + m;
            const bool valid = b < b_hi;
            const bool ok = mbar_wait(&ctl->t_full[acc], acc_phase, abort, dev_flags);
            if (!__all_sync(0xffffffffu, ok)) break;
            tc_fence_after();
#pragma unroll 1
            for (int cc = 0; cc < H / 32; ++cc) {
                float v[32];
                tmem_ld_32x32b_x32(tmem + (static_cast<uint32_t>(32 * q) << 16) + static_cast<uint32_t>(acc * H + cc * 32),
                                   v);
#pragma unroll
                for (int e = 0; e < kSMaxE; ++e) {
                    if (e >= E) break;
                    const float n = static_cast<float>(cnt[e]);
                    if (!__any_sync(0xffffffffu, n != 0.0f)) continue;
                    const float4* bs = reinterpret_cast<const float4*>(bias_s + e * H + cc * 32);
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        const float4 bb = bs[j];
                        v[4 * j] = fmaf(n, bb.x, v[4 * j]);
                        v[4 * j + 1] = fmaf(n, bb.y, v[4 * j + 1]);
                        v[4 * j + 2] = fmaf(n, bb.z, v[4 * j + 2]);
                        v[4 * j + 3] = fmaf(n, bb.w, v[4 * j + 3]);
                    }
                }
                if (valid) {
                    float4* dst = reinterpret_cast<float4*>(out + b * H + cc * 32);
#pragma unroll
                    for (int j = 0; j < 8; ++j)
                        __stcs(dst + j, make_float4(v[4 * j] * inv_nh, v[4 * j + 1] * inv_nh, v[4 * j + 2] * inv_nh,
                                                    v[4 * j + 3] * inv_nh));
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&ctl->t_empty[acc]);
            if (C::D_BUFS > 1) acc ^= 1;
            if (acc == 0) acc_phase ^= 1;
#pragma unroll
            for (int f = 0; f < kSMaxE; ++f) cnt[f] = cnt_next[f];
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == kSMmaWarp) {
        tc_fence_after();
        tmem_dealloc(tmem, C::TMEM_COLS);
    }
}

template <typename K>
cudaError_t set_smem(K kernel, int bytes) {
    return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
}

}  // namespace

cudaError_t launch_hmean_fwd_tf32(const float* x, const float* W, const float* bias, const int32_t* expert_idx,
                                  int64_t B, int N_H, int E, int H, float* out, uint32_t* dev_flags, int num_sms,
                                  cudaStream_t s) {
    const int raw_bytes = kSRowsPerStage * N_H * 64;
    int raw_stages = SCfg<256>::RAW_BUDGET / raw_bytes;
    if (raw_stages > kSRawMaxStages) raw_stages = kSRawMaxStages;
    raw_stages -= raw_stages % kSReducers;  // a multiple of the reducer warps (N_H <= 16: at least 8)
    if (E <= kSMaxE && N_H <= kSMaxHorizon && raw_stages >= kSReducers) {
        // raw rows staged by TMA; every CTA owns B / grid batch rows
        CUtensorMap tm_x, tm_w;
        const uint64_t T = static_cast<uint64_t>(B) * N_H;
        if (!make_map_2d(&tm_x, x, T, H, 16, static_cast<uint32_t>(kSRowsPerStage * N_H), kMapSw64) ||
            !make_map_2d(&tm_w, W, static_cast<uint64_t>(E) * H, H, 16, H, kMapSw64))
            return cudaErrorInvalidValue;
        const int grid = static_cast<int>(B < num_sms ? B : num_sms);
        const float inv_nh = static_cast<float>(1.0 / static_cast<double>(N_H));
        if (H == 256)
            launch_pdl(hmean_fwd_tf32_sum_kernel<256>, dim3(grid), dim3(kSThreads), SCfg<256>::SMEM_BYTES, s,
                       tm_x, tm_w, bias, expert_idx, static_cast<int>(B), N_H, E, inv_nh, raw_stages, out, dev_flags);
        else
            launch_pdl(hmean_fwd_tf32_sum_kernel<128>, dim3(grid), dim3(kSThreads), SCfg<128>::SMEM_BYTES, s,
                       tm_x, tm_w, bias, expert_idx, static_cast<int>(B), N_H, E, inv_nh, raw_stages, out, dev_flags);
        return cudaGetLastError();
    }
    CUtensorMap tm_b;
    if (!make_map_2d(&tm_b, W, static_cast<uint64_t>(E) * H, H, 32, H)) return cudaErrorInvalidValue;
    const int64_t tiles = (B + 127) / 128;
    const int grid = static_cast<int>(tiles < num_sms ? tiles : num_sms);
    const float inv_nh = static_cast<float>(1.0 / static_cast<double>(N_H));
    if (H == 256)
        launch_pdl(hmean_fwd_tf32_kernel<256>, dim3(grid), dim3(kThreadsHmean), HCfg<256>::SMEM_BYTES, s,
                   x, tm_b, bias, expert_idx, static_cast<int>(B), N_H, E, inv_nh, out, dev_flags);
    else
        launch_pdl(hmean_fwd_tf32_kernel<128>, dim3(grid), dim3(kThreadsHmean), HCfg<128>::SMEM_BYTES, s,
                   x, tm_b, bias, expert_idx, static_cast<int>(B), N_H, E, inv_nh, out, dev_flags);
    return cudaGetLastError();
}

cudaError_t hmean_set_smem_limits() {
    cudaError_t e = set_smem(hmean_fwd_tf32_kernel<256>, HCfg<256>::SMEM_BYTES);
    if (e == cudaSuccess) e = set_smem(hmean_fwd_tf32_kernel<128>, HCfg<128>::SMEM_BYTES);
    if (e == cudaSuccess) e = set_smem(hmean_fwd_tf32_sum_kernel<256>, SCfg<256>::SMEM_BYTES);
    if (e == cudaSuccess) e = set_smem(hmean_fwd_tf32_sum_kernel<128>, SCfg<128>::SMEM_BYTES);
    return e;
}

}  // namespace moe
