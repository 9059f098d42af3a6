// gemm_tf32.cu -- tcgen05 (5th-generation tensor core) TF32 kernels of the
// expert contractions, accumulating in tensor memory (TMEM).
//
// foxhunt commit 11b96dac6a ("Top-1 Mixture-of-Experts gate per Switch
// Transformer"), kernel list / PERFORMANCE: the forward applies the selected
// expert's [H, H] linear (routed[t,o] = sum_i W[e*,o,i] x[t,i] + b[e*,o]); the
// backward runs the chain rule through the selected expert only
// (d_x[t,i] = sum_o W[e*,o,i] d_out[t,o]; dW[e,o,i] = sum_{t in e} d_out[t,o]
// x[t,i]; db[e,o] = sum_{t in e} d_out[t,o]). The pages give one block per
// token and one thread per output channel; here the tokens of an expert are
// contiguous in the routing permutation, so each expert is a dense GEMM whose
// token rows are gathered on the fly.
//
// Row gathers use cp.async (16 bytes per lane, eight lanes per 128-byte row
// segment) into the swizzled shared-memory layout the MMA reads: measured on
// the B200 with one CTA per SM and 96 KiB in flight, this path streams rows at
// ~6.1 TB/s, where TMA tile::gather4 (512 bytes per operation) reaches
// ~2.0 TB/s. The dense expert-weight operand is loaded by TMA.
//
//   grouped_tf32_kernel : persistent, one CTA per SM; a tile is 128 sorted
//     tokens x all H outputs. Warps 8-11 gather the tile's rows (K-major,
//     128-byte swizzle) into a 6-deep ring; warp 13 streams the expert's weight
//     slab by TMA into a 3-deep ring (it comes from L2; K-major for the
//     forward, MN-major straight from W for d_x); one thread of warp 12 issues
//     tcgen05.mma kind::tf32 (M=128, N=H, K=8) into one of two TMEM
//     accumulators; warps 0-7 drain the other accumulator (tcgen05.ld), add
//     the bias, transpose through shared memory and store the rows to their
//     original token positions, 4 rows x 128 bytes per warp instruction. The
//     COLLAPSE instances serve the backward through the horizon mean (gradient
//     row t / N_H, result scaled by 1 / N_H).
//
//   wgrad_tf32_kernel : one CTA per range of the sorted token list (range c of
//     expert e -> partial-sum slot c + e). Tokens are the contraction index, so
//     both operands are MN-major, which for TF32 needs the 128-byte swizzle with
//     32-byte granules. Warps 4-7 gather 32 tokens of d_out and x per stage;
//     warp 8 issues M=128 x N=H MMAs with the whole dW[e] (H x H fp32) in TMEM;
//     warps 0-3 sum d_out over the staged tokens for db, then drain dW into the
//     slot. A separate kernel adds the slots in a fixed pairwise order (no
//     atomics: foxhunt commit b23f8f2efa, Discipline).
//
// The tensor core reads each fp32 operand as TF32 (its 10 leading mantissa
// bits, the low 13 bits dropped) and accumulates in fp32. Every pipeline wait
// is bounded (common.cuh).
#include <cstdint>

#include "common.cuh"
#include "internal.h"

namespace moe {
namespace {

// Weight gradient: warps 0-3 db + epilogue (TMEM lane quadrant = warp), 4-7
// row-gather producers, 8 MMA issuer + TMEM owner.
constexpr int kThreads = 288;
constexpr int kProducer0 = 128;
constexpr int kMmaWarp = 8;
// Grouped GEMM: warps 0-7 epilogue (warp w drains TMEM lane quadrant w % 4,
// column half w / 4), 8-11 row-gather producers, 12 MMA issuer + TMEM owner,
// 13 weight-slab TMA loader.
constexpr int kThreadsGrouped = 448;
constexpr int kGEpiWarps = 8;
constexpr int kGProducer0 = 256;
constexpr int kGMmaWarp = 12;
constexpr int kGBLoadWarp = 13;
constexpr int kMaxStages = 8;

struct __align__(8) Ctl {
    uint64_t full[kMaxStages];
    uint64_t empty[kMaxStages];
    uint64_t tfull[2];
    uint64_t tempty[2];
    uint32_t tmem_base;
    int abort;
    int off[33];
    int tstart[33];
};

// ------------------------------------------------------------------ grouped GEMM
// Two shared-memory rings: the gathered token rows (A, from HBM, long latency:
// deep ring) and the expert's weight slab (B, from L2: shallow ring). Each
// k-chunk is 32 fp32 = one 128-byte swizzle row of K.
// Barriers of the grouped GEMM: one full/empty pair per stage of each ring,
// and the full/empty pair of each TMEM accumulator.
struct __align__(8) GCtl {
    uint64_t afull[kMaxStages];
    uint64_t aempty[kMaxStages];
    uint64_t bfull[kMaxStages];
    uint64_t bempty[kMaxStages];
    uint64_t tfull[2];
    uint64_t tempty[2];
    uint32_t tmem_base;
    int abort;
    int off[33];
    int tstart[33];
};

template <int H>
struct GCfg {
    static constexpr int BM = 128;
    static constexpr int KCH = H / 32;
    static constexpr int A_BYTES = BM * 128;          // 16 KiB
    static constexpr int B_BYTES = H * 128;           // 16 / 32 KiB
    static constexpr int A_STAGES = (H == 256) ? 6 : 8;
    static constexpr int B_STAGES = (H == 256) ? 3 : 4;
    static constexpr int RING_BYTES = A_STAGES * A_BYTES + B_STAGES * B_BYTES;
    static constexpr int STG_BYTES = kGEpiWarps * 32 * 128;  // epilogue staging: 32 rows x 128 B per warp
    static constexpr int TMEM_COLS = 2 * H;                  // two accumulators
    static constexpr int SMEM_BYTES = 1024 + RING_BYTES + STG_BYTES + static_cast<int>(sizeof(GCtl));
    static_assert(A_STAGES <= kMaxStages && B_STAGES <= kMaxStages, "stages");
    static_assert(SMEM_BYTES <= 227 * 1024, "shared memory");
};

__device__ __forceinline__ int find_expert(const int* tstart, int E, int tile) {
    int e = 0;
    while (e + 1 < E && tstart[e + 1] <= tile) ++e;
    return e;
}

// B_MN = false: the weight operand is K-major in memory (B_e[n][k] = W[e][n][k],
// the forward). B_MN = true: it is read MN-major straight from W (B_e[n][k] =
// W[e][k][n], the input gradient), in 32-row x 128-byte boxes with the 32-byte
// granule swizzle that tcgen05 requires for an MN-major TF32 operand.
// COLLAPSE: token t's source row is t / src_div and each result is multiplied
// by out_scale (the backward through the horizon mean); without it both are 1
// and the code is the plain contraction's.
template <int H, bool B_MN, bool COLLAPSE>
__global__ void __launch_bounds__(kThreadsGrouped, 1)
grouped_tf32_kernel(const float* __restrict__ src, const __grid_constant__ CUtensorMap tm_b,
                    const float* __restrict__ bias, const int32_t* __restrict__ offsets,
                    const int32_t* __restrict__ perm, int E, int accumulate, int src_div, float out_scale,
                    float* __restrict__ out, uint32_t* __restrict__ dev_flags) {
    using C = GCfg<H>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* aring = smem;
    uint8_t* bring = smem + C::A_STAGES * C::A_BYTES;
    float* stg = reinterpret_cast<float*>(smem + C::RING_BYTES);
    GCtl* ctl = reinterpret_cast<GCtl*>(smem + C::RING_BYTES + C::STG_BYTES);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::A_STAGES; ++s) {
            mbar_init(&ctl->afull[s], 128);  // 128 gather threads
            mbar_init(&ctl->aempty[s], 1);   // tcgen05.commit
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
    if (warp == kGBLoadWarp && lane == 0) tma_prefetch_desc(&tm_b);
    if (warp == kGMmaWarp) {
        tmem_alloc(&ctl->tmem_base, C::TMEM_COLS);
        tmem_relinquish();
    }
    griddep_wait();  // the prologue above overlaps the previous kernel; global memory from here on
    if (threadIdx.x <= E) ctl->off[threadIdx.x] = offsets[threadIdx.x];
    __syncthreads();
    if (threadIdx.x == 0) {
        int ts = 0;
        for (int e = 0; e < E; ++e) {
            ctl->tstart[e] = ts;
            ts += (ctl->off[e + 1] - ctl->off[e] + C::BM - 1) / C::BM;
        }
        ctl->tstart[E] = ts;
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = ctl->tmem_base;
    const int ntiles = ctl->tstart[E];
    volatile int* abort = &ctl->abort;

    if (warp >= kGProducer0 / 32 && warp < kGProducer0 / 32 + 4) {
        // ---------------- producers: cp.async row gather
        const int ptid = threadIdx.x - kGProducer0;  // 0..127
        const int prow = ptid >> 3, pg = ptid & 7;  // row within a 16-row block, 16-byte granule
        int tok[8], nxt[8];
        auto load_tokens = [&](int tile, int (&t)[8]) {
            const int e = find_expert(ctl->tstart, E, tile);
            const int row0 = ctl->off[e] + (tile - ctl->tstart[e]) * C::BM;
            const int nrows = min(C::BM, ctl->off[e + 1] - row0);
#pragma unroll
            for (int it = 0; it < 8; ++it) {
                const int r = it * 16 + prow;
                const int tk = (r < nrows) ? perm[row0 + r] : -1;
                t[it] = (COLLAPSE && tk >= 0) ? tk / src_div : tk;  // the token's source row
            }
        };
        if (static_cast<int>(blockIdx.x) < ntiles) load_tokens(blockIdx.x, tok);
        int sa = 0;
        uint32_t pa = 0;
        bool ok = true;
        for (int tile = blockIdx.x; tile < ntiles && ok; tile += gridDim.x) {
            if (tile + static_cast<int>(gridDim.x) < ntiles) load_tokens(tile + gridDim.x, nxt);
            for (int kc = 0; kc < C::KCH; ++kc) {
                if (!(ok = mbar_wait(&ctl->aempty[sa], pa ^ 1, abort, dev_flags))) break;
                const uint32_t a_u32 = smem_u32(aring + sa * C::A_BYTES);
#pragma unroll
                for (int it = 0; it < 8; ++it) {
                    const int r = it * 16 + prow;
                    const int t = tok[it];
                    const float* gsrc = src + static_cast<int64_t>(t < 0 ? 0 : t) * H + kc * 32 + pg * 4;
                    cp_async_16_l2_256(a_u32 + r * 128 + ((pg ^ (r & 7)) << 4), gsrc, t < 0 ? 0u : 16u);
                }
                cp_async_arrive_noinc(&ctl->afull[sa]);
                if (++sa == C::A_STAGES) {
                    sa = 0;
                    pa ^= 1;
                }
            }
#pragma unroll
            for (int it = 0; it < 8; ++it) tok[it] = nxt[it];
        }
    } else if (warp == kGBLoadWarp) {
        // ---------------- weight-slab loader: TMA, at most B_STAGES chunks ahead of the MMA
        if (lane == 0) {
            int sb = 0;
            uint32_t pb = 0;
            bool ok = true;
            for (int tile = blockIdx.x; tile < ntiles && ok; tile += gridDim.x) {
                const int e = find_expert(ctl->tstart, E, tile);
                for (int kc = 0; kc < C::KCH; ++kc) {
                    if (!(ok = mbar_wait(&ctl->bempty[sb], pb ^ 1, abort, dev_flags))) break;
                    mbar_arrive_expect_tx(&ctl->bfull[sb], C::B_BYTES);
                    if (B_MN) {
                        // k-chunk = rows kc*32 .. +31 of W[e]; one box per 32 output columns
#pragma unroll
                        for (int g = 0; g < H / 32; ++g)
                            tma_load_2d(bring + sb * C::B_BYTES + g * 32 * 128, &tm_b, g * 32, e * H + kc * 32,
                                        &ctl->bfull[sb]);
                    } else {
                        tma_load_2d(bring + sb * C::B_BYTES, &tm_b, kc * 32, e * H, &ctl->bfull[sb]);
                    }
                    if (++sb == C::B_STAGES) {
                        sb = 0;
                        pb ^= 1;
                    }
                }
            }
        }
        __syncwarp();
    } else if (warp == kGMmaWarp) {
        // ---------------- MMA issuer (one thread)
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_tf32(128, H, 0, B_MN ? 1 : 0);
            int sa = 0, sb = 0;
            uint32_t pa = 0, pb = 0;
            int acc = 0;
            uint32_t acc_phase = 0;
            bool ok = true;
            for (int tile = blockIdx.x; tile < ntiles && ok; tile += gridDim.x) {
                if (!(ok = mbar_wait(&ctl->tempty[acc], acc_phase ^ 1, abort, dev_flags))) break;
                tc_fence_after();
                const uint32_t d = tmem + static_cast<uint32_t>(acc * H);
                for (int kc = 0; kc < C::KCH; ++kc) {
                    if (!(ok = mbar_wait(&ctl->afull[sa], pa, abort, dev_flags))) break;
                    if (!(ok = mbar_wait(&ctl->bfull[sb], pb, abort, dev_flags))) break;
                    fence_proxy_async_smem();
                    tc_fence_after();
                    const uint32_t a_addr = smem_u32(aring + sa * C::A_BYTES);
                    const uint32_t b_addr = smem_u32(bring + sb * C::B_BYTES);
#pragma unroll
                    for (int ks = 0; ks < 4; ++ks) {
                        const uint64_t bdesc = B_MN ? sw128_32b_mn_desc(b_addr + ks * 1024, 32 * 128, 512)
                                                    : sw128_desc(b_addr + ks * 32, 16, 1024);
                        mma_tf32(d, sw128_desc(a_addr + ks * 32, 16, 1024), bdesc, idesc, (kc | ks) != 0 ? 1u : 0u);
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
                if (!ok) break;
                mma_commit(&ctl->tfull[acc]);
                acc ^= 1;
                if (acc == 0) acc_phase ^= 1;
            }
        }
        __syncwarp();
    } else if (warp < kGEpiWarps) {
        // ---------------- epilogue: TMEM -> registers -> smem transpose -> rows.
        // Warp w owns TMEM lanes 32 (w % 4) .. +31 (tile rows) and the column half w / 4.
        constexpr int HALF = H / 2;
        const int q = warp & 3;
        const int c0 = (warp >> 2) * HALF;
        const uint32_t my_u32 = smem_u32(stg + warp * 32 * 32);  // this warp's 32 x 32 transpose buffer
        const int j = lane & 7;
        const int myrow = 32 * q + lane;
        // This lane's token of a tile: loaded one tile ahead, so that the DRAM
        // latency of perm[] is never exposed between two tiles.
        auto tile_token = [&](int tile) -> int {
            const int e = find_expert(ctl->tstart, E, tile);
            const int row0 = ctl->off[e] + (tile - ctl->tstart[e]) * C::BM;
            return (myrow < ctl->off[e + 1] - row0) ? perm[row0 + myrow] : -1;
        };
        int tok_next = static_cast<int>(blockIdx.x) < ntiles ? tile_token(blockIdx.x) : -1;
        // the bias this lane adds in each 32-column chunk; reloaded only when the expert changes
        float4 bv[HALF / 32];
        int bias_e = -1;
        int acc = 0;
        uint32_t acc_phase = 0;
        for (int tile = blockIdx.x; tile < ntiles; tile += gridDim.x) {
            const int e = find_expert(ctl->tstart, E, tile);
            const int tok_mine = tok_next;
            if (tile + static_cast<int>(gridDim.x) < ntiles) tok_next = tile_token(tile + gridDim.x);
            if (e != bias_e) {
#pragma unroll
                for (int c = 0; c < HALF / 32; ++c)
                    bv[c] = bias ? __ldg(reinterpret_cast<const float4*>(bias + static_cast<int64_t>(e) * H + c0 + c * 32) + j)
                                 : make_float4(0.f, 0.f, 0.f, 0.f);
                bias_e = e;
            }
            if (!mbar_wait(&ctl->tfull[acc], acc_phase, abort, dev_flags)) break;
            __syncwarp();
            tc_fence_after();
            // 32-column chunks, double-buffered: the TMEM load of chunk c + 1 is in
            // flight while chunk c is transposed and stored
            constexpr int NCH = HALF / 32;
            const uint32_t tbase = tmem + (static_cast<uint32_t>(32 * q) << 16) + static_cast<uint32_t>(acc * H + c0);
            uint32_t buf[2][32];
            tmem_ld_32x32b_x32_async(tbase, buf[0]);
            tmem_ld_wait_tied(buf[0]);
#pragma unroll
            for (int c = 0; c < NCH; ++c) {
                if (c + 1 < NCH) tmem_ld_32x32b_x32_async(tbase + static_cast<uint32_t>((c + 1) * 32), buf[(c + 1) & 1]);
                float v[32];
#pragma unroll
                for (int i = 0; i < 32; ++i) v[i] = COLLAPSE ? __uint_as_float(buf[c & 1][i]) * out_scale
                                                             : __uint_as_float(buf[c & 1][i]);
                {
#pragma unroll
                    for (int jj = 0; jj < 8; ++jj)
                        st_shared_v4(my_u32 + 4 * (lane * 32 + ((jj ^ (lane & 7)) * 4)), v[4 * jj], v[4 * jj + 1],
                                     v[4 * jj + 2], v[4 * jj + 3]);
                    __syncwarp();
                    if (accumulate) {
#pragma unroll
                        for (int it = 0; it < 8; ++it) {
                            const int R = it * 4 + (lane >> 3);
                            const float4 val = ld_shared_v4(my_u32 + 4 * (R * 32 + ((j ^ (R & 7)) * 4)));
                            const int tok = __shfl_sync(0xffffffffu, tok_mine, R);
                            if (tok >= 0) {
                                float4* dst = reinterpret_cast<float4*>(out + static_cast<int64_t>(tok) * H + c0 +
                                                                        c * 32 + j * 4);
                                float4 o = *dst;
                                o.x += val.x + bv[c].x;
                                o.y += val.y + bv[c].y;
                                o.z += val.z + bv[c].z;
                                o.w += val.w + bv[c].w;
                                *dst = o;
                            }
                        }
                    } else {
                        // padding rows (tok < 0) only occur in an expert's last tile; the
                        // stores are predicated rather than branched around
#pragma unroll
                        for (int it = 0; it < 8; ++it) {
                            const int R = it * 4 + (lane >> 3);
                            float4 val = ld_shared_v4(my_u32 + 4 * (R * 32 + ((j ^ (R & 7)) * 4)));
                            const int tok = __shfl_sync(0xffffffffu, tok_mine, R);
                            val.x += bv[c].x;
                            val.y += bv[c].y;
                            val.z += bv[c].z;
                            val.w += bv[c].w;
                            st_global_cs_v4_pred(out + static_cast<int64_t>(tok < 0 ? 0 : tok) * H + c0 + c * 32 + j * 4,
                                                 val, tok >= 0);
                        }
                    }
                    __syncwarp();
                }
                if (c + 1 < NCH) tmem_ld_wait_tied(buf[(c + 1) & 1]);
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
    if (warp == kGMmaWarp) {
        tc_fence_after();
        tmem_dealloc(tmem, C::TMEM_COLS);
    }
}

// ------------------------------------------------------------------ weight gradient
template <int H>
struct WCfg {
    static constexpr int KT = 32;                    // tokens per stage (4 MMAs of K = 8)
    static constexpr int G = H / 32;                 // 128-byte column groups
    static constexpr int LOG_G = (G == 8) ? 3 : 2;
    static constexpr int GROUP_BYTES = KT * 128;     // one group: KT rows x 128 B (4 KiB)
    static constexpr int OP_BYTES = G * GROUP_BYTES; // one operand per stage
    static constexpr int STAGE_BYTES = 2 * OP_BYTES; // d_out then x
    static constexpr int STAGES = (H == 256) ? 3 : 6;
    static constexpr int MH = H / 128;               // 128-row halves of dW
    static constexpr int TMEM_COLS = MH * H;
    static constexpr int STG_BYTES = 4 * 32 * 128;
    static constexpr int PER_THREAD = KT * G * 8 / 128;  // 16-byte granules per operand per producer thread
    static constexpr int SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + STG_BYTES + static_cast<int>(sizeof(Ctl));
    static_assert(G == 4 || G == 8, "H");
    static_assert(STAGES <= kMaxStages, "stages");
    static_assert(SMEM_BYTES <= 227 * 1024, "shared memory");
};

template <int H>
__global__ void __launch_bounds__(kThreads, 1)
wgrad_tf32_kernel(const float* __restrict__ g_src, const float* __restrict__ x_src,
                  const int32_t* __restrict__ offsets, const int32_t* __restrict__ perm, int T, int E, int P,
                  int g_div, float* __restrict__ part, float* __restrict__ part_db, uint32_t* __restrict__ dev_flags) {
    using C = WCfg<H>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* stages = smem;
    float* stg = reinterpret_cast<float*>(smem + C::STAGES * C::STAGE_BYTES);
    Ctl* ctl = reinterpret_cast<Ctl*>(smem + C::STAGES * C::STAGE_BYTES + C::STG_BYTES);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int c = blockIdx.x;

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::STAGES; ++s) {
            mbar_init(&ctl->full[s], 128);     // 128 gather threads
            mbar_init(&ctl->empty[s], 1 + 4);  // tcgen05.commit + the four db warps
        }
        mbar_init(&ctl->tfull[0], 1);
        mbar_init(&ctl->tempty[0], 4);
        ctl->abort = 0;
        fence_mbar_init();
    }
    if (warp == kMmaWarp) {
        tmem_alloc(&ctl->tmem_base, C::TMEM_COLS);
        tmem_relinquish();
    }
    griddep_wait();  // the prologue above overlaps the previous kernel; global memory from here on
    if (threadIdx.x <= E) ctl->off[threadIdx.x] = offsets[threadIdx.x];
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = ctl->tmem_base;
    volatile int* abort = &ctl->abort;
    const int lo = static_cast<int>(split_lo(c, T, P)), hi = static_cast<int>(split_lo(c + 1, T, P));

    if (warp >= 4 && warp < 8) {
        // ---------------- producers: 32 tokens of d_out and x per stage, MN-major,
        // 128-byte swizzle with 32-byte granules (granule index ^ row % 4)
        const int ptid = threadIdx.x - kProducer0;  // 0..127
        const int q16 = ptid & 7;                   // 16-byte granule within a 128-byte group row
        const int g = (ptid >> 3) & (C::G - 1);     // column group
        const int rsub = ptid >> (3 + C::LOG_G);    // row offset inside one pass
        constexpr int ROWS_PER_PASS = 128 / (8 * C::G);
        int stage = 0;
        uint32_t phase = 0;
        bool ok = true;
        // perm[] of the next stage is loaded one stage ahead (the range's sorted
        // positions are contiguous, so the next stage starts at p0 + KT or, past
        // an expert boundary, at that boundary; entries past hi are not loaded)
        int next_lane = (lo + lane < hi) ? perm[lo + lane] : -1;
        int next_p0 = lo;
        for (int e = 0; e < E && ok; ++e) {
            const int s = max(lo, ctl->off[e]), t = min(hi, ctl->off[e + 1]);
            for (int p0 = s; p0 < t; p0 += C::KT) {
                int tok_lane = (p0 + lane >= t) ? -1 : (p0 == next_p0) ? next_lane : perm[p0 + lane];
                // the lane's gradient row, one division per lane and stage (none for g_div = 1)
                const int gtok_lane = (g_div == 1 || tok_lane < 0) ? tok_lane : tok_lane / g_div;
                next_p0 = (p0 + C::KT < t) ? p0 + C::KT : t;
                next_lane = (next_p0 + lane < hi) ? perm[next_p0 + lane] : -1;
                if (!(ok = mbar_wait(&ctl->empty[stage], phase ^ 1, abort, dev_flags))) break;
                const uint32_t base = smem_u32(stages + stage * C::STAGE_BYTES);
#pragma unroll
                for (int it = 0; it < C::PER_THREAD; ++it) {
                    const int r = it * ROWS_PER_PASS + rsub;
                    const int tk = __shfl_sync(0xffffffffu, tok_lane, r);
                    const int gtk = __shfl_sync(0xffffffffu, gtok_lane, r);
                    const uint32_t off = g * C::GROUP_BYTES + r * 128 + ((((q16 >> 1) ^ (r & 3)) << 5) | ((q16 & 1) << 4));
                    const int64_t col = g * 32 + q16 * 4;
                    const int64_t row = static_cast<int64_t>(tk < 0 ? 0 : tk) * H + col;
                    const int64_t grow = static_cast<int64_t>(tk < 0 ? 0 : gtk) * H + col;  // gradient source row
                    const uint32_t nb = tk < 0 ? 0u : 16u;
                    cp_async_16(base + off, g_src + grow, nb);
                    cp_async_16(base + C::OP_BYTES + off, x_src + row, nb);
                }
                cp_async_arrive_noinc(&ctl->full[stage]);
                if (++stage == C::STAGES) {
                    stage = 0;
                    phase ^= 1;
                }
            }
        }
    } else if (warp == kMmaWarp) {
        // ---------------- MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_tf32(128, H, 1, 1);  // both operands MN-major
            int stage = 0;
            uint32_t phase = 0;
            uint32_t acc_phase = 0;
            bool ok = true;
            for (int e = 0; e < E && ok; ++e) {
                const int s = max(lo, ctl->off[e]), t = min(hi, ctl->off[e + 1]);
                if (s >= t) continue;
                if (!(ok = mbar_wait(&ctl->tempty[0], acc_phase ^ 1, abort, dev_flags))) break;
                tc_fence_after();
                bool first = true;
                for (int p0 = s; p0 < t; p0 += C::KT) {
                    if (!(ok = mbar_wait(&ctl->full[stage], phase, abort, dev_flags))) break;
                    fence_proxy_async_smem();
                    tc_fence_after();
                    const uint32_t g_addr = smem_u32(stages + stage * C::STAGE_BYTES);
                    const uint32_t x_addr = g_addr + C::OP_BYTES;
#pragma unroll
                    for (int ks = 0; ks < 4; ++ks) {
#pragma unroll
                        for (int mh = 0; mh < C::MH; ++mh) {
                            const uint64_t adesc =
                                sw128_32b_mn_desc(g_addr + mh * 4 * C::GROUP_BYTES + ks * 1024, C::GROUP_BYTES, 512);
                            const uint64_t bdesc = sw128_32b_mn_desc(x_addr + ks * 1024, C::GROUP_BYTES, 512);
                            mma_tf32(tmem + static_cast<uint32_t>(mh * H), adesc, bdesc, idesc,
                                     (first && ks == 0) ? 0u : 1u);
                        }
                    }
                    first = false;
                    mma_commit(&ctl->empty[stage]);
                    if (++stage == C::STAGES) {
                        stage = 0;
                        phase ^= 1;
                    }
                }
                if (!ok) break;
                mma_commit(&ctl->tfull[0]);
                acc_phase ^= 1;
            }
        }
        __syncwarp();
    } else if (warp < 4) {
        // ---------------- db over the staged d_out rows, then drain dW to the slot
        const int tid = threadIdx.x;  // 0..127: owns d_out column o = tid (and tid + 128)
        const int q = warp;
        float* my = stg + warp * 32 * 32;
        int stage = 0;
        uint32_t phase = 0;
        uint32_t acc_phase = 0;
        bool ok = true;
        for (int e = 0; e < E && ok; ++e) {
            const int s = max(lo, ctl->off[e]), t = min(hi, ctl->off[e + 1]);
            if (s >= t) continue;
            float db0 = 0.0f, db1 = 0.0f;
            for (int p0 = s; p0 < t; p0 += C::KT) {
                if (!(ok = mbar_wait(&ctl->full[stage], phase, abort, dev_flags))) break;
                const uint8_t* gt = stages + stage * C::STAGE_BYTES;
#pragma unroll
                for (int h = 0; h < C::MH; ++h) {
                    const int o = tid + 128 * h;
                    const int g = o >> 5, jo = o & 31;
                    // 32-byte granule (jo / 8) of row rr sits at granule (jo / 8) ^ (rr % 4)
                    const uint8_t* colbase = gt + g * C::GROUP_BYTES + (jo & 7) * 4;
                    float acc = 0.0f;
#pragma unroll 8
                    for (int rr = 0; rr < C::KT; ++rr)
                        acc += *reinterpret_cast<const float*>(colbase + rr * 128 + (((jo >> 3) ^ (rr & 3)) << 5));
                    if (h == 0) db0 += acc; else db1 += acc;
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&ctl->empty[stage]);
                if (++stage == C::STAGES) {
                    stage = 0;
                    phase ^= 1;
                }
            }
            if (!ok) break;
            if (!(ok = mbar_wait(&ctl->tfull[0], acc_phase, abort, dev_flags))) break;
            __syncwarp();
            tc_fence_after();
            const int64_t slot = static_cast<int64_t>(c) + e;
            const int j = lane & 7;
#pragma unroll 1
            for (int mh = 0; mh < C::MH; ++mh) {
#pragma unroll 1
                for (int cc = 0; cc < H / 32; ++cc) {
                    float v[32];
                    tmem_ld_32x32b_x32(tmem + (static_cast<uint32_t>(32 * q) << 16) + static_cast<uint32_t>(mh * H + cc * 32), v);
#pragma unroll
                    for (int jj = 0; jj < 8; ++jj)
                        *reinterpret_cast<float4*>(my + lane * 32 + ((jj ^ (lane & 7)) * 4)) =
                            make_float4(v[4 * jj], v[4 * jj + 1], v[4 * jj + 2], v[4 * jj + 3]);
                    __syncwarp();
#pragma unroll
                    for (int it = 0; it < 8; ++it) {
                        const int R = it * 4 + (lane >> 3);
                        const float4 val = *reinterpret_cast<const float4*>(my + R * 32 + ((j ^ (R & 7)) * 4));
                        const int o = mh * 128 + 32 * q + R;
                        *reinterpret_cast<float4*>(part + (slot * H + o) * H + cc * 32 + j * 4) = val;
                    }
                    __syncwarp();
                }
            }
            part_db[slot * H + tid] = db0;
            if (C::MH == 2) part_db[slot * H + tid + 128] = db1;
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&ctl->tempty[0]);
            acc_phase ^= 1;
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == kMmaWarp) {
        tc_fence_after();
        tmem_dealloc(tmem, C::TMEM_COLS);
    }
}

template <typename K>
cudaError_t set_smem(K kernel, int bytes) {
    return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
}

}  // namespace

template <int H, bool B_MN>
cudaError_t launch_grouped_tf32_t(const float* src, const CUtensorMap& tm_b, const float* bias,
                                  const int32_t* offsets, const int32_t* perm, int E, int accumulate, int src_div,
                                  float out_scale, float* out, uint32_t* dev_flags, int grid, cudaStream_t s) {
    if (src_div != 1 || out_scale != 1.0f)
        launch_pdl(grouped_tf32_kernel<H, B_MN, true>, dim3(grid), dim3(kThreadsGrouped), GCfg<H>::SMEM_BYTES, s,
                   src, tm_b, bias, offsets, perm, E, accumulate, src_div, out_scale, out, dev_flags);
    else
        launch_pdl(grouped_tf32_kernel<H, B_MN, false>, dim3(grid), dim3(kThreadsGrouped), GCfg<H>::SMEM_BYTES, s,
                   src, tm_b, bias, offsets, perm, E, accumulate, 1, 1.0f, out, dev_flags);
    return cudaGetLastError();
}

cudaError_t launch_grouped_tf32(const float* src, const float* W, const float* bias, const int32_t* offsets,
                                const int32_t* perm, int64_t T, int E, int H, int w_transposed, int accumulate,
                                int src_div, float out_scale, float* out, uint32_t* dev_flags, int num_sms,
                                cudaStream_t s) {
    CUtensorMap tm_b;
    const bool ok = w_transposed ? make_map_2d(&tm_b, W, static_cast<uint64_t>(E) * H, H, 32, 32, kMapSw128Atom32)
                                 : make_map_2d(&tm_b, W, static_cast<uint64_t>(E) * H, H, 32, H);
    if (!ok) return cudaErrorInvalidValue;
    const int64_t tiles = (T + 127) / 128 + E;
    const int grid = static_cast<int>(tiles < num_sms ? tiles : num_sms);
    if (H == 256)
        return w_transposed ? launch_grouped_tf32_t<256, true>(src, tm_b, bias, offsets, perm, E, accumulate,
                                                               src_div, out_scale, out, dev_flags, grid, s)
                            : launch_grouped_tf32_t<256, false>(src, tm_b, bias, offsets, perm, E, accumulate,
                                                                src_div, out_scale, out, dev_flags, grid, s);
    return w_transposed ? launch_grouped_tf32_t<128, true>(src, tm_b, bias, offsets, perm, E, accumulate,
                                                           src_div, out_scale, out, dev_flags, grid, s)
                        : launch_grouped_tf32_t<128, false>(src, tm_b, bias, offsets, perm, E, accumulate,
                                                            src_div, out_scale, out, dev_flags, grid, s);
}

cudaError_t launch_wgrad_tf32(const float* x, const float* d_out, const int32_t* offsets, const int32_t* perm,
                              int64_t T, int E, int H, int g_div, float* part, float* part_db, uint32_t* dev_flags,
                              cudaStream_t s) {
    const int P = wgrad_splits(T);
    if (H == 256) {
        launch_pdl(wgrad_tf32_kernel<256>, dim3(P), dim3(kThreads), WCfg<256>::SMEM_BYTES, s,
                   d_out, x, offsets, perm, static_cast<int>(T), E, P, g_div, part, part_db, dev_flags);
    } else {
        launch_pdl(wgrad_tf32_kernel<128>, dim3(P), dim3(kThreads), WCfg<128>::SMEM_BYTES, s,
                   d_out, x, offsets, perm, static_cast<int>(T), E, P, g_div, part, part_db, dev_flags);
    }
    return cudaGetLastError();
}

// The dynamic shared-memory limits of every tcgen05 kernel, set once per device
// (before the first launch there) instead of at every launch.
cudaError_t tf32_set_smem_limits() {
    cudaError_t e = set_smem(grouped_tf32_kernel<256, false, false>, GCfg<256>::SMEM_BYTES);
    if (e == cudaSuccess) e = set_smem(grouped_tf32_kernel<256, true, false>, GCfg<256>::SMEM_BYTES);
    if (e == cudaSuccess) e = set_smem(grouped_tf32_kernel<256, false, true>, GCfg<256>::SMEM_BYTES);
    if (e == cudaSuccess) e = set_smem(grouped_tf32_kernel<256, true, true>, GCfg<256>::SMEM_BYTES);
    if (e == cudaSuccess) e = set_smem(grouped_tf32_kernel<128, false, false>, GCfg<128>::SMEM_BYTES);
    if (e == cudaSuccess) e = set_smem(grouped_tf32_kernel<128, true, false>, GCfg<128>::SMEM_BYTES);
    if (e == cudaSuccess) e = set_smem(grouped_tf32_kernel<128, false, true>, GCfg<128>::SMEM_BYTES);
    if (e == cudaSuccess) e = set_smem(grouped_tf32_kernel<128, true, true>, GCfg<128>::SMEM_BYTES);
    if (e == cudaSuccess) e = set_smem(wgrad_tf32_kernel<256>, WCfg<256>::SMEM_BYTES);
    if (e == cudaSuccess) e = set_smem(wgrad_tf32_kernel<128>, WCfg<128>::SMEM_BYTES);
    return e;
}

}  // namespace moe
