// route.cu -- top-1 routing: argmax per token, per-expert counts and offsets,
// and the stable expert-sorted token permutation.
//
// foxhunt commit 11b96dac6a ("Top-1 Mixture-of-Experts gate per Switch
// Transformer"), kernel list and PERFORMANCE: the expert of a token is the
// argmax of its gate logits, picked by one thread scanning e = 0, 1, ... and
// moving only on a strictly greater value. Here a group of lanes shares one
// token and reduces (value, index) pairs with a combiner that yields exactly
// that scan's result: NaN entries are never chosen, equal values keep the lower
// index, and a NaN at e = 0 pins the result to 0.
//
// Three launches, all integer-exact and deterministic:
//   1. route_count   : argmax of 1024 tokens per block, per-block expert counts
//                      (warp ballots, no atomics).
//   2. route_scan    : one block: counts, offsets and every block's base
//                      position inside each expert's segment.
//   3. route_scatter : per-token rank inside its block (warp ballots in token
//                      order), perm[base + rank] = t.
#include <cstdint>

#include "common.cuh"
#include "internal.h"

namespace moe {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kTokPerWarp = kRouteTokPerBlk / kWarps;  // 128

__device__ __forceinline__ void combine(float& v, int& e, bool& ok, float ov, int oe, bool ook) {
    const bool take = ook && (!ok || ov > v || (ov == v && oe < e));
    if (take) {
        v = ov;
        e = oe;
        ok = true;
    }
}

template <int LPT>  // lanes per token: a power of two >= E
__global__ void __launch_bounds__(kThreads) route_count_kernel(const float* __restrict__ logits, int64_t T, int E,
                                                              int32_t* __restrict__ expert_idx,
                                                              int32_t* __restrict__ blk_counts) {
    __shared__ int s_idx[kRouteTokPerBlk];
    __shared__ int s_wcnt[kWarps][32];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t t0 = static_cast<int64_t>(blockIdx.x) * kRouteTokPerBlk;
    constexpr int TPW = 32 / LPT;  // tokens per warp per step
    const int sub = lane % LPT;
    for (int base = warp * TPW; base < kRouteTokPerBlk; base += kWarps * TPW) {
        const int tl = base + lane / LPT;
        const int64_t t = t0 + tl;
        const bool in = (t < T) && (sub < E);
        const float raw = in ? __ldg(logits + t * E + sub) : 0.0f;
        float v = raw;
        int e = sub;
        bool ok = in && !isnan(raw);
        const bool nan0 = __shfl_sync(0xffffffffu, in && isnan(raw), lane & ~(LPT - 1));
#pragma unroll
        for (int off = LPT / 2; off >= 1; off >>= 1) {
            const float ov = __shfl_xor_sync(0xffffffffu, v, off);
            const int oe = __shfl_xor_sync(0xffffffffu, e, off);
            const bool ook = __shfl_xor_sync(0xffffffffu, ok, off);
            combine(v, e, ok, ov, oe, ook);
        }
        const int k = nan0 ? 0 : e;
        if (sub == 0) {
            s_idx[tl] = (t < T) ? k : -1;
            if (t < T) expert_idx[t] = k;
        }
    }
    __syncthreads();
    // per-warp counts over the warp's 128 consecutive tokens; lane e keeps expert e
    int cnt = 0;
#pragma unroll
    for (int it = 0; it < kTokPerWarp / 32; ++it) {
        const int k = s_idx[warp * kTokPerWarp + it * 32 + lane];
        for (int e = 0; e < E; ++e) {
            const int c = __popc(__ballot_sync(0xffffffffu, k == e));
            if (lane == e) cnt += c;
        }
    }
    s_wcnt[warp][lane] = cnt;
    __syncthreads();
    if (threadIdx.x < E) {
        int total = 0;
        for (int w = 0; w < kWarps; ++w) total += s_wcnt[w][threadIdx.x];
        blk_counts[static_cast<int64_t>(blockIdx.x) * E + threadIdx.x] = total;
    }
}

// Exclusive scan of blk_counts[.][e] over blocks for every expert, plus counts
// and offsets. One block of 1024 threads walks the blocks in chunks of 1024.
__global__ void __launch_bounds__(1024) route_scan_kernel(const int32_t* __restrict__ blk_counts, int64_t nblk,
                                                         int E, int32_t* __restrict__ counts,
                                                         int32_t* __restrict__ offsets,
                                                         int32_t* __restrict__ blk_base) {
    __shared__ int s_warp[32];
    __shared__ int s_tot[33];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // totals per expert
    for (int e = 0; e < E; ++e) {
        int acc = 0;
        for (int64_t b = threadIdx.x; b < nblk; b += blockDim.x) acc += blk_counts[b * E + e];
#pragma unroll
        for (int off = 16; off >= 1; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
        if (lane == 0) s_warp[warp] = acc;
        __syncthreads();
        if (threadIdx.x == 0) {
            int tot = 0;
            for (int w = 0; w < (int)(blockDim.x >> 5); ++w) tot += s_warp[w];
            s_tot[e] = tot;
        }
        __syncthreads();
    }
    if (threadIdx.x == 0) {
        int run = 0;
        for (int e = 0; e < E; ++e) {
            counts[e] = s_tot[e];
            offsets[e] = run;
            s_warp[e] = run;  // reuse as the running base of expert e
            run += s_tot[e];
        }
        offsets[E] = run;
        for (int e = 0; e < E; ++e) s_tot[e] = s_warp[e];
    }
    __syncthreads();
    for (int e = 0; e < E; ++e) {
        int carry = s_tot[e];
        for (int64_t c0 = 0; c0 < nblk; c0 += blockDim.x) {
            const int64_t b = c0 + threadIdx.x;
            const int v = (b < nblk) ? blk_counts[b * E + e] : 0;
            int incl = v;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const int u = __shfl_up_sync(0xffffffffu, incl, off);
                if (lane >= off) incl += u;
            }
            if (lane == 31) s_warp[warp] = incl;
            __syncthreads();
            if (warp == 0) {
                const int nw = blockDim.x >> 5;
                int w = (lane < nw) ? s_warp[lane] : 0;
                int wi = w;
#pragma unroll
                for (int off = 1; off < 32; off <<= 1) {
                    const int u = __shfl_up_sync(0xffffffffu, wi, off);
                    if (lane >= off) wi += u;
                }
                if (lane < nw) s_warp[lane] = wi - w;  // exclusive warp prefix
                if (lane == nw - 1) s_tot[32] = wi;    // chunk total
            }
            __syncthreads();
            if (b < nblk) blk_base[b * E + e] = carry + s_warp[warp] + incl - v;
            carry += s_tot[32];
            __syncthreads();
        }
    }
}

__global__ void __launch_bounds__(kThreads) route_scatter_kernel(const int32_t* __restrict__ expert_idx, int64_t T,
                                                                int E, const int32_t* __restrict__ blk_base,
                                                                int32_t* __restrict__ perm) {
    __shared__ int s_wcnt[kWarps][32];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t t0 = static_cast<int64_t>(blockIdx.x) * kRouteTokPerBlk + warp * kTokPerWarp;
    constexpr int IT = kTokPerWarp / 32;
    int k[IT];
    int cnt = 0;
#pragma unroll
    for (int it = 0; it < IT; ++it) {
        const int64_t t = t0 + it * 32 + lane;
        k[it] = (t < T) ? expert_idx[t] : -1;
        for (int e = 0; e < E; ++e) {
            const int c = __popc(__ballot_sync(0xffffffffu, k[it] == e));
            if (lane == e) cnt += c;
        }
    }
    s_wcnt[warp][lane] = cnt;
    __syncthreads();
    // lane e: first free position of expert e for this warp
    int run = 0;
    if (lane < E) {
        run = blk_base[static_cast<int64_t>(blockIdx.x) * E + lane];
        for (int w = 0; w < warp; ++w) run += s_wcnt[w][lane];
    }
    const unsigned lt = (1u << lane) - 1u;
#pragma unroll
    for (int it = 0; it < IT; ++it) {
        const int kk = k[it];
        const unsigned same = __match_any_sync(0xffffffffu, kk);
        const int base = __shfl_sync(0xffffffffu, run, kk < 0 ? 0 : kk);
        if (kk >= 0) perm[base + __popc(same & lt)] = static_cast<int32_t>(t0 + it * 32 + lane);
        for (int e = 0; e < E; ++e) {
            const int c = __popc(__ballot_sync(0xffffffffu, kk == e));
            if (lane == e) run += c;
        }
    }
}

}  // namespace

cudaError_t launch_route(const float* logits, int64_t T, int E, int32_t* expert_idx, int32_t* counts,
                         int32_t* offsets, int32_t* perm, int32_t* blk_counts, int32_t* blk_base,
                         cudaStream_t s) {
    const int64_t nblk = (T + kRouteTokPerBlk - 1) / kRouteTokPerBlk;
    if (E <= 4)
        route_count_kernel<4><<<(unsigned)nblk, kThreads, 0, s>>>(logits, T, E, expert_idx, blk_counts);
    else if (E <= 8)
        route_count_kernel<8><<<(unsigned)nblk, kThreads, 0, s>>>(logits, T, E, expert_idx, blk_counts);
    else if (E <= 16)
        route_count_kernel<16><<<(unsigned)nblk, kThreads, 0, s>>>(logits, T, E, expert_idx, blk_counts);
    else
        route_count_kernel<32><<<(unsigned)nblk, kThreads, 0, s>>>(logits, T, E, expert_idx, blk_counts);
    route_scan_kernel<<<1, 1024, 0, s>>>(blk_counts, nblk, E, counts, offsets, blk_base);
    route_scatter_kernel<<<(unsigned)nblk, kThreads, 0, s>>>(expert_idx, T, E, blk_base, perm);
    return cudaGetLastError();
}

}  // namespace moe
