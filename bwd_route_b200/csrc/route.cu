// route.cu -- top-1 routing: argmax per token, per-expert counts and offsets,
// and the stable expert-sorted token permutation.
//
// foxhunt commit 11b96dac6a ("Top-1 Mixture-of-Experts gate per Switch
// Transformer"), kernel list and PERFORMANCE: the expert of a token is the
// argmax of its gate logits, picked by one thread scanning e = 0, 1, ... and
// moving only on a strictly greater value. Here a group of lanes shares one
// token: a shuffle butterfly finds the maximum over the non-NaN entries and a
// ballot picks the lowest expert index holding it, which is exactly that
// scan's result (equal values, -0 / +0 included, keep the lower index; NaN
// entries are never chosen; a NaN at e = 0 pins the result to 0).
//
// Three launches, all integer-exact and deterministic:
//   1. route_count   : each warp loads its 128 tokens' logits (a lane group of
//                      LPT lanes per token, 16 steps in flight), takes the
//                      group maximum with xor shuffles and the lowest index
//                      holding it with a ballot; per-block expert counts come
//                      from warp ballots (no atomics).
//   2. route_scan    : one block, one warp per expert: counts, offsets and every
//                      block's base position inside each expert's segment.
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

template <int LPT>  // lanes per token: a power of two >= E
__global__ void __launch_bounds__(kThreads) route_count_kernel(const float* __restrict__ logits, int64_t T, int E,
                                                              int32_t* __restrict__ expert_idx,
                                                              int32_t* __restrict__ blk_counts) {
    __shared__ int s_idx[kRouteTokPerBlk];
    __shared__ int s_wcnt[kWarps][32];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t t0 = static_cast<int64_t>(blockIdx.x) * kRouteTokPerBlk;
    const int ntok = static_cast<int>((T - t0 < kRouteTokPerBlk) ? (T - t0) : kRouteTokPerBlk);
    constexpr int TPW = 32 / LPT;              // tokens per warp per step
    constexpr int STEPS = kTokPerWarp / TPW;   // steps for the warp's 128 consecutive tokens
    constexpr int BATCH = STEPS < 16 ? STEPS : 16;
    const int sub = lane % LPT;
    const int wt0 = warp * kTokPerWarp;
    const int g0 = (lane / LPT) * LPT;            // first lane of this token's group
    const uint32_t gmask = (LPT == 32 ? 0xffffffffu : ((1u << LPT) - 1u)) << g0;
    for (int b0 = 0; b0 < STEPS; b0 += BATCH) {
        float v[BATCH];
#pragma unroll
        for (int j = 0; j < BATCH; ++j) {  // all loads of the batch first
            const int tl = wt0 + (b0 + j) * TPW + lane / LPT;
            v[j] = (tl < ntok && sub < E) ? __ldg(logits + (t0 + tl) * E + sub) : __int_as_float(0x7fc00000);
        }
#pragma unroll
        for (int j = 0; j < BATCH; ++j) {
            const int tl = wt0 + (b0 + j) * TPW + lane / LPT;
            // the group's maximum over its valid entries (fmaxf skips NaN; padding lanes hold NaN)
            float m = v[j];
#pragma unroll
            for (int off = LPT / 2; off >= 1; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
            // the lowest expert index holding that maximum (-0 == +0 tie); a NaN at
            // e = 0 wins outright, as in a scan that never moves off its NaN start
            const bool nan0 = (sub == 0) && isnan(v[j]) && (tl < ntok);
            const uint32_t hit = __ballot_sync(0xffffffffu, v[j] == m) & gmask;
            const uint32_t n0 = __ballot_sync(0xffffffffu, nan0) & gmask;
            const int k = (n0 || !hit) ? 0 : __ffs(hit >> g0) - 1;
            if (sub == 0) s_idx[tl] = (tl < ntok) ? k : -1;
        }
    }
    __syncthreads();
    // expert_idx written coalesced; per-warp counts over its 128 tokens, lane e keeps expert e
    int cnt = 0;
#pragma unroll
    for (int it = 0; it < kTokPerWarp / 32; ++it) {
        const int tl = wt0 + it * 32 + lane;
        const int k = s_idx[tl];
        if (tl < ntok) expert_idx[t0 + tl] = k;
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

// One block, warp e scans the per-block counts of expert e: blk_base[b][e] =
// offsets[e] + sum_{b' < b} blk_counts[b'][e]; also counts and offsets. Two
// passes over the counts (totals, then the scan with the expert's offset), each
// with batches of independent loads.
__global__ void __launch_bounds__(1024) route_scan_kernel(const int32_t* __restrict__ blk_counts, int64_t nblk,
                                                         int E, int32_t* __restrict__ counts,
                                                         int32_t* __restrict__ offsets,
                                                         int32_t* __restrict__ blk_base) {
    // Each expert gets Q = 32 / E warps; warp q of expert e owns a contiguous
    // run of routing blocks. Pass 1 sums each run, one thread turns the run sums
    // into the expert totals, the offsets and each run's starting base, and pass
    // 2 scans each run from its base. The first batch of a run stays in
    // registers between the passes, so a run of up to 256 blocks (every expert at
    // 262144 tokens for E = 8) reads the per-block counts once.
    __shared__ int s_part[32];
    __shared__ int s_base[32];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int Q = 32 / E;
    const int e = warp / Q, q = warp - e * Q;
    constexpr int kBatch = 8;  // chunks of 32 blocks loaded before they are used
    const int64_t run = (nblk + Q - 1) / Q;
    const int64_t lo = q * run;
    const int64_t hi = lo + run < nblk ? lo + run : nblk;
    auto load = [&](int64_t c0, int (&v)[kBatch]) {
#pragma unroll
        for (int j = 0; j < kBatch; ++j) {
            const int64_t b = c0 + j * 32 + lane;
            v[j] = (b < hi) ? blk_counts[b * E + e] : 0;
        }
    };
    int v0[kBatch];
    if (e < E) {
        int tot = 0;
        load(lo, v0);
#pragma unroll
        for (int j = 0; j < kBatch; ++j) tot += v0[j];
        for (int64_t c0 = lo + 32 * kBatch; c0 < hi; c0 += 32 * kBatch) {
            int v[kBatch];
            load(c0, v);
#pragma unroll
            for (int j = 0; j < kBatch; ++j) tot += v[j];
        }
#pragma unroll
        for (int off = 16; off >= 1; off >>= 1) tot += __shfl_xor_sync(0xffffffffu, tot, off);
        if (lane == 0) s_part[warp] = tot;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        int acc = 0;
        for (int ee = 0; ee < E; ++ee) {
            offsets[ee] = acc;
            const int first = acc;
            for (int qq = 0; qq < Q; ++qq) {
                s_base[ee * Q + qq] = acc;
                acc += s_part[ee * Q + qq];
            }
            counts[ee] = acc - first;
        }
        offsets[E] = acc;
    }
    __syncthreads();
    if (e < E) {
        int carry = s_base[warp];
        auto scan = [&](int64_t c0, const int (&v)[kBatch]) {
#pragma unroll
            for (int j = 0; j < kBatch; ++j) {
                int incl = v[j];
#pragma unroll
                for (int off = 1; off < 32; off <<= 1) {
                    const int u = __shfl_up_sync(0xffffffffu, incl, off);
                    if (lane >= off) incl += u;
                }
                const int64_t b = c0 + j * 32 + lane;
                if (b < hi) blk_base[b * E + e] = carry + incl - v[j];
                carry += __shfl_sync(0xffffffffu, incl, 31);
            }
        };
        scan(lo, v0);
        for (int64_t c0 = lo + 32 * kBatch; c0 < hi; c0 += 32 * kBatch) {
            int v[kBatch];
            load(c0, v);
            scan(c0, v);
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

// The routing kernels use static shared memory only; kept so that callers that
// prepare a device once have a single place to do it.
cudaError_t route_set_smem_limits() { return cudaSuccess; }

}  // namespace moe
