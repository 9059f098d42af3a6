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
// Three launches (two while nblk x E <= 32768: the scan then runs inside every
// scatter block), all integer-exact and deterministic:
//   1. route_count   : E a multiple of 4: one thread per token scans its row
//                      (128-bit loads); other E: each warp loads its 128
//                      tokens' logits (a lane group of LPT lanes per token, 16
//                      steps in flight), takes the group maximum with xor
//                      shuffles and the lowest index holding it with a ballot.
//                      Per-block expert counts (exact integer sums).
//   2. route_scan    : one block, one warp per expert: counts, offsets and every
//                      block's base position inside each expert's segment.
//   3. route_scatter : per-token rank inside its block (lanes grouped by
//                      expert in token order), perm[base + rank] = t.
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
    griddep_wait();  // every global access below comes after the previous grid
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

// The same result when E is a multiple of 4 (E = 4, 8, 16, 32): one thread per
// token reads its row with 128-bit loads and runs the pages' scan as written
// (start at e = 0, move only on a strictly greater value), which fixes ties,
// -0 / +0 and NaN exactly as the definition does. Thread i of the block takes
// tokens i, i + 256, i + 512, i + 768 (rows of neighbouring lanes are
// contiguous, so every load instruction is coalesced); TOK of them have their
// rows in flight at once, few enough that 8 blocks fit on an SM. Per-block expert counts: per-warp aggregated integer
// adds into shared memory (exact, order-free).
template <int E>
__global__ void __launch_bounds__(kThreads, 8) route_count_vec_kernel(const float* __restrict__ logits, int64_t T,
                                                                  int32_t* __restrict__ expert_idx,
                                                                  int32_t* __restrict__ blk_counts) {
    griddep_wait();  // every global access below comes after the previous grid
    constexpr int Q = E / 4;                               // float4s per row
    constexpr int TOK = (Q == 1) ? 4 : (Q == 2 ? 2 : 1);   // tokens in flight per thread
    constexpr int PER = kRouteTokPerBlk / kThreads;         // 4 tokens per thread
    __shared__ int s_cnt[E];
    if (threadIdx.x < E) s_cnt[threadIdx.x] = 0;
    __syncthreads();
    const int64_t t0 = static_cast<int64_t>(blockIdx.x) * kRouteTokPerBlk;
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int p0 = 0; p0 < PER; p0 += TOK) {
        float4 v[TOK][Q];
#pragma unroll
        for (int j = 0; j < TOK; ++j) {
            const int64_t t = t0 + (p0 + j) * kThreads + threadIdx.x;
            const float4* row = reinterpret_cast<const float4*>(logits + (t < T ? t : 0) * E);
#pragma unroll
            for (int q = 0; q < Q; ++q) v[j][q] = __ldg(row + q);
        }
#pragma unroll
        for (int j = 0; j < TOK; ++j) {
            const int64_t t = t0 + (p0 + j) * kThreads + threadIdx.x;
            float best = v[j][0].x;
            int k = 0;
#pragma unroll
            for (int q = 0; q < Q; ++q) {
                const float x[4] = {v[j][q].x, v[j][q].y, v[j][q].z, v[j][q].w};
#pragma unroll
                for (int r = 0; r < 4; ++r) {
                    if (q == 0 && r == 0) continue;
                    if (x[r] > best) {
                        best = x[r];
                        k = 4 * q + r;
                    }
                }
            }
            const bool valid = t < T;
            if (valid) expert_idx[t] = k;
            const unsigned vmask = __ballot_sync(0xffffffffu, valid);
            const unsigned same = __match_any_sync(0xffffffffu, valid ? k : -1) & vmask;
            if (valid && lane == __ffs(same) - 1) atomicAdd(&s_cnt[k], __popc(same));
        }
    }
    __syncthreads();
    if (threadIdx.x < E) blk_counts[static_cast<int64_t>(blockIdx.x) * E + threadIdx.x] = s_cnt[threadIdx.x];
}

// One block, warp e scans the per-block counts of expert e: blk_base[b][e] =
// offsets[e] + sum_{b' < b} blk_counts[b'][e]; also counts and offsets. Two
// passes over the counts (totals, then the scan with the expert's offset), each
// with batches of independent loads.
__global__ void __launch_bounds__(1024) route_scan_kernel(const int32_t* __restrict__ blk_counts, int64_t nblk,
                                                         int E, int32_t* __restrict__ counts,
                                                         int32_t* __restrict__ offsets,
                                                         int32_t* __restrict__ blk_base) {
    griddep_wait();  // every global access below comes after the previous grid
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
    griddep_wait();  // every global access below comes after the previous grid
    // s_pos[w][e]: first the number of warp w's tokens on expert e, then warp w's
    // next free position in expert e's segment. Lanes holding the same expert are
    // grouped with __match_any_sync: a token's rank is the number of lower lanes
    // in its group, and the group's lowest lane advances the position.
    __shared__ int s_pos[kWarps][32];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    s_pos[warp][lane] = 0;
    __syncwarp();
    const int64_t t0 = static_cast<int64_t>(blockIdx.x) * kRouteTokPerBlk + warp * kTokPerWarp;
    constexpr int IT = kTokPerWarp / 32;
    const unsigned lt = (1u << lane) - 1u;
    int k[IT];
#pragma unroll
    for (int it = 0; it < IT; ++it) {
        const int64_t t = t0 + it * 32 + lane;
        k[it] = (t < T) ? expert_idx[t] : -1;
    }
#pragma unroll
    for (int it = 0; it < IT; ++it) {
        const unsigned same = __match_any_sync(0xffffffffu, k[it]);
        if (k[it] >= 0 && (same & lt) == 0) s_pos[warp][k[it]] += __popc(same);
        __syncwarp();
    }
    __syncthreads();
    int run = 0;
    if (lane < E) {
        run = blk_base[static_cast<int64_t>(blockIdx.x) * E + lane];
        for (int w = 0; w < warp; ++w) run += s_pos[w][lane];
    }
    __syncthreads();
    if (lane < E) s_pos[warp][lane] = run;
    __syncwarp();
#pragma unroll
    for (int it = 0; it < IT; ++it) {
        const int kk = k[it];
        const unsigned same = __match_any_sync(0xffffffffu, kk);
        const int base = kk >= 0 ? s_pos[warp][kk] : 0;
        if (kk >= 0) perm[base + __popc(same & lt)] = static_cast<int32_t>(t0 + it * 32 + lane);
        __syncwarp();
        if (kk >= 0 && (same & lt) == 0) s_pos[warp][kk] = base + __popc(same);
        __syncwarp();
    }
}

// The scan folded into the scatter: every block reads the per-block counts of
// all blocks (nblk x E integers, L2-resident) and computes, with exact integer
// sums, the expert totals and its own base in each expert's segment:
//   base[b][e] = offsets[e] + sum_{b' < b} blk_counts[b'][e],
//   offsets[e] = sum_{e' < e} counts[e'],   counts[e] = sum_{b'} blk_counts[b'][e];
// block 0 also writes counts and offsets. Thread i reads expert e = i % EP
// (EP = E rounded up to a power of two, so a thread always sees the same expert)
// of blocks i / EP, i / EP + 256 / EP, ...; lanes of one expert combine with xor
// shuffles, warps through shared-memory integer adds. Then the tokens are
// scattered exactly as route_scatter_kernel does. Used while nblk x E is small
// enough that reading it in every block is cheaper than a separate scan launch.
constexpr int64_t kPrefixMaxEntries = 32768;

__global__ void __launch_bounds__(kThreads) route_scatter_prefix_kernel(const int32_t* __restrict__ expert_idx,
                                                                       int64_t T, int E, int EP, int64_t nblk,
                                                                       const int32_t* __restrict__ blk_counts,
                                                                       int32_t* __restrict__ counts,
                                                                       int32_t* __restrict__ offsets,
                                                                       int32_t* __restrict__ perm) {
    griddep_wait();  // every global access below comes after the previous grid
    __shared__ int s_before[32], s_total[32], s_base[32];
    __shared__ int s_pos[kWarps][32];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x < 32) {
        s_before[threadIdx.x] = 0;
        s_total[threadIdx.x] = 0;
    }
    __syncthreads();
    {
        const int e = threadIdx.x % EP;
        const int step = kThreads / EP;
        int before = 0, total = 0;
        if (e < E) {
            for (int64_t b = threadIdx.x / EP; b < nblk; b += step) {
                const int v = blk_counts[b * E + e];
                total += v;
                if (b < static_cast<int64_t>(blockIdx.x)) before += v;
            }
        }
        // lanes e, e + EP, e + 2 EP, ... of this warp hold expert e (EP <= 32)
        for (int off = 16; off >= EP; off >>= 1) {
            before += __shfl_xor_sync(0xffffffffu, before, off);
            total += __shfl_xor_sync(0xffffffffu, total, off);
        }
        if (lane < EP && e < E) {
            atomicAdd(&s_before[e], before);
            atomicAdd(&s_total[e], total);
        }
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        int acc = 0;
        for (int e = 0; e < E; ++e) {
            if (blockIdx.x == 0) {
                offsets[e] = acc;
                counts[e] = s_total[e];
            }
            s_base[e] = acc + s_before[e];
            acc += s_total[e];
        }
        if (blockIdx.x == 0) offsets[E] = acc;
    }
    s_pos[warp][lane] = 0;
    __syncthreads();
    const int64_t t0 = static_cast<int64_t>(blockIdx.x) * kRouteTokPerBlk + warp * kTokPerWarp;
    constexpr int IT = kTokPerWarp / 32;
    const unsigned lt = (1u << lane) - 1u;
    int k[IT];
#pragma unroll
    for (int it = 0; it < IT; ++it) {
        const int64_t t = t0 + it * 32 + lane;
        k[it] = (t < T) ? expert_idx[t] : -1;
    }
#pragma unroll
    for (int it = 0; it < IT; ++it) {
        const unsigned same = __match_any_sync(0xffffffffu, k[it]);
        if (k[it] >= 0 && (same & lt) == 0) s_pos[warp][k[it]] += __popc(same);
        __syncwarp();
    }
    __syncthreads();
    int run = 0;
    if (lane < E) {
        run = s_base[lane];
        for (int w = 0; w < warp; ++w) run += s_pos[w][lane];
    }
    __syncthreads();
    if (lane < E) s_pos[warp][lane] = run;
    __syncwarp();
#pragma unroll
    for (int it = 0; it < IT; ++it) {
        const int kk = k[it];
        const unsigned same = __match_any_sync(0xffffffffu, kk);
        const int base = kk >= 0 ? s_pos[warp][kk] : 0;
        if (kk >= 0) perm[base + __popc(same & lt)] = static_cast<int32_t>(t0 + it * 32 + lane);
        __syncwarp();
        if (kk >= 0 && (same & lt) == 0) s_pos[warp][kk] = base + __popc(same);
        __syncwarp();
    }
}

}  // namespace

cudaError_t launch_route(const float* logits, int64_t T, int E, int32_t* expert_idx, int32_t* counts,
                         int32_t* offsets, int32_t* perm, int32_t* blk_counts, int32_t* blk_base,
                         cudaStream_t s) {
    const int64_t nblk = (T + kRouteTokPerBlk - 1) / kRouteTokPerBlk;
    if (E == 4)
        launch_pdl(route_count_vec_kernel<4>, dim3((unsigned)nblk), dim3(kThreads), 0, s,
                   logits, T, expert_idx, blk_counts);
    else if (E == 8)
        launch_pdl(route_count_vec_kernel<8>, dim3((unsigned)nblk), dim3(kThreads), 0, s,
                   logits, T, expert_idx, blk_counts);
    else if (E == 16)
        launch_pdl(route_count_vec_kernel<16>, dim3((unsigned)nblk), dim3(kThreads), 0, s,
                   logits, T, expert_idx, blk_counts);
    else if (E == 32)
        launch_pdl(route_count_vec_kernel<32>, dim3((unsigned)nblk), dim3(kThreads), 0, s,
                   logits, T, expert_idx, blk_counts);
    else if (E <= 4)
        launch_pdl(route_count_kernel<4>, dim3((unsigned)nblk), dim3(kThreads), 0, s,
                   logits, T, E, expert_idx, blk_counts);
    else if (E <= 8)
        launch_pdl(route_count_kernel<8>, dim3((unsigned)nblk), dim3(kThreads), 0, s,
                   logits, T, E, expert_idx, blk_counts);
    else if (E <= 16)
        launch_pdl(route_count_kernel<16>, dim3((unsigned)nblk), dim3(kThreads), 0, s,
                   logits, T, E, expert_idx, blk_counts);
    else
        launch_pdl(route_count_kernel<32>, dim3((unsigned)nblk), dim3(kThreads), 0, s,
                   logits, T, E, expert_idx, blk_counts);
    if (nblk * E <= kPrefixMaxEntries) {
        int ep = 1;
        while (ep < E) ep <<= 1;
        launch_pdl(route_scatter_prefix_kernel, dim3((unsigned)nblk), dim3(kThreads), 0, s,
                   expert_idx, T, E, ep, nblk, blk_counts, counts, offsets, perm);
        return cudaGetLastError();
    }
    launch_pdl(route_scan_kernel, dim3(1), dim3(1024), 0, s,
               blk_counts, nblk, E, counts, offsets, blk_base);
    launch_pdl(route_scatter_kernel, dim3((unsigned)nblk), dim3(kThreads), 0, s,
               expert_idx, T, E, blk_base, perm);
    return cudaGetLastError();
}

// The routing kernels use static shared memory only; kept so that callers that
// prepare a device once have a single place to do it.
cudaError_t route_set_smem_limits() { return cudaSuccess; }

}  // namespace moe
