// check_routing.cu -- validation of a routing handed to the library from
// outside moe_top1_route.
//
// The contraction kernels index the activations through offsets and perm
// without checking them (a check per token costs them about 5 % of their
// time), so a routing that is wrong -- an uninitialised buffer, another batch's
// routing, a buffer sized for another T -- can make them read and write outside
// their arrays. foxhunt commit 9170d24fe3 ("Single source of truth for the
// attention path"), BUG CAUGHT DURING WIRING, records the same class of fault:
// a scratch sized for the wrong count (n_tail) that only showed up as wrong
// memory traffic. This kernel lets a caller that does not produce its routing
// with moe_top1_route check it once, before the first contraction uses it. It
// reads only the four routing arrays, within their declared sizes, and records
// MOE_FLAG_BAD_ROUTING in the workspace flag word when any rule below fails:
//   offsets[0] = 0, offsets[E] = T, offsets non-decreasing,
//   counts[e] = offsets[e+1] - offsets[e],
//   every perm entry in [0, T), strictly ascending inside its expert's
//   segment, and expert_idx[perm[k]] = e for every position k of segment e.
// Together these make perm a permutation of 0..T-1 that groups the tokens by
// expert in ascending t, with every expert index in [0, E).
#include <cstdint>

#include "common.cuh"
#include "internal.h"
#include "moe_top1.h"

namespace moe {
namespace {

constexpr int kThreads = 256;
constexpr int64_t kMaxT = (int64_t{1} << 31) - 256;

__global__ void __launch_bounds__(kThreads)
check_routing_kernel(const int32_t* __restrict__ expert_idx, const int32_t* __restrict__ counts,
                     const int32_t* __restrict__ offsets, const int32_t* __restrict__ perm, int64_t T, int E,
                     uint32_t* __restrict__ flags) {
    griddep_wait();  // every global access below comes after the previous grid
    __shared__ int32_t s_off[33];
    __shared__ int s_offsets_ok;
    if (threadIdx.x == 0) {
        bool ok = offsets[0] == 0 && static_cast<int64_t>(offsets[E]) == T;
        bool counts_ok = true;
        for (int e = 0; e <= E; ++e) s_off[e] = offsets[e];
        for (int e = 0; e < E; ++e) {
            if (s_off[e + 1] < s_off[e]) ok = false;
            if (counts[e] != s_off[e + 1] - s_off[e]) counts_ok = false;
        }
        s_offsets_ok = ok ? 1 : 0;
        if (blockIdx.x == 0 && !(ok && counts_ok)) atomicOr(flags, MOE_FLAG_BAD_ROUTING);
    }
    __syncthreads();
    if (!s_offsets_ok) return;  // segments undefined: already recorded
    bool bad = false;
    const int64_t stride = static_cast<int64_t>(gridDim.x) * kThreads;
    for (int64_t k = static_cast<int64_t>(blockIdx.x) * kThreads + threadIdx.x; k < T; k += stride) {
        // expert segment of position k: the largest e with offsets[e] <= k
        int lo = 0, hi = E;  // offsets[lo] <= k < offsets[hi]
        while (hi - lo > 1) {
            const int mid = (lo + hi) >> 1;
            if (s_off[mid] <= k) lo = mid; else hi = mid;
        }
        const int32_t p = perm[k];
        if (p < 0 || static_cast<int64_t>(p) >= T) {
            bad = true;
            continue;
        }
        if (expert_idx[p] != lo) bad = true;
        if (k + 1 < s_off[lo + 1] && !(perm[k + 1] > p)) bad = true;
    }
    if (__syncthreads_or(bad) && threadIdx.x == 0) atomicOr(flags, MOE_FLAG_BAD_ROUTING);
}

bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3) == 0; }

}  // namespace
}  // namespace moe

extern "C" moe_status_t moe_top1_check_routing(const moe_routing_t* routing, int64_t T, int32_t E, void* workspace,
                                               size_t workspace_bytes, void* stream) {
    using namespace moe;
    if (!routing || T < 0) return MOE_ERR_INVALID_ARG;
    if (T >= kMaxT || E < 1 || E > 32) return MOE_ERR_UNSUPPORTED_SHAPE;
    if (!routing->counts || !routing->offsets) return MOE_ERR_INVALID_ARG;
    if (T > 0 && (!routing->expert_idx || !routing->perm)) return MOE_ERR_INVALID_ARG;
    if (!aligned4(routing->expert_idx) || !aligned4(routing->counts) || !aligned4(routing->offsets) ||
        !aligned4(routing->perm))
        return MOE_ERR_MISALIGNED;
    if (!workspace) return MOE_ERR_WORKSPACE;
    if ((reinterpret_cast<uintptr_t>(workspace) & 255) != 0) return MOE_ERR_MISALIGNED;
    if (workspace_bytes < 256) return MOE_ERR_WORKSPACE;
    int dev = 0, num_sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&num_sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return MOE_ERR_CUDA;
    const int64_t want = (T + kThreads - 1) / kThreads;
    const int64_t cap = static_cast<int64_t>(num_sms) * 8;
    const int grid = static_cast<int>(want < 1 ? 1 : (want < cap ? want : cap));
    launch_pdl(check_routing_kernel, dim3(grid), dim3(kThreads), 0, static_cast<cudaStream_t>(stream),
               routing->expert_idx, routing->counts, routing->offsets, routing->perm, T, E, static_cast<uint32_t*>(workspace));
    return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}
