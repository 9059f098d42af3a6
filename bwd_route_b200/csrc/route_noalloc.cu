// route_noalloc.cu -- the routing entry point for callers that cannot allocate
// device memory.
//
// moe_top1_route needs a caller-provided workspace for its per-block expert
// counts and bases. Some callers cannot provide one: a host framework that hands
// a plug-in only its input and output tensors and owns every byte of device
// memory through its own allocator, or a runtime that plans all device memory
// up front and forbids allocations once it is running. For them this file keeps
// that scratch in a fixed, file-scope device array instead, so the call needs
// nothing but its inputs and outputs. The routing kernels are the same ones
// moe_top1_route launches.
#include <cstdint>

#include "internal.h"
#include "moe_top1.h"

namespace moe {

namespace {

constexpr int64_t kNoAllocMaxBlocks = MOE_NOALLOC_MAX_TOKENS / kRouteTokPerBlk;  // 2048
constexpr int kNoAllocMaxExperts = 32;
static_assert(MOE_NOALLOC_MAX_TOKENS % kRouteTokPerBlk == 0, "whole routing blocks");

// Per-block expert counts followed by per-block expert bases: 2 x 2048 x 32
// int32 = 512 KiB. Every GPU that loads the library holds this until the
// process exits. Host code must not use the array's name as a device address
// (on the host it is only a stand-in); it uses the address that
// cudaGetSymbolAddress returns in the current context.
static __device__ __align__(256) int32_t g_route_scratch[2 * kNoAllocMaxBlocks * kNoAllocMaxExperts];

// The array's device address in the CUDA context current on the calling thread.
// A module-scope __device__ variable has one copy per context that loads the
// library's module, and that copy's address belongs to the context: a context
// created after a cudaDeviceReset, or a non-primary context a host made current
// on the same device, has its own copy at its own address. So the address is
// looked up on every call (a host-side table lookup that allocates nothing and
// enqueues no work) instead of being cached per device number.
cudaError_t scratch_of_current_context(int32_t** out) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_route_scratch);
    if (e != cudaSuccess) return e;
    *out = static_cast<int32_t*>(p);
    return cudaSuccess;
}

bool is_aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

bool overlaps(const void* a, size_t na, const void* b, size_t nb) {
    if (!a || !b || na == 0 || nb == 0) return false;
    const uintptr_t a0 = reinterpret_cast<uintptr_t>(a), b0 = reinterpret_cast<uintptr_t>(b);
    return a0 < b0 + nb && b0 < a0 + na;
}

}  // namespace
}  // namespace moe

extern "C" moe_status_t moe_top1_route_noalloc(const float* gate_logits, int64_t B, int64_t N_H, int32_t E,
                                               const moe_routing_t* out, void* stream) {
    using namespace moe;
    if (B < 0 || N_H < 0) return MOE_ERR_INVALID_ARG;
    if (N_H != 0 && B > MOE_NOALLOC_MAX_TOKENS / N_H) return MOE_ERR_UNSUPPORTED_SHAPE;
    const int64_t T = B * N_H;
    if (T > MOE_NOALLOC_MAX_TOKENS) return MOE_ERR_UNSUPPORTED_SHAPE;  // beyond the fixed scratch
    if (E < 1 || E > kNoAllocMaxExperts) return MOE_ERR_UNSUPPORTED_SHAPE;
    if (!out || !out->counts || !out->offsets) return MOE_ERR_INVALID_ARG;
    if (T > 0 && (!gate_logits || !out->expert_idx || !out->perm)) return MOE_ERR_INVALID_ARG;
    if (T > 0 && !is_aligned(gate_logits, 16)) return MOE_ERR_MISALIGNED;
    if (!is_aligned(out->counts, 4) || !is_aligned(out->offsets, 4) || !is_aligned(out->expert_idx, 4) ||
        !is_aligned(out->perm, 4))
        return MOE_ERR_MISALIGNED;
    const void* o[4] = {out->expert_idx, out->counts, out->offsets, out->perm};
    const size_t n[4] = {sizeof(int32_t) * T, sizeof(int32_t) * E, sizeof(int32_t) * (E + 1), sizeof(int32_t) * T};
    for (int i = 0; i < 4; ++i) {
        if (overlaps(o[i], n[i], gate_logits, sizeof(float) * T * E)) return MOE_ERR_ALIAS;
        for (int j = i + 1; j < 4; ++j)
            if (overlaps(o[i], n[i], o[j], n[j])) return MOE_ERR_ALIAS;
    }
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (T == 0) {
        cudaError_t e = cudaMemsetAsync(out->counts, 0, sizeof(int32_t) * E, s);
        if (e == cudaSuccess) e = cudaMemsetAsync(out->offsets, 0, sizeof(int32_t) * (E + 1), s);
        return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
    }
    int32_t* scratch = nullptr;
    if (scratch_of_current_context(&scratch) != cudaSuccess) return MOE_ERR_CUDA;
    // The count kernel writes every per-block count the scan reads, and the scan
    // writes every base the scatter reads: nothing in the scratch has to start at 0.
    const int64_t nblk = (T + kRouteTokPerBlk - 1) / kRouteTokPerBlk;
    const cudaError_t e = launch_route(gate_logits, T, E, out->expert_idx, out->counts, out->offsets, out->perm,
                                       scratch, scratch + nblk * E, s);
    return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}
