// internal.h -- host-side declarations shared by the kernel files and the C ABI.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

namespace moe {

// Tokens handled by one block of the routing kernels; the fewest tokens one
// block of the aux kernel handles (the workspace has a partial-sum row for
// every such block).
constexpr int kRouteTokPerBlk = 1024;
constexpr int kAuxMinTokPerBlk = 256;

// Weight-gradient contraction: the expert-sorted token list is cut into
// `wgrad_splits(T)` equal ranges (further cut at expert boundaries); range c
// of expert e produces partial sum slot c + e. The split count depends on T
// only, so the reduction tree -- and hence every bit of dW and db -- is fixed
// for a given routing.
constexpr int kWgradMaxSplits = 148;
constexpr int kWgradMinTokPerSplit = 128;  // one 128-token tile: more CTAs at small T
// The TF32 backward strategy when the caller does not ask for one: a single pass
// over d_out (d_x and the dW / db partial sums together) for the horizon-mean
// gradient at H = 256, and at H = 128 above 65,536 tokens; two passes otherwise.
// Measured on a B200 (backward call, CUDA graph), two passes against one: H 128,
// 40,960 tokens 27.7 / 29.5 us, 65,535: 36.3 / 37.6, 81,920: 45.1 / 40.9,
// 131,070: 64.1 / 53.6, 262,144: 110.5 / 88.8, 1,048,576: 396 / 327; H 256,
// 1,048,576 tokens, per-token gradient 0.735 / 0.792 ms, horizon-mean gradient
// 0.757 / 0.733 ms.
constexpr int64_t kBwdSinglePassMinT128 = 65536;
inline bool bwd_single_pass_default(int H, int64_t T, bool collapse) {
    return (collapse && H == 256) || (H == 128 && T > kBwdSinglePassMinT128);
}
inline int wgrad_splits(int64_t T) {
    int64_t p = (T + kWgradMinTokPerSplit - 1) / kWgradMinTokPerSplit;
    if (p < 1) p = 1;
    if (p > kWgradMaxSplits) p = kWgradMaxSplits;
    return static_cast<int>(p);
}
// First sorted position of split c (floor(c * T / P)); ranges are [lo(c), lo(c+1)).
__host__ __device__ inline int64_t split_lo(int c, int64_t T, int P) { return (static_cast<int64_t>(c) * T) / P; }

// Byte offset, inside the workspace's 256-byte head, of the aux kernel's ticket
// counter (the flag word is at 0).
constexpr size_t kWsTicketOffset = 64;

struct WsLayout {
    size_t flags = 0;        // uint32 flag word (256 B reserved)
    size_t route_counts = 0; // int32 [nblk_route][E]
    size_t route_base = 0;   // int32 [nblk_route][E]
    size_t aux_psum = 0;     // float [nblk_aux][E]
    size_t wg_part = 0;      // float [P + E][H][H] dW partial sums
    size_t wg_part_db = 0;   // float [P + E][H]    db partial sums
    size_t route_end = 0;    // bytes the routing / aux calls need
    size_t total = 0;        // bytes every call needs
};

inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

inline WsLayout ws_layout(int64_t T, int E, int H) {
    WsLayout L;
    const int64_t nr = T > 0 ? (T + kRouteTokPerBlk - 1) / kRouteTokPerBlk : 1;
    const int64_t na = T > 0 ? (T + kAuxMinTokPerBlk - 1) / kAuxMinTokPerBlk : 1;
    const int P = wgrad_splits(T);
    size_t off = 0;
    L.flags = off;
    off += 256;
    L.route_counts = off;
    off = align_up(off + sizeof(int32_t) * nr * E, 256);
    L.route_base = off;
    off = align_up(off + sizeof(int32_t) * nr * E, 256);
    L.aux_psum = off;
    off = align_up(off + sizeof(float) * na * E, 256);
    L.route_end = off;
    if (H > 0) {
        L.wg_part = off;
        off = align_up(off + sizeof(float) * static_cast<size_t>(P + E) * H * H, 256);
        L.wg_part_db = off;
        off = align_up(off + sizeof(float) * static_cast<size_t>(P + E) * H, 256);
    }
    L.total = off;
    return L;
}

// ---------------------------------------------------------------- launchers
// Each returns the cudaError_t of its launch(es).
cudaError_t launch_route(const float* logits, int64_t T, int E, int32_t* expert_idx, int32_t* counts,
                         int32_t* offsets, int32_t* perm, int32_t* blk_counts, int32_t* blk_base,
                         cudaStream_t s);

// The adaptive-lambda update that can follow the aux loss in the same launch:
// out = floor + extra * max(0, target - *ent_ema) / target. out == nullptr: none.
struct LambdaNext {
    const float* ent_ema = nullptr;
    float floor = 0.0f, extra = 0.0f, target = 1.0f;
    float* out = nullptr;
};

// ticket: a uint32 of the workspace's reserved head (zeroed by
// moe_top1_workspace_init); the aux kernel's last block resets it after use.
// With next.out set, the last block also writes the next lambda once every block
// has read lambda_eff (next.out may be lambda_eff).
cudaError_t launch_aux(const float* logits, const int32_t* counts, int64_t T, int E, const float* lambda_eff,
                       float* d_logits, float* loss_out, float* mean_p, float* stats, float* blk_psum,
                       uint32_t* ticket, LambdaNext next, cudaStream_t s);

cudaError_t launch_usage_entropy_ema(const int32_t* counts, int64_t T, int E, float alpha, int reset,
                                     float* usage_ema, float* ent_ema, float* ent_step, cudaStream_t s);

cudaError_t launch_lambda_eff(const float* ent_ema, float lambda_floor, float lambda_max_extra, float ent_target,
                              float* lambda_eff, cudaStream_t s);

// out[perm[r], n] = out_scale * sum_k src[perm[r] / src_div, k] * B_e[n, k]
// (+ bias[e, n]) for the sorted rows r of expert e (src_div = 1, out_scale = 1:
// the plain contraction; src_div = N_H: every horizon token of a batch row reads
// that row's gradient). b_kmajor = 1: B_e[n, k] = Wsrc[e][n][k] (forward);
// b_kmajor = 0: B_e[n, k] = Wsrc[e][k][n] (input gradient).
cudaError_t launch_grouped_ffma(const float* src, const float* Wsrc, const float* bias, const int32_t* offsets,
                                const int32_t* perm, int64_t T, int E, int H, int b_kmajor, int accumulate,
                                int src_div, float out_scale, float* out, cudaStream_t s);

// Same contraction on tcgen05 (TF32 in, FP32 accumulate), straight from W
// [E][H][H]: w_transposed = 0: B_e[n, k] = W[e][n][k] (forward);
// w_transposed = 1: B_e[n, k] = W[e][k][n] (input gradient).
cudaError_t launch_grouped_tf32(const float* src, const float* W, const float* bias, const int32_t* offsets,
                                const int32_t* perm, int64_t T, int E, int H, int w_transposed, int accumulate,
                                int src_div, float out_scale, float* out, uint32_t* dev_flags, int num_sms,
                                cudaStream_t s);

// Per-range partial sums of dW / db into the slot buffers (see wgrad_splits);
// token t's gradient row is d_out[t / g_div].
cudaError_t launch_wgrad_ffma(const float* x, const float* d_out, const int32_t* offsets, const int32_t* perm,
                              int64_t T, int E, int H, int g_div, float* part, float* part_db, cudaStream_t s);
cudaError_t launch_wgrad_tf32(const float* x, const float* d_out, const int32_t* offsets, const int32_t* perm,
                              int64_t T, int E, int H, int g_div, float* part, float* part_db, uint32_t* dev_flags,
                              cudaStream_t s);
// Fixed-order pairwise sum of the slots of each expert, times scale, into dW / db
// (either may be null). P: the number of ranges the partial sums were cut into
// (wgrad_splits(T) for the weight-gradient kernels, the pair count for the
// fused backward).
cudaError_t launch_wgrad_reduce(const float* part, const float* part_db, const int32_t* offsets, int64_t T,
                                int E, int H, int P, float scale, float* dW, float* db, int acc_dw, int acc_db,
                                cudaStream_t s);

// The fused TF32 backward (d_x, and dW / db partial sums into the slots, in one
// pass over d_out and x): H = 256 on P pairs of CTAs, H = 128 on P single CTAs;
// range c of expert e gives slot c + e. Token t's gradient row is
// g_src[t / g_div]; d_x is scaled by out_scale (the slot reduction applies it to
// dW and db).
constexpr int kFusedMaxPairs = 74;
cudaError_t launch_bwd_fused_tf32(const float* x, const float* W, const float* g_src, const int32_t* offsets,
                                  const int32_t* perm, int64_t T, int E, int H, int P, int g_div, float out_scale,
                                  int acc_dx, float* d_x, float* part, float* part_db, uint32_t* dev_flags,
                                  cudaStream_t s);
// Pairs that run at once on the current device (at most kFusedMaxPairs).
cudaError_t bwd_fused_max_pairs(int* out);
// Pairs used for T tokens: one per 512 tokens, at most max_pairs (<= wgrad_splits(T),
// so the slots fit the workspace).
int bwd_fused_pairs(int64_t T, int max_pairs);
cudaError_t bwd_fused_set_smem_limits();

// Driver entry point for tensor-map encoding (resolved at run time, so the
// library does not link libcuda).
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn get_encode_tiled();

// Shared-memory layouts a 2D tensor map writes its boxes in.
enum MapLayout : int {
    kMapSw128 = 0,        // 128-byte swizzle, 16-byte granules (box_cols = 32 floats)
    kMapSw128Atom32 = 1,  // 128-byte swizzle, 32-byte granules (box_cols = 32 floats)
    kMapSw64 = 2,         // 64-byte swizzle, 16-byte granules (box_cols = 16 floats)
    kMapPlain = 3         // no swizzle: rows of box_cols floats, back to back
};
// 2D fp32 tensor [rows][cols] with a box of box_cols x box_rows in the given
// layout. make_map_2d returns a cached copy when the same map was encoded before
// on this device; encode_map_2d always encodes.
// Every library kernel is launched with programmatic stream serialization: it may
// be scheduled while the kernel before it in the stream is still tearing down, runs
// its prologue (barrier init, tensor-memory allocation, tensor-map prefetch), and
// waits (griddep_wait in common.cuh: all of the previous grid complete and its
// memory visible) before its first global-memory access. After a kernel that is
// not the library's it behaves like a plain launch.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s, Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

bool make_map_2d(CUtensorMap* map, const float* base, uint64_t rows, uint64_t cols, uint32_t box_cols,
                 uint32_t box_rows, int layout = kMapSw128);
bool encode_map_2d(CUtensorMap* map, const float* base, uint64_t rows, uint64_t cols, uint32_t box_cols,
                   uint32_t box_rows, int layout);

}  // namespace moe
