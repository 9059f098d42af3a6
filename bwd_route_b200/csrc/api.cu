// api.cu -- the C ABI declared in include/moe_top1.h: argument validation on
// the host (nothing is launched for a bad call), workspace layout, and the
// launches of the kernels in route.cu, aux.cu, gemm_ffma.cu and gemm_tf32.cu.
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "hmean.h"
#include "internal.h"
#include "moe_top1.h"

namespace moe {

cudaError_t aux_set_smem_limits();
cudaError_t route_set_smem_limits();
cudaError_t tf32_set_smem_limits();

namespace {

constexpr int64_t kMaxT = (int64_t{1} << 31) - 256;
constexpr int kMaxDevices = 64;

struct DeviceInfo {
    int num_sms = 0;
    int fused_pairs = 0;  // CTA pairs of the fused backward that run at once
    bool aux_ready = false;
};
DeviceInfo g_dev[kMaxDevices];
std::mutex g_mu;

cudaError_t device_info(DeviceInfo** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_mu);
    DeviceInfo& d = g_dev[dev];
    if (d.num_sms == 0) {
        e = cudaDeviceGetAttribute(&d.num_sms, cudaDevAttrMultiProcessorCount, dev);
        if (e != cudaSuccess) return e;
    }
    if (!d.aux_ready) {
        e = aux_set_smem_limits();
        if (e == cudaSuccess) e = route_set_smem_limits();
        if (e == cudaSuccess) e = tf32_set_smem_limits();
        if (e == cudaSuccess) e = hmean_set_smem_limits();
        if (e == cudaSuccess) e = bwd_fused_set_smem_limits();
        if (e != cudaSuccess) return e;
        // pairs of the fused backward that fit at once; a failed query only
        // disables that call (it then returns MOE_ERR_CUDA), not the others
        if (bwd_fused_max_pairs(&d.fused_pairs) != cudaSuccess) {
            d.fused_pairs = 0;
            (void)cudaGetLastError();
        }
        d.aux_ready = true;
    }
    *out = &d;
    return cudaSuccess;
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

struct Range {
    const void* p;
    size_t bytes;
};

bool overlap(Range a, Range b) {
    if (!a.p || !b.p || a.bytes == 0 || b.bytes == 0) return false;
    const uintptr_t a0 = reinterpret_cast<uintptr_t>(a.p), b0 = reinterpret_cast<uintptr_t>(b.p);
    return a0 < b0 + b.bytes && b0 < a0 + a.bytes;
}

// Every output must be disjoint from every other output and from every input.
bool any_alias(const Range* outs, int n_out, const Range* ins, int n_in) {
    for (int i = 0; i < n_out; ++i) {
        for (int j = i + 1; j < n_out; ++j)
            if (overlap(outs[i], outs[j])) return true;
        for (int j = 0; j < n_in; ++j)
            if (overlap(outs[i], ins[j])) return true;
    }
    return false;
}

moe_status_t tokens(int64_t B, int64_t N_H, int64_t* T) {
    if (B < 0 || N_H < 0) return MOE_ERR_INVALID_ARG;
    if (N_H != 0 && B > kMaxT / N_H) return MOE_ERR_UNSUPPORTED_SHAPE;
    *T = B * N_H;
    if (*T >= kMaxT) return MOE_ERR_UNSUPPORTED_SHAPE;
    return MOE_OK;
}

bool h_supported(int H, moe_math_t math) {
    if (math == MOE_MATH_TF32) return H == 128 || H == 256;
    if (math == MOE_MATH_FFMA) return H >= 32 && H <= 256 && H % 32 == 0;
    return false;
}

moe_status_t cuda_status(cudaError_t e) { return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA; }

EncodeTiledFn g_encode = nullptr;

}  // namespace

EncodeTiledFn get_encode_tiled() {
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_encode) {
        void* fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            g_encode = reinterpret_cast<EncodeTiledFn>(fn);
    }
    return g_encode;
}

namespace {

// Recently encoded tensor maps (a map depends only on the arguments and the
// device, so the same weight tensor reuses its map on every call).
struct MapKey {
    const float* base;
    uint64_t rows, cols;
    uint32_t box_cols, box_rows;
    int layout;
    int dev;
    bool operator==(const MapKey& o) const {
        return base == o.base && rows == o.rows && cols == o.cols && box_cols == o.box_cols &&
               box_rows == o.box_rows && layout == o.layout && dev == o.dev;
    }
};
constexpr int kMapCache = 16;
MapKey g_map_key[kMapCache];
CUtensorMap g_map_val[kMapCache];
int g_map_n = 0, g_map_next = 0;
std::mutex g_map_mu;

}  // namespace

bool make_map_2d(CUtensorMap* map, const float* base, uint64_t rows, uint64_t cols, uint32_t box_cols,
                 uint32_t box_rows, int layout) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return false;
    const MapKey key{base, rows, cols, box_cols, box_rows, layout, dev};
    {
        std::lock_guard<std::mutex> lock(g_map_mu);
        for (int i = 0; i < g_map_n; ++i)
            if (g_map_key[i] == key) {
                *map = g_map_val[i];
                return true;
            }
    }
    if (!encode_map_2d(map, base, rows, cols, box_cols, box_rows, layout)) return false;
    std::lock_guard<std::mutex> lock(g_map_mu);
    const int slot = g_map_n < kMapCache ? g_map_n++ : (g_map_next++ % kMapCache);
    g_map_key[slot] = key;
    g_map_val[slot] = *map;
    return true;
}

bool encode_map_2d(CUtensorMap* map, const float* base, uint64_t rows, uint64_t cols, uint32_t box_cols,
                   uint32_t box_rows, int layout) {
    EncodeTiledFn enc = get_encode_tiled();
    if (!enc) return false;
    const CUtensorMapSwizzle swz = layout == kMapSw128Atom32 ? CU_TENSOR_MAP_SWIZZLE_128B_ATOM_32B
                                   : layout == kMapSw64      ? CU_TENSOR_MAP_SWIZZLE_64B
                                   : layout == kMapPlain     ? CU_TENSOR_MAP_SWIZZLE_NONE
                                                             : CU_TENSOR_MAP_SWIZZLE_128B;
    const cuuint64_t dims[2] = {cols, rows};
    const cuuint64_t strides[1] = {cols * sizeof(float)};
    const cuuint32_t box[2] = {box_cols, box_rows};
    const cuuint32_t estr[2] = {1, 1};
    const CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<float*>(base), dims, strides, box, estr,
                           CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// Body of both backward entry points: token t's output gradient is
// g_scale * d_out[t / g_div] (d_out has g_rows rows; collapse: the [B, H]
// gradient of the horizon mean).
moe_status_t bwd_impl(const float* x, const float* W, const float* d_out, int64_t g_rows, int g_div, float g_scale,
                      bool collapse, const moe_routing_t* routing,
                          int64_t B, int64_t N_H, int32_t E, int32_t H, moe_math_t math, float* d_x, float* dW,
                          float* db, uint32_t accumulate_flags, void* workspace, size_t workspace_bytes,
                          void* stream) {
    int64_t T = 0;
    moe_status_t st = tokens(B, N_H, &T);
    if (st != MOE_OK) return st;
    if (math != MOE_MATH_TF32 && math != MOE_MATH_FFMA) return MOE_ERR_INVALID_ARG;
    if (accumulate_flags & ~(MOE_ACC_DX | MOE_ACC_DW | MOE_ACC_DB | MOE_BWD_SINGLE_PASS)) return MOE_ERR_INVALID_ARG;
    if (E < 1 || E > 32 || !h_supported(H, math)) return MOE_ERR_UNSUPPORTED_SHAPE;
    if (!routing) return MOE_ERR_INVALID_ARG;
    if (!d_x && !dW && !db) return MOE_OK;
    if (T > 0 && (!d_out || !routing->offsets || !routing->perm)) return MOE_ERR_INVALID_ARG;
    if (d_x && !W) return MOE_ERR_INVALID_ARG;
    if (T > 0 && (dW || db) && !x) return MOE_ERR_INVALID_ARG;
    if (!aligned(x, 16) || !aligned(W, 16) || !aligned(d_out, 16) || !aligned(d_x, 16) || !aligned(dW, 16) ||
        !aligned(db, 16))
        return MOE_ERR_MISALIGNED;
    const size_t act = sizeof(float) * T * H;
    const size_t wbytes = sizeof(float) * E * H * H;
    const Range outs[3] = {{d_x, act}, {dW, wbytes}, {db, sizeof(float) * E * H}};
    const Range ins[6] = {{x, act},
                          {W, wbytes},
                          {d_out, sizeof(float) * static_cast<size_t>(g_rows) * H},
                          {routing->offsets, sizeof(int32_t) * (E + 1)},
                          {routing->perm, sizeof(int32_t) * T},
                          {workspace, workspace ? workspace_bytes : 0}};
    if (any_alias(outs, 3, ins, 6)) return MOE_ERR_ALIAS;
    const WsLayout L = ws_layout(T, E, H);
    const bool need_ws = (dW || db) || (d_x && math == MOE_MATH_TF32);  // TF32 d_x: the flag word
    if (need_ws) {
        if (!workspace) return MOE_ERR_WORKSPACE;
        if (!aligned(workspace, 256)) return MOE_ERR_MISALIGNED;
        if (workspace_bytes < L.total) return MOE_ERR_WORKSPACE;
    }
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const int acc_dx = (accumulate_flags & MOE_ACC_DX) ? 1 : 0;
    const int acc_dw = (accumulate_flags & MOE_ACC_DW) ? 1 : 0;
    const int acc_db = (accumulate_flags & MOE_ACC_DB) ? 1 : 0;
    if (T == 0) {
        cudaError_t e = cudaSuccess;
        if (dW && !acc_dw) e = cudaMemsetAsync(dW, 0, wbytes, s);
        if (e == cudaSuccess && db && !acc_db) e = cudaMemsetAsync(db, 0, sizeof(float) * E * H, s);
        return cuda_status(e);
    }
    DeviceInfo* dev = nullptr;
    cudaError_t e = device_info(&dev);
    if (e != cudaSuccess) return MOE_ERR_CUDA;
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    uint32_t* flags = reinterpret_cast<uint32_t*>(ws);
    // One pass over d_out (d_x and the dW / db partial sums together), or two (d_x,
    // then dW / db): bwd_single_pass_default gives the measured rule, and
    // MOE_BWD_SINGLE_PASS asks for the single pass at every size.
    const bool single_pass = math == MOE_MATH_TF32 && d_x && (dW || db) &&
                             ((accumulate_flags & MOE_BWD_SINGLE_PASS) || bwd_single_pass_default(H, T, collapse));
    if (single_pass) {
        // H = 256: pairs of CTAs (as many as run at once); H = 128: single CTAs, one
        // per wgrad_splits(T) range
        float* part = reinterpret_cast<float*>(ws + L.wg_part);
        float* part_db = reinterpret_cast<float*>(ws + L.wg_part_db);
        if (H == 256 && dev->fused_pairs < 1) return MOE_ERR_CUDA;
        const int P = H == 256 ? bwd_fused_pairs(T, dev->fused_pairs) : wgrad_splits(T);
        e = launch_bwd_fused_tf32(x, W, d_out, routing->offsets, routing->perm, T, E, H, P, g_div, g_scale, acc_dx, d_x,
                                  part, part_db, flags, s);
        if (e == cudaSuccess)
            e = launch_wgrad_reduce(part, part_db, routing->offsets, T, E, H, P, g_scale, dW, db, acc_dw, acc_db, s);
        return cuda_status(e);
    }
    if (d_x) {
        if (math == MOE_MATH_TF32) {
            e = launch_grouped_tf32(d_out, W, nullptr, routing->offsets, routing->perm, T, E, H, 1, acc_dx, g_div,
                                    g_scale, d_x, flags, dev->num_sms, s);
        } else {
            e = launch_grouped_ffma(d_out, W, nullptr, routing->offsets, routing->perm, T, E, H, 0, acc_dx, g_div,
                                    g_scale, d_x, s);
        }
        if (e != cudaSuccess) return MOE_ERR_CUDA;
    }
    if (dW || db) {
        float* part = reinterpret_cast<float*>(ws + L.wg_part);
        float* part_db = reinterpret_cast<float*>(ws + L.wg_part_db);
        if (math == MOE_MATH_TF32)
            e = launch_wgrad_tf32(x, d_out, routing->offsets, routing->perm, T, E, H, g_div, part, part_db, flags, s);
        else
            e = launch_wgrad_ffma(x, d_out, routing->offsets, routing->perm, T, E, H, g_div, part, part_db, s);
        if (e == cudaSuccess)
            e = launch_wgrad_reduce(part, part_db, routing->offsets, T, E, H, wgrad_splits(T), g_scale, dW, db, acc_dw,
                                    acc_db, s);
        if (e != cudaSuccess) return MOE_ERR_CUDA;
    }
    return MOE_OK;
}

namespace {

// Argument checks of the adaptive-lambda update (shared by the separate call and
// the one folded into the aux launch).
moe_status_t check_lambda_args(const float* ent_ema, float lambda_floor, float lambda_max_extra, float ent_target,
                               const float* lambda_out) {
    if (!ent_ema || !lambda_out) return MOE_ERR_INVALID_ARG;
    if (!aligned(ent_ema, 4) || !aligned(lambda_out, 4)) return MOE_ERR_MISALIGNED;
    if (!std::isfinite(ent_target) || !(ent_target > 0.0f)) return MOE_ERR_INVALID_ARG;
    if (!std::isfinite(lambda_floor) || !(lambda_floor >= 0.0f)) return MOE_ERR_INVALID_ARG;
    if (!std::isfinite(lambda_max_extra) || !(lambda_max_extra >= 0.0f)) return MOE_ERR_INVALID_ARG;
    return MOE_OK;
}

moe_status_t aux_impl(const float* gate_logits, const int32_t* counts, int64_t B, int64_t N_H, int32_t E,
                      const float* lambda_eff, float* d_logits, float* loss_out, float* mean_p, float* stats,
                      const LambdaNext& next, void* workspace, size_t workspace_bytes, void* stream) {
    int64_t T = 0;
    moe_status_t st = tokens(B, N_H, &T);
    if (st != MOE_OK) return st;
    if (E < 1 || E > 32) return MOE_ERR_UNSUPPORTED_SHAPE;
    if (!counts || !lambda_eff || !loss_out || !mean_p) return MOE_ERR_INVALID_ARG;
    if (T > 0 && !gate_logits) return MOE_ERR_INVALID_ARG;
    if (!aligned(gate_logits, 16) || !aligned(d_logits, 16) || !aligned(counts, 4) || !aligned(lambda_eff, 4) ||
        !aligned(loss_out, 4) || !aligned(mean_p, 4) || !aligned(stats, 4))
        return MOE_ERR_MISALIGNED;
    const size_t lbytes = sizeof(float) * T * E;
    // the next lambda may replace lambda_eff (read by every block before the last
    // one writes it) or ent_ema (read by the thread that writes it), nothing else
    const Range outs[5] = {{d_logits, lbytes},
                           {loss_out, 2 * sizeof(float)},
                           {mean_p, sizeof(float) * E},
                           {stats, sizeof(float) * (3 * E + 4)},
                           {next.out, next.out ? sizeof(float) : 0}};
    const bool next_is_lambda = next.out && next.out == lambda_eff;
    const Range ins[4] = {{gate_logits, lbytes},
                          {counts, sizeof(int32_t) * E},
                          {next_is_lambda ? nullptr : lambda_eff, next_is_lambda ? 0 : sizeof(float)},
                          {workspace, workspace ? workspace_bytes : 0}};
    if (any_alias(outs, 5, ins, 4)) return MOE_ERR_ALIAS;
    if (next_is_lambda) {  // lambda_eff is then an output too: disjoint from the other outputs
        const Range lam[1] = {{lambda_eff, sizeof(float)}};
        if (any_alias(outs, 4, lam, 1)) return MOE_ERR_ALIAS;
    }
    if (next.out) {
        const Range ema[1] = {{next.ent_ema, sizeof(float)}};
        if (any_alias(outs, 4, ema, 1)) return MOE_ERR_ALIAS;
    }
    // the kernel writes the workspace (per-block sums, ticket) while other blocks
    // still read the inputs: none of them may lie inside it
    const Range wsr{workspace, workspace ? workspace_bytes : 0};
    if (overlap(wsr, ins[0]) || overlap(wsr, ins[1]) || overlap(wsr, {lambda_eff, sizeof(float)}) ||
        (next.out && overlap(wsr, {next.ent_ema, sizeof(float)})))
        return MOE_ERR_ALIAS;
    const WsLayout L = ws_layout(T, E, 0);
    if (!workspace) return MOE_ERR_WORKSPACE;
    if (!aligned(workspace, 256)) return MOE_ERR_MISALIGNED;
    if (workspace_bytes < L.route_end) return MOE_ERR_WORKSPACE;
    DeviceInfo* dev = nullptr;
    if (device_info(&dev) != cudaSuccess) return MOE_ERR_CUDA;
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    return cuda_status(launch_aux(gate_logits, counts, T, E, lambda_eff, d_logits, loss_out, mean_p, stats,
                                  reinterpret_cast<float*>(ws + L.aux_psum),
                                  reinterpret_cast<uint32_t*>(ws + kWsTicketOffset), next,
                                  static_cast<cudaStream_t>(stream)));
}

}  // namespace

}  // namespace moe

using namespace moe;

extern "C" {

int32_t moe_top1_abi_version(void) { return MOE_TOP1_ABI_VERSION; }

const char* moe_status_string(moe_status_t s) {
    switch (s) {
        case MOE_OK: return "MOE_OK";
        case MOE_ERR_INVALID_ARG: return "MOE_ERR_INVALID_ARG";
        case MOE_ERR_UNSUPPORTED_SHAPE: return "MOE_ERR_UNSUPPORTED_SHAPE";
        case MOE_ERR_MISALIGNED: return "MOE_ERR_MISALIGNED";
        case MOE_ERR_ALIAS: return "MOE_ERR_ALIAS";
        case MOE_ERR_WORKSPACE: return "MOE_ERR_WORKSPACE";
        case MOE_ERR_CUDA: return "MOE_ERR_CUDA";
        case MOE_ERR_DEVICE_CHECK: return "MOE_ERR_DEVICE_CHECK";
    }
    return "MOE_ERR_UNKNOWN";
}

size_t moe_top1_workspace_bytes(int64_t T, int32_t E, int32_t H) {
    if (T < 0 || E < 1 || E > 32 || H < 0) return 0;
    return ws_layout(T, E, H).total;
}

moe_status_t moe_top1_workspace_init(void* workspace, size_t workspace_bytes, void* stream) {
    if (!workspace) return MOE_ERR_INVALID_ARG;
    if (!aligned(workspace, 256)) return MOE_ERR_MISALIGNED;
    if (workspace_bytes < 256) return MOE_ERR_WORKSPACE;
    return cuda_status(cudaMemsetAsync(workspace, 0, 256, static_cast<cudaStream_t>(stream)));
}

moe_status_t moe_top1_device_flags(void* workspace, size_t workspace_bytes, void* stream, uint32_t* flags_out) {
    if (!workspace || !flags_out) return MOE_ERR_INVALID_ARG;
    if (!aligned(workspace, 256)) return MOE_ERR_MISALIGNED;
    if (workspace_bytes < 256) return MOE_ERR_WORKSPACE;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    uint32_t host = 0;
    cudaError_t e = cudaMemcpyAsync(&host, workspace, sizeof(uint32_t), cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e == cudaSuccess) e = cudaMemsetAsync(workspace, 0, sizeof(uint32_t), s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return MOE_ERR_CUDA;
    *flags_out = host;
    return host ? MOE_ERR_DEVICE_CHECK : MOE_OK;
}

moe_status_t moe_top1_route(const float* gate_logits, int64_t B, int64_t N_H, int32_t E, const moe_routing_t* out,
                            void* workspace, size_t workspace_bytes, void* stream) {
    int64_t T = 0;
    moe_status_t st = tokens(B, N_H, &T);
    if (st != MOE_OK) return st;
    if (E < 1 || E > 32) return MOE_ERR_UNSUPPORTED_SHAPE;
    if (!out || !out->counts || !out->offsets) return MOE_ERR_INVALID_ARG;
    if (T > 0 && (!gate_logits || !out->expert_idx || !out->perm)) return MOE_ERR_INVALID_ARG;
    if (T > 0 && !aligned(gate_logits, 16)) return MOE_ERR_MISALIGNED;
    if (!aligned(out->counts, 4) || !aligned(out->offsets, 4) || !aligned(out->expert_idx, 4) ||
        !aligned(out->perm, 4))
        return MOE_ERR_MISALIGNED;
    const WsLayout L = ws_layout(T, E, 0);
    const Range outs[4] = {{out->expert_idx, sizeof(int32_t) * T},
                           {out->counts, sizeof(int32_t) * E},
                           {out->offsets, sizeof(int32_t) * (E + 1)},
                           {out->perm, sizeof(int32_t) * T}};
    const Range ins[2] = {{gate_logits, sizeof(float) * T * E}, {workspace, workspace ? workspace_bytes : 0}};
    if (any_alias(outs, 4, ins, 2)) return MOE_ERR_ALIAS;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (T == 0) {
        cudaError_t e = cudaMemsetAsync(out->counts, 0, sizeof(int32_t) * E, s);
        if (e == cudaSuccess) e = cudaMemsetAsync(out->offsets, 0, sizeof(int32_t) * (E + 1), s);
        return cuda_status(e);
    }
    if (!workspace) return MOE_ERR_WORKSPACE;
    if (!aligned(workspace, 256)) return MOE_ERR_MISALIGNED;
    if (workspace_bytes < L.route_end) return MOE_ERR_WORKSPACE;
    DeviceInfo* dev = nullptr;
    if (device_info(&dev) != cudaSuccess) return MOE_ERR_CUDA;
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    return cuda_status(launch_route(gate_logits, T, E, out->expert_idx, out->counts, out->offsets, out->perm,
                                    reinterpret_cast<int32_t*>(ws + L.route_counts),
                                    reinterpret_cast<int32_t*>(ws + L.route_base), s));
}

moe_status_t moe_top1_fwd(const float* x, const float* W, const float* bias, const moe_routing_t* routing,
                          int64_t B, int64_t N_H, int32_t E, int32_t H, moe_math_t math, float* routed,
                          void* workspace, size_t workspace_bytes, void* stream) {
    int64_t T = 0;
    moe_status_t st = tokens(B, N_H, &T);
    if (st != MOE_OK) return st;
    if (math != MOE_MATH_TF32 && math != MOE_MATH_FFMA) return MOE_ERR_INVALID_ARG;
    if (E < 1 || E > 32 || !h_supported(H, math)) return MOE_ERR_UNSUPPORTED_SHAPE;
    if (!routing || !W || !bias) return MOE_ERR_INVALID_ARG;
    if (T > 0 && (!x || !routed || !routing->offsets || !routing->perm)) return MOE_ERR_INVALID_ARG;
    if (!aligned(x, 16) || !aligned(W, 16) || !aligned(bias, 16) || !aligned(routed, 16)) return MOE_ERR_MISALIGNED;
    const size_t act = sizeof(float) * T * H;
    const Range outs[1] = {{routed, act}};
    const Range ins[6] = {{x, act},
                          {W, sizeof(float) * E * H * H},
                          {bias, sizeof(float) * E * H},
                          {routing->offsets, sizeof(int32_t) * (E + 1)},
                          {routing->perm, sizeof(int32_t) * T},
                          {workspace, workspace ? workspace_bytes : 0}};
    if (any_alias(outs, 1, ins, 6)) return MOE_ERR_ALIAS;
    if (math == MOE_MATH_TF32) {
        if (!workspace) return MOE_ERR_WORKSPACE;
        if (!aligned(workspace, 256)) return MOE_ERR_MISALIGNED;
        if (workspace_bytes < 256) return MOE_ERR_WORKSPACE;
    }
    if (T == 0) return MOE_OK;
    DeviceInfo* dev = nullptr;
    cudaError_t e = device_info(&dev);
    if (e != cudaSuccess) return MOE_ERR_CUDA;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (math == MOE_MATH_TF32)
        return cuda_status(launch_grouped_tf32(x, W, bias, routing->offsets, routing->perm, T, E, H, 0, 0, 1, 1.0f, routed,
                                               static_cast<uint32_t*>(workspace), dev->num_sms, s));
    return cuda_status(launch_grouped_ffma(x, W, bias, routing->offsets, routing->perm, T, E, H, 1, 0, 1, 1.0f, routed, s));
}

moe_status_t moe_top1_fwd_mean_collapse(const float* x, const float* W, const float* bias,
                                        const moe_routing_t* routing, int64_t B, int64_t N_H, int32_t E, int32_t H,
                                        moe_math_t math, float* ctx_mean, void* workspace, size_t workspace_bytes,
                                        void* stream) {
    int64_t T = 0;
    moe_status_t st = tokens(B, N_H, &T);
    if (st != MOE_OK) return st;
    if (math != MOE_MATH_TF32 && math != MOE_MATH_FFMA) return MOE_ERR_INVALID_ARG;
    if (E < 1 || E > 32 || !h_supported(H, math)) return MOE_ERR_UNSUPPORTED_SHAPE;
    if (B > 0 && (N_H < 1 || N_H > 32)) return MOE_ERR_UNSUPPORTED_SHAPE;
    if (!routing || !W || !bias) return MOE_ERR_INVALID_ARG;
    if (B > 0 && (!x || !ctx_mean || !routing->expert_idx)) return MOE_ERR_INVALID_ARG;
    if (!aligned(x, 16) || !aligned(W, 16) || !aligned(bias, 16) || !aligned(ctx_mean, 16)) return MOE_ERR_MISALIGNED;
    if (!aligned(routing->expert_idx, 4)) return MOE_ERR_MISALIGNED;
    const Range outs[1] = {{ctx_mean, sizeof(float) * B * H}};
    const Range ins[5] = {{x, sizeof(float) * T * H},
                          {W, sizeof(float) * E * H * H},
                          {bias, sizeof(float) * E * H},
                          {routing->expert_idx, sizeof(int32_t) * T},
                          {workspace, workspace ? workspace_bytes : 0}};
    if (any_alias(outs, 1, ins, 5)) return MOE_ERR_ALIAS;
    if (math == MOE_MATH_TF32) {
        if (!workspace) return MOE_ERR_WORKSPACE;
        if (!aligned(workspace, 256)) return MOE_ERR_MISALIGNED;
        if (workspace_bytes < 256) return MOE_ERR_WORKSPACE;
    }
    if (B == 0) return MOE_OK;
    DeviceInfo* dev = nullptr;
    cudaError_t e = device_info(&dev);
    if (e != cudaSuccess) return MOE_ERR_CUDA;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const int nh = static_cast<int>(N_H);
    if (math == MOE_MATH_TF32)
        return cuda_status(launch_hmean_fwd_tf32(x, W, bias, routing->expert_idx, B, nh, E, H, ctx_mean,
                                                 static_cast<uint32_t*>(workspace), dev->num_sms, s));
    return cuda_status(launch_hmean_fwd_ffma(x, W, bias, routing->expert_idx, B, nh, E, H, ctx_mean, s));
}

moe_status_t moe_top1_bwd(const float* x, const float* W, const float* d_out, const moe_routing_t* routing,
                          int64_t B, int64_t N_H, int32_t E, int32_t H, moe_math_t math, float* d_x, float* dW,
                          float* db, uint32_t accumulate_flags, void* workspace, size_t workspace_bytes,
                          void* stream) {
    int64_t T = 0;
    moe_status_t st = tokens(B, N_H, &T);
    if (st != MOE_OK) return st;
    return bwd_impl(x, W, d_out, T, 1, 1.0f, false, routing, B, N_H, E, H, math, d_x, dW, db, accumulate_flags,
                    workspace, workspace_bytes, stream);
}

moe_status_t moe_top1_bwd_mean_collapse(const float* x, const float* W, const float* grad_ctx_mean,
                                        const moe_routing_t* routing, int64_t B, int64_t N_H, int32_t E, int32_t H,
                                        moe_math_t math, float* d_x, float* dW, float* db, uint32_t accumulate_flags,
                                        void* workspace, size_t workspace_bytes, void* stream) {
    int64_t T = 0;
    moe_status_t st = tokens(B, N_H, &T);
    if (st != MOE_OK) return st;
    if (N_H > (int64_t{1} << 30)) return MOE_ERR_UNSUPPORTED_SHAPE;
    const int g_div = T > 0 ? static_cast<int>(N_H) : 1;
    const float g_scale = T > 0 ? static_cast<float>(1.0 / static_cast<double>(N_H)) : 1.0f;
    return bwd_impl(x, W, grad_ctx_mean, B, g_div, g_scale, true, routing, B, N_H, E, H, math, d_x, dW, db,
                    accumulate_flags, workspace, workspace_bytes, stream);
}

moe_status_t moe_aux_loss_fwd_bwd(const float* gate_logits, const int32_t* counts, int64_t B, int64_t N_H,
                                  int32_t E, const float* lambda_eff, float* d_logits, float* loss_out,
                                  float* mean_p, float* stats, void* workspace, size_t workspace_bytes,
                                  void* stream) {
    return aux_impl(gate_logits, counts, B, N_H, E, lambda_eff, d_logits, loss_out, mean_p, stats, LambdaNext{},
                    workspace, workspace_bytes, stream);
}

moe_status_t moe_aux_loss_fwd_bwd_lambda_update(const float* gate_logits, const int32_t* counts, int64_t B,
                                                int64_t N_H, int32_t E, const float* lambda_eff, float* d_logits,
                                                float* loss_out, float* mean_p, float* stats, const float* ent_ema,
                                                float lambda_floor, float lambda_max_extra, float ent_target,
                                                float* lambda_next, void* workspace, size_t workspace_bytes,
                                                void* stream) {
    moe_status_t st = check_lambda_args(ent_ema, lambda_floor, lambda_max_extra, ent_target, lambda_next);
    if (st != MOE_OK) return st;
    LambdaNext next;
    next.ent_ema = ent_ema;
    next.floor = lambda_floor;
    next.extra = lambda_max_extra;
    next.target = ent_target;
    next.out = lambda_next;
    return aux_impl(gate_logits, counts, B, N_H, E, lambda_eff, d_logits, loss_out, mean_p, stats, next, workspace,
                    workspace_bytes, stream);
}

moe_status_t moe_lambda_eff_update(const float* ent_ema, float lambda_floor, float lambda_max_extra,
                                   float ent_target, float* lambda_eff, void* stream) {
    moe_status_t st = check_lambda_args(ent_ema, lambda_floor, lambda_max_extra, ent_target, lambda_eff);
    if (st != MOE_OK) return st;
    return cuda_status(launch_lambda_eff(ent_ema, lambda_floor, lambda_max_extra, ent_target, lambda_eff,
                                         static_cast<cudaStream_t>(stream)));
}

moe_status_t moe_usage_entropy_ema_update(const int32_t* counts, int64_t T, int32_t E, float alpha,
                                          int32_t reset, float* usage_ema, float* ent_ema, float* ent_step,
                                          void* stream) {
    if (T < 0) return MOE_ERR_INVALID_ARG;
    if (E < 1 || E > 32) return MOE_ERR_UNSUPPORTED_SHAPE;
    if (!counts || !usage_ema || !ent_ema) return MOE_ERR_INVALID_ARG;
    if (!(alpha >= 0.0f && alpha <= 1.0f)) return MOE_ERR_INVALID_ARG;  // NaN fails too
    if (!aligned(counts, 4) || !aligned(usage_ema, 4) || !aligned(ent_ema, 4) || (ent_step && !aligned(ent_step, 4)))
        return MOE_ERR_MISALIGNED;
    const Range outs[3] = {{usage_ema, sizeof(float) * static_cast<size_t>(E)},
                           {ent_ema, sizeof(float)},
                           {ent_step, ent_step ? sizeof(float) : 0}};
    const Range ins[1] = {{counts, sizeof(int32_t) * static_cast<size_t>(E)}};
    if (any_alias(outs, 3, ins, 1)) return MOE_ERR_ALIAS;
    return cuda_status(launch_usage_entropy_ema(counts, T, E, alpha, reset ? 1 : 0, usage_ema, ent_ema, ent_step,
                                                static_cast<cudaStream_t>(stream)));
}

}  // extern "C"
