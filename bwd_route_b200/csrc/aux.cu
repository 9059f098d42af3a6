// aux.cu -- load-balance auxiliary loss with its logit gradient, and the
// adaptive lambda controller.
//
// foxhunt commit 11b96dac6a ("Top-1 Mixture-of-Experts gate per Switch
// Transformer"), kernel list and ARCHITECTURE: a softmax of the gate logits and
// the balance loss aux = E * sum_e frac_e * mean_p_e, where frac comes from the
// non-differentiable top-1 choice (straight-through: only mean_p carries
// gradient). foxhunt commit 2d0e6b6bdc ("Replace static moe_lambda=0.01 with a
// GPU-driven controller"): lambda_eff = floor + max_extra * max(0, target -
// ent_ema) / target, read by the loss kernel from device memory. foxhunt commit
// 6cfd7e6691 (softmax + cross-entropy kernel), Kernel: the softmax is shifted
// by the row max.
//
// The logit gradient of token t needs only its own softmax row and the global
// frac, so one streaming pass reads the logits once, writes d_logits and leaves
// per-block sums of p (warps work on 32-token chunks staged in their own shared
// buffers); the last block to finish then sums those in a fixed order (mean_p,
// aux, loss, stats). No floating-point atomics: every bit is reproducible.
#include <cstdint>

#include "common.cuh"
#include "internal.h"

namespace moe {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kChunk = 32;                                   // tokens a warp handles at a time
// Tokens per block: 256 up to kAuxSmallT tokens (more blocks, a shorter chain in
// each), 1024 above (fewer per-block partial sums for the last block to add).
// Measured on a B200: at 81,920 tokens the small blocks take 1 us less per step;
// at 262,144 tokens they take 20.6 us against 16.2 (cold, under a profiler).
constexpr int kAuxTokPerBlkSmall = kWarps * kChunk;      // one chunk per warp
constexpr int kAuxTokPerBlkLarge = 4 * kWarps * kChunk;  // four chunks per warp
constexpr int64_t kAuxSmallT = 131072;
static_assert(kAuxTokPerBlkSmall >= kAuxMinTokPerBlk, "the workspace holds a row per block");
inline int aux_tok_per_blk(int64_t T) { return T <= kAuxSmallT ? kAuxTokPerBlkSmall : kAuxTokPerBlkLarge; }

// Shared-memory slot of float4 q (experts 4q..4q+3) of token row t when a row
// holds Q = EMAX / 4 float4s: the XOR swizzle spreads the 8 rows read by one
// quarter-warp over distinct banks, so row reads and writes are conflict-free.
template <int EMAX>
__device__ __forceinline__ int row_slot(int t, int q) {
    constexpr int Q = EMAX / 4;
    if (Q == 1) return t;
    constexpr int SH = (Q == 2) ? 2 : (Q == 4) ? 1 : 0;
    return t * Q + (q ^ ((t >> SH) & (Q - 1)));
}

__device__ void aux_finalize_block(const float* blk_psum, int64_t nblk,
                                   const int32_t* __restrict__ counts, int64_t T, int E,
                                   const float* lambda_eff, float* __restrict__ loss_out,
                                   float* __restrict__ mean_p, float* __restrict__ stats);

// The adaptive lambda of the next step from the gate-entropy EMA (a NaN EMA gives
// the floor): floor + extra * max(0, target - ent_ema) / target.
__device__ __forceinline__ float lambda_from_ema(float ent_ema, float floor, float extra, float target) {
    float deficit = target - ent_ema;
    if (!(deficit > 0.0f)) deficit = 0.0f;  // max(0, .); NaN gives 0
    return floor + extra * deficit / target;
}

// Called by every thread of the block that finalized: after the barrier no
// thread of it reads lambda_eff any more (the other blocks read it before they
// took their tickets), so next.out may be lambda_eff.
__device__ __forceinline__ void write_lambda_next(const LambdaNext& next) {
    if (!next.out) return;
    __syncthreads();
    if (threadIdx.x == 0) *next.out = lambda_from_ema(__ldcg(next.ent_ema), next.floor, next.extra, next.target);
}

// One block per CPW x 256 consecutive tokens (CPW = 1 or 4); warp w handles
// chunks w, w + 8, ... of 32 tokens. The warp stages all its chunks' logits in its own
// shared buffer (128-bit loads, every load in flight before the first use, no
// block barrier for the data), lane t computes token t of each chunk reading
// its row as float4s, and the gradients go back out with 128-bit stores. When
// E is not a multiple of 4 the rows are moved one float at a time.
// With four chunks per warp and rows of at most 8 experts a block holds 32 KB of
// shared memory, so 7 blocks fit an SM if each thread keeps to 32 registers: the
// 1024 blocks of 1,048,576 tokens then run in one wave instead of two.
template <int EMAX, int kChunksPerWarp>
__global__ void __launch_bounds__(kThreads, (kChunksPerWarp == 4 && EMAX <= 8) ? 7 : 1) aux_kernel(const float* __restrict__ logits,
                                                      const int32_t* __restrict__ counts, int64_t T, int E,
                                                      const float* lambda_eff,
                                                      float* __restrict__ d_logits, float* __restrict__ blk_psum,
                                                      uint32_t* __restrict__ ticket, float* __restrict__ loss_out,
                                                      float* __restrict__ mean_p, float* __restrict__ stats,
                                                      LambdaNext next) {
    griddep_wait();  // every global access below comes after the previous grid
    constexpr int Q = EMAX / 4;          // float4s per staged row
    constexpr int BUF4 = kChunk * Q;     // float4s per chunk buffer
    extern __shared__ float4 s_dyn4[];   // kWarps x kChunksPerWarp chunk buffers
    __shared__ float s_frac[EMAX];
    __shared__ float s_part[kWarps][EMAX];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x < EMAX)
        s_frac[threadIdx.x] = threadIdx.x < E ? static_cast<float>(counts[threadIdx.x]) / static_cast<float>(T) : 0.0f;
    // through L2: the last block may overwrite lambda_eff (next.out) once every block has used it
    const float lam = __ldcg(lambda_eff);
    const float scale = lam * static_cast<float>(E) / static_cast<float>(T);
    const bool vec = (E == EMAX);        // rows move as whole float4s
    float4* wbuf = s_dyn4 + warp * kChunksPerWarp * BUF4;
    int64_t c0[kChunksPerWarp];
    int n[kChunksPerWarp];
#pragma unroll
    for (int j = 0; j < kChunksPerWarp; ++j) {
        c0[j] = static_cast<int64_t>(blockIdx.x) * (kChunksPerWarp * kWarps * kChunk) + (j * kWarps + warp) * kChunk;
        n[j] = c0[j] >= T ? 0 : static_cast<int>((T - c0[j] < kChunk) ? (T - c0[j]) : kChunk);
    }
    if (vec) {
        // cp.async straight into the swizzled rows: all of the warp's copies (Q per
        // lane per chunk) are in flight before the warp waits once; rows past the
        // end of a ragged chunk are zero-filled and never used.
#pragma unroll
        for (int j = 0; j < kChunksPerWarp; ++j) {
            const float4* src4 = reinterpret_cast<const float4*>(logits + (n[j] > 0 ? c0[j] : 0) * E);
            const uint32_t b32 = smem_u32(wbuf + j * BUF4);
#pragma unroll
            for (int u = 0; u < Q; ++u) {
                const int i = lane + 32 * u;  // float4 i of the chunk: row i / Q, quarter i % Q
                cp_async_16(b32 + 16 * row_slot<EMAX>(i / Q, i % Q), src4 + (i < n[j] * Q ? i : 0),
                            i < n[j] * Q ? 16u : 0u);
            }
        }
        cp_async_wait_all();
        __syncwarp();
    }
#pragma unroll
    for (int j = 0; j < kChunksPerWarp && !vec; ++j) {
        float4* buf = wbuf + j * BUF4;
        {
            float* b = reinterpret_cast<float*>(buf);
            for (int i = lane; i < n[j] * E; i += 32) {
                const int t = i / E, e = i % E;
                b[row_slot<EMAX>(t, e / 4) * 4 + (e & 3)] = __ldg(logits + c0[j] * E + i);
            }
        }
    }
    __syncthreads();  // s_frac (the chunk buffers are per warp)
    float psum[EMAX];
#pragma unroll
    for (int e = 0; e < EMAX; ++e) psum[e] = 0.0f;
#pragma unroll
    for (int j = 0; j < kChunksPerWarp; ++j) {
        if (lane < n[j]) {
            float4* buf = wbuf + j * BUF4;
            float x[EMAX];
#pragma unroll
            for (int q = 0; q < Q; ++q) {
                const float4 v = buf[row_slot<EMAX>(lane, q)];
                x[4 * q] = v.x;
                x[4 * q + 1] = v.y;
                x[4 * q + 2] = v.z;
                x[4 * q + 3] = v.w;
            }
            float m = x[0];
#pragma unroll
            for (int e = 1; e < EMAX; ++e)
                if (e < E && x[e] > m) m = x[e];
            float sum = 0.0f;
#pragma unroll
            for (int e = 0; e < EMAX; ++e) {
                if (e < E) {
                    x[e] = expf(x[e] - m);
                    sum += x[e];
                }
            }
            const float rs = __frcp_rn(sum);  // correctly rounded 1 / sum
            float g = 0.0f;
#pragma unroll
            for (int e = 0; e < EMAX; ++e) {
                if (e < E) {
                    x[e] = x[e] * rs;
                    g += s_frac[e] * x[e];
                }
            }
#pragma unroll
            for (int e = 0; e < EMAX; ++e) {
                if (e < E) {
                    psum[e] += x[e];
                    x[e] = scale * (x[e] * (s_frac[e] - g));
                }
            }
#pragma unroll
            for (int q = 0; q < Q; ++q)
                buf[row_slot<EMAX>(lane, q)] = make_float4(x[4 * q], x[4 * q + 1], x[4 * q + 2], x[4 * q + 3]);
        }
    }
    __syncwarp();
    if (d_logits) {
#pragma unroll
        for (int j = 0; j < kChunksPerWarp; ++j) {
            const float4* buf = wbuf + j * BUF4;
            if (vec) {
                float4* dst4 = reinterpret_cast<float4*>(d_logits + c0[j] * E);
                for (int i = lane; i < n[j] * Q; i += 32) dst4[i] = buf[row_slot<EMAX>(i / Q, i % Q)];
            } else {
                const float* b = reinterpret_cast<const float*>(buf);
                for (int i = lane; i < n[j] * E; i += 32) {
                    const int t = i / E, e = i % E;
                    d_logits[c0[j] * E + i] = b[row_slot<EMAX>(t, e / 4) * 4 + (e & 3)];
                }
            }
        }
    }
    // fixed-order block sum of p: xor-butterfly inside each warp, then warps in order
#pragma unroll
    for (int e = 0; e < EMAX; ++e) {
        float v = psum[e];
#pragma unroll
        for (int off = 16; off >= 1; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
        if (lane == 0) s_part[warp][e] = v;
    }
    __syncthreads();
    if (threadIdx.x < E) {
        float acc = s_part[0][threadIdx.x];
        for (int w = 1; w < kWarps; ++w) acc += s_part[w][threadIdx.x];
        blk_psum[static_cast<int64_t>(blockIdx.x) * E + threadIdx.x] = acc;
        __threadfence();  // this block's partials are visible before its ticket is taken
    }
    // The block that takes the last ticket (an integer counter in the workspace)
    // finalizes: every other block's partials are in memory by then. The order of
    // the sums does not depend on which block is last. The counter is reset for
    // the next call.
    __shared__ int s_last;
    __syncthreads();
    if (threadIdx.x == 0) s_last = (atomicAdd(ticket, 1u) == gridDim.x - 1) ? 1 : 0;
    __syncthreads();
    if (s_last) {
        __threadfence();
        aux_finalize_block(blk_psum, gridDim.x, counts, T, E, lambda_eff, loss_out, mean_p, stats);
        if (threadIdx.x == 0) *ticket = 0u;
        write_lambda_next(next);
    }
}

// One block: mean_p from the per-block sums (double, fixed order), then aux,
// loss, stats. Warp w takes experts w, w + nwarps, ...; lane l of it sums the
// expert's per-block partials l, l + 32, l + 64, ... in block order (eight
// loads in flight), then an xor butterfly combines the lanes.
__device__ void aux_finalize_block(const float* blk_psum, int64_t nblk,
                                   const int32_t* __restrict__ counts, int64_t T, int E,
                                   const float* lambda_eff, float* __restrict__ loss_out,
                                   float* __restrict__ mean_p, float* __restrict__ stats) {
    __shared__ double s_sum[32];
    __shared__ float s_mean[32];
    __shared__ double s_hf[32], s_hm[32];
    __shared__ int s_cnt[32];
    __shared__ float s_lam;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nwarps = blockDim.x >> 5;
    if (threadIdx.x == 0) s_lam = __ldcg(lambda_eff);
    if (threadIdx.x < E) s_cnt[threadIdx.x] = counts[threadIdx.x];
    for (int e = warp; e < E; e += nwarps) {
        double acc = 0.0;
        for (int64_t b0 = lane; b0 < nblk; b0 += 8 * 32) {
            float v[8];  // eight independent loads, then added in block order
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int64_t b = b0 + static_cast<int64_t>(u) * 32;
                // written by other blocks of the same launch: read through L2 (coherent), not the
                // non-coherent read-only path
                v[u] = (b < nblk) ? __ldcg(blk_psum + b * E + e) : 0.0f;
            }
#pragma unroll
            for (int u = 0; u < 8; ++u)
                if (b0 + static_cast<int64_t>(u) * 32 < nblk) acc += static_cast<double>(v[u]);
        }
#pragma unroll
        for (int off = 16; off >= 1; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
        if (lane == 0) s_sum[e] = acc;
    }
    __syncthreads();
    if (threadIdx.x < E) {
        const int x = threadIdx.x;
        const float m = T > 0 ? static_cast<float>(s_sum[x] / static_cast<double>(T)) : 0.0f;
        s_mean[x] = m;
        // entropy terms of expert x (0 ln 0 = 0)
        const double f = T > 0 ? static_cast<double>(s_cnt[x]) / static_cast<double>(T) : 0.0;
        s_hf[x] = f > 0.0 ? f * log(f) : 0.0;
        s_hm[x] = m > 0.0f ? static_cast<double>(m) * log(static_cast<double>(m)) : 0.0;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        const float lam = s_lam;
        double acc = 0.0, hf = 0.0, hm = 0.0;
        for (int e = 0; e < E; ++e) {
            acc += static_cast<double>(s_cnt[e]) * static_cast<double>(s_mean[e]);
            hf -= s_hf[e];
            hm -= s_hm[e];
        }
        const float aux_raw = T > 0 ? static_cast<float>(static_cast<double>(E) * acc / static_cast<double>(T)) : 0.0f;
        loss_out[0] = aux_raw;
        loss_out[1] = lam * aux_raw;
        for (int e = 0; e < E; ++e) mean_p[e] = s_mean[e];
        if (stats) {
            for (int e = 0; e < E; ++e) {
                stats[e] = T > 0 ? static_cast<float>(s_cnt[e]) / static_cast<float>(T) : 0.0f;
                stats[E + e] = s_mean[e];
                stats[2 * E + e] = static_cast<float>(s_cnt[e]);
            }
            stats[3 * E + 0] = aux_raw;
            stats[3 * E + 1] = lam;
            stats[3 * E + 2] = static_cast<float>(hf);
            stats[3 * E + 3] = static_cast<float>(hm);
        }
    }
}

// The empty batch: only the finalize (zeros, and lambda in the stats).
__global__ void __launch_bounds__(kThreads) aux_finalize_kernel(const int32_t* __restrict__ counts, int E,
                                                               const float* lambda_eff,
                                                               float* __restrict__ loss_out, float* __restrict__ mean_p,
                                                               float* __restrict__ stats, LambdaNext next) {
    griddep_wait();  // every global access below comes after the previous grid
    aux_finalize_block(nullptr, 0, counts, 0, E, lambda_eff, loss_out, mean_p, stats);
    write_lambda_next(next);
}

__global__ void lambda_eff_kernel(const float* __restrict__ ent_ema, float lambda_floor, float lambda_max_extra,
                                  float ent_target, float* __restrict__ lambda_eff) {
    griddep_wait();  // every global access below comes after the previous grid
    *lambda_eff = lambda_from_ema(*ent_ema, lambda_floor, lambda_max_extra, ent_target);
}

// Producer of the gate-entropy signal the lambda controller reads (one warp;
// lane e owns expert e): H = -sum_e frac_e ln frac_e over this step's argmax
// usage fractions, then the caller-weighted moving averages of frac and H, or
// the cold-start state on a reset. Double inside, fp32 in memory; the sum over
// experts is one fixed xor butterfly, read from lane 0.
__global__ void usage_entropy_ema_kernel(const int32_t* __restrict__ counts, int64_t T, int E, float alpha,
                                         int reset, float* __restrict__ usage_ema, float* __restrict__ ent_ema,
                                         float* __restrict__ ent_step) {
    griddep_wait();  // every global access below comes after the previous grid
    const int lane = threadIdx.x;
    const bool on = lane < E;
    const double f = (on && T > 0) ? static_cast<double>(counts[lane]) / static_cast<double>(T) : 0.0;
    double h = f > 0.0 ? -f * log(f) : 0.0;
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) h += __shfl_xor_sync(0xffffffffu, h, off);
    if (reset) {
        if (on) usage_ema[lane] = static_cast<float>(1.0 / static_cast<double>(E));
        if (lane == 0) *ent_ema = static_cast<float>(log(static_cast<double>(E)));
    } else if (T > 0) {
        const double a = alpha;
        if (on) usage_ema[lane] = static_cast<float>((1.0 - a) * static_cast<double>(usage_ema[lane]) + a * f);
        if (lane == 0) *ent_ema = static_cast<float>((1.0 - a) * static_cast<double>(*ent_ema) + a * h);
    }
    if (lane == 0 && ent_step) *ent_step = static_cast<float>(h);
}

}  // namespace

cudaError_t launch_usage_entropy_ema(const int32_t* counts, int64_t T, int E, float alpha, int reset,
                                     float* usage_ema, float* ent_ema, float* ent_step, cudaStream_t s) {
    launch_pdl(usage_entropy_ema_kernel, dim3(1), dim3(32), 0, s,
               counts, T, E, alpha, reset, usage_ema, ent_ema, ent_step);
    return cudaGetLastError();
}

cudaError_t launch_aux(const float* logits, const int32_t* counts, int64_t T, int E, const float* lambda_eff,
                       float* d_logits, float* loss_out, float* mean_p, float* stats, float* blk_psum,
                       uint32_t* ticket, LambdaNext next, cudaStream_t s) {
    if (T == 0) {
        launch_pdl(aux_finalize_kernel, dim3(1), dim3(kThreads), 0, s,
                   counts, E, lambda_eff, loss_out, mean_p, stats, next);
        return cudaGetLastError();
    }
    const int tpb = aux_tok_per_blk(T);
    const int64_t nblk = (T + tpb - 1) / tpb;
    const int cpw = tpb / (kWarps * kChunk);
    const int emax = E <= 4 ? 4 : E <= 8 ? 8 : E <= 16 ? 16 : 32;
    const size_t smem = sizeof(float) * kWarps * cpw * kChunk * emax;
#define MOE_AUX_LAUNCH(EM, CPW)                                                                              \
    launch_pdl(aux_kernel<EM, CPW>, dim3((unsigned)nblk), dim3(kThreads), smem, s, logits, counts, T, E,     \
               lambda_eff, d_logits, blk_psum, ticket, loss_out, mean_p, stats, next)
    if (cpw == 1) {
        if (emax == 4) MOE_AUX_LAUNCH(4, 1);
        else if (emax == 8) MOE_AUX_LAUNCH(8, 1);
        else if (emax == 16) MOE_AUX_LAUNCH(16, 1);
        else MOE_AUX_LAUNCH(32, 1);
    } else {
        if (emax == 4) MOE_AUX_LAUNCH(4, 4);
        else if (emax == 8) MOE_AUX_LAUNCH(8, 4);
        else if (emax == 16) MOE_AUX_LAUNCH(16, 4);
        else MOE_AUX_LAUNCH(32, 4);
    }
#undef MOE_AUX_LAUNCH
    return cudaGetLastError();
}

cudaError_t launch_lambda_eff(const float* ent_ema, float lambda_floor, float lambda_max_extra, float ent_target,
                              float* lambda_eff, cudaStream_t s) {
    launch_pdl(lambda_eff_kernel, dim3(1), dim3(1), 0, s,
               ent_ema, lambda_floor, lambda_max_extra, ent_target, lambda_eff);
    return cudaGetLastError();
}

cudaError_t aux_set_smem_limits() {
    // 8 warps x 4 chunks x 32 tokens x 32 experts x 4 bytes = 128 KiB for the widest instance
    cudaError_t e = cudaFuncSetAttribute(aux_kernel<16, 4>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(sizeof(float) * kWarps * 4 * kChunk * 16));
    if (e != cudaSuccess) return e;
    return cudaFuncSetAttribute(aux_kernel<32, 4>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                static_cast<int>(sizeof(float) * kWarps * 4 * kChunk * 32));
}

}  // namespace moe
