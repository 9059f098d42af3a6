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
// per-block sums of p; a one-block kernel then sums those in a fixed order
// (mean_p, aux, loss, stats). No atomics: every bit is reproducible.
#include <cstdint>

#include "common.cuh"
#include "internal.h"

namespace moe {
namespace {

constexpr int kThreads = kAuxTokPerBlk;  // one token per thread
constexpr int kWarps = kThreads / 32;

template <int EMAX>
__global__ void __launch_bounds__(kThreads, 1) aux_kernel(const float* __restrict__ logits,
                                                      const int32_t* __restrict__ counts, int64_t T, int E,
                                                      const float* __restrict__ lambda_eff,
                                                      float* __restrict__ d_logits, float* __restrict__ blk_psum) {
    extern __shared__ float4 s_tile4[];  // kAuxTokPerBlk * E floats (logits, then gradients)
    float* s_tile = reinterpret_cast<float*>(s_tile4);
    __shared__ float s_frac[32];
    __shared__ float s_part[kWarps][EMAX];
    const int64_t t0 = static_cast<int64_t>(blockIdx.x) * kAuxTokPerBlk;
    const int64_t ntok = (T - t0 < kAuxTokPerBlk) ? (T - t0) : kAuxTokPerBlk;
    const int64_t nflt = ntok * E;
    const float* src = logits + t0 * E;
    // coalesced 128-bit staging (the block's first float is 16-byte aligned: 1024 * E * 4 bytes per block)
    const int64_t n4 = nflt / 4;
    stage_f4<2>(s_tile4, reinterpret_cast<const float4*>(src), static_cast<int>(n4), threadIdx.x, kThreads);
    for (int64_t i = n4 * 4 + threadIdx.x; i < nflt; i += kThreads) s_tile[i] = __ldg(src + i);
    if (threadIdx.x < E) s_frac[threadIdx.x] = static_cast<float>(counts[threadIdx.x]) / static_cast<float>(T);
    __syncthreads();
    const float lam = *lambda_eff;
    const float scale = lam * static_cast<float>(E) / static_cast<float>(T);
    float psum[EMAX];
#pragma unroll
    for (int e = 0; e < EMAX; ++e) psum[e] = 0.0f;
    const int tl = threadIdx.x;  // this thread's token in the block
    if (tl < ntok) {
        float* row = s_tile + static_cast<int64_t>(tl) * E;
        float p[EMAX];
        float m = row[0];
#pragma unroll
        for (int e = 1; e < EMAX; ++e)
            if (e < E && row[e] > m) m = row[e];
        float s = 0.0f;
#pragma unroll
        for (int e = 0; e < EMAX; ++e) {
            if (e < E) {
                p[e] = expf(row[e] - m);
                s += p[e];
            }
        }
        float g = 0.0f;
#pragma unroll
        for (int e = 0; e < EMAX; ++e) {
            if (e < E) {
                p[e] = p[e] / s;
                g += s_frac[e] * p[e];
            }
        }
#pragma unroll
        for (int e = 0; e < EMAX; ++e) {
            if (e < E) {
                psum[e] = p[e];
                row[e] = scale * (p[e] * (s_frac[e] - g));
            }
        }
    }
    // fixed-order block sum of p: xor-butterfly inside each warp, then warps in order
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
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
    }
    if (d_logits) {
        float* dst = d_logits + t0 * E;
        for (int64_t i = threadIdx.x; i < n4; i += kThreads) reinterpret_cast<float4*>(dst)[i] = s_tile4[i];
        for (int64_t i = n4 * 4 + threadIdx.x; i < nflt; i += kThreads) dst[i] = s_tile[i];
    }
}

// One block: mean_p from the per-block sums (double, fixed order: warp e sums
// expert e with lane-strided partials and an xor butterfly), then aux, loss and
// stats.
__global__ void __launch_bounds__(1024) aux_finalize_kernel(const float* __restrict__ blk_psum, int64_t nblk,
                                                           const int32_t* __restrict__ counts, int64_t T, int E,
                                                           const float* __restrict__ lambda_eff,
                                                           float* __restrict__ loss_out, float* __restrict__ mean_p,
                                                           float* __restrict__ stats) {
    __shared__ float s_mean[32];
    __shared__ double s_hf[32], s_hm[32];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (warp < E) {
        double acc = 0.0;
        for (int64_t b0 = 0; b0 < nblk; b0 += 8 * 32) {
            float v[8];  // eight independent loads, then added in block order
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int64_t b = b0 + u * 32 + lane;
                v[u] = (b < nblk) ? blk_psum[b * E + warp] : 0.0f;
            }
#pragma unroll
            for (int u = 0; u < 8; ++u)
                if (b0 + u * 32 + lane < nblk) acc += static_cast<double>(v[u]);
        }
#pragma unroll
        for (int off = 16; off >= 1; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
        if (lane == 0) {
            const float m = T > 0 ? static_cast<float>(acc / static_cast<double>(T)) : 0.0f;
            s_mean[warp] = m;
            // entropy terms of expert `warp` (0 ln 0 = 0)
            const double f = T > 0 ? static_cast<double>(counts[warp]) / static_cast<double>(T) : 0.0;
            s_hf[warp] = f > 0.0 ? f * log(f) : 0.0;
            s_hm[warp] = m > 0.0f ? static_cast<double>(m) * log(static_cast<double>(m)) : 0.0;
        }
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        const float lam = *lambda_eff;
        double acc = 0.0, hf = 0.0, hm = 0.0;
        for (int e = 0; e < E; ++e) {
            acc += static_cast<double>(counts[e]) * static_cast<double>(s_mean[e]);
            hf -= s_hf[e];
            hm -= s_hm[e];
        }
        const float aux_raw = T > 0 ? static_cast<float>(static_cast<double>(E) * acc / static_cast<double>(T)) : 0.0f;
        loss_out[0] = aux_raw;
        loss_out[1] = lam * aux_raw;
        for (int e = 0; e < E; ++e) mean_p[e] = s_mean[e];
        if (stats) {
            for (int e = 0; e < E; ++e) {
                stats[e] = T > 0 ? static_cast<float>(counts[e]) / static_cast<float>(T) : 0.0f;
                stats[E + e] = s_mean[e];
                stats[2 * E + e] = static_cast<float>(counts[e]);
            }
            stats[3 * E + 0] = aux_raw;
            stats[3 * E + 1] = lam;
            stats[3 * E + 2] = static_cast<float>(hf);
            stats[3 * E + 3] = static_cast<float>(hm);
        }
    }
}

__global__ void lambda_eff_kernel(const float* __restrict__ ent_ema, float lambda_floor, float lambda_max_extra,
                                  float ent_target, float* __restrict__ lambda_eff) {
    float deficit = ent_target - *ent_ema;
    if (!(deficit > 0.0f)) deficit = 0.0f;  // max(0, .); a NaN entropy gives the floor
    *lambda_eff = lambda_floor + lambda_max_extra * deficit / ent_target;
}

}  // namespace

cudaError_t launch_aux(const float* logits, const int32_t* counts, int64_t T, int E, const float* lambda_eff,
                       float* d_logits, float* loss_out, float* mean_p, float* stats, float* blk_psum,
                       cudaStream_t s) {
    const int64_t nblk = T > 0 ? (T + kAuxTokPerBlk - 1) / kAuxTokPerBlk : 0;
    if (T > 0) {
        const size_t smem = sizeof(float) * kAuxTokPerBlk * E;
        if (E <= 4)
            aux_kernel<4><<<(unsigned)nblk, kThreads, smem, s>>>(logits, counts, T, E, lambda_eff, d_logits, blk_psum);
        else if (E <= 8)
            aux_kernel<8><<<(unsigned)nblk, kThreads, smem, s>>>(logits, counts, T, E, lambda_eff, d_logits, blk_psum);
        else if (E <= 16)
            aux_kernel<16><<<(unsigned)nblk, kThreads, smem, s>>>(logits, counts, T, E, lambda_eff, d_logits, blk_psum);
        else
            aux_kernel<32><<<(unsigned)nblk, kThreads, smem, s>>>(logits, counts, T, E, lambda_eff, d_logits, blk_psum);
        const cudaError_t err = cudaGetLastError();
        if (err != cudaSuccess) return err;
    }
    aux_finalize_kernel<<<1, 1024, 0, s>>>(blk_psum, nblk, counts, T, E, lambda_eff, loss_out, mean_p, stats);
    return cudaGetLastError();
}

cudaError_t launch_lambda_eff(const float* ent_ema, float lambda_floor, float lambda_max_extra, float ent_target,
                              float* lambda_eff, cudaStream_t s) {
    lambda_eff_kernel<<<1, 1, 0, s>>>(ent_ema, lambda_floor, lambda_max_extra, ent_target, lambda_eff);
    return cudaGetLastError();
}

cudaError_t aux_set_smem_limits() {
    cudaError_t e = cudaFuncSetAttribute(aux_kernel<16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(sizeof(float) * kAuxTokPerBlk * 16));
    if (e != cudaSuccess) return e;
    return cudaFuncSetAttribute(aux_kernel<32>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                static_cast<int>(sizeof(float) * kAuxTokPerBlk * 32));
}

}  // namespace moe
