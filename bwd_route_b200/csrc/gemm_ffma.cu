// gemm_ffma.cu -- FP32 fused-multiply-add variants of the expert contractions,
// and the fixed-order reduction of the weight-gradient partial sums.
//
// foxhunt commit 11b96dac6a ("Top-1 Mixture-of-Experts gate per Switch
// Transformer"): forward routed[t,o] = sum_i W[e*,o,i] x[t,i] + b[e*,o]
// (PERFORMANCE: one output channel per dot product over H inputs); backward
// through the selected expert only (d_x[t,i] = sum_o W[e*,o,i] d_out[t,o]; dW and
// db summed over the expert's tokens, zero for inactive experts). foxhunt
// commit b23f8f2efa ("Local L40S profile"), reduce_axis0 / Discipline: sums over
// tokens are block tree-reductions without atomicAdd. Here the sum over an
// expert's tokens is split into fixed ranges of the expert-sorted token list
// (partial sums, one slot per range) and the slots are added in a fixed
// pairwise order, so no [tokens, E, H, H] scratch exists and every bit is
// reproducible.
#include <cstdint>

#include "common.cuh"
#include "hmean.h"
#include "internal.h"

namespace moe {
namespace {

// ---------------------------------------------------------------- grouped GEMM (FFMA)
constexpr int kGBM = 128, kGBN = 32, kGBK = 32, kGThreads = 256;

// Tile `tile` of the expert-sorted rows (kGBM rows per tile, tiles of one expert
// contiguous): returns the expert or -1 past the last tile.
__device__ __forceinline__ int find_tile(const int* s_tstart, int E, int tile) {
    if (tile >= s_tstart[E]) return -1;
    int e = 0;
    while (e + 1 < E && s_tstart[e + 1] <= tile) ++e;
    return e;
}

__global__ void __launch_bounds__(kGThreads) grouped_ffma_kernel(const float* __restrict__ src,
                                                                const float* __restrict__ Wsrc,
                                                                const float* __restrict__ bias,
                                                                const int32_t* __restrict__ offsets,
                                                                const int32_t* __restrict__ perm, int E,
                                                                int H, int b_kmajor, int accumulate, int src_div,
                                                                float out_scale, float* __restrict__ out) {
    griddep_wait();  // every global access below comes after the previous grid
    __shared__ int s_off[33];
    __shared__ int s_tstart[33];
    __shared__ int s_tok[kGBM];
    __shared__ __align__(16) float sA[kGBK][kGBM + 4];  // A^T: [k][row]
    __shared__ __align__(16) float sB[kGBK][kGBN + 4];  // [k][n]
    const int tid = threadIdx.x;
    if (tid <= E) s_off[tid] = offsets[tid];
    __syncthreads();
    if (tid == 0) {
        int ts = 0;
        for (int e = 0; e < E; ++e) {
            s_tstart[e] = ts;
            ts += (s_off[e + 1] - s_off[e] + kGBM - 1) / kGBM;
        }
        s_tstart[E] = ts;
    }
    __syncthreads();
    const int tile = blockIdx.x;
    const int e = find_tile(s_tstart, E, tile);
    if (e < 0) return;
    const int row0 = s_off[e] + (tile - s_tstart[e]) * kGBM;
    const int nrows = min(kGBM, s_off[e + 1] - row0);
    const int n0 = blockIdx.y * kGBN;
    for (int m = tid; m < kGBM; m += kGThreads) s_tok[m] = (m < nrows) ? perm[row0 + m] : -1;
    __syncthreads();
    const float* We = Wsrc + static_cast<int64_t>(e) * H * H;
    const int tm = tid / 8, tn = tid % 8;  // rows tm*4.., cols tn*4..
    float acc[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = 0.0f;
    for (int k0 = 0; k0 < H; k0 += kGBK) {
        // A: kGBM rows x kGBK cols, 8 float4 per row
#pragma unroll
        for (int q = 0; q < (kGBM * kGBK / 4) / kGThreads; ++q) {
            const int idx = tid + q * kGThreads;
            const int m = idx / 8, kq = idx % 8;
            const int tok = s_tok[m];
            float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
            if (tok >= 0)
                v = __ldg(reinterpret_cast<const float4*>(src + static_cast<int64_t>(src_div == 1 ? tok : tok / src_div) * H +
                                                          k0) + kq);
            sA[kq * 4 + 0][m] = v.x;
            sA[kq * 4 + 1][m] = v.y;
            sA[kq * 4 + 2][m] = v.z;
            sA[kq * 4 + 3][m] = v.w;
        }
        // B: kGBK x kGBN
        {
            if (b_kmajor) {  // B[k][n] = We[n0+n][k0+k]
                const int n = tid / 8, kq = tid % 8;
                const float4 v = __ldg(reinterpret_cast<const float4*>(We + static_cast<int64_t>(n0 + n) * H + k0) + kq);
                sB[kq * 4 + 0][n] = v.x;
                sB[kq * 4 + 1][n] = v.y;
                sB[kq * 4 + 2][n] = v.z;
                sB[kq * 4 + 3][n] = v.w;
            } else {  // B[k][n] = We[k0+k][n0+n]
                const int k = tid / 8, nq = tid % 8;
                const float4 v = __ldg(reinterpret_cast<const float4*>(We + static_cast<int64_t>(k0 + k) * H + n0) + nq);
                *reinterpret_cast<float4*>(&sB[k][nq * 4]) = v;
            }
        }
        __syncthreads();
#pragma unroll 8
        for (int k = 0; k < kGBK; ++k) {
            const float4 a = *reinterpret_cast<const float4*>(&sA[k][tm * 4]);
            const float4 b = *reinterpret_cast<const float4*>(&sB[k][tn * 4]);
            const float av[4] = {a.x, a.y, a.z, a.w};
            const float bv[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
        }
        __syncthreads();
    }
    float4 bvec = make_float4(0.f, 0.f, 0.f, 0.f);
    if (bias) bvec = __ldg(reinterpret_cast<const float4*>(bias + static_cast<int64_t>(e) * H + n0 + tn * 4));
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int m = tm * 4 + i;
        const int tok = s_tok[m];
        if (tok < 0) continue;
        float4 v = make_float4(acc[i][0] * out_scale + bvec.x, acc[i][1] * out_scale + bvec.y,
                               acc[i][2] * out_scale + bvec.z, acc[i][3] * out_scale + bvec.w);
        float4* dst = reinterpret_cast<float4*>(out + static_cast<int64_t>(tok) * H + n0 + tn * 4);
        if (accumulate) {
            const float4 o = *dst;
            v.x += o.x;
            v.y += o.y;
            v.z += o.z;
            v.w += o.w;
        }
        *dst = v;
    }
}

// ---------------------------------------------------------------- forward through the horizon mean (FFMA)
// ctx_mean[b] = (1/N_H) (sum_e W[e] X_be + sum_e n_be bias[e]) with
// X_be = sum_{h : e_bh = e} x[b,h] summed in ascending h ("Single source of
// truth for the attention path", MHA additions). Block = 128 batch rows x 32
// outputs; the K loop runs over (e, 32-wide k-chunk) in a fixed order.
__global__ void __launch_bounds__(kGThreads) hmean_fwd_ffma_kernel(const float* __restrict__ x,
                                                                  const float* __restrict__ W,
                                                                  const float* __restrict__ bias,
                                                                  const int32_t* __restrict__ expert_idx, int B,
                                                                  int N_H, int E, int H, float inv_nh,
                                                                  float* __restrict__ out) {
    griddep_wait();  // every global access below comes after the previous grid
    __shared__ uint32_t s_mask[kGBM][32];  // [row][e], bit h: horizon token h (N_H <= 32) chose expert e
    __shared__ __align__(16) float sA[kGBK][kGBM + 4];    // X_be^T: [k][row]
    __shared__ __align__(16) float sB[kGBK][kGBN + 4];    // [k][n]
    const int tid = threadIdx.x;
    const int b0 = blockIdx.x * kGBM;
    const int n0 = blockIdx.y * kGBN;
    for (int m = tid; m < kGBM; m += kGThreads) {
        uint32_t mk[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) mk[e] = 0u;
        const int b = b0 + m;
        if (b < B) {
            for (int h = 0; h < N_H; ++h) {
                const int e = expert_idx[static_cast<int64_t>(b) * N_H + h];
#pragma unroll
                for (int f = 0; f < 32; ++f)
                    if (f == e) mk[f] |= 1u << h;
            }
        }
#pragma unroll
        for (int e = 0; e < 32; ++e) s_mask[m][e] = mk[e];
    }
    __syncthreads();
    const int tm = tid / 8, tn = tid % 8;  // rows tm*4.., cols tn*4..
    float acc[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = 0.0f;
    for (int e = 0; e < E; ++e) {
        const float* We = W + static_cast<int64_t>(e) * H * H;
        for (int k0 = 0; k0 < H; k0 += kGBK) {
#pragma unroll
            for (int q = 0; q < (kGBM * kGBK / 4) / kGThreads; ++q) {
                const int idx = tid + q * kGThreads;
                const int m = idx / 8, kq = idx % 8;
                uint32_t mk = s_mask[m][e];
                float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
                if (mk) {
                    const float* xr = x + static_cast<int64_t>(b0 + m) * N_H * H + k0 + kq * 4;
                    v = __ldg(reinterpret_cast<const float4*>(xr + static_cast<int64_t>(__ffs(mk) - 1) * H));
                    for (mk &= mk - 1; mk; mk &= mk - 1) {
                        const float4 u = __ldg(reinterpret_cast<const float4*>(xr + static_cast<int64_t>(__ffs(mk) - 1) * H));
                        v.x += u.x;
                        v.y += u.y;
                        v.z += u.z;
                        v.w += u.w;
                    }
                }
                sA[kq * 4 + 0][m] = v.x;
                sA[kq * 4 + 1][m] = v.y;
                sA[kq * 4 + 2][m] = v.z;
                sA[kq * 4 + 3][m] = v.w;
            }
            {  // B[k][n] = W[e][n0+n][k0+k]
                const int n = tid / 8, kq = tid % 8;
                const float4 v = __ldg(reinterpret_cast<const float4*>(We + static_cast<int64_t>(n0 + n) * H + k0) + kq);
                sB[kq * 4 + 0][n] = v.x;
                sB[kq * 4 + 1][n] = v.y;
                sB[kq * 4 + 2][n] = v.z;
                sB[kq * 4 + 3][n] = v.w;
            }
            __syncthreads();
#pragma unroll 8
            for (int k = 0; k < kGBK; ++k) {
                const float4 a = *reinterpret_cast<const float4*>(&sA[k][tm * 4]);
                const float4 b = *reinterpret_cast<const float4*>(&sB[k][tn * 4]);
                const float av[4] = {a.x, a.y, a.z, a.w};
                const float bv[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
                for (int i = 0; i < 4; ++i)
#pragma unroll
                    for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
            }
            __syncthreads();
        }
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int m = tm * 4 + i;
        const int b = b0 + m;
        if (b >= B) continue;
        float r[4] = {acc[i][0], acc[i][1], acc[i][2], acc[i][3]};
        for (int e = 0; e < E; ++e) {
            const uint32_t mk = s_mask[m][e];
            if (!mk) continue;
            const float n = static_cast<float>(__popc(mk));
            const float4 bb = __ldg(reinterpret_cast<const float4*>(bias + static_cast<int64_t>(e) * H + n0 + tn * 4));
            r[0] = fmaf(n, bb.x, r[0]);
            r[1] = fmaf(n, bb.y, r[1]);
            r[2] = fmaf(n, bb.z, r[2]);
            r[3] = fmaf(n, bb.w, r[3]);
        }
        *reinterpret_cast<float4*>(out + static_cast<int64_t>(b) * H + n0 + tn * 4) =
            make_float4(r[0] * inv_nh, r[1] * inv_nh, r[2] * inv_nh, r[3] * inv_nh);
    }
}

// ---------------------------------------------------------------- weight gradient (FFMA)
// CTA (c, o-tile, i-tile): for every expert piece of range c, accumulate the
// 32 x 32 block of d_out^T x over the piece's tokens (ascending sorted order),
// write it to slot c + e. The i-tile-0 CTAs also sum d_out for db.
constexpr int kWT = 32, kWChunk = 64, kWThreads = 64;

__global__ void __launch_bounds__(kWThreads) wgrad_ffma_kernel(const float* __restrict__ x,
                                                              const float* __restrict__ d_out,
                                                              const int32_t* __restrict__ offsets,
                                                              const int32_t* __restrict__ perm, int64_t T, int E,
                                                              int H, int P, int g_div, float* __restrict__ part,
                                                              float* __restrict__ part_db) {
    griddep_wait();  // every global access below comes after the previous grid
    __shared__ __align__(16) float sG[kWChunk][kWT];  // d_out rows
    __shared__ __align__(16) float sX[kWChunk][kWT];  // x rows
    __shared__ int s_tok[kWChunk];
    const int c = blockIdx.x;
    const int o0 = blockIdx.y * kWT, i0 = blockIdx.z * kWT;
    const int tid = threadIdx.x;
    const int to = tid / 8, ti = tid % 8;  // outputs o0+to*4.., i0+ti*4..
    const int64_t lo = split_lo(c, T, P), hi = split_lo(c + 1, T, P);
    for (int e = 0; e < E; ++e) {
        const int64_t s = max(lo, static_cast<int64_t>(offsets[e]));
        const int64_t t = min(hi, static_cast<int64_t>(offsets[e + 1]));
        if (s >= t) continue;
        float acc[4][4];
#pragma unroll
        for (int a = 0; a < 4; ++a)
#pragma unroll
            for (int b = 0; b < 4; ++b) acc[a][b] = 0.0f;
        float dbacc = 0.0f;
        for (int64_t p0 = s; p0 < t; p0 += kWChunk) {
            const int n = static_cast<int>(min(static_cast<int64_t>(kWChunk), t - p0));
            if (tid < kWChunk) s_tok[tid] = (tid < n) ? perm[p0 + tid] : -1;
            __syncthreads();
            for (int idx = tid; idx < kWChunk * kWT / 4; idx += kWThreads) {
                const int r = idx / (kWT / 4), q = idx % (kWT / 4);
                const int tok = s_tok[r];
                float4 g = make_float4(0.f, 0.f, 0.f, 0.f), v = g;
                if (tok >= 0) {
                    g = __ldg(reinterpret_cast<const float4*>(d_out + static_cast<int64_t>(g_div == 1 ? tok : tok / g_div) * H +
                                                              o0) + q);
                    v = __ldg(reinterpret_cast<const float4*>(x + static_cast<int64_t>(tok) * H + i0) + q);
                }
                *reinterpret_cast<float4*>(&sG[r][q * 4]) = g;
                *reinterpret_cast<float4*>(&sX[r][q * 4]) = v;
            }
            __syncthreads();
            // two-level sum: each chunk of kWChunk tokens is summed on its own and
            // then added to the piece total, which keeps the fp32 rounding error of
            // sums over many thousands of tokens near that of a 64-term sum
            float cacc[4][4];
#pragma unroll
            for (int a = 0; a < 4; ++a)
#pragma unroll
                for (int b = 0; b < 4; ++b) cacc[a][b] = 0.0f;
            for (int r = 0; r < n; ++r) {
                const float4 g = *reinterpret_cast<const float4*>(&sG[r][to * 4]);
                const float4 v = *reinterpret_cast<const float4*>(&sX[r][ti * 4]);
                const float gv[4] = {g.x, g.y, g.z, g.w};
                const float xv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                for (int a = 0; a < 4; ++a)
#pragma unroll
                    for (int b = 0; b < 4; ++b) cacc[a][b] = fmaf(gv[a], xv[b], cacc[a][b]);
            }
#pragma unroll
            for (int a = 0; a < 4; ++a)
#pragma unroll
                for (int b = 0; b < 4; ++b) acc[a][b] += cacc[a][b];
            if (blockIdx.z == 0 && tid < kWT) {
                float cdb = 0.0f;
                for (int r = 0; r < n; ++r) cdb += sG[r][tid];
                dbacc += cdb;
            }
            __syncthreads();
        }
        const int64_t slot = c + e;
#pragma unroll
        for (int a = 0; a < 4; ++a) {
            float* dst = part + (slot * H + o0 + to * 4 + a) * H + i0 + ti * 4;
            *reinterpret_cast<float4*>(dst) = make_float4(acc[a][0], acc[a][1], acc[a][2], acc[a][3]);
        }
        if (blockIdx.z == 0 && tid < kWT) part_db[slot * H + o0 + tid] = dbacc;
    }
}

// ---------------------------------------------------------------- fixed-order reduction
// Sum of n values in the pairwise tree of a binary counter: value k merges with
// the completed block to its left whenever bit j of k is set. Deterministic.
struct PairwiseSum {
    float4 lvl[9];
    int n = 0;
    __device__ void add(float4 v) {
        int j = 0;
        while ((n >> j) & 1) {
            v = make_float4(lvl[j].x + v.x, lvl[j].y + v.y, lvl[j].z + v.z, lvl[j].w + v.w);
            ++j;
        }
        lvl[j] = v;
        ++n;
    }
    __device__ float4 result() const {
        float4 r = make_float4(0.f, 0.f, 0.f, 0.f);
        bool any = false;
        for (int j = 8; j >= 0; --j) {
            if ((n >> j) & 1) {
                r = any ? make_float4(r.x + lvl[j].x, r.y + lvl[j].y, r.z + lvl[j].z, r.w + lvl[j].w) : lvl[j];
                any = true;
            }
        }
        return r;
    }
};

__device__ __forceinline__ float4 add4(float4 a, float4 b) {
    return make_float4(a.x + b.x, a.y + b.y, a.z + b.z, a.w + b.w);
}

// Sum of the n slots of each element in a fixed tree: slots are taken in groups
// of eight added as ((s0+s1)+(s2+s3))+((s4+s5)+(s6+s7)) (missing slots of the last
// group count as 0), and the group sums are added pairwise in order
// (PairwiseSum). The group sums are independent: a block covers S chunks of 32
// float4 elements, and its 8 warps compute the S x ng (chunk, group) sums at once
// (eight loads in flight each); one thread per element then combines its groups
// in order. S adapts to the expert's group count ng so that a block holds about
// eight such sums: S = 8 for one group, down to S = 1 from five groups on, so an
// expert with few slots uses few blocks and one with many spreads over many.
// grid.x: one block per 32-element chunk of dW[e], then of db[e] (the most S = 1
// needs; with S > 1 the blocks past the last chunk return at once); grid.y = E.
constexpr int kRedElems = 32;
constexpr int kRedWarps = 8;
constexpr int kRedMaxGroups = (kWgradMaxSplits + 7) / 8;  // slots of one expert <= ranges <= kWgradMaxSplits
constexpr int kRedMaxItems = kRedMaxGroups > kRedWarps ? kRedMaxGroups : kRedWarps;
__global__ void __launch_bounds__(kRedWarps * 32) wgrad_reduce_kernel(const float* __restrict__ part,
                                                                     const float* __restrict__ part_db,
                                                                     const int32_t* __restrict__ offsets, int64_t T,
                                                                     int E, int H, int P, float scale,
                                                                     float* __restrict__ dW, float* __restrict__ db,
                                                                     int acc_dw, int acc_db) {
    griddep_wait();  // every global access below comes after the previous grid
    __shared__ int s_c[2];
    __shared__ float4 s_g[kRedMaxItems][kRedElems];
    const int e = blockIdx.y;
    // the ranges c that overlap expert e's tokens [a, b) are contiguous: thread c
    // tests range c (P <= blockDim.x) and the first / last overlapping one record it
    const int64_t a = offsets[e], b = offsets[e + 1];
    if (threadIdx.x == 0) {
        s_c[0] = 0;
        s_c[1] = -1;
    }
    __syncthreads();
    if (a < b && static_cast<int>(threadIdx.x) < P) {
        const int c = threadIdx.x;
        const int64_t lo = split_lo(c, T, P), hi = split_lo(c + 1, T, P);
        if (lo < b && hi > a) {
            if (lo <= a) s_c[0] = c;      // the range that holds token a
            if (hi >= b) s_c[1] = c;      // the range that holds token b - 1
        }
    }
    __syncthreads();
    const int c_lo = s_c[0], c_hi = s_c[1];
    const int n = c_hi - c_lo + 1;  // slots of expert e (0 for an expert with no tokens)
    const int ng = (n + 7) / 8;
    const int S = ng <= 1 ? 8 : ng == 2 ? 4 : ng <= 4 ? 2 : 1;  // chunks per block: S x ng <= 8 up to 8 groups
    const int64_t HH = static_cast<int64_t>(H) * H;
    const int nb_w = static_cast<int>((HH / 4 + kRedElems - 1) / kRedElems);
    const bool is_w = static_cast<int>(blockIdx.x) < nb_w;
    if (is_w ? !dW : !db) return;  // block-uniform
    const int64_t count = is_w ? HH / 4 : H / 4;  // float4 elements of dW[e] or db[e]
    const int64_t chunk0 = static_cast<int64_t>(is_w ? blockIdx.x : blockIdx.x - nb_w) * S;
    if (chunk0 * kRedElems >= count) return;  // block-uniform: past the last chunk at this S
    const float4* src = is_w ? reinterpret_cast<const float4*>(part + (static_cast<int64_t>(c_lo) + e) * HH)
                             : reinterpret_cast<const float4*>(part_db + (static_cast<int64_t>(c_lo) + e) * H);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const float4 z = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int i = warp; i < S * ng; i += kRedWarps) {  // (chunk i % S, group i / S)
        const int g = i / S;
        const int64_t j = (chunk0 + i % S) * kRedElems + lane;
        const bool valid = j < count;
        float4 v[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int k = g * 8 + u;
            v[u] = (valid && k < n) ? __ldg(src + static_cast<int64_t>(k) * count + j) : z;
        }
        s_g[i][lane] = add4(add4(add4(v[0], v[1]), add4(v[2], v[3])), add4(add4(v[4], v[5]), add4(v[6], v[7])));
    }
    __syncthreads();
    if (static_cast<int>(threadIdx.x) >= S * kRedElems) return;
    const int ch = threadIdx.x / kRedElems;
    const int64_t j = (chunk0 + ch) * kRedElems + lane;
    if (j >= count) return;
    PairwiseSum ps;
    for (int g = 0; g < ng; ++g) ps.add(s_g[g * S + ch][lane]);
    float4 r = ps.result();
    r = make_float4(r.x * scale, r.y * scale, r.z * scale, r.w * scale);
    float4* dst = is_w ? reinterpret_cast<float4*>(dW + e * HH) + j : reinterpret_cast<float4*>(db + static_cast<int64_t>(e) * H) + j;
    if (is_w ? acc_dw : acc_db) {
        const float4 o = *dst;
        r = make_float4(o.x + r.x, o.y + r.y, o.z + r.z, o.w + r.w);
    }
    *dst = r;
}

}  // namespace

cudaError_t launch_grouped_ffma(const float* src, const float* Wsrc, const float* bias, const int32_t* offsets,
                                const int32_t* perm, int64_t T, int E, int H, int b_kmajor, int accumulate,
                                int src_div, float out_scale, float* out, cudaStream_t s) {
    const int64_t tiles = (T + kGBM - 1) / kGBM + E;  // upper bound; extra CTAs exit
    dim3 grid(static_cast<unsigned>(tiles), H / kGBN);
    launch_pdl(grouped_ffma_kernel, dim3(grid), dim3(kGThreads), 0, s,
               src, Wsrc, bias, offsets, perm, E, H, b_kmajor, accumulate, src_div, out_scale, out);
    return cudaGetLastError();
}

cudaError_t launch_hmean_fwd_ffma(const float* x, const float* W, const float* bias, const int32_t* expert_idx,
                                  int64_t B, int N_H, int E, int H, float* out, cudaStream_t s) {
    const dim3 grid(static_cast<unsigned>((B + kGBM - 1) / kGBM), static_cast<unsigned>(H / kGBN));
    const float inv_nh = static_cast<float>(1.0 / static_cast<double>(N_H));
    launch_pdl(hmean_fwd_ffma_kernel, dim3(grid), dim3(kGThreads), 0, s,
               x, W, bias, expert_idx, static_cast<int>(B), N_H, E, H, inv_nh, out);
    return cudaGetLastError();
}

cudaError_t launch_wgrad_ffma(const float* x, const float* d_out, const int32_t* offsets, const int32_t* perm,
                              int64_t T, int E, int H, int g_div, float* part, float* part_db, cudaStream_t s) {
    const int P = wgrad_splits(T);
    dim3 grid(P, H / kWT, H / kWT);
    launch_pdl(wgrad_ffma_kernel, dim3(grid), dim3(kWThreads), 0, s,
               x, d_out, offsets, perm, T, E, H, P, g_div, part, part_db);
    return cudaGetLastError();
}

cudaError_t launch_wgrad_reduce(const float* part, const float* part_db, const int32_t* offsets, int64_t T,
                                int E, int H, int P, float scale, float* dW, float* db, int acc_dw, int acc_db,
                                cudaStream_t s) {
    const int64_t HH = static_cast<int64_t>(H) * H;
    const int nb_w = static_cast<int>((HH / 4 + kRedElems - 1) / kRedElems);
    const int nb_b = (H / 4 + kRedElems - 1) / kRedElems;
    if (P < 1 || P > kWgradMaxSplits) return cudaErrorInvalidValue;  // the group sums of one expert fit s_g
    dim3 grid(nb_w + nb_b, E);
    launch_pdl(wgrad_reduce_kernel, dim3(grid), dim3(kRedWarps * 32), 0, s,
               part, part_db, offsets, T, E, H, P, scale, dW, db, acc_dw, acc_db);
    return cudaGetLastError();
}

}  // namespace moe
