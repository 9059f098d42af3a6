// gemm_tf32_bwd.cu -- the whole backward of the expert path (d_x, dW and db) in
// one pass over d_out and x: at H = 256 on pairs of CTAs that share one tcgen05
// MMA (cta_group::2), at H = 128 on single CTAs.
//
// foxhunt commit 11b96dac6a ("Top-1 Mixture-of-Experts gate per Switch
// Transformer"), kernel list: one backward kernel produces the input gradient
// (d_fused_ctx) and the expert weight and bias gradients together:
//   d_x[t, i]   = sum_o W[e*, o, i] d_out[t, o]
//   dW[e, o, i] = sum_{t in e} d_out[t, o] x[t, i],   db[e, o] = sum_{t in e} d_out[t, o].
// Both contractions read the same d_out rows, so doing them in one kernel reads
// d_out from memory once instead of twice.
//
// Tensor memory decides the shape. At H = 256 one expert's dW is 256 x 256 fp32
// = all 512 columns of one SM's tensor memory, leaving nothing for d_x. A pair
// of CTAs (a cluster of 2 on two SMs) shares every MMA: the accumulator's rows
// are split between the two CTAs' tensor memories, so each CTA holds half of
// dW's rows (256 columns) and the d_x rows of its own 128 tokens (256 columns).
//
// Work split. The expert-sorted token list is cut into P equal ranges (cut
// again at expert boundaries), one per pair; range c of expert e gives the
// partial-sum slot c + e, which the fixed-order slot reduction adds up (no
// atomics: foxhunt commit b23f8f2efa, Discipline). A pair walks its range in
// pair-tiles of 256 tokens of one expert; CTA v owns tokens 128 v .. 128 v +
// 127 of each pair-tile. Per pair-tile the even CTA's MMA thread issues
//   d_x: M = 256 tokens x N = 256 i x K = 256 o (8 stages of 32 o), A = the
//        d_out rows of each CTA's tokens (K-major), B = W[e] read MN-major, CTA
//        v holding the columns i in [128 v, 128 v + 128);
//   dW:  M = 256 o x N = 256 i x K = the 256 tokens (8 stages of 32 tokens),
//        A = d_out with CTA v holding the rows o in [128 v, +128), B = x with
//        CTA v holding the columns i in [128 v, +128) (both MN-major).
// d_out rows therefore reach shared memory twice (one copy per operand layout:
// the tensor core takes TF32 K-major operands only with the 16-byte-granule
// swizzle and MN-major ones only with the 32-byte-granule swizzle), but from
// HBM once: the second read, by the same or the peer CTA, hits L2.
//
// Warp roles (each CTA): 0-7 drain the d_x accumulator (TMEM -> transpose in
// shared memory -> token rows); 8-9 gather the X stages' rows and 10-11 the W
// stages' rows with cp.async (each pair of warps fills the stages of its kind and
// passes the others, see the ring below); 12: the
// MMA issuer (even CTA) or the relay (odd CTA: once its stage has landed, it
// makes it visible to the tensor core and arrives on the even CTA's barrier);
// 13 loads the W[e] slab by TMA; 14-17 sum d_out over the staged tokens for db
// and drain dW into the slot at the end of an expert's run.
//
// At H = 128 a CTA's tensor memory holds all of dW (128 columns) and its d_x
// (128 columns), so the same kernel runs on single CTAs: 128-token tiles, one
// range per CTA (slot c + e as above), M = 128 MMAs, no relay, and every
// barrier arrival local.
//
// Every wait is bounded (common.cuh); a CTA that gives up records
// MOE_FLAG_WAIT_TIMEOUT, waits for its own TMA loads in flight and leaves
// through the pair's final cluster barrier, after the MMAs it issued are done.
#include <cstdint>

#include "common.cuh"
#include "internal.h"

namespace moe {
namespace {

constexpr int kHalf = 128;         // operand width each CTA holds (columns of B, rows of dW's A)
constexpr int kThreads = 576;
constexpr int kEpiWarps = 8;     // warps 0-7
constexpr int kProducer0 = 256;  // warps 8-11
constexpr int kMmaWarp = 12;
constexpr int kWLoadWarp = 13;
constexpr int kDbWarp0 = 14;     // warps 14-17
// One ring of stages, filled and consumed in the MMA's order: each tile's X
// stages (d_x: 32 o each), then its W stages (dW: 32 tokens each). A single
// ring keeps all of its slots loading whichever kind of stage comes next.
// Every role that waits on a slot's empty barrier passes every stage in order,
// the ones it does not fill included, and arrives on that stage's full (ready)
// barrier: a stage cannot be consumed before each such role has reached it, so
// no role is ever more than one phase away from a slot's current phase and the
// parity waits stay unambiguous. (A role that skipped the other kind's stages
// could reach a slot two phases on and see a stale phase as its own.)
constexpr int kStages = 6;
// full / ready arrivals: the 64 threads that gather the stage's rows (cp.async),
// the 64 threads of the other producer kind and the W-slab loader
constexpr int kFullArrivals = 64 + 64 + 1;
constexpr int kStageBytes = 32768;  // region 0 (A) and region 1 (B), 16 KiB each
constexpr int kRegion = 16384;
constexpr int kGroupBytes = 4096;   // MN-major: 32 rows x 128 bytes per 32-wide column group
constexpr int kStgBytes = kEpiWarps * 32 * 128;

struct __align__(8) Ctl {
    uint64_t full[kStages];   // even CTA: kFullArrivals + the odd CTA's relay
    uint64_t ready[kStages];  // odd CTA: kFullArrivals
    uint64_t tma[kStages];    // each CTA: its own W-slab TMA of an X stage (arrival + bytes)
    uint64_t empty[kStages];  // each CTA: the pair's MMA commit + its 4 db warps
    uint64_t dx_full;         // each CTA: MMA commit
    uint64_t dx_empty;        // even CTA: the 8 d_x drain warps of both CTAs
    uint64_t dw_full;         // each CTA: MMA commit
    uint64_t dw_empty;        // even CTA: the 4 db / dW warps of both CTAs
    uint64_t done;            // even CTA: the last commit
    uint32_t tmem_base;
    int abort;
    int off[33];
};

constexpr int kSmemBytes = 1024 + kStages * kStageBytes + kStgBytes + static_cast<int>(sizeof(Ctl));
static_assert(kSmemBytes <= 227 * 1024, "shared memory");

// The tiles of range [lo, hi) of the sorted token list, in order: expert e's
// run is [max(lo, off[e]), min(hi, off[e + 1])), cut into TILE-token tiles.
template <int TILE>
struct TileIter {
    int e, p0, s, t;
    __device__ void first(const int* off, int E, int lo, int hi) {
        e = -1;
        t = 0;
        p0 = 0;
        next_run(off, E, lo, hi);
    }
    __device__ void next_run(const int* off, int E, int lo, int hi) {
        for (++e; e < E; ++e) {
            s = max(lo, off[e]);
            t = min(hi, off[e + 1]);
            if (s < t) {
                p0 = s;
                return;
            }
        }
    }
    __device__ void next(const int* off, int E, int lo, int hi) {
        p0 += TILE;
        if (p0 >= t) next_run(off, E, lo, hi);
    }
    __device__ bool valid(int E) const { return e < E; }
    __device__ int ntok() const { return min(TILE, t - p0); }
    __device__ bool first_in_run() const { return p0 == s; }
    __device__ bool last_in_run() const { return p0 + TILE >= t; }
};

// Ring slot and phase parity of the k-th stage of the launch.
__device__ __forceinline__ int slot_of(int k) { return k % kStages; }
__device__ __forceinline__ uint32_t parity_of(int k) { return static_cast<uint32_t>((k / kStages) & 1); }

// One arrival on the even CTA's barrier `bar` (PAIR), or on this CTA's.
template <bool PAIR>
__device__ __forceinline__ void arrive_on_leader(uint64_t* bar) {
    if (PAIR)
        mbar_arrive_cluster(mapa_shared(smem_u32(bar), 0));
    else
        mbar_arrive(bar);
}

// g_src: d_out, or the [B, H] gradient of the horizon mean (COLLAPSE: token t
// reads row t / g_div and every result is scaled by out_scale).
template <int H, bool PAIR, bool COLLAPSE>
__device__ __forceinline__ void bwd_fused_body(const float* __restrict__ x, const float* __restrict__ g_src,
                                               const CUtensorMap* tm_w, const int32_t* __restrict__ offsets,
                                               const int32_t* __restrict__ perm, int T, int E, int P, int g_div,
                                               float out_scale, int acc_dx, float* __restrict__ d_x,
                                               float* __restrict__ part, float* __restrict__ part_db,
                                               uint32_t* __restrict__ dev_flags) {
    static_assert((PAIR && H == 256) || (!PAIR && H == 128), "pairs at H = 256, single CTAs at H = 128");
    constexpr int kH = H;
    constexpr int kTileTok = PAIR ? 256 : 128;   // tokens per (pair-)tile
    constexpr int kTmemCols = 2 * H;             // [0, H) d_x, [H, 2H) dW
    constexpr int kM = PAIR ? 256 : 128;         // MMA rows: tokens (d_x) or o (dW)
    using Iter = TileIter<kTileTok>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* ring = smem;
    float* stg = reinterpret_cast<float*>(smem + kStages * kStageBytes);
    Ctl* ctl = reinterpret_cast<Ctl*>(smem + kStages * kStageBytes + kStgBytes);
    constexpr int nX = kH / 32;  // X stages per tile
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t v = PAIR ? cluster_ctarank() : 0u;  // 0: the even CTA, which issues the MMAs
    const bool leader = (v == 0);
    const int c = PAIR ? static_cast<int>(cluster_id_x()) : static_cast<int>(blockIdx.x);

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&ctl->full[s], kFullArrivals + (PAIR ? 1 : 0));
            mbar_init(&ctl->ready[s], kFullArrivals);
            mbar_init(&ctl->tma[s], 1);
            mbar_init(&ctl->empty[s], 1 + 4);
        }
        mbar_init(&ctl->dx_full, 1);
        mbar_init(&ctl->dx_empty, (PAIR ? 2 : 1) * kEpiWarps);
        mbar_init(&ctl->dw_full, 1);
        mbar_init(&ctl->dw_empty, (PAIR ? 2 : 1) * 4);
        mbar_init(&ctl->done, 1);
        ctl->abort = 0;
        fence_mbar_init();
    }
    if (warp == kWLoadWarp && lane == 0) tma_prefetch_desc(tm_w);
    if (warp == kMmaWarp) {
        if (PAIR) {
            tmem_alloc_pair(&ctl->tmem_base, kTmemCols);
            tmem_relinquish_pair();
        } else {
            tmem_alloc(&ctl->tmem_base, kTmemCols);
            tmem_relinquish();
        }
    }
    griddep_wait();  // the prologue above overlaps the previous kernel; global memory from here on
    if (threadIdx.x <= E) ctl->off[threadIdx.x] = offsets[threadIdx.x];
    tc_fence_before();
    if (PAIR)
        cluster_sync_all();  // barriers initialised in both CTAs before any remote arrival
    else
        __syncthreads();
    tc_fence_after();
    const uint32_t tmem = ctl->tmem_base;
    volatile int* abort = &ctl->abort;
    const int lo = static_cast<int>(split_lo(c, T, P)), hi = static_cast<int>(split_lo(c + 1, T, P));
    const int* off = ctl->off;

    if (warp >= kProducer0 / 32 && warp < kProducer0 / 32 + 2) {
        // ---------------- X-stage producers (warps 8-9): A = the d_out rows of this
        // CTA's 128 tokens, 32 o per stage, K-major (128-byte swizzle).
        const int ptid = threadIdx.x - kProducer0;  // 0..63
        const int prow = ptid >> 3, pg = ptid & 7;  // row within an 8-row block, 16-byte granule
        int kbase = 0;  // the stage index of the tile's first X stage
        bool ok = true;
        Iter it;
        it.first(off, E, lo, hi);
        while (ok && it.valid(E)) {
            const int n = it.ntok();
            int tx[16];  // the token of rows r = j * 8 + prow
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                const int r = kHalf * static_cast<int>(v) + j * 8 + prow;
                tx[j] = (r < n) ? perm[it.p0 + r] : -1;
                if (COLLAPSE && tx[j] >= 0) tx[j] = tx[j] / g_div;  // the token's gradient row
            }
            for (int kc = 0; kc < nX && ok; ++kc) {
                const int k = kbase + kc, sl = slot_of(k);
                if (!(ok = mbar_wait(&ctl->empty[sl], parity_of(k) ^ 1, abort, dev_flags))) break;
                const uint32_t a_u32 = smem_u32(ring + sl * kStageBytes);
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    const int r = j * 8 + prow;
                    const int gr = tx[j];
                    const float* src = g_src + static_cast<int64_t>(gr < 0 ? 0 : gr) * kH + kc * 32 + pg * 4;
                    cp_async_16_l2_256(a_u32 + r * 128 + ((pg ^ (r & 7)) << 4), src, gr < 0 ? 0u : 16u);
                }
                cp_async_arrive_noinc(leader ? &ctl->full[sl] : &ctl->ready[sl]);
            }
            const int ntc = (n + 31) / 32;
            for (int tc = 0; tc < ntc && ok; ++tc) {  // pass the W stages
                const int k = kbase + nX + tc, sl = slot_of(k);
                if (!(ok = mbar_wait(&ctl->empty[sl], parity_of(k) ^ 1, abort, dev_flags))) break;
                mbar_arrive(leader ? &ctl->full[sl] : &ctl->ready[sl]);
            }
            kbase += nX + ntc;
            it.next(off, E, lo, hi);
        }
        cp_async_wait_all();  // nothing in flight into this CTA's shared memory when it leaves
    } else if (warp >= kProducer0 / 32 + 2 && warp < kProducer0 / 32 + 4) {
        // ---------------- W-stage producers (warps 10-11): 32 tokens per stage; A =
        // d_out[., o-half v], B = x[., i-half v], MN-major (32-byte granules)
        const int ptid = threadIdx.x - kProducer0 - 64;  // 0..63
        const int q16 = ptid & 7, gq = (ptid >> 3) & 3, rsub = ptid >> 5;
        int kbase = 0;  // the stage index of the tile's first X stage
        bool ok = true;
        Iter it;
        it.first(off, E, lo, hi);
        while (ok && it.valid(E)) {
            const int n = it.ntok();
            int tw[8];  // lane l: the token at position 32 tc + l of the tile
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const int q = j * 32 + lane;
                tw[j] = (q < n) ? perm[it.p0 + q] : -1;
            }
            const int ntc = (n + 31) / 32;
            for (int kc = 0; kc < nX && ok; ++kc) {  // pass the X stages
                const int k = kbase + kc, sl = slot_of(k);
                if (!(ok = mbar_wait(&ctl->empty[sl], parity_of(k) ^ 1, abort, dev_flags))) break;
                mbar_arrive(leader ? &ctl->full[sl] : &ctl->ready[sl]);
            }
            for (int tc = 0; tc < ntc && ok; ++tc) {
                const int k = kbase + nX + tc, sl = slot_of(k);
                ok = mbar_wait(&ctl->empty[sl], parity_of(k) ^ 1, abort, dev_flags);
                if (!(ok = __all_sync(0xffffffffu, ok))) break;  // the gather below shuffles across the warp
                const uint32_t a_u32 = smem_u32(ring + sl * kStageBytes);
                int tok_l = tw[0];
#pragma unroll
                for (int j = 1; j < 8; ++j)
                    if (j == tc) tok_l = tw[j];
                const int gtok_l = (COLLAPSE && tok_l >= 0) ? tok_l / g_div : tok_l;
                const int64_t col = kHalf * static_cast<int64_t>(v) + gq * 32 + q16 * 4;
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    const int r = j * 2 + rsub;
                    const int tk = __shfl_sync(0xffffffffu, tok_l, r);
                    const int gtk = __shfl_sync(0xffffffffu, gtok_l, r);
                    const uint32_t o = gq * kGroupBytes + r * 128 + ((((q16 >> 1) ^ (r & 3)) << 5) | ((q16 & 1) << 4));
                    const uint32_t nb = tk < 0 ? 0u : 16u;
                    cp_async_16(a_u32 + o, g_src + static_cast<int64_t>(tk < 0 ? 0 : gtk) * kH + col, nb);
                    cp_async_16(a_u32 + kRegion + o, x + static_cast<int64_t>(tk < 0 ? 0 : tk) * kH + col, nb);
                }
                cp_async_arrive_noinc(leader ? &ctl->full[sl] : &ctl->ready[sl]);
            }
            kbase += nX + ntc;
            it.next(off, E, lo, hi);
        }
        cp_async_wait_all();
    } else if (warp == kWLoadWarp) {
        // ---------------- W[e] slab (columns i of this CTA's half) for the X stages, by TMA
        if (lane == 0) {
            int kbase = 0;
            uint32_t tbits = 0;     // bit s: parity of slot s's next W-slab load
            uint32_t issued = 0;    // bit s: slot s has had a load
            bool ok = true;
            Iter it;
            it.first(off, E, lo, hi);
            while (ok && it.valid(E)) {
                for (int kc = 0; kc < nX && ok; ++kc) {
                    const int k = kbase + kc, sl = slot_of(k);
                    if (!(ok = mbar_wait(&ctl->empty[sl], parity_of(k) ^ 1, abort, dev_flags))) break;
                    mbar_arrive_expect_tx(&ctl->tma[sl], kRegion);
                    uint8_t* dst = ring + sl * kStageBytes + kRegion;
#pragma unroll
                    for (int g = 0; g < kHalf / 32; ++g)
                        tma_load_2d(dst + g * kGroupBytes, tm_w, kHalf * static_cast<int>(v) + g * 32,
                                    it.e * kH + kc * 32, &ctl->tma[sl]);
                    tbits ^= 1u << sl;
                    issued |= 1u << sl;
                    mbar_arrive(leader ? &ctl->full[sl] : &ctl->ready[sl]);
                }
                const int ntc = (it.ntok() + 31) / 32;
                for (int tc = 0; tc < ntc && ok; ++tc) {  // pass the W stages
                    const int k = kbase + nX + tc, sl = slot_of(k);
                    if (!(ok = mbar_wait(&ctl->empty[sl], parity_of(k) ^ 1, abort, dev_flags))) break;
                    mbar_arrive(leader ? &ctl->full[sl] : &ctl->ready[sl]);
                }
                kbase += nX + ntc;
                it.next(off, E, lo, hi);
            }
            // let this CTA's loads land before it can leave (already so unless a wait gave up)
            for (int sl = 0; sl < kStages; ++sl)
                if ((issued >> sl) & 1u)
                    mbar_wait_drain(&ctl->tma[sl], ((tbits >> sl) & 1u) ^ 1u, kWaitLimitCycles);
        }
        __syncwarp();
    } else if (warp == kMmaWarp) {
        if (leader && lane == 0) {
            // ---------------- MMA issuer: one thread of the even CTA, for both CTAs
            constexpr uint32_t idesc_dx = idesc_tf32(kM, kH, 0, 1);  // A K-major, B MN-major
            constexpr uint32_t idesc_dw = idesc_tf32(kM, kH, 1, 1);  // both MN-major
            const uint32_t tmem_dx = tmem, tmem_dw = tmem + kH;
            // completion of the MMAs issued so far -> the barrier in every CTA of the pair
            auto commit_all = [](uint64_t* bar) {
                if (PAIR)
                    mma_commit_pair_mc(bar, 0x3);
                else
                    mma_commit(bar);
            };
            int kbase = 0;
            uint32_t tbits = 0;  // bit s: parity of slot s's next W-slab load
            uint32_t dx_phase = 0, dw_phase = 0;
            bool ok = true;
            Iter it;
            it.first(off, E, lo, hi);
            while (ok && it.valid(E)) {
                // d_x of this pair-tile: the accumulator must have been drained by both CTAs
                if (!(ok = mbar_wait_cl(&ctl->dx_empty, dx_phase ^ 1, abort, dev_flags))) break;
                tc_fence_after();
                for (int kc = 0; kc < nX; ++kc) {
                    const int k = kbase + kc, sl = slot_of(k);
                    if (!(ok = mbar_wait_cl(&ctl->full[sl], parity_of(k), abort, dev_flags))) break;
                    if (!(ok = mbar_wait(&ctl->tma[sl], (tbits >> sl) & 1u, abort, dev_flags))) break;
                    tbits ^= 1u << sl;
                    fence_proxy_async_smem();
                    tc_fence_after();
                    const uint32_t a_addr = smem_u32(ring + sl * kStageBytes);
#pragma unroll
                    for (int ks = 0; ks < 4; ++ks) {
                        const uint64_t ad = sw128_desc(a_addr + ks * 32, 16, 1024);
                        const uint64_t bd = sw128_32b_mn_desc(a_addr + kRegion + ks * 1024, kGroupBytes, 512);
                        const uint32_t accumulate = (kc | ks) != 0 ? 1u : 0u;
                        if (PAIR)
                            mma_tf32_pair(tmem_dx, ad, bd, idesc_dx, accumulate);
                        else
                            mma_tf32(tmem_dx, ad, bd, idesc_dx, accumulate);
                    }
                    commit_all(&ctl->empty[sl]);
                }
                if (!ok) break;
                commit_all(&ctl->dx_full);
                dx_phase ^= 1;
                // dW of this pair-tile, accumulated over the expert's run
                if (it.first_in_run()) {
                    if (!(ok = mbar_wait_cl(&ctl->dw_empty, dw_phase ^ 1, abort, dev_flags))) break;
                    tc_fence_after();
                }
                const int ntc = (it.ntok() + 31) / 32;
                for (int tc = 0; tc < ntc; ++tc) {
                    const int k = kbase + nX + tc, sl = slot_of(k);
                    if (!(ok = mbar_wait_cl(&ctl->full[sl], parity_of(k), abort, dev_flags))) break;
                    fence_proxy_async_smem();
                    tc_fence_after();
                    const uint32_t a_addr = smem_u32(ring + sl * kStageBytes);
#pragma unroll
                    for (int ks = 0; ks < 4; ++ks) {
                        const uint64_t ad = sw128_32b_mn_desc(a_addr + ks * 1024, kGroupBytes, 512);
                        const uint64_t bd = sw128_32b_mn_desc(a_addr + kRegion + ks * 1024, kGroupBytes, 512);
                        const uint32_t accumulate = (it.first_in_run() && tc == 0 && ks == 0) ? 0u : 1u;
                        if (PAIR)
                            mma_tf32_pair(tmem_dw, ad, bd, idesc_dw, accumulate);
                        else
                            mma_tf32(tmem_dw, ad, bd, idesc_dw, accumulate);
                    }
                    commit_all(&ctl->empty[sl]);
                }
                if (!ok) break;
                if (it.last_in_run()) {
                    commit_all(&ctl->dw_full);
                    dw_phase ^= 1;
                }
                kbase += nX + ntc;
                it.next(off, E, lo, hi);
            }
            // every MMA issued (and every commit arrival on the odd CTA) is done before the pair may leave
            if (PAIR)
                mma_commit_pair(&ctl->done);
            else
                mma_commit(&ctl->done);
            mbar_wait_drain(&ctl->done, 0, kWaitLimitCycles);
        } else if (PAIR && !leader && lane == 0) {
            // ---------------- relay (odd CTA): this CTA's stage has landed -> the even CTA's barrier
            const uint32_t full0 = mapa_shared(smem_u32(&ctl->full[0]), 0);
            int kbase = 0;
            uint32_t tbits = 0;
            bool ok = true;
            Iter it;
            it.first(off, E, lo, hi);
            while (ok && it.valid(E)) {
                for (int kc = 0; kc < nX; ++kc) {
                    const int k = kbase + kc, sl = slot_of(k);
                    if (!(ok = mbar_wait(&ctl->ready[sl], parity_of(k), abort, dev_flags))) break;
                    if (!(ok = mbar_wait(&ctl->tma[sl], (tbits >> sl) & 1u, abort, dev_flags))) break;
                    tbits ^= 1u << sl;
                    fence_proxy_async_smem();
                    mbar_arrive_cluster(full0 + sl * 8);
                }
                if (!ok) break;
                const int ntc = (it.ntok() + 31) / 32;
                for (int tc = 0; tc < ntc; ++tc) {
                    const int k = kbase + nX + tc, sl = slot_of(k);
                    if (!(ok = mbar_wait(&ctl->ready[sl], parity_of(k), abort, dev_flags))) break;
                    fence_proxy_async_smem();
                    mbar_arrive_cluster(full0 + sl * 8);
                }
                kbase += nX + ntc;
                it.next(off, E, lo, hi);
            }
        }
        __syncwarp();
    } else if (warp < kEpiWarps) {
        // ---------------- d_x drain: TMEM -> registers -> shared-memory transpose -> token rows.
        // Warp w reads TMEM lanes 32 (w % 4) .. +31 (this CTA's tile rows) and the column half w / 4.
        constexpr int kCols = kH / 2;  // d_x columns this warp drains
        const int q = warp & 3;
        const int c0 = (warp >> 2) * kCols;
        const uint32_t my_u32 = smem_u32(stg + warp * 32 * 32);
        const int j = lane & 7;
        const int myrow = kHalf * static_cast<int>(v) + 32 * q + lane;  // position within the (pair-)tile
        uint32_t dx_phase = 0;
        Iter it;
        it.first(off, E, lo, hi);
        int tok_next = it.valid(E) ? ((myrow < it.ntok()) ? perm[it.p0 + myrow] : -1) : -1;
        while (it.valid(E)) {
            const int tok_mine = tok_next;
            Iter nx = it;
            nx.next(off, E, lo, hi);
            tok_next = nx.valid(E) ? ((myrow < nx.ntok()) ? perm[nx.p0 + myrow] : -1) : -1;
            if (!mbar_wait_cl(&ctl->dx_full, dx_phase, abort, dev_flags)) break;
            __syncwarp();
            tc_fence_after();
            // 32-column chunks, double-buffered: the TMEM load of chunk cc + 1 is in
            // flight while chunk cc is transposed and stored
            constexpr int NCH = kCols / 32;
            const uint32_t tbase = tmem + (static_cast<uint32_t>(32 * q) << 16) + static_cast<uint32_t>(c0);
            uint32_t buf[2][32];
            tmem_ld_32x32b_x32_async(tbase, buf[0]);
            tmem_ld_wait_tied(buf[0]);
#pragma unroll
            for (int cc = 0; cc < NCH; ++cc) {
                if (cc + 1 < NCH)
                    tmem_ld_32x32b_x32_async(tbase + static_cast<uint32_t>((cc + 1) * 32), buf[(cc + 1) & 1]);
                float vals[32];
#pragma unroll
                for (int i = 0; i < 32; ++i) vals[i] = COLLAPSE ? __uint_as_float(buf[cc & 1][i]) * out_scale
                                                                : __uint_as_float(buf[cc & 1][i]);
#pragma unroll
                for (int jj = 0; jj < 8; ++jj)
                    st_shared_v4(my_u32 + 4 * (lane * 32 + ((jj ^ (lane & 7)) * 4)), vals[4 * jj], vals[4 * jj + 1],
                                 vals[4 * jj + 2], vals[4 * jj + 3]);
                __syncwarp();
#pragma unroll
                for (int r8 = 0; r8 < 8; ++r8) {
                    const int R = r8 * 4 + (lane >> 3);
                    float4 val = ld_shared_v4(my_u32 + 4 * (R * 32 + ((j ^ (R & 7)) * 4)));
                    const int tok = __shfl_sync(0xffffffffu, tok_mine, R);
                    float* dst = d_x + static_cast<int64_t>(tok < 0 ? 0 : tok) * kH + c0 + cc * 32 + j * 4;
                    if (acc_dx) {
                        if (tok >= 0) {
                            const float4 o = *reinterpret_cast<const float4*>(dst);
                            val.x += o.x;
                            val.y += o.y;
                            val.z += o.z;
                            val.w += o.w;
                            *reinterpret_cast<float4*>(dst) = val;
                        }
                    } else {
                        st_global_cs_v4_pred(dst, val, tok >= 0);
                    }
                }
                __syncwarp();
                if (cc + 1 < NCH) tmem_ld_wait_tied(buf[(cc + 1) & 1]);
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) arrive_on_leader<PAIR>(&ctl->dx_empty);
            dx_phase ^= 1;
            it = nx;
        }
    } else if (warp >= kDbWarp0 && warp < kDbWarp0 + 4) {
        // ---------------- db over the staged d_out rows (column o = 128 v + tdb), and
        // the dW drain of TMEM lane quadrant warp % 4 at the end of each expert run
        const int tdb = threadIdx.x - kDbWarp0 * 32;  // 0..127
        const int dq = warp & 3;
        const int g = tdb >> 5, jo = tdb & 31;
        int kbase = 0;
        uint32_t dw_phase = 0;
        float db_run = 0.0f;
        bool ok = true;
        Iter it;
        it.first(off, E, lo, hi);
        while (ok && it.valid(E)) {
            // every stage of the ring passes here once (its slot is released by the MMA's
            // commit and these four warps); only the W stages hold d_out rows to sum
            const int ntc = (it.ntok() + 31) / 32;
            for (int j = 0; j < nX + ntc; ++j) {
                const int k = kbase + j, sl = slot_of(k);
                ok = leader ? mbar_wait_cl(&ctl->full[sl], parity_of(k), abort, dev_flags)
                            : mbar_wait(&ctl->ready[sl], parity_of(k), abort, dev_flags);
                if (!ok) break;
                if (j >= nX) {
                    const uint8_t* colbase = ring + sl * kStageBytes + g * kGroupBytes + (jo & 7) * 4;
                    float acc = 0.0f;
#pragma unroll 8
                    for (int rr = 0; rr < 32; ++rr)
                        acc += *reinterpret_cast<const float*>(colbase + rr * 128 + (((jo >> 3) ^ (rr & 3)) << 5));
                    db_run += acc;
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&ctl->empty[sl]);
            }
            kbase += nX + ntc;
            if (!ok) break;
            if (it.last_in_run()) {
                if (!(ok = mbar_wait_cl(&ctl->dw_full, dw_phase, abort, dev_flags))) break;
                __syncwarp();
                tc_fence_after();
                const int64_t slot = static_cast<int64_t>(c) + it.e;
                const int o = kHalf * static_cast<int>(v) + 32 * dq + lane;  // dW row of this TMEM lane
                float* prow = part + (slot * kH + o) * kH;
#pragma unroll 1
                for (int cc = 0; cc < kH / 32; ++cc) {
                    float vals[32];
                    tmem_ld_32x32b_x32(tmem + kH + (static_cast<uint32_t>(32 * dq) << 16) + static_cast<uint32_t>(cc * 32),
                                       vals);
#pragma unroll
                    for (int k4 = 0; k4 < 8; ++k4)
                        *reinterpret_cast<float4*>(prow + cc * 32 + 4 * k4) =
                            make_float4(vals[4 * k4], vals[4 * k4 + 1], vals[4 * k4 + 2], vals[4 * k4 + 3]);
                }
                part_db[slot * kH + kHalf * static_cast<int>(v) + tdb] = db_run;
                db_run = 0.0f;
                tc_fence_before();
                __syncwarp();
                if (lane == 0) arrive_on_leader<PAIR>(&ctl->dw_empty);
                dw_phase ^= 1;
            }
            it.next(off, E, lo, hi);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (PAIR) cluster_sync_all();  // no CTA leaves while the peer may still arrive on its barriers
    if (warp == kMmaWarp) {
        tc_fence_after();
        if (PAIR)
            tmem_dealloc_pair(tmem, kTmemCols);
        else
            tmem_dealloc(tmem, kTmemCols);
    }
}

#define BWD_FUSED_ARGS                                                                                           \
    const float* __restrict__ x, const float* __restrict__ g_src, const __grid_constant__ CUtensorMap tm_w,      \
        const int32_t* __restrict__ offsets, const int32_t* __restrict__ perm, int T, int E, int P, int g_div,   \
        float out_scale, int acc_dx, float* __restrict__ d_x, float* __restrict__ part,                          \
        float* __restrict__ part_db, uint32_t* __restrict__ dev_flags

template <bool COLLAPSE>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1) bwd_fused_pair_kernel(BWD_FUSED_ARGS) {
    bwd_fused_body<256, true, COLLAPSE>(x, g_src, &tm_w, offsets, perm, T, E, P, g_div, out_scale, acc_dx, d_x, part,
                                        part_db, dev_flags);
}

template <bool COLLAPSE>
__global__ void __launch_bounds__(kThreads, 1) bwd_fused_single_kernel(BWD_FUSED_ARGS) {
    bwd_fused_body<128, false, COLLAPSE>(x, g_src, &tm_w, offsets, perm, T, E, P, g_div, out_scale, acc_dx, d_x, part,
                                         part_db, dev_flags);
}

#undef BWD_FUSED_ARGS

}  // namespace

// Pairs (clusters of 2) that fit on the device at once, at most kFusedMaxPairs.
cudaError_t bwd_fused_max_pairs(int* out) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * kFusedMaxPairs, 1, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = kSmemBytes;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    const cudaError_t e = cudaOccupancyMaxActiveClusters(&n, bwd_fused_pair_kernel<false>, &cfg);
    if (e != cudaSuccess) return e;
    *out = n < 1 ? 1 : (n > kFusedMaxPairs ? kFusedMaxPairs : n);
    return cudaSuccess;
}

int bwd_fused_pairs(int64_t T, int max_pairs) {
    int64_t p = (T + 511) / 512;
    if (p < 1) p = 1;
    if (p > max_pairs) p = max_pairs;
    return static_cast<int>(p);
}

cudaError_t launch_bwd_fused_tf32(const float* x, const float* W, const float* g_src, const int32_t* offsets,
                                  const int32_t* perm, int64_t T, int E, int H, int P, int g_div, float out_scale,
                                  int acc_dx, float* d_x, float* part, float* part_db, uint32_t* dev_flags,
                                  cudaStream_t s) {
    CUtensorMap tm_w;
    if (!make_map_2d(&tm_w, W, static_cast<uint64_t>(E) * H, H, 32, 32, kMapSw128Atom32)) return cudaErrorInvalidValue;
    const bool collapse = g_div != 1 || out_scale != 1.0f;
    const int Ti = static_cast<int>(T);
    if (H == 256) {
        if (collapse)
            launch_pdl(bwd_fused_pair_kernel<true>, dim3(2 * P), dim3(kThreads), kSmemBytes, s,
                       x, g_src, tm_w, offsets, perm, Ti, E, P, g_div, out_scale, acc_dx, d_x, part, part_db, dev_flags);
        else
            launch_pdl(bwd_fused_pair_kernel<false>, dim3(2 * P), dim3(kThreads), kSmemBytes, s,
                       x, g_src, tm_w, offsets, perm, Ti, E, P, 1, 1.0f, acc_dx, d_x, part, part_db, dev_flags);
    } else {
        if (collapse)
            launch_pdl(bwd_fused_single_kernel<true>, dim3(P), dim3(kThreads), kSmemBytes, s,
                       x, g_src, tm_w, offsets, perm, Ti, E, P, g_div, out_scale, acc_dx, d_x, part, part_db, dev_flags);
        else
            launch_pdl(bwd_fused_single_kernel<false>, dim3(P), dim3(kThreads), kSmemBytes, s,
                       x, g_src, tm_w, offsets, perm, Ti, E, P, 1, 1.0f, acc_dx, d_x, part, part_db, dev_flags);
    }
    return cudaGetLastError();
}

cudaError_t bwd_fused_set_smem_limits() {
    cudaError_t e = cudaSuccess;
    const void* kernels[4] = {reinterpret_cast<const void*>(bwd_fused_pair_kernel<false>),
                              reinterpret_cast<const void*>(bwd_fused_pair_kernel<true>),
                              reinterpret_cast<const void*>(bwd_fused_single_kernel<false>),
                              reinterpret_cast<const void*>(bwd_fused_single_kernel<true>)};
    for (const void* k : kernels)
        if (e == cudaSuccess) e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    return e;
}

}  // namespace moe
