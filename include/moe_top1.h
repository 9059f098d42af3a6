/*
 * moe_top1.h -- C ABI of the B200 (sm_100a) top-1 mixture-of-experts gate.
 *
 * The gate routes each of T = B * N_H context tokens to the expert whose gate
 * logit is largest and applies that expert's [H, H] linear with bias; its
 * backward sends gradients through the selected expert only; a load-balance
 * auxiliary loss, scaled by an adaptive lambda, gives the gate its gradient.
 *
 * Sources (page title, section):
 *   [P1] foxhunt commit 11b96dac6a, "Top-1 Mixture-of-Experts gate per Switch
 *        Transformer": kernel list, ARCHITECTURE, PERFORMANCE.
 *   [P2] foxhunt commit 2d0e6b6bdc, "Replace static moe_lambda=0.01 with a
 *        GPU-driven controller": formula, Wiring.
 *   [P3] foxhunt commit b23f8f2efa, "Local L40S profile": reduce_axis0 and
 *        Discipline (block tree-reduce, no atomicAdd).
 *   [P5] foxhunt commit 9170d24fe3, "Single source of truth for the attention
 *        path": MHA additions (d_ctx must not alias other gradients),
 *        PerceptionTrainer integration (capture-safe zero_grads at step start).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * Layout.  All tensors are dense, row-major, fp32 unless stated. Token t of
 *   sample b and horizon h is row t = b * N_H + h. gate_logits [T, E];
 *   x, d_out, routed, d_x [T, H]; W [E, H, H] with W[e][o][i] (row o = output
 *   channel, column i = input channel, so y = W x); bias, db [E, H];
 *   dW [E, H, H] like W.
 * Pointers.  Every tensor pointer is a DEVICE pointer owned by the caller; the
 *   library never allocates, frees or copies to the host, and never
 *   synchronises (except moe_top1_device_flags). Float tensors must be 16-byte
 *   aligned. `stream` is a cudaStream_t (NULL = legacy default stream); all work
 *   is enqueued on it in order, so the calls can be captured in a CUDA graph.
 * Workspace.  `workspace` is caller-owned device memory of at least
 *   moe_top1_workspace_bytes(T, E, H) bytes, 256-byte aligned, initialised once
 *   with moe_top1_workspace_init. Calls that share a workspace must be ordered
 *   on one stream.
 * Shapes.  1 <= E <= 32; 0 <= T < 2^31 - 256; H a multiple of 32 with
 *   32 <= H <= 256 for MOE_MATH_FFMA, H = 128 or 256 for MOE_MATH_TF32.
 * Errors.  Arguments are validated on the host before anything is launched; a
 *   bad argument returns a status and enqueues nothing. A launch error returns
 *   MOE_ERR_CUDA. A kernel that gives up on a bounded wait records a bit in the
 *   workspace flag word (read with moe_top1_device_flags) instead of hanging.
 * Determinism.  For the same inputs, math mode and device every output is
 *   bitwise identical from run to run: reductions use fixed-order trees and no
 *   floating-point atomics ([P3] Discipline).
 */
#ifndef MOE_TOP1_H
#define MOE_TOP1_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* 1: routing, forward, backward, aux loss, lambda update.
 * 2: adds moe_usage_entropy_ema_update and moe_top1_bwd_mean_collapse (every
 *    version-1 call is unchanged).
 * 3: adds moe_top1_fwd_mean_collapse (every earlier call is unchanged).
 * 4: adds moe_top1_check_routing and MOE_FLAG_BAD_ROUTING (every earlier call is
 *    unchanged).
 * 5: adds the MOE_BWD_SINGLE_PASS flag of the backward calls; moe_top1_bwd with
 *    TF32 and every output requested takes two contraction passes by default
 *    (results within fp32 rounding of version 4's single pass).
 * 6: the TF32 backward takes the single pass by default at H = 128 above 65,536
 *    tokens; the weight-gradient ranges hold 128 tokens or more (256 before), so
 *    dW / db below 18,944 tokens sum in another fixed order; adds moe_aux_loss_fwd_bwd_lambda_update (the aux loss and the lambda update
 *    in one launch); the aux loss's per-block sums of p cover 256 tokens up to
 *    131,072 tokens (mean_p within fp32 rounding of version 5 there). */
#define MOE_TOP1_ABI_VERSION 6

typedef enum {
    MOE_OK = 0,
    MOE_ERR_INVALID_ARG = 1,       /* null pointer where one is required, negative size, bad scalar */
    MOE_ERR_UNSUPPORTED_SHAPE = 2, /* E, H or T outside the supported range */
    MOE_ERR_MISALIGNED = 3,        /* a float tensor or the workspace is not aligned */
    MOE_ERR_ALIAS = 4,             /* an output overlaps another output or an input */
    MOE_ERR_WORKSPACE = 5,         /* workspace missing or smaller than required */
    MOE_ERR_CUDA = 6,              /* a CUDA runtime call or launch failed */
    MOE_ERR_DEVICE_CHECK = 7       /* (moe_top1_device_flags) a kernel recorded a failure */
} moe_status_t;

typedef enum {
    MOE_MATH_TF32 = 0, /* tcgen05 tensor cores, TF32 inputs, FP32 accumulation */
    MOE_MATH_FFMA = 1  /* FP32 fused multiply-add on the CUDA cores */
} moe_math_t;

/* Bits of the device flag word. */
#define MOE_FLAG_WAIT_TIMEOUT 0x1u  /* a pipeline wait ran past its bound */
#define MOE_FLAG_BAD_ROUTING  0x2u  /* moe_top1_check_routing found a malformed routing */

/* Routing result: caller-owned device buffers. The forward, backward and aux
 * entry points take a routing as an input and trust it: it must be what
 * moe_top1_route (or moe_top1_route_noalloc) wrote for the same tokens. The
 * contraction kernels index activations with offsets and perm without checking
 * them again (a check per token costs about 5 % of their time), so a routing
 * from anywhere else -- an uninitialised buffer, another batch -- can make them
 * read and write outside the arrays. A caller that builds or receives a routing
 * some other way checks it first with moe_top1_check_routing. */
typedef struct {
    int32_t* expert_idx; /* [T]     selected expert of each token */
    int32_t* counts;     /* [E]     tokens routed to each expert */
    int32_t* offsets;    /* [E + 1] exclusive prefix sum of counts; offsets[E] = T */
    int32_t* perm;       /* [T]     tokens grouped by expert, ascending t inside a group */
} moe_routing_t;

/* Bytes of workspace that every entry point below needs for T tokens, E experts,
 * H channels (the maximum over all entry points and math modes). */
size_t moe_top1_workspace_bytes(int64_t T, int32_t E, int32_t H);

/* Clears the workspace flag word (enqueued on `stream`). */
moe_status_t moe_top1_workspace_init(void* workspace, size_t workspace_bytes, void* stream);

/*
 * Routing. [P1] kernel list (the forward picks one expert per token from the
 * gate logits) and PERFORMANCE (one thread per block makes that choice): the
 * expert of token t is the argmax over e of gate_logits[t, e]; on a tie the lowest index wins (the
 * result of a scan from e = 0 that moves only on a strictly greater value, so a
 * NaN at e = 0 selects expert 0 and a NaN elsewhere is never selected).
 * Also writes counts, offsets and the stable permutation perm (the r-th token
 * of expert e, in ascending t, is perm[offsets[e] + r]). Integer results are
 * exact. Needs the workspace.
 */
moe_status_t moe_top1_route(const float* gate_logits, int64_t B, int64_t N_H, int32_t E,
                            const moe_routing_t* out, void* workspace, size_t workspace_bytes,
                            void* stream);

/*
 * Routing without a workspace. The pages have no counterpart: this entry point
 * exists for callers that cannot allocate device memory -- a plug-in whose host
 * framework hands it only input and output tensors and owns every byte of
 * device memory, or a runtime that plans all of its device memory up front and
 * allows no allocation while it runs. Same arguments (minus the workspace),
 * outputs and exact results as moe_top1_route; the per-block scratch of the
 * routing kernels lives in a fixed device array inside the library instead:
 * 512 KiB on every GPU that loads the library, held until the process exits.
 * Limits: T = B * N_H <= MOE_NOALLOC_MAX_TOKENS and E <= 32; a larger call
 * returns MOE_ERR_UNSUPPORTED_SHAPE and launches nothing.
 * Every call looks up the array's address in the CUDA context current on the
 * calling thread (cudaGetSymbolAddress: a host-side lookup that allocates
 * nothing) and uses that context's copy of the array, so a context created
 * after a cudaDeviceReset, or a non-primary context a host makes current, gets
 * its own copy. The first call in a context may make the runtime load the
 * library's device code into it; make that first call before any stream capture.
 * All calls share the one array: calls that can run on the GPU at the same time
 * (other streams, other host threads) race on it, so the caller must order them.
 * The array keeps the last call's contents; the kernels overwrite every entry
 * they read, so nothing needs clearing between calls. Allocates nothing (no
 * cudaMalloc, cudaFree or allocating library call).
 */
#define MOE_NOALLOC_MAX_TOKENS 2097152
moe_status_t moe_top1_route_noalloc(const float* gate_logits, int64_t B, int64_t N_H, int32_t E,
                                    const moe_routing_t* out, void* stream);

/*
 * Validation of a routing that did not come from moe_top1_route. [P5] BUG
 * CAUGHT DURING WIRING records a scratch sized for the wrong count that only
 * showed up as wrong memory traffic; the contraction kernels here trust offsets
 * and perm the same way, so a caller holding a routing from anywhere else (its
 * own sort, a file, another process) checks it once before the first
 * contraction uses it. One kernel reads the four arrays of `routing` (device
 * pointers, none NULL when T > 0; counts and offsets always), within their
 * declared sizes only, and sets MOE_FLAG_BAD_ROUTING in the workspace flag word
 * unless all of these hold:
 *   offsets[0] = 0, offsets[E] = T, offsets non-decreasing;
 *   counts[e] = offsets[e + 1] - offsets[e];
 *   every perm entry lies in [0, T), entries of one expert's segment
 *   [offsets[e], offsets[e + 1]) strictly ascend, and expert_idx[perm[k]] = e
 *   for every position k of segment e.
 * These make perm a permutation of 0..T-1 grouping the tokens by expert in
 * ascending t, with every expert index in [0, E): exactly what moe_top1_route
 * writes (whose routings always pass). The result is read with
 * moe_top1_device_flags (MOE_ERR_DEVICE_CHECK, bit MOE_FLAG_BAD_ROUTING), which
 * synchronises; the check itself is enqueued on `stream` and touches no
 * activation. Needs 256 bytes of workspace (the flag word), 256-byte aligned.
 * 0 <= T < 2^31 - 256, 1 <= E <= 32.
 */
moe_status_t moe_top1_check_routing(const moe_routing_t* routing, int64_t T, int32_t E, void* workspace,
                                    size_t workspace_bytes, void* stream);

/*
 * Forward. [P1] kernel list (the chosen expert's [H, H] linear is applied to
 * the token's context vector) and PERFORMANCE (one output channel = a dot
 * product over the H inputs):
 *   routed[t, o] = sum_i W[e*, o, i] * x[t, i] + bias[e*, o],  e* = expert_idx[t].
 * `routing` is the result of moe_top1_route on the same tokens (device
 * pointers; only offsets and perm are read). routed is overwritten and must
 * not overlap x, W or bias. MOE_MATH_TF32 rounds x and W to TF32 inside the
 * tensor core and accumulates in FP32; MOE_MATH_FFMA multiplies in FP32.
 */
moe_status_t moe_top1_fwd(const float* x, const float* W, const float* bias,
                          const moe_routing_t* routing, int64_t B, int64_t N_H, int32_t E,
                          int32_t H, moe_math_t math, float* routed, void* workspace,
                          size_t workspace_bytes, void* stream);

/*
 * Forward with the horizon mean-collapse folded in. [P5] MHA additions and the
 * horizon_mean_collapse kernel: the MoE output [B, N_H, H] is averaged over the
 * horizon axis into ctx_mean [B, H]:
 *   ctx_mean[b, o] = (1/N_H) sum_h routed[b * N_H + h, o]
 * with routed as in moe_top1_fwd, without that [T, H] array ever existing. The
 * horizon tokens of row b that chose expert e are summed first (ascending h,
 * fp32), so ctx_mean[b] = (1/N_H) (sum_e W[e] X_be + sum_e n_be bias[e]) is one
 * contraction per row with K = E * H, accumulated over the experts in a fixed
 * order (deterministic, no atomics). Reads only routing->expert_idx. ctx_mean
 * [B, H] is overwritten and must not overlap any input. 1 <= N_H <= 32 when
 * B > 0 (MOE_ERR_UNSUPPORTED_SHAPE otherwise). MOE_MATH_TF32 rounds the summed
 * rows and W to TF32 inside the tensor core; MOE_MATH_FFMA multiplies in FP32.
 * An expert index outside [0, E) contributes nothing. Same workspace rule as
 * moe_top1_fwd (TF32: the flag word).
 */
moe_status_t moe_top1_fwd_mean_collapse(const float* x, const float* W, const float* bias,
                                        const moe_routing_t* routing, int64_t B, int64_t N_H, int32_t E,
                                        int32_t H, moe_math_t math, float* ctx_mean, void* workspace,
                                        size_t workspace_bytes, void* stream);

/* Accumulate flags of moe_top1_bwd: a set bit adds the result to the output
 * buffer instead of overwriting it ([P1] kernel list calls d_fused_ctx an
 * accumulator; [P5] zeroes the gradients at step start). */
#define MOE_ACC_DX 0x1u
#define MOE_ACC_DW 0x2u
#define MOE_ACC_DB 0x4u
/* Strategy bit of the same argument. With MOE_MATH_TF32 and d_x and dW (or db)
 * requested, the backward runs either two contraction passes (d_x; then dW and
 * db) or a single pass that computes all three from one read of d_out (or
 * grad_ctx_mean) and x ([P1] kernel list: one backward produces d_fused_ctx and
 * dW / db). The single pass moves about a third less DRAM traffic. On a B200 it is
 * the faster at H = 128 above 65,536 tokens, and for the horizon-mean gradient at
 * H = 256, so both calls take it there by default and the two passes elsewhere
 * (at H = 256 the two passes are the faster for the per-token gradient). This bit
 * requests the single pass in both calls at every size. The
 * two strategies add the dW / db partial sums in different fixed orders: each is
 * bitwise reproducible, and they agree to fp32 rounding. Ignored for FFMA. */
#define MOE_BWD_SINGLE_PASS 0x100u

/*
 * Backward (straight-through). [P1] kernel list (gradients flow only through
 * the selected expert's weights and bias; the other experts receive nothing)
 * and ARCHITECTURE (the top-1 choice is not differentiable, so the expert path
 * gives the gate logits no gradient):
 *   d_x[t, i]   = sum_o W[e*, o, i] * d_out[t, o]
 *   dW[e, o, i] = sum_{t : e*(t) = e} d_out[t, o] * x[t, i]
 *   db[e, o]    = sum_{t : e*(t) = e} d_out[t, o]
 * An expert with no tokens gets exactly 0 in dW and db. No gradient is written
 * for the gate logits (only the aux loss below produces one). Any of d_x, dW,
 * db may be NULL to skip it. Outputs are overwritten unless the matching
 * MOE_ACC_* bit is set. The sums over tokens are per-expert contractions
 * reduced in a fixed-order tree (replacing [P3]'s per-token scratch and
 * reduce_axis0). Outputs must not overlap each other or any input ([P5]).
 */
moe_status_t moe_top1_bwd(const float* x, const float* W, const float* d_out,
                          const moe_routing_t* routing, int64_t B, int64_t N_H, int32_t E,
                          int32_t H, moe_math_t math, float* d_x, float* dW, float* db,
                          uint32_t accumulate_flags, void* workspace, size_t workspace_bytes,
                          void* stream);

/*
 * Backward with the horizon mean-collapse folded in. [P5] MHA additions and the
 * horizon_mean_collapse kernel: the MoE output [B, N_H, H] is averaged over the
 * horizon axis into ctx_mean [B, H], so the gradient reaching token (b, h) is
 * grad_ctx_mean[b, :] / N_H. This call is moe_top1_bwd with
 *   d_out[b * N_H + h, :] = grad_ctx_mean[b, :] / N_H
 * without that [T, H] array ever existing: the contraction kernels read row b of
 * grad_ctx_mean [B, H] for every horizon token of batch row b, and the 1 / N_H
 * is applied once to each result (exact when N_H is a power of two; otherwise
 * within one rounding of the definition). Same arguments, outputs, flags,
 * workspace and errors as moe_top1_bwd; grad_ctx_mean must not overlap any
 * output. The forward half is moe_top1_fwd_mean_collapse.
 */
moe_status_t moe_top1_bwd_mean_collapse(const float* x, const float* W, const float* grad_ctx_mean,
                                        const moe_routing_t* routing, int64_t B, int64_t N_H, int32_t E,
                                        int32_t H, moe_math_t math, float* d_x, float* dW, float* db,
                                        uint32_t accumulate_flags, void* workspace, size_t workspace_bytes,
                                        void* stream);

/*
 * Load-balance auxiliary loss and its logit gradient. [P1] kernel list (a
 * softmax of the gate logits feeds a balance loss built from the usage
 * fraction, the mean probability and the expert count), ARCHITECTURE (the
 * usage fraction comes from the non-differentiable top-1 choice, so only the
 * mean probability carries gradient) and [P2] Wiring (the loss kernel reads
 * lambda from device memory):
 *   p[t, e]   = softmax_e(gate_logits[t, :])  (shifted by the row max)
 *   frac[e]   = counts[e] / T,   mean_p[e] = (1/T) sum_t p[t, e]
 *   aux_raw   = E * (sum_e counts[e] * mean_p[e]) / T
 *   d_logits[t, j] = lambda * (E / T) * p[t, j] * (frac[j] - sum_e frac[e] p[t, e])
 * with lambda = *lambda_eff (device scalar). Writes loss_out[0] = aux_raw,
 * loss_out[1] = lambda * aux_raw, mean_p [E], d_logits [T, E] (overwritten;
 * may be NULL) and, if stats is not NULL, stats [3E + 4] = frac[E], mean_p[E],
 * counts[E] (as float), aux_raw, lambda, H(frac), H(mean_p) where
 * H(q) = -sum q ln q (0 ln 0 = 0). T = 0 gives zeros everywhere. counts must be
 * the routing of the same tokens. Needs the workspace; gate_logits, counts and
 * lambda_eff must not lie inside it (the kernel writes it while they are read:
 * MOE_ERR_ALIAS).
 */
moe_status_t moe_aux_loss_fwd_bwd(const float* gate_logits, const int32_t* counts, int64_t B,
                                  int64_t N_H, int32_t E, const float* lambda_eff,
                                  float* d_logits, float* loss_out, float* mean_p, float* stats,
                                  void* workspace, size_t workspace_bytes, void* stream);

/*
 * moe_aux_loss_fwd_bwd and then moe_lambda_eff_update in one launch (the order of
 * a training step: this step's loss uses the current weight, the controller then
 * sets the next one). Every output of moe_aux_loss_fwd_bwd is computed with
 * lambda = *lambda_eff as it was when the call began; then
 *   *lambda_next = lambda_floor + lambda_max_extra * max(0, ent_target - *ent_ema) / ent_target
 * is written by the block that finishes last, after every block has read
 * lambda_eff. lambda_next may be lambda_eff (the weight for the next step replaces
 * this step's) or ent_ema, and must not overlap any other output; ent_ema must not
 * lie inside the workspace. Arguments,
 * requirements and errors are those of the two calls; every bit of every output
 * is the same as theirs.
 */
moe_status_t moe_aux_loss_fwd_bwd_lambda_update(const float* gate_logits, const int32_t* counts, int64_t B,
                                                int64_t N_H, int32_t E, const float* lambda_eff,
                                                float* d_logits, float* loss_out, float* mean_p, float* stats,
                                                const float* ent_ema, float lambda_floor,
                                                float lambda_max_extra, float ent_target, float* lambda_next,
                                                void* workspace, size_t workspace_bytes, void* stream);

/*
 * Adaptive load-balance weight. [P2] opening paragraph:
 *   lambda_eff = lambda_floor + lambda_max_extra * max(0, ent_target - ent_ema) / ent_target
 * ent_ema and lambda_eff are device scalars (lambda_eff may equal ent_ema's
 * buffer only if the caller no longer needs ent_ema); a NaN ent_ema gives the
 * floor. ent_target must be finite and > 0 ([P2] uses 0.7 * ln E); the
 * floor and the extra must be finite and >= 0.
 */
moe_status_t moe_lambda_eff_update(const float* ent_ema, float lambda_floor,
                                   float lambda_max_extra, float ent_target, float* lambda_eff,
                                   void* stream);

/*
 * Producer of the gate-entropy signal ent_ema that moe_lambda_eff_update reads.
 * [P2] opening paragraph (ent_ema comes from an existing producer) and Wiring
 * (the constructor puts 1/K in every per-expert usage slot and ln K in the
 * entropy slot; lambda returns to its floor at a fold boundary). The pages name
 * neither the entropy's input nor the averaging weight; this call uses the
 * entropy of the step's argmax usage fractions and a caller-set weight:
 *   frac[e] = counts[e] / T,   H = -sum_e frac[e] ln frac[e]   (0 ln 0 = 0)
 *   usage_ema[e] <- (1 - alpha) usage_ema[e] + alpha frac[e]
 *   ent_ema      <- (1 - alpha) ent_ema      + alpha H
 * reset != 0 writes the cold-start state instead: usage_ema[e] = 1/E,
 * ent_ema = ln E (so the next lambda is the floor). T = 0 leaves the state as it
 * is (no observation). counts [E] int32 (the routing's counts), usage_ema [E]
 * and ent_ema (device scalar) float, read and written in place; ent_step
 * (device scalar) receives H, or NULL. alpha in [0, 1]; 1 <= E <= 32; outputs
 * must not overlap each other or counts. Computed in double, stored as float;
 * one warp, deterministic. No workspace.
 */
moe_status_t moe_usage_entropy_ema_update(const int32_t* counts, int64_t T, int32_t E, float alpha,
                                          int32_t reset, float* usage_ema, float* ent_ema, float* ent_step,
                                          void* stream);

/* Diagnostic (no counterpart on the pages): launches one thread that waits on
 * a barrier nothing arrives on, through the same bounded wait as the tensor-core
 * kernels, with a limit of limit_cycles SM clock cycles (1 .. 4e9). The wait
 * gives up, sets MOE_FLAG_WAIT_TIMEOUT in the workspace flag word and the
 * kernel returns; no fault, the context stays usable. Lets a test check the
 * failure path end to end: afterwards moe_top1_device_flags reports the bit. */
moe_status_t moe_top1_selftest_wait_timeout(void* workspace, size_t workspace_bytes, int64_t limit_cycles,
                                            void* stream);

/* Synchronises `stream`, returns the workspace flag word in *flags_out and
 * clears it. MOE_ERR_DEVICE_CHECK if any bit was set. (Debug / tests.) */
moe_status_t moe_top1_device_flags(void* workspace, size_t workspace_bytes, void* stream,
                                   uint32_t* flags_out);

/* Human-readable name of a status. Never NULL. */
const char* moe_status_string(moe_status_t status);

/* MOE_TOP1_ABI_VERSION of the built library. */
int32_t moe_top1_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* MOE_TOP1_H */
