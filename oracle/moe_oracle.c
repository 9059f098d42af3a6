/*
 * moe_oracle.c -- plain, slow, CPU oracle of the top-1 (Switch-style) MoE gate.
 *
 * TEST INFRASTRUCTURE ONLY. Only the tests, the smoke check and the CPU-baseline
 * leg of the benchmark may load this file. The product path (the CUDA library
 * and its Python binding) never calls it, and it includes nothing of theirs.
 *
 * Every floating-point result is accumulated in double and returned in double,
 * so a caller sees the exact sum of the fp32 products up to fp64 rounding.
 * Loops follow the definitions in their plainest order; nothing is blocked,
 * fused or reordered.
 *
 * Sources (page title, section):
 *   [P1] foxhunt commit 11b96dac6a, "Top-1 Mixture-of-Experts gate per Switch
 *        Transformer": kernel list, ARCHITECTURE, PERFORMANCE.
 *   [P2] foxhunt commit 2d0e6b6bdc, "Replace static moe_lambda=0.01 with a
 *        GPU-driven controller": the lambda_eff formula and its unit test; the
 *        constructor bootstrap and fold-boundary reset of the controller state.
 *   [P4] foxhunt commit 6cfd7e6691, "Per-(batch, horizon) softmax + cross-entropy
 *        loss + gradient": Kernel section (numerically stable softmax).
 *
 * Pinned by tests/test_oracle_pins.py; see the header comment of each function.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------------- */
/* TF32 input rounding.                                                       */
/*                                                                           */
/* The pages never mention TF32. A TF32 value is an fp32 bit pattern whose    */
/* low 13 mantissa bits are zero (1 sign, 8 exponent, 10 mantissa bits).      */
/* mode 0: no rounding (plain fp32)                                           */
/* mode 1: round toward zero (drop the 13 low bits)                           */
/* mode 2: round to nearest, ties away from zero                              */
/* mode 3: round to nearest, ties to even                                     */
/* Inf and NaN pass through unchanged.                                        */
/* ------------------------------------------------------------------------- */
float oracle_tf32_round(float v, int32_t mode)
{
    uint32_t u;
    memcpy(&u, &v, 4);
    if (((u >> 23) & 0xFFu) == 0xFFu || mode == 0) return v;
    if (mode == 2) {
        u += 0x1000u;
    } else if (mode == 3) {
        u += 0x0FFFu + ((u >> 13) & 1u);
    }
    u &= 0xFFFFE000u;
    memcpy(&v, &u, 4);
    return v;
}

static double tf(float v, int32_t mode) { return (double)oracle_tf32_round(v, mode); }

/* ------------------------------------------------------------------------- */
/* Routing. [P1] kernel list and PERFORMANCE: the top-1 expert is the argmax  */
/* of the token's gate logits, picked by one thread that scans the logits.    */
/* A sequential scan from e = 0 with a strict '>' keeps the lowest index on a */
/* tie. counts[e] = number of tokens routed to e; offsets = exclusive prefix  */
/* sum of counts (E + 1 entries); perm lists the tokens of expert 0 in        */
/* ascending t, then those of expert 1, and so on (a stable counting sort).   */
/* ------------------------------------------------------------------------- */
void oracle_route(const float* logits, int64_t T, int32_t E, int32_t* expert_idx,
                  int32_t* counts, int32_t* offsets, int32_t* perm)
{
    for (int64_t t = 0; t < T; ++t) {
        float best = logits[t * E];
        int32_t k = 0;
        for (int32_t e = 1; e < E; ++e) {
            if (logits[t * E + e] > best) {
                best = logits[t * E + e];
                k = e;
            }
        }
        expert_idx[t] = k;
    }
    for (int32_t e = 0; e < E; ++e) counts[e] = 0;
    for (int64_t t = 0; t < T; ++t) counts[expert_idx[t]] += 1;
    offsets[0] = 0;
    for (int32_t e = 0; e < E; ++e) offsets[e + 1] = offsets[e] + counts[e];
    int32_t* next = (int32_t*)malloc(sizeof(int32_t) * (size_t)(E > 0 ? E : 1));
    for (int32_t e = 0; e < E; ++e) next[e] = offsets[e];
    for (int64_t t = 0; t < T; ++t) {
        int32_t e = expert_idx[t];
        perm[next[e]] = (int32_t)t;
        next[e] += 1;
    }
    free(next);
}

/* ------------------------------------------------------------------------- */
/* Forward. [P1] kernel list, ARCHITECTURE and PERFORMANCE: each expert is an */
/* [H, H] linear with bias; one output channel o is the dot product of row o  */
/* of the selected expert's W with the token's input:                         */
/*   routed[t, o] = sum_i W[e*, o, i] * x[t, i] + bias[e*, o].                */
/* tf32_mode rounds x and W (not bias) before multiplying.                    */
/* ------------------------------------------------------------------------- */
void oracle_fwd(const float* x, const float* W, const float* bias, const int32_t* expert_idx,
                int64_t T, int32_t E, int32_t H, int32_t tf32_mode, double* routed)
{
    (void)E;
    for (int64_t t = 0; t < T; ++t) {
        const int32_t e = expert_idx[t];
        const float* We = W + (int64_t)e * H * H;
        for (int32_t o = 0; o < H; ++o) {
            double acc = 0.0;
            for (int32_t i = 0; i < H; ++i)
                acc += tf(We[(int64_t)o * H + i], tf32_mode) * tf(x[t * H + i], tf32_mode);
            routed[t * H + o] = acc + (double)bias[(int64_t)e * H + o];
        }
    }
}

/* ------------------------------------------------------------------------- */
/* Forward followed by the horizon mean. [P5] MHA additions: the gate's      */
/* output [B, N_H, H] is averaged over the horizon axis into ctx_mean [B, H]: */
/*   ctx_mean[b, o] = (1/N_H) sum_h routed[b*N_H + h, o],                     */
/* routed being the forward above (exact products, no TF32 rounding), the    */
/* horizon tokens visited in ascending h. Also returns the size of the terms,*/
/*   mag[b, o] = (1/N_H) sum_h (sum_i |W[e,o,i] x[t,i]| + |bias[e,o]|),       */
/* which bounds what rounding the inputs or the partial sums can change.     */
/* ------------------------------------------------------------------------- */
void oracle_fwd_mean_collapse(const float* x, const float* W, const float* bias, const int32_t* expert_idx,
                              int64_t B, int32_t N_H, int32_t E, int32_t H, double* ctx_mean, double* mag)
{
    (void)E;
    for (int64_t b = 0; b < B; ++b) {
        for (int32_t o = 0; o < H; ++o) {
            double sum = 0.0, size = 0.0;
            for (int32_t h = 0; h < N_H; ++h) {
                const int64_t t = b * N_H + h;
                const int32_t e_t = expert_idx[t];
                const float* w_row = W + ((int64_t)e_t * H + o) * H;
                double acc = 0.0, acc_abs = 0.0;
                for (int32_t i = 0; i < H; ++i) {
                    const double term = (double)w_row[i] * (double)x[t * H + i];
                    acc += term;
                    acc_abs += fabs(term);
                }
                const double b_o = (double)bias[(int64_t)e_t * H + o];
                sum += acc + b_o;
                size += acc_abs + fabs(b_o);
            }
            ctx_mean[b * H + o] = sum / (double)N_H;
            if (mag) mag[b * H + o] = size / (double)N_H;
        }
    }
}

/* ------------------------------------------------------------------------- */
/* The same horizon mean, written as a contraction over summed inputs, with  */
/* the contraction's operands rounded like a TF32 tensor core rounds them.   */
/* The forward is linear in x, so the horizon tokens of row b that chose     */
/* expert e can be summed before the expert's matrix is applied:              */
/*   ctx_mean[b, o] = (1/N_H) sum_e (sum_i W[e, o, i] X_be[i] + n_be bias[e, o])*/
/*   X_be = sum_{h : e*(b*N_H + h) = e} x[b*N_H + h],  n_be = that count.     */
/* Reading for the TF32 mode: X_be is formed in fp32, adding the horizon      */
/* tokens in ascending h, and then X_be and W are the operands that           */
/* tf32_mode rounds (bias and the counts are not rounded). Products are      */
/* exact in double and every other sum is in double. An expert index outside */
/* [0, E) contributes nothing.                                                */
/* ------------------------------------------------------------------------- */
void oracle_fwd_mean_collapse_presum(const float* x, const float* W, const float* bias, const int32_t* expert_idx,
                                     int64_t B, int32_t N_H, int32_t E, int32_t H, int32_t tf32_mode,
                                     double* ctx_mean)
{
    float* X = (float*)malloc(sizeof(float) * (size_t)H);
    double* acc = (double*)malloc(sizeof(double) * (size_t)H);
    for (int64_t b = 0; b < B; ++b) {
        for (int32_t o = 0; o < H; ++o) acc[o] = 0.0;
        for (int32_t e = 0; e < E; ++e) {
            int32_t n_be = 0;
            for (int32_t h = 0; h < N_H; ++h) {
                const int64_t t = b * N_H + h;
                if (expert_idx[t] != e) continue;
                for (int32_t i = 0; i < H; ++i) X[i] = (n_be == 0) ? x[t * H + i] : X[i] + x[t * H + i];
                ++n_be;
            }
            if (n_be == 0) continue;
            for (int32_t o = 0; o < H; ++o) {
                const float* w_row = W + ((int64_t)e * H + o) * H;
                double dot = 0.0;
                for (int32_t i = 0; i < H; ++i) dot += tf(w_row[i], tf32_mode) * tf(X[i], tf32_mode);
                acc[o] += dot + (double)n_be * (double)bias[(int64_t)e * H + o];
            }
        }
        for (int32_t o = 0; o < H; ++o) ctx_mean[b * H + o] = acc[o] / (double)N_H;
    }
    free(X);
    free(acc);
}

/* ------------------------------------------------------------------------- */
/* Backward, input gradient. [P1] kernel list and PERFORMANCE: the chain rule */
/* runs through the selected expert only, and the weight column lines up     */
/* with the input index:  d_x[t, i] = sum_o W[e*, o, i] * d_out[t, o].        */
/* ------------------------------------------------------------------------- */
void oracle_bwd_dx(const float* W, const float* d_out, const int32_t* expert_idx,
                   int64_t T, int32_t E, int32_t H, int32_t tf32_mode, double* d_x)
{
    (void)E;
    for (int64_t t = 0; t < T; ++t) {
        const int32_t e = expert_idx[t];
        const float* We = W + (int64_t)e * H * H;
        for (int32_t i = 0; i < H; ++i) {
            double acc = 0.0;
            for (int32_t o = 0; o < H; ++o)
                acc += tf(We[(int64_t)o * H + i], tf32_mode) * tf(d_out[t * H + o], tf32_mode);
            d_x[t * H + i] = acc;
        }
    }
}

/* ------------------------------------------------------------------------- */
/* Backward, weight and bias gradients. [P1] kernel list: only the selected  */
/* expert of a token receives gradient from it; the others receive nothing:  */
/*   dW[e, o, i] = sum_{t : e*(t) = e} d_out[t, o] * x[t, i]                  */
/*   db[e, o]    = sum_{t : e*(t) = e} d_out[t, o].                           */
/* Tokens are visited in ascending t. An expert with no tokens gets exactly 0.*/
/* Also returns the magnitude scale of each sum, the root of the sum of the   */
/* squared terms (dW_scale, db_scale), used to judge fp32 cancellation.       */
/* tf32_mode rounds d_out and x in dW (db is a plain sum, never rounded).     */
/* ------------------------------------------------------------------------- */
void oracle_bwd_dw(const float* x, const float* d_out, const int32_t* expert_idx,
                   int64_t T, int32_t E, int32_t H, int32_t tf32_mode,
                   double* dW, double* db, double* dW_scale, double* db_scale)
{
    const int64_t HH = (int64_t)H * H;
    memset(dW, 0, sizeof(double) * (size_t)(E * HH));
    memset(db, 0, sizeof(double) * (size_t)(E * H));
    if (dW_scale) memset(dW_scale, 0, sizeof(double) * (size_t)(E * HH));
    if (db_scale) memset(db_scale, 0, sizeof(double) * (size_t)(E * H));
    for (int64_t t = 0; t < T; ++t) {
        const int32_t e = expert_idx[t];
        for (int32_t o = 0; o < H; ++o) {
            const double g = (double)d_out[t * H + o];
            const double gt = tf(d_out[t * H + o], tf32_mode);
            db[(int64_t)e * H + o] += g;
            if (db_scale) db_scale[(int64_t)e * H + o] += g * g;
            double* row = dW + (int64_t)e * HH + (int64_t)o * H;
            double* srow = dW_scale ? dW_scale + (int64_t)e * HH + (int64_t)o * H : NULL;
            for (int32_t i = 0; i < H; ++i) {
                const double term = gt * tf(x[t * H + i], tf32_mode);
                row[i] += term;
                if (srow) srow[i] += term * term;
            }
        }
    }
    if (dW_scale)
        for (int64_t k = 0; k < E * HH; ++k) dW_scale[k] = sqrt(dW_scale[k]);
    if (db_scale)
        for (int64_t k = 0; k < (int64_t)E * H; ++k) db_scale[k] = sqrt(db_scale[k]);
}

/* db alone (the second sum above), for full-size workloads.                  */
void oracle_bwd_db(const float* d_out, const int32_t* expert_idx, int64_t T, int32_t E, int32_t H,
                   double* db, double* db_scale)
{
    memset(db, 0, sizeof(double) * (size_t)(E * H));
    memset(db_scale, 0, sizeof(double) * (size_t)(E * H));
    for (int64_t t = 0; t < T; ++t) {
        const int32_t e = expert_idx[t];
        for (int32_t o = 0; o < H; ++o) {
            const double g = (double)d_out[t * H + o];
            db[(int64_t)e * H + o] += g;
            db_scale[(int64_t)e * H + o] += g * g;
        }
    }
    for (int64_t k = 0; k < (int64_t)E * H; ++k) db_scale[k] = sqrt(db_scale[k]);
}

/* The same sums for a list of n single entries (e, o, i) -- for full-size     */
/* workloads, where the whole dW is too slow on one core.                      */
void oracle_bwd_dw_entries(const float* x, const float* d_out, const int32_t* expert_idx,
                           int64_t T, int32_t H, int32_t tf32_mode, int64_t n,
                           const int32_t* e_list, const int32_t* o_list, const int32_t* i_list,
                           double* dW, double* dW_scale)
{
    for (int64_t k = 0; k < n; ++k) {
        double acc = 0.0, sq = 0.0;
        for (int64_t t = 0; t < T; ++t) {
            if (expert_idx[t] != e_list[k]) continue;
            const double term = tf(d_out[t * H + o_list[k]], tf32_mode) *
                                tf(x[t * H + i_list[k]], tf32_mode);
            acc += term;
            sq += term * term;
        }
        dW[k] = acc;
        dW_scale[k] = sqrt(sq);
    }
}

/* ------------------------------------------------------------------------- */
/* Load-balance auxiliary loss and its logit gradient.                        */
/* [P1] kernel list: softmax of gate_logits, aux = frac . prob_mean x N_E.    */
/* [P1] ARCHITECTURE: the gate gets no gradient from the expert path (STE);   */
/*      the aux loss is its only differentiable signal, so frac (a count of   */
/*      argmax results) is a constant and only prob_mean is differentiated.   */
/* [P2] Wiring: the loss kernel reads lambda from device memory; the loss is  */
/*      lambda_eff * aux.                                                      */
/* [P4] Kernel: softmax shifted by the row max, exponentiated, divided by the */
/*      row sum.                                                               */
/*   p[t, e]   = exp(l[t, e] - max_e l[t, e]) / sum_e exp(...)                 */
/*   frac[e]   = counts[e] / T                                                 */
/*   mean_p[e] = (1/T) sum_t p[t, e]                                           */
/*   aux       = E * (sum_e counts[e] * mean_p[e]) / T  (= E sum_e frac mean_p)*/
/*   loss      = lambda_eff * aux                                              */
/*   d_logits[t, j] = lambda_eff * (E/T) * p[t, j]                            */
/*                    * (frac[j] - sum_e frac[e] p[t, e])                     */
/* d_logits_unscaled holds d_logits / (lambda_eff * E / T).                    */
/* T = 0: every output is 0.                                                   */
/* ------------------------------------------------------------------------- */
void oracle_aux(const float* logits, const int32_t* counts, int64_t T, int32_t E,
                float lambda_eff, double* mean_p, double* aux_raw, double* loss,
                double* d_logits, double* d_logits_unscaled)
{
    double* p = (double*)malloc(sizeof(double) * (size_t)(E > 0 ? E : 1));
    double* frac = (double*)malloc(sizeof(double) * (size_t)(E > 0 ? E : 1));
    for (int32_t e = 0; e < E; ++e) {
        mean_p[e] = 0.0;
        frac[e] = T > 0 ? (double)counts[e] / (double)T : 0.0;
    }
    const double lam = (double)lambda_eff;
    const double scale = T > 0 ? lam * (double)E / (double)T : 0.0;
    for (int64_t t = 0; t < T; ++t) {
        double m = (double)logits[t * E];
        for (int32_t e = 1; e < E; ++e)
            if ((double)logits[t * E + e] > m) m = (double)logits[t * E + e];
        double s = 0.0;
        for (int32_t e = 0; e < E; ++e) {
            p[e] = exp((double)logits[t * E + e] - m);
            s += p[e];
        }
        for (int32_t e = 0; e < E; ++e) p[e] /= s;
        double g = 0.0;
        for (int32_t e = 0; e < E; ++e) g += frac[e] * p[e];
        for (int32_t e = 0; e < E; ++e) {
            mean_p[e] += p[e];
            const double u = p[e] * (frac[e] - g);
            if (d_logits_unscaled) d_logits_unscaled[t * E + e] = u;
            if (d_logits) d_logits[t * E + e] = scale * u;
        }
    }
    double acc = 0.0;
    for (int32_t e = 0; e < E; ++e) {
        mean_p[e] = T > 0 ? mean_p[e] / (double)T : 0.0;
        acc += (double)counts[e] * mean_p[e];
    }
    *aux_raw = T > 0 ? (double)E * acc / (double)T : 0.0;
    *loss = lam * *aux_raw;
    free(p);
    free(frac);
}

/* ------------------------------------------------------------------------- */
/* Adaptive load-balance weight. [P2] opening paragraph:                      */
/*   lambda_eff = floor + max_extra * max(0, target - ent_ema) / target       */
/* with target = entropy_target_frac * ln(E) (config knobs 0.01, 0.09, 0.7).  */
/* ------------------------------------------------------------------------- */
double oracle_lambda_eff(double ent_ema, double lambda_floor, double lambda_max_extra,
                         double ent_target)
{
    double deficit = ent_target - ent_ema;
    if (!(deficit > 0.0)) deficit = 0.0;
    return lambda_floor + lambda_max_extra * deficit / ent_target;
}

/* ------------------------------------------------------------------------- */
/* Producer of ent_ema, the gate-entropy signal the lambda controller reads.  */
/* [P2] opening paragraph and Wiring: ent_ema comes from an existing          */
/* producer; the constructor puts 1/K in every per-expert usage slot and ln K */
/* in the entropy slot (cold start), and the lambda slot goes back to its     */
/* floor at a fold boundary. The pages name neither the entropy's input nor   */
/* the averaging weight. Reading used: the entropy of this step's argmax      */
/* usage fractions frac_e = counts[e] / T,                                    */
/*   H = - sum_e frac_e ln frac_e          (a term with frac_e = 0 is 0),     */
/* averaged with a caller-set weight alpha of the newest step:                */
/*   usage_ema[e] <- (1 - alpha) usage_ema[e] + alpha frac_e                  */
/*   ent_ema      <- (1 - alpha) ent_ema      + alpha H                       */
/* reset != 0 writes the cold-start state instead (1/E per expert, ln E).     */
/* T == 0 is no observation: the state is left as it is and H is 0.           */
/* ------------------------------------------------------------------------- */
void oracle_usage_entropy_ema(const int32_t* counts, int64_t T, int32_t E, double alpha, int32_t reset,
                              double* usage_ema, double* ent_ema, double* ent_step)
{
    double h = 0.0;
    for (int32_t e = 0; e < E && T > 0; ++e) {
        const double f = (double)counts[e] / (double)T;
        if (f > 0.0) h -= f * log(f);
    }
    *ent_step = h;
    if (reset) {
        for (int32_t e = 0; e < E; ++e) usage_ema[e] = 1.0 / (double)E;
        *ent_ema = log((double)E);
        return;
    }
    if (T <= 0) return;
    for (int32_t e = 0; e < E; ++e)
        usage_ema[e] = (1.0 - alpha) * usage_ema[e] + alpha * ((double)counts[e] / (double)T);
    *ent_ema = (1.0 - alpha) * *ent_ema + alpha * h;
}
