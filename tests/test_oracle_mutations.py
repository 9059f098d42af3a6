"""The oracle's pins catch plausible mistakes.

Each case plants one mistake in a copy of oracle/moe_oracle.c (a flipped
comparison, a dropped term, a wrong sign, a swapped index, a transposed
operand), compiles it with gcc into a temporary library, points the oracle
wrapper at it, and runs the pin tests of test_oracle_pins.py: at least one pin
must fail for every planted mistake. Everything runs on the CPU.
"""
import ctypes
import inspect
import os
import subprocess

import pytest

import oracle
import test_oracle_pins as pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "moe_oracle.c")

# (name, exact source text, replacement)
MUTATIONS = [
    ("argmax keeps the last maximum", "if (logits[t * E + e] > best) {", "if (logits[t * E + e] >= best) {"),
    ("permutation not stable", "perm[next[e]] = (int32_t)t;",
     "perm[offsets[e + 1] - 1 - (next[e] - offsets[e])] = (int32_t)t;"),
    ("forward uses W transposed",
     "acc += tf(We[(int64_t)o * H + i], tf32_mode) * tf(x[t * H + i], tf32_mode);",
     "acc += tf(We[(int64_t)i * H + o], tf32_mode) * tf(x[t * H + i], tf32_mode);"),
    ("forward drops the bias", "routed[t * H + o] = acc + (double)bias[(int64_t)e * H + o];",
     "routed[t * H + o] = acc;"),
    ("d_x uses W untransposed",
     "acc += tf(We[(int64_t)o * H + i], tf32_mode) * tf(d_out[t * H + o], tf32_mode);",
     "acc += tf(We[(int64_t)i * H + o], tf32_mode) * tf(d_out[t * H + o], tf32_mode);"),
    ("dW pairs the wrong x channel", "const double term = gt * tf(x[t * H + i], tf32_mode);",
     "const double term = gt * tf(x[t * H + o], tf32_mode);"),
    ("db drops the gradient", "            db[(int64_t)e * H + o] += g;\n            if (db_scale)",
     "            db[(int64_t)e * H + o] += 0.5 * g;\n            if (db_scale)"),
    ("aux gradient sign flipped", "const double u = p[e] * (frac[e] - g);", "const double u = p[e] * (g - frac[e]);"),
    ("aux without the expert count", "*aux_raw = T > 0 ? (double)E * acc / (double)T : 0.0;",
     "*aux_raw = T > 0 ? acc / (double)T : 0.0;"),
    ("mean_p not averaged", "mean_p[e] = T > 0 ? mean_p[e] / (double)T : 0.0;", "mean_p[e] = mean_p[e];"),
    ("frac from the wrong expert", "frac[e] = T > 0 ? (double)counts[e] / (double)T : 0.0;",
     "frac[e] = T > 0 ? (double)counts[0] / (double)T : 0.0;"),
    ("lambda deficit sign flipped", "double deficit = ent_target - ent_ema;", "double deficit = ent_ema - ent_target;"),
    ("lambda deficit not normalised", "return lambda_floor + lambda_max_extra * deficit / ent_target;",
     "return lambda_floor + lambda_max_extra * deficit;"),
    ("tf32 keeps all bits", "    u &= 0xFFFFE000u;", "    u &= 0xFFFFFFFFu;"),
    ("usage entropy sign flipped", "if (f > 0.0) h -= f * log(f);", "if (f > 0.0) h += f * log(f);"),
    ("entropy average weights swapped", "*ent_ema = (1.0 - alpha) * *ent_ema + alpha * h;",
     "*ent_ema = alpha * *ent_ema + (1.0 - alpha) * h;"),
    ("usage average from the wrong expert", "usage_ema[e] = (1.0 - alpha) * usage_ema[e] + alpha * ((double)counts[e] / (double)T);",
     "usage_ema[e] = (1.0 - alpha) * usage_ema[e] + alpha * ((double)counts[0] / (double)T);"),
    ("cold start entropy wrong", "*ent_ema = log((double)E);", "*ent_ema = 1.0 / (double)E;"),
    ("horizon mean not divided by N_H", "ctx_mean[b * H + o] = sum / (double)N_H;", "ctx_mean[b * H + o] = sum;"),
    ("horizon mean drops the bias", "sum += acc + b_o;", "sum += acc;"),
    ("horizon mean uses W transposed", "const double term = (double)w_row[i] * (double)x[t * H + i];",
     "const double term = (double)W[((int64_t)e_t * H + i) * H + o] * (double)x[t * H + i];"),
    ("horizon mean takes the first token's expert", "const int32_t e_t = expert_idx[t];",
     "const int32_t e_t = expert_idx[b * N_H];"),
    ("horizon mean reads token 0's input", "(double)w_row[i] * (double)x[t * H + i];",
     "(double)w_row[i] * (double)x[b * N_H * H + i];"),
    ("horizon mean magnitude keeps signs", "acc_abs += fabs(term);", "acc_abs += term;"),
    ("summed horizon mean adds each bias once per row", "acc[o] += dot + (double)n_be * (double)bias[(int64_t)e * H + o];",
     "acc[o] += dot + (double)bias[(int64_t)e * H + o];"),
    ("summed horizon mean leaves X_be unrounded", "dot += tf(w_row[i], tf32_mode) * tf(X[i], tf32_mode);",
     "dot += tf(w_row[i], tf32_mode) * (double)X[i];"),
    ("summed horizon mean keeps only the last token", "X[i] = (n_be == 0) ? x[t * H + i] : X[i] + x[t * H + i];",
     "X[i] = x[t * H + i];"),
    ("summed horizon mean not divided by N_H", "ctx_mean[b * H + o] = acc[o] / (double)N_H;",
     "ctx_mean[b * H + o] = acc[o];"),
]


def _pin_tests():
    return [f for name, f in inspect.getmembers(pins, inspect.isfunction)
            if name.startswith("test_") and not inspect.signature(f).parameters]


def _first_failing_pin(lib):
    saved = oracle._lib
    oracle._lib = lib
    try:
        for f in _pin_tests():
            try:
                f()
            except Exception:  # an assertion (or a crash of the mutated arithmetic)
                return f.__name__
        return None
    finally:
        oracle._lib = saved


def test_every_mutation_applies_to_the_source():
    src = open(SRC).read()
    for name, old, _ in MUTATIONS:
        assert src.count(old) == 1, name


@pytest.mark.parametrize("name,old,new", MUTATIONS, ids=[m[0] for m in MUTATIONS])
def test_pins_catch_planted_mistake(name, old, new, tmp_path):
    src = open(SRC).read()
    mutated = tmp_path / "moe_oracle_mutant.c"
    mutated.write_text(src.replace(old, new))
    so = tmp_path / "libmutant.so"
    subprocess.check_call(["gcc", "-O2", "-std=c99", "-fPIC", "-shared", "-o", str(so), str(mutated), "-lm"])
    caught = _first_failing_pin(oracle.configure(ctypes.CDLL(str(so))))
    assert caught is not None, f"no pin catches: {name}"


def test_unmutated_oracle_passes_every_pin():
    assert _first_failing_pin(oracle._load()) is None
