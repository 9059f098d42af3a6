"""Seeded synthetic inputs for the top-1 MoE gate.

This module only draws random numbers: it holds none of the gate's arithmetic, so
both the CUDA path and the CPU oracle can be fed from it.

Shapes and distributions follow the workloads of the gate described in "foxhunt
commit 11b96dac6a: Top-1 Mixture-of-Experts gate per Switch Transformer"
(ARCHITECTURE: N_EXPERTS experts, each an [H, H] linear with bias, over
[B, N_H, H] context tokens) and the expert-collapse observation of "foxhunt
commit 2d0e6b6bdc: GPU-driven lambda controller" (Motivation: one expert at ~81%
utilisation), which the skewed workload imitates.

Recipe (numpy PCG64, one seed per workload, draws in this order):
  gate_logits [T, E] ~ N(0, 1)         (T = B * N_H tokens, t = b * N_H + h)
  x           [T, H] ~ N(0, 1)
  d_out       [T, H] ~ N(0, 1)
  W           [E, H, H] ~ N(0, 1/H)    (std 1/sqrt(H); W[e][o][i], y = W x)
  bias        [E, H] ~ N(0, 0.01)      (0.01 read as the variance: std 0.1)
Workload-specific changes to the logits are listed in WORKLOADS.
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np

LAMBDA_FLOOR = 0.01
LAMBDA_MAX_EXTRA = 0.09
ENTROPY_TARGET_FRAC = 0.7


@dataclasses.dataclass(frozen=True)
class Spec:
    name: str
    B: int
    N_H: int
    E: int
    H: int
    seed: int
    logits: str = "normal"          # "normal" | "zeros" | "binary"
    skew_expert: int = -1           # expert that gets +skew_value on its logit
    skew_value: float = 0.0
    identity_weights: bool = False  # W[e] = I, bias = 0

    @property
    def T(self) -> int:
        return self.B * self.N_H


# The five gate workloads and their sub-cases.
WORKLOADS = {
    # 40 tokens: small enough for brute force.
    "tiny_b8_e4_h128": Spec("tiny_b8_e4_h128", 8, 5, 4, 128, 1001),
    # all logits 0: every softmax row is uniform, every token ties.
    "tiny_uniform_b8_e4_h128": Spec("tiny_uniform_b8_e4_h128", 8, 5, 4, 128, 1001, logits="zeros"),
    # identity experts: routed must equal x.
    "tiny_identity_b8_e4_h128": Spec("tiny_identity_b8_e4_h128", 8, 5, 4, 128, 1001,
                                     identity_weights=True),
    # 5,120 tokens.
    "small_b1024_e4_h128": Spec("small_b1024_e4_h128", 1024, 5, 4, 128, 1002),
    # 20,480 tokens, +2.0 on expert 4: about 71% of tokens pick it.
    "skewed_b4096_e8_h128": Spec("skewed_b4096_e8_h128", 4096, 5, 8, 128, 1003,
                                 skew_expert=4, skew_value=2.0),
    # 1,048,576 tokens, H = 256: the throughput workload.
    "large_b65536_e8_h256": Spec("large_b65536_e8_h256", 65536, 16, 8, 256, 1004),
    # 262,144 tokens, H = 256: the throughput workload's shape at a quarter of the
    # tokens (activations still larger than L2), for profiler captures.
    "mid_b16384_e8_h256": Spec("mid_b16384_e8_h256", 16384, 16, 8, 256, 1006),
    # 81,920 tokens with logits in {0, 1}: frequent argmax ties.
    "ties_b16384_e4_h128": Spec("ties_b16384_e4_h128", 16384, 5, 4, 128, 1005, logits="binary"),
    # the same with +10 on expert 0: every token collapses onto expert 0.
    "collapsed_b16384_e4_h128": Spec("collapsed_b16384_e4_h128", 16384, 5, 4, 128, 1005,
                                     logits="binary", skew_expert=0, skew_value=10.0),
}

THROUGHPUT_WORKLOAD = "large_b65536_e8_h256"


@dataclasses.dataclass
class Inputs:
    spec: Spec
    gate_logits: np.ndarray  # [T, E] float32
    x: np.ndarray            # [T, H] float32
    d_out: np.ndarray        # [T, H] float32
    W: np.ndarray            # [E, H, H] float32
    bias: np.ndarray         # [E, H] float32
    lambda_floor: float = LAMBDA_FLOOR
    lambda_max_extra: float = LAMBDA_MAX_EXTRA
    ent_target: float = 0.0
    ent_ema: float = 0.0


def make_spec(name: str, B: int, N_H: int, E: int, H: int, seed: int, **kw) -> Spec:
    """An ad-hoc workload (edge cases in tests: ragged token counts, E = 1, ...)."""
    return Spec(name, B, N_H, E, H, seed, **kw)


def generate(spec: Spec, with_activations: bool = True) -> Inputs:
    """Draw the inputs of one workload. Deterministic in spec.seed."""
    rng = np.random.Generator(np.random.PCG64(spec.seed))
    T, E, H = spec.T, spec.E, spec.H
    if spec.logits == "normal":
        logits = rng.standard_normal((T, E), dtype=np.float32)
    elif spec.logits == "zeros":
        rng.standard_normal((T, E), dtype=np.float32)  # keep the stream aligned
        logits = np.zeros((T, E), dtype=np.float32)
    elif spec.logits == "binary":
        logits = rng.integers(0, 2, size=(T, E)).astype(np.float32)
    else:
        raise ValueError(spec.logits)
    if spec.skew_expert >= 0:
        logits[:, spec.skew_expert] += np.float32(spec.skew_value)
    if with_activations:
        x = rng.standard_normal((T, H), dtype=np.float32)
        d_out = rng.standard_normal((T, H), dtype=np.float32)
    else:
        x = np.empty((0, H), np.float32)
        d_out = np.empty((0, H), np.float32)
        rng.standard_normal((T, H), dtype=np.float32)
        rng.standard_normal((T, H), dtype=np.float32)
    W = rng.standard_normal((E, H, H), dtype=np.float32) * np.float32(1.0 / math.sqrt(H))
    bias = rng.standard_normal((E, H), dtype=np.float32) * np.float32(0.1)
    if spec.identity_weights:
        W = np.broadcast_to(np.eye(H, dtype=np.float32), (E, H, H)).copy()
        bias = np.zeros((E, H), np.float32)
    ent_target = ENTROPY_TARGET_FRAC * math.log(E) if E > 1 else 1.0
    # The entropy EMA fed to the lambda controller: half the target, so that the
    # controller sits between its floor and its ceiling.
    ent_ema = 0.5 * ent_target
    return Inputs(spec, logits, x, d_out, W, bias, LAMBDA_FLOOR, LAMBDA_MAX_EXTRA,
                  ent_target, ent_ema)


def token_sample(inp: Inputs, n_tokens: int) -> Inputs:
    """The first n_tokens tokens of a workload (a bounded sample for CPU timing)."""
    n = min(n_tokens, inp.spec.T)
    spec = dataclasses.replace(inp.spec, name=inp.spec.name + f"_first{n}", B=n, N_H=1)
    return dataclasses.replace(inp, spec=spec, gate_logits=inp.gate_logits[:n],
                               x=inp.x[:n], d_out=inp.d_out[:n])
