"""Shared helpers of the GPU parity tests: run the C ABI on a workload with
guard bands around every output, and compare against the CPU oracle."""
from __future__ import annotations

import numpy as np
import torch

import oracle
from bwd_route_b200 import ops

# How the tensor core turns an fp32 operand into TF32 (the pages say nothing
# about TF32). Established on the B200 by test_tf32_operand_rounding_rule: an
# identity expert returns each input with its 13 low mantissa bits cleared,
# i.e. rounded toward zero.
TF32_RULE = oracle.TF32_RZ

# Tolerances: FFMA |g - o| <= 1e-5 + 1e-5 |o|; TF32 (against the TF32-rounded
# oracle) |g - o| <= 1e-4 + 2e-3 |o|. For sums over tokens (dW, db) |o| is read
# as the magnitude of the sum, max(|o|, S), S = root-sum-of-squares of its terms.
TOL = {ops.MOE_MATH_FFMA: (1e-5, 1e-5), ops.MOE_MATH_TF32: (1e-4, 2e-3)}

SENTINEL = 0x7FBADBAD  # a NaN payload no kernel writes
PAD = 64


class Guarded:
    """A device buffer whose n elements sit between two guard bands of sentinels."""

    def __init__(self, n: int, dtype=torch.float32, shape=None):
        self.n = n
        self.buf = torch.empty(n + 2 * PAD, dtype=dtype, device="cuda")
        self.buf.view(torch.int32).fill_(SENTINEL)
        self.t = self.buf[PAD:PAD + n]
        if shape is not None:
            self.t = self.t.view(*shape)

    def guards_intact(self) -> bool:
        g = self.buf.view(torch.int32)
        return bool((g[:PAD] == SENTINEL).all() and (g[PAD + self.n:] == SENTINEL).all())

    def host(self) -> np.ndarray:
        return self.t.cpu().numpy()


def dev(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def run_gpu(inp, math: int, lam: float, parts=("route", "fwd", "bwd", "aux"), acc_flags: int = 0,
            preset: dict | None = None):
    """Runs the library on a workload; returns host arrays and the guard check."""
    s = inp.spec
    B, N_H, E, H, T = s.B, s.N_H, s.E, s.H, s.T
    out = {}
    g = {
        "expert_idx": Guarded(T, torch.int32), "counts": Guarded(E, torch.int32),
        "offsets": Guarded(E + 1, torch.int32), "perm": Guarded(T, torch.int32),
        "routed": Guarded(T * H, shape=(T, H)), "d_x": Guarded(T * H, shape=(T, H)),
        "dW": Guarded(E * H * H, shape=(E, H, H)), "db": Guarded(E * H, shape=(E, H)),
        "d_logits": Guarded(T * E, shape=(T, E)), "loss": Guarded(2), "mean_p": Guarded(E),
        "stats": Guarded(3 * E + 4),
    }
    if preset:
        for k, v in preset.items():
            g[k].t.copy_(dev(v).view_as(g[k].t))
    routing = ops.Routing(g["expert_idx"].t, g["counts"].t, g["offsets"].t, g["perm"].t)
    logits, x, d_out = dev(inp.gate_logits), dev(inp.x), dev(inp.d_out)
    W, bias = dev(inp.W), dev(inp.bias)
    lam_t = torch.tensor([lam], dtype=torch.float32, device="cuda")
    ws = ops.new_workspace(T, E, H, "cuda")
    if "route" in parts:
        ops.moe_top1_route(logits, B, N_H, E, routing, ws)
    if "fwd" in parts:
        ops.moe_top1_fwd(x, W, bias, routing, B, N_H, E, H, math, g["routed"].t, ws)
    if "bwd" in parts:
        ops.moe_top1_bwd(x, W, d_out, routing, B, N_H, E, H, math, g["d_x"].t, g["dW"].t, g["db"].t,
                         acc_flags, ws)
    if "aux" in parts:
        ops.moe_aux_loss_fwd_bwd(logits, routing.counts, B, N_H, E, lam_t, g["d_logits"].t, g["loss"].t,
                                 g["mean_p"].t, g["stats"].t, ws)
    torch.cuda.synchronize()
    out["flags"] = ops.moe_top1_device_flags(ws)
    out["guards_ok"] = all(v.guards_intact() for v in g.values())
    for k, v in g.items():
        out[k] = v.host()
    return out


def assert_close(name, g, o, atol, rtol, scale=None, max_report=5):
    """|g - o| <= atol + rtol * max(|o|, scale) elementwise."""
    g = np.asarray(g, np.float64)
    o = np.asarray(o, np.float64)
    mag = np.abs(o) if scale is None else np.maximum(np.abs(o), scale)
    err = np.abs(g - o)
    bad = ~(err <= atol + rtol * mag)
    if bad.any():
        idx = np.argwhere(bad)[:max_report]
        lines = [f"{tuple(i)}: gpu={g[tuple(i)]!r} oracle={o[tuple(i)]!r}" for i in idx]
        raise AssertionError(f"{name}: {int(bad.sum())} of {bad.size} elements outside "
                             f"{atol} + {rtol}*|o|; max err {err.max():.3e}\n" + "\n".join(lines))


def tf32_mode(math: int) -> int:
    return TF32_RULE if math == ops.MOE_MATH_TF32 else oracle.TF32_NONE
