"""CPU oracle of the top-1 MoE gate (ctypes wrapper around moe_oracle.c).

TEST INFRASTRUCTURE ONLY: imported by tests/, by the smoke check in
__graft_entry__.py and by the CPU-baseline leg of bench.py -- nowhere else. The
product path (bwd_route_b200 and its CUDA library) never imports this package,
and this package imports nothing from the product.

Every function returns float64 numpy arrays (integers for routing). The C file
says, per function, which page passage it restates.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moe_oracle.c")
_LIB = os.path.join(_HERE, "libmoe_oracle.so")

TF32_NONE, TF32_RZ, TF32_RNA, TF32_RNE = 0, 1, 2, 3


def build(force: bool = False) -> str:
    """Compile moe_oracle.c with gcc (plain -O2, single thread)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c99", "-fPIC", "-shared", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def configure(lib: ctypes.CDLL) -> ctypes.CDLL:
    """Declares the C signatures on a loaded copy of the oracle library."""
    P = ctypes.c_void_p
    i64, i32 = ctypes.c_int64, ctypes.c_int32
    lib.oracle_tf32_round.restype = ctypes.c_float
    lib.oracle_tf32_round.argtypes = [ctypes.c_float, i32]
    lib.oracle_route.argtypes = [P, i64, i32, P, P, P, P]
    lib.oracle_fwd.argtypes = [P, P, P, P, i64, i32, i32, i32, P]
    lib.oracle_bwd_dx.argtypes = [P, P, P, i64, i32, i32, i32, P]
    lib.oracle_bwd_dw.argtypes = [P, P, P, i64, i32, i32, i32, P, P, P, P]
    lib.oracle_bwd_db.argtypes = [P, P, i64, i32, i32, P, P]
    lib.oracle_bwd_dw_entries.argtypes = [P, P, P, i64, i32, i32, i64, P, P, P, P, P]
    lib.oracle_fwd_mean_collapse.argtypes = [P, P, P, P, i64, i32, i32, i32, P, P]
    lib.oracle_fwd_mean_collapse_presum.argtypes = [P, P, P, P, i64, i32, i32, i32, i32, P]
    lib.oracle_aux.argtypes = [P, P, i64, i32, ctypes.c_float, P, P, P, P, P]
    lib.oracle_lambda_eff.restype = ctypes.c_double
    lib.oracle_lambda_eff.argtypes = [ctypes.c_double] * 4
    lib.oracle_usage_entropy_ema.argtypes = [P, i64, i32, ctypes.c_double, i32, P, P, P]
    return lib


def _load():
    global _lib
    if _lib is None:
        _lib = configure(ctypes.CDLL(build()))
    return _lib


def _p(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _f32(a) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=np.float32)


def _i32(a) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=np.int32)


def tf32_round(v: float, mode: int) -> float:
    return float(_load().oracle_tf32_round(float(v), int(mode)))


def route(gate_logits):
    """-> (expert_idx [T], counts [E], offsets [E+1], perm [T]) as int32."""
    lg = _f32(gate_logits)
    T, E = lg.shape
    idx = np.empty(T, np.int32)
    counts = np.empty(E, np.int32)
    offsets = np.empty(E + 1, np.int32)
    perm = np.empty(T, np.int32)
    _load().oracle_route(_p(lg), T, E, _p(idx), _p(counts), _p(offsets), _p(perm))
    return idx, counts, offsets, perm


def fwd(x, W, bias, expert_idx, tf32_mode: int = TF32_NONE):
    x, W, bias, idx = _f32(x), _f32(W), _f32(bias), _i32(expert_idx)
    T, H = x.shape
    E = W.shape[0]
    out = np.empty((T, H), np.float64)
    _load().oracle_fwd(_p(x), _p(W), _p(bias), _p(idx), T, E, H, tf32_mode, _p(out))
    return out


def bwd_dx(W, d_out, expert_idx, tf32_mode: int = TF32_NONE):
    W, d_out, idx = _f32(W), _f32(d_out), _i32(expert_idx)
    T, H = d_out.shape
    E = W.shape[0]
    out = np.empty((T, H), np.float64)
    _load().oracle_bwd_dx(_p(W), _p(d_out), _p(idx), T, E, H, tf32_mode, _p(out))
    return out


def bwd_dw(x, d_out, expert_idx, E: int, tf32_mode: int = TF32_NONE):
    """-> (dW [E,H,H], db [E,H], dW_scale, db_scale), all float64."""
    x, d_out, idx = _f32(x), _f32(d_out), _i32(expert_idx)
    T, H = x.shape
    dW = np.empty((E, H, H), np.float64)
    db = np.empty((E, H), np.float64)
    sW = np.empty((E, H, H), np.float64)
    sb = np.empty((E, H), np.float64)
    _load().oracle_bwd_dw(_p(x), _p(d_out), _p(idx), T, E, H, tf32_mode,
                          _p(dW), _p(db), _p(sW), _p(sb))
    return dW, db, sW, sb


def bwd_db(d_out, expert_idx, E: int):
    """-> (db [E,H], db_scale [E,H]) float64."""
    d_out, idx = _f32(d_out), _i32(expert_idx)
    T, H = d_out.shape
    db = np.empty((E, H), np.float64)
    sb = np.empty((E, H), np.float64)
    _load().oracle_bwd_db(_p(d_out), _p(idx), T, E, H, _p(db), _p(sb))
    return db, sb


def fwd_mean_collapse(x, W, bias, expert_idx, N_H: int):
    """Forward of the gate followed by the horizon mean [B, N_H, H] -> [B, H]
    ("Single source of truth for the attention path" page, MHA additions):
    ctx_mean[b] = (1/N_H) sum_h routed[b*N_H + h], exact products in double.
    -> (ctx_mean [B,H], mag [B,H]) float64; mag is (1/N_H) sum_h of the absolute
    terms, sum_i |W x| + |bias|."""
    x, W, bias, idx = _f32(x), _f32(W), _f32(bias), _i32(expert_idx)
    T, H = x.shape
    E = W.shape[0]
    N_H = int(N_H)
    if N_H < 1 or T % N_H:
        raise ValueError("T must be a multiple of N_H >= 1")
    B = T // N_H
    out = np.empty((B, H), np.float64)
    mag = np.empty((B, H), np.float64)
    _load().oracle_fwd_mean_collapse(_p(x), _p(W), _p(bias), _p(idx), B, N_H, E, H, _p(out), _p(mag))
    return out, mag


def fwd_mean_collapse_presum(x, W, bias, expert_idx, N_H: int, tf32_mode: int = TF32_NONE):
    """The horizon mean of the forward computed as one contraction per batch row
    over the per-(row, expert) sums of the horizon tokens' inputs, X_be, formed in
    fp32 in ascending h; tf32_mode rounds X_be and W (the operands a TF32 tensor
    core is given). -> ctx_mean [B, H] float64."""
    x, W, bias, idx = _f32(x), _f32(W), _f32(bias), _i32(expert_idx)
    T, H = x.shape
    E = W.shape[0]
    N_H = int(N_H)
    if N_H < 1 or T % N_H:
        raise ValueError("T must be a multiple of N_H >= 1")
    B = T // N_H
    out = np.empty((B, H), np.float64)
    _load().oracle_fwd_mean_collapse_presum(_p(x), _p(W), _p(bias), _p(idx), B, N_H, E, H, int(tf32_mode), _p(out))
    return out


def bwd_mean_collapse(x, W, grad_ctx_mean, expert_idx, N_H: int, E: int, tf32_mode: int = TF32_NONE,
                      with_dw: bool = True):
    """Backward of the gate followed by the horizon mean [B, N_H, H] -> [B, H]
    ("Single source of truth for the attention path" page, MHA additions and the
    horizon_mean_collapse kernel): every horizon token h of batch row b receives
    grad_ctx_mean[b] / N_H. Computed as the plain backward on the broadcast rows
    grad_ctx_mean[b] (the contraction's operand; TF32 mode rounds it), each
    result divided by N_H in double.
    -> dict d_x [T,H], and with_dw: dW, db, dW_scale, db_scale (float64)."""
    g = _f32(grad_ctx_mean)
    g_rep = np.repeat(g, int(N_H), axis=0)
    out = {"d_x": bwd_dx(W, g_rep, expert_idx, tf32_mode) / N_H}
    if with_dw:
        dW, db, sW, sb = bwd_dw(x, g_rep, expert_idx, E, tf32_mode)
        out.update(dW=dW / N_H, db=db / N_H, dW_scale=sW / N_H, db_scale=sb / N_H)
    return out


def bwd_dw_entries(x, d_out, expert_idx, e_list, o_list, i_list, tf32_mode: int = TF32_NONE):
    """dW at single entries (e, o, i) -> (values, scales), float64 [n]."""
    x, d_out, idx = _f32(x), _f32(d_out), _i32(expert_idx)
    e_list, o_list, i_list = _i32(e_list), _i32(o_list), _i32(i_list)
    T, H = x.shape
    n = len(e_list)
    vals = np.empty(n, np.float64)
    scales = np.empty(n, np.float64)
    _load().oracle_bwd_dw_entries(_p(x), _p(d_out), _p(idx), T, H, tf32_mode, n,
                                  _p(e_list), _p(o_list), _p(i_list), _p(vals), _p(scales))
    return vals, scales


def aux(gate_logits, counts, lambda_eff: float):
    """-> dict(mean_p [E], aux_raw, loss, d_logits [T,E], d_logits_unscaled [T,E])."""
    lg, c = _f32(gate_logits), _i32(counts)
    T, E = lg.shape
    mean_p = np.empty(E, np.float64)
    aux_raw = np.empty(1, np.float64)
    loss = np.empty(1, np.float64)
    d = np.empty((T, E), np.float64)
    du = np.empty((T, E), np.float64)
    _load().oracle_aux(_p(lg), _p(c), T, E, float(np.float32(lambda_eff)),
                       _p(mean_p), _p(aux_raw), _p(loss), _p(d), _p(du))
    return {"mean_p": mean_p, "aux_raw": float(aux_raw[0]), "loss": float(loss[0]),
            "d_logits": d, "d_logits_unscaled": du}


def lambda_eff(ent_ema: float, lambda_floor: float, lambda_max_extra: float, ent_target: float) -> float:
    return float(_load().oracle_lambda_eff(ent_ema, lambda_floor, lambda_max_extra, ent_target))


def usage_entropy_ema(counts, T: int, alpha: float, reset: bool, usage_ema, ent_ema: float):
    """One update of the gate-entropy producer: returns (usage_ema', ent_ema', H of this step)."""
    c = np.ascontiguousarray(counts, dtype=np.int32)
    E = c.shape[0]
    u = np.array(usage_ema, dtype=np.float64).reshape(E).copy()
    ent = ctypes.c_double(float(ent_ema))
    h = ctypes.c_double(0.0)
    _load().oracle_usage_entropy_ema(_p(c), int(T), E, float(alpha), int(bool(reset)), _p(u), ctypes.byref(ent),
                                     ctypes.byref(h))
    return u, ent.value, h.value


def step(inp, lambda_eff_value: float | None = None, tf32_mode: int = TF32_NONE, with_dw: bool = True):
    """One full pass of the gate on a workload (routing, forward, backward, aux)."""
    idx, counts, offsets, perm = route(inp.gate_logits)
    out = {"expert_idx": idx, "counts": counts, "offsets": offsets, "perm": perm}
    out["routed"] = fwd(inp.x, inp.W, inp.bias, idx, tf32_mode)
    out["d_x"] = bwd_dx(inp.W, inp.d_out, idx, tf32_mode)
    if with_dw:
        out["dW"], out["db"], out["dW_scale"], out["db_scale"] = bwd_dw(
            inp.x, inp.d_out, idx, inp.W.shape[0], tf32_mode)
    lam = lambda_eff_value
    if lam is None:
        lam = lambda_eff(inp.ent_ema, inp.lambda_floor, inp.lambda_max_extra, inp.ent_target)
    out["lambda_eff"] = lam
    out.update(aux(inp.gate_logits, counts, lam))
    return out
