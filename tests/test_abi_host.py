"""Host-side checks of the C ABI (no GPU needed).

The library must load without a GPU, export every function that
include/moe_top1.h declares, and reject bad arguments with the documented
status before anything touches the GPU (validation happens on the host, so
these calls never reach the CUDA runtime).
"""
import ctypes
import os
import re

import pytest

from bwd_route_b200 import build as libbuild
from bwd_route_b200 import ops

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moe_top1.h")

OK, INVALID, SHAPE, MISALIGNED, ALIAS, WORKSPACE = 0, 1, 2, 3, 4, 5

# Fake device addresses: validation only compares and aligns them, never dereferences.
A = 0x7F0000000000


def _p(v):
    return ctypes.c_void_p(v) if v else None


@pytest.fixture(scope="module")
def L():
    libbuild.build()
    return ops.lib()


def header_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?\w+\**\s+\**(moe_\w+)\s*\(", text, flags=re.M)))


def test_header_declares_the_five_entry_points():
    fns = header_functions()
    for name in ["moe_top1_route", "moe_top1_fwd", "moe_top1_bwd", "moe_aux_loss_fwd_bwd", "moe_lambda_eff_update"]:
        assert name in fns


def test_library_exports_every_declared_symbol(L):
    fns = header_functions()
    assert sorted(fns) == sorted(ops.EXPORTED)
    for name in fns:
        assert hasattr(L, name), name


def test_abi_version_and_status_strings(L):
    assert L.moe_top1_abi_version() == 6
    for s, name in enumerate(ops._STATUS):
        assert L.moe_status_string(s).decode() == name
    assert L.moe_status_string(99).decode() == "MOE_ERR_UNKNOWN"


def test_workspace_bytes(L):
    a = L.moe_top1_workspace_bytes(1_048_576, 8, 256)
    b = L.moe_top1_workspace_bytes(40, 4, 128)
    assert a > b > 0
    assert a % 256 == 0
    # dW partial slots for (148 ranges + 8 experts) x 256 x 256 fp32 dominate
    assert a >= (148 + 8) * 256 * 256 * 4
    assert L.moe_top1_workspace_bytes(10, 0, 128) == 0
    assert L.moe_top1_workspace_bytes(10, 33, 128) == 0
    assert L.moe_top1_workspace_bytes(-1, 4, 128) == 0


def _routing(base):
    return ops.RoutingC(_p(base), _p(base + 0x100000), _p(base + 0x200000), _p(base + 0x300000))


def test_route_rejects_bad_arguments_before_launch(L):
    r = _routing(A + 0x10000000)
    ws, wsb = _p(A + 0x20000000), 1 << 20
    lg = _p(A)
    assert L.moe_top1_route(lg, -1, 5, 4, ctypes.byref(r), ws, wsb, None) == INVALID
    assert L.moe_top1_route(lg, 8, 5, 0, ctypes.byref(r), ws, wsb, None) == SHAPE
    assert L.moe_top1_route(lg, 8, 5, 33, ctypes.byref(r), ws, wsb, None) == SHAPE
    assert L.moe_top1_route(lg, 1 << 40, 1 << 20, 4, ctypes.byref(r), ws, wsb, None) == SHAPE
    assert L.moe_top1_route(None, 8, 5, 4, ctypes.byref(r), ws, wsb, None) == INVALID
    assert L.moe_top1_route(lg, 8, 5, 4, None, ws, wsb, None) == INVALID
    assert L.moe_top1_route(_p(A + 4), 8, 5, 4, ctypes.byref(r), ws, wsb, None) == MISALIGNED
    # perm overlapping expert_idx
    bad = ops.RoutingC(_p(A + 0x10000000), _p(A + 0x10100000), _p(A + 0x10200000), _p(A + 0x10000000 + 64))
    assert L.moe_top1_route(lg, 8, 5, 4, ctypes.byref(bad), ws, wsb, None) == ALIAS
    # an output inside the logits
    bad = ops.RoutingC(_p(A + 16), _p(A + 0x10100000), _p(A + 0x10200000), _p(A + 0x10300000))
    assert L.moe_top1_route(lg, 8, 5, 4, ctypes.byref(bad), ws, wsb, None) == ALIAS
    assert L.moe_top1_route(lg, 8, 5, 4, ctypes.byref(r), None, 0, None) == WORKSPACE
    assert L.moe_top1_route(lg, 8, 5, 4, ctypes.byref(r), ws, 64, None) == WORKSPACE
    assert L.moe_top1_route(lg, 8, 5, 4, ctypes.byref(r), _p(A + 0x20000010), wsb, None) == MISALIGNED


def test_fwd_bwd_reject_bad_arguments_before_launch(L):
    r = _routing(A + 0x10000000)
    x, W, b, out = _p(A), _p(A + 0x1000000), _p(A + 0x2000000), _p(A + 0x3000000)
    ws, wsb = _p(A + 0x40000000), 1 << 30
    tf32, ffma = 0, 1
    f = L.moe_top1_fwd
    assert f(x, W, b, ctypes.byref(r), 8, 5, 4, 96, tf32, out, ws, wsb, None) == SHAPE   # TF32: H in {128, 256}
    assert f(x, W, b, ctypes.byref(r), 8, 5, 4, 100, ffma, out, ws, wsb, None) == SHAPE  # FFMA: H % 32
    assert f(x, W, b, ctypes.byref(r), 8, 5, 4, 512, ffma, out, ws, wsb, None) == SHAPE
    assert f(x, W, b, ctypes.byref(r), 8, 5, 4, 128, 7, out, ws, wsb, None) == INVALID
    assert f(x, None, b, ctypes.byref(r), 8, 5, 4, 128, tf32, out, ws, wsb, None) == INVALID
    assert f(x, W, b, ctypes.byref(r), 8, 5, 4, 128, tf32, _p(A + 0x3000008), ws, wsb, None) == MISALIGNED
    assert f(x, W, b, ctypes.byref(r), 8, 5, 4, 128, tf32, _p(A + 64), ws, wsb, None) == ALIAS   # routed on x
    assert f(x, W, b, ctypes.byref(r), 8, 5, 4, 128, tf32, out, None, 0, None) == WORKSPACE
    g = L.moe_top1_bwd
    dx, dW, db = _p(A + 0x5000000), _p(A + 0x6000000), _p(A + 0x7000000)
    assert g(x, W, x, ctypes.byref(r), 8, 5, 4, 128, tf32, dx, dW, db, 0x8, ws, wsb, None) == INVALID
    assert g(x, W, x, ctypes.byref(r), 8, 5, 4, 128, tf32, dx, dW, db, 0x200, ws, wsb, None) == INVALID
    # the single-pass bit is a known flag: the call gets past argument checks to the aliasing check
    assert g(x, W, x, ctypes.byref(r), 8, 5, 4, 128, tf32, dx, dx, db, 0x100, ws, wsb, None) == ALIAS
    assert g(x, W, x, ctypes.byref(r), 8, 5, 4, 128, tf32, dx, dx, db, 0, ws, wsb, None) == ALIAS  # dW on d_x
    assert g(x, W, x, ctypes.byref(r), 8, 5, 4, 128, tf32, x, dW, db, 0, ws, wsb, None) == ALIAS   # d_x on x
    assert g(x, W, x, ctypes.byref(r), 8, 5, 4, 128, tf32, dx, dW, db, 0, ws, 4096, None) == WORKSPACE
    assert g(x, None, x, ctypes.byref(r), 8, 5, 4, 128, tf32, dx, None, None, 0, ws, wsb, None) == INVALID
    # nothing requested: nothing to do, no launch
    assert g(x, W, x, ctypes.byref(r), 8, 5, 4, 128, tf32, None, None, None, 0, ws, wsb, None) == OK


def test_aux_and_lambda_reject_bad_arguments(L):
    lg, cnt, lam = _p(A), _p(A + 0x1000000), _p(A + 0x1000100)
    d, loss, mp, st = _p(A + 0x2000000), _p(A + 0x3000000), _p(A + 0x3000100), _p(A + 0x3000200)
    ws, wsb = _p(A + 0x40000000), 1 << 20
    a = L.moe_aux_loss_fwd_bwd
    assert a(lg, cnt, 8, 5, 0, lam, d, loss, mp, st, ws, wsb, None) == SHAPE
    assert a(lg, None, 8, 5, 4, lam, d, loss, mp, st, ws, wsb, None) == INVALID
    assert a(lg, cnt, 8, 5, 4, None, d, loss, mp, st, ws, wsb, None) == INVALID
    assert a(lg, cnt, 8, 5, 4, lam, _p(A + 0x2000004), loss, mp, st, ws, wsb, None) == MISALIGNED
    assert a(lg, cnt, 8, 5, 4, lam, d, loss, _p(A + 0x3000004), st, ws, wsb, None) == ALIAS  # mean_p on loss
    assert a(lg, cnt, 8, 5, 4, lam, d, loss, mp, st, ws, 16, None) == WORKSPACE
    u = L.moe_lambda_eff_update
    e, out = _p(A), _p(A + 256)
    assert u(None, 0.01, 0.09, 1.0, out, None) == INVALID
    assert u(e, 0.01, 0.09, 0.0, out, None) == INVALID
    assert u(e, 0.01, 0.09, float("nan"), out, None) == INVALID
    assert u(e, -0.01, 0.09, 1.0, out, None) == INVALID
    assert u(e, 0.01, float("inf"), 1.0, out, None) == INVALID
    assert u(_p(A + 2), 0.01, 0.09, 1.0, out, None) == MISALIGNED


def test_aux_with_lambda_update_rejects_bad_arguments(L):
    """The folded call checks the arguments of both calls; the next lambda may be
    lambda_eff or ent_ema and nothing else the call touches (the aliasing checks
    run before the workspace check, so a too-small workspace marks a call that
    got past them)."""
    lg, cnt, lam = _p(A), _p(A + 0x1000000), _p(A + 0x1000100)
    d, loss, mp, st = _p(A + 0x2000000), _p(A + 0x3000000), _p(A + 0x3000100), _p(A + 0x3000200)
    ema, nxt = _p(A + 0x1000200), _p(A + 0x1000300)
    ws, wsb = _p(A + 0x40000000), 1 << 20
    f = L.moe_aux_loss_fwd_bwd_lambda_update

    def call(**k):
        return f(k.get("lg", lg), cnt, 8, 5, k.get("E", 4), k.get("lam", lam), k.get("d", d), loss,
                 k.get("mp", mp), st, k.get("ema", ema), k.get("floor", 0.01), k.get("extra", 0.09),
                 k.get("target", 1.0), k.get("nxt", nxt), ws, k.get("wsb", wsb), None)

    assert call(E=0) == SHAPE
    assert call(ema=None) == INVALID
    assert call(nxt=None) == INVALID
    assert call(target=0.0) == INVALID
    assert call(target=float("nan")) == INVALID
    assert call(floor=-0.01) == INVALID
    assert call(extra=float("inf")) == INVALID
    assert call(nxt=_p(A + 0x1000302)) == MISALIGNED
    assert call(nxt=loss) == ALIAS                      # next lambda on loss_out
    assert call(nxt=_p(A + 0x2000000 + 32)) == ALIAS    # next lambda inside d_logits
    assert call(nxt=_p(A + 16)) == ALIAS                # next lambda inside the logits
    assert call(nxt=cnt) == ALIAS                       # next lambda on counts
    assert call(lam=mp, nxt=mp) == ALIAS                # lambda_eff (written) on mean_p
    assert call(ema=d) == ALIAS                         # ent_ema inside d_logits
    assert call(ema=_p(A + 0x40000100)) == ALIAS        # ent_ema inside the workspace
    assert call(lam=_p(A + 0x40000100)) == ALIAS        # lambda_eff inside the workspace
    assert call(wsb=16) == WORKSPACE                    # separate buffers
    assert call(nxt=lam, wsb=16) == WORKSPACE           # next lambda replaces lambda_eff
    assert call(nxt=ema, wsb=16) == WORKSPACE           # next lambda replaces ent_ema


def test_bwd_mean_collapse_rejects_bad_arguments(L):
    b = L.moe_top1_bwd_mean_collapse
    R = ops.RoutingC(_p(A + 0x100000), _p(A + 0x200000), _p(A + 0x300000), _p(A + 0x400000))
    x, W, g = _p(A + 0x1000000), _p(A + 0x2000000), _p(A + 0x3000000)
    dx, dW, db = _p(A + 0x4000000), _p(A + 0x5000000), _p(A + 0x6000000)
    ws, wsb = _p(A + 0x40000000), 1 << 30
    args = lambda **k: [k.get("x", x), W, k.get("g", g), ctypes.byref(R), 8, 5, 4, k.get("H", 128), 0,
                        k.get("dx", dx), dW, db, 0, ws, wsb, None]
    assert b(*args(H=100)) == SHAPE
    assert b(*args(g=None)) == INVALID
    assert b(*args(g=_p(A + 0x3000004))) == MISALIGNED
    # d_x overlapping the last row of grad_ctx_mean [B, H] = 8 x 128 floats
    assert b(*args(dx=_p(A + 0x3000000 + 4 * 128 * 7))) == ALIAS


def test_fwd_mean_collapse_rejects_bad_arguments(L):
    f = L.moe_top1_fwd_mean_collapse
    R = ops.RoutingC(_p(A + 0x100000), _p(A + 0x200000), _p(A + 0x300000), _p(A + 0x400000))
    x, W, b, out = _p(A + 0x1000000), _p(A + 0x2000000), _p(A + 0x3000000), _p(A + 0x4000000)
    ws, wsb = _p(A + 0x40000000), 1 << 30
    args = lambda **k: [x, k.get("W", W), b, ctypes.byref(R), k.get("B", 8), k.get("N_H", 5), 4, k.get("H", 128),
                        k.get("math", 0), k.get("out", out), k.get("ws", ws), wsb, None]
    assert f(*args(N_H=33)) == SHAPE      # one mask bit per horizon token
    assert f(*args(N_H=0)) == SHAPE       # a mean over no tokens
    assert f(*args(H=96)) == SHAPE
    assert f(*args(math=7)) == INVALID
    assert f(*args(W=None)) == INVALID
    assert f(*args(out=_p(A + 0x4000008))) == MISALIGNED
    assert f(*args(out=_p(A + 0x1000000 + 4 * 128 * 39))) == ALIAS   # ctx_mean on the last row of x [40, 128]
    assert f(*args(ws=None)) == WORKSPACE
    assert f(*args(B=0)) == OK            # nothing to compute: returns before any launch


def test_usage_entropy_update_rejects_bad_arguments(L):
    u = L.moe_usage_entropy_ema_update
    cnt, ue, ee, hs = _p(A), _p(A + 0x100), _p(A + 0x200), _p(A + 0x300)
    assert u(cnt, 100, 0, 0.1, 0, ue, ee, hs, None) == SHAPE
    assert u(cnt, 100, 33, 0.1, 0, ue, ee, hs, None) == SHAPE
    assert u(cnt, -1, 8, 0.1, 0, ue, ee, hs, None) == INVALID
    assert u(None, 100, 8, 0.1, 0, ue, ee, hs, None) == INVALID
    assert u(cnt, 100, 8, 0.1, 0, None, ee, hs, None) == INVALID
    assert u(cnt, 100, 8, 0.1, 0, ue, None, hs, None) == INVALID
    for bad in (-0.1, 1.5, float("nan")):
        assert u(cnt, 100, 8, bad, 0, ue, ee, hs, None) == INVALID
    assert u(cnt, 100, 8, 0.1, 0, _p(A + 0x102), ee, hs, None) == MISALIGNED
    assert u(cnt, 100, 8, 0.1, 0, ue, _p(A + 0x104), hs, None) == ALIAS      # ent_ema inside usage_ema [8]
    assert u(cnt, 100, 8, 0.1, 0, ue, ee, _p(A + 0x200), None) == ALIAS      # ent_step on ent_ema
    assert u(cnt, 100, 8, 0.1, 0, _p(A + 0x10), ee, hs, None) == ALIAS      # usage_ema over counts [8]


def test_python_binding_refuses_cpu_tensors():
    import torch
    with pytest.raises(ValueError):
        ops._ptr(torch.zeros(4))


def test_check_routing_rejects_bad_arguments(L):
    r = ops.RoutingC(_p(A), _p(A + 0x100000), _p(A + 0x200000), _p(A + 0x300000))
    ws = _p(A + 0x400000)
    f = L.moe_top1_check_routing
    assert f(None, 10, 4, ws, 256, None) == INVALID
    assert f(ctypes.byref(r), -1, 4, ws, 256, None) == INVALID
    assert f(ctypes.byref(r), 10, 0, ws, 256, None) == SHAPE
    assert f(ctypes.byref(r), 10, 33, ws, 256, None) == SHAPE
    assert f(ctypes.byref(r), 2 ** 31, 4, ws, 256, None) == SHAPE
    assert f(ctypes.byref(r), 10, 4, None, 256, None) == WORKSPACE
    assert f(ctypes.byref(r), 10, 4, ws, 255, None) == WORKSPACE
    assert f(ctypes.byref(r), 10, 4, _p(A + 0x400010), 256, None) == MISALIGNED
    bad = ops.RoutingC(_p(A + 2), _p(A + 0x100000), _p(A + 0x200000), _p(A + 0x300000))
    assert f(ctypes.byref(bad), 10, 4, ws, 256, None) == MISALIGNED
    nul = ops.RoutingC(None, _p(A + 0x100000), _p(A + 0x200000), None)
    assert f(ctypes.byref(nul), 10, 4, ws, 256, None) == INVALID
