"""Thin ctypes binding of libmoe_top1.so (C ABI: include/moe_top1.h).

Argument marshalling only: every function takes torch tensors that already
live on the GPU, checks their dtype / contiguity, and passes data pointers and
the current CUDA stream to the C entry point of the same name. All arithmetic
happens in the library's CUDA kernels. There is no CPU fallback: without the
built library every call raises.
"""
from __future__ import annotations

import ctypes
import dataclasses
import os

import torch

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libmoe_top1.so")

MOE_MATH_TF32 = 0
MOE_MATH_FFMA = 1
MOE_ACC_DX, MOE_ACC_DW, MOE_ACC_DB = 0x1, 0x2, 0x4
MOE_BWD_SINGLE_PASS = 0x100  # one pass over d_out for d_x, dW and db (TF32)
MOE_FLAG_WAIT_TIMEOUT = 0x1
MOE_FLAG_BAD_ROUTING = 0x2

_STATUS = ["MOE_OK", "MOE_ERR_INVALID_ARG", "MOE_ERR_UNSUPPORTED_SHAPE", "MOE_ERR_MISALIGNED",
           "MOE_ERR_ALIAS", "MOE_ERR_WORKSPACE", "MOE_ERR_CUDA", "MOE_ERR_DEVICE_CHECK"]

# Symbols declared in include/moe_top1.h.
EXPORTED = [
    "moe_top1_workspace_bytes", "moe_top1_workspace_init", "moe_top1_route", "moe_top1_fwd",
    "moe_top1_bwd", "moe_aux_loss_fwd_bwd", "moe_lambda_eff_update", "moe_top1_device_flags",
    "moe_status_string", "moe_top1_abi_version", "moe_top1_route_noalloc", "moe_top1_selftest_wait_timeout",
    "moe_usage_entropy_ema_update", "moe_top1_bwd_mean_collapse", "moe_top1_fwd_mean_collapse",
    "moe_top1_check_routing", "moe_aux_loss_fwd_bwd_lambda_update",
]
MOE_NOALLOC_MAX_TOKENS = 2097152


class MoeError(RuntimeError):
    def __init__(self, fn: str, status: int):
        name = _STATUS[status] if 0 <= status < len(_STATUS) else f"status {status}"
        super().__init__(f"{fn}: {name}")
        self.status = status
        self.status_name = name


class RoutingC(ctypes.Structure):
    _fields_ = [("expert_idx", ctypes.c_void_p), ("counts", ctypes.c_void_p),
                ("offsets", ctypes.c_void_p), ("perm", ctypes.c_void_p)]


_lib = None


def library_path() -> str:
    return _LIB_PATH


def lib() -> ctypes.CDLL:
    """Loads libmoe_top1.so (raises if it was not built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(_LIB_PATH):
            raise RuntimeError(f"{_LIB_PATH} is missing: build it with `python -m bwd_route_b200.build`")
        L = ctypes.CDLL(_LIB_PATH)
        P, I64, I32, U32, SZ = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_uint32, ctypes.c_size_t
        L.moe_top1_workspace_bytes.restype = SZ
        L.moe_top1_workspace_bytes.argtypes = [I64, I32, I32]
        L.moe_top1_workspace_init.restype = I32
        L.moe_top1_workspace_init.argtypes = [P, SZ, P]
        L.moe_top1_route.restype = I32
        L.moe_top1_route.argtypes = [P, I64, I64, I32, ctypes.POINTER(RoutingC), P, SZ, P]
        L.moe_top1_fwd.restype = I32
        L.moe_top1_fwd.argtypes = [P, P, P, ctypes.POINTER(RoutingC), I64, I64, I32, I32, I32, P, P, SZ, P]
        L.moe_top1_fwd_mean_collapse.restype = I32
        L.moe_top1_fwd_mean_collapse.argtypes = L.moe_top1_fwd.argtypes
        L.moe_top1_bwd.restype = I32
        L.moe_top1_bwd.argtypes = [P, P, P, ctypes.POINTER(RoutingC), I64, I64, I32, I32, I32, P, P, P, U32,
                                   P, SZ, P]
        L.moe_top1_bwd_mean_collapse.restype = I32
        L.moe_top1_bwd_mean_collapse.argtypes = L.moe_top1_bwd.argtypes
        L.moe_aux_loss_fwd_bwd.restype = I32
        L.moe_aux_loss_fwd_bwd.argtypes = [P, P, I64, I64, I32, P, P, P, P, P, P, SZ, P]
        L.moe_aux_loss_fwd_bwd_lambda_update.restype = I32
        L.moe_aux_loss_fwd_bwd_lambda_update.argtypes = [P, P, I64, I64, I32, P, P, P, P, P, P, ctypes.c_float,
                                                         ctypes.c_float, ctypes.c_float, P, P, SZ, P]
        L.moe_lambda_eff_update.restype = I32
        L.moe_lambda_eff_update.argtypes = [P, ctypes.c_float, ctypes.c_float, ctypes.c_float, P, P]
        L.moe_top1_device_flags.restype = I32
        L.moe_top1_device_flags.argtypes = [P, SZ, P, ctypes.POINTER(U32)]
        L.moe_status_string.restype = ctypes.c_char_p
        L.moe_status_string.argtypes = [I32]
        L.moe_top1_abi_version.restype = I32
        L.moe_top1_abi_version.argtypes = []
        L.moe_top1_selftest_wait_timeout.restype = I32
        L.moe_top1_selftest_wait_timeout.argtypes = [P, SZ, I64, P]
        L.moe_usage_entropy_ema_update.restype = I32
        L.moe_usage_entropy_ema_update.argtypes = [P, I64, I32, ctypes.c_float, I32, P, P, P, P]
        L.moe_top1_check_routing.restype = I32
        L.moe_top1_check_routing.argtypes = [ctypes.POINTER(RoutingC), I64, I32, P, SZ, P]
        L.moe_top1_route_noalloc.restype = I32
        L.moe_top1_route_noalloc.argtypes = [P, I64, I64, I32, ctypes.POINTER(RoutingC), P]
        _lib = L
    return _lib


def _ptr(t: torch.Tensor | None, dtype=None):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("expected a CUDA tensor")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"expected {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError("expected a contiguous tensor")
    return ctypes.c_void_p(t.data_ptr())


_raw_stream = getattr(torch._C, "_cuda_getCurrentRawStream", None)


def _stream(stream) -> ctypes.c_void_p:
    """The CUDA stream handle to launch on: the given torch stream, else the
    current stream of the current device (read without building a Stream object)."""
    if stream is not None:
        return ctypes.c_void_p(stream.cuda_stream)
    if _raw_stream is not None:
        return ctypes.c_void_p(_raw_stream(torch.cuda.current_device()))
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _check(fn: str, status: int):
    if status != 0:
        raise MoeError(fn, status)


@dataclasses.dataclass
class Routing:
    expert_idx: torch.Tensor  # [T] int32
    counts: torch.Tensor      # [E] int32
    offsets: torch.Tensor     # [E+1] int32
    perm: torch.Tensor        # [T] int32

    @staticmethod
    def empty(T: int, E: int, device) -> "Routing":
        i32 = torch.int32
        return Routing(torch.empty(T, dtype=i32, device=device), torch.empty(E, dtype=i32, device=device),
                       torch.empty(E + 1, dtype=i32, device=device), torch.empty(T, dtype=i32, device=device))

    def c(self) -> RoutingC:
        return RoutingC(_ptr(self.expert_idx, torch.int32), _ptr(self.counts, torch.int32),
                        _ptr(self.offsets, torch.int32), _ptr(self.perm, torch.int32))


def moe_top1_workspace_bytes(T: int, E: int, H: int) -> int:
    return int(lib().moe_top1_workspace_bytes(T, E, H))


def new_workspace(T: int, E: int, H: int, device, stream=None) -> torch.Tensor:
    """Allocates (torch) and initialises a workspace for every call on T, E, H."""
    n = moe_top1_workspace_bytes(T, E, H)
    ws = torch.empty(max(n, 256), dtype=torch.uint8, device=device)
    moe_top1_workspace_init(ws, stream)
    return ws


def moe_top1_workspace_init(ws: torch.Tensor, stream=None):
    _check("moe_top1_workspace_init", lib().moe_top1_workspace_init(_ptr(ws), ws.numel(), _stream(stream)))


def moe_top1_route(gate_logits: torch.Tensor, B: int, N_H: int, E: int, routing: Routing, ws: torch.Tensor,
                   stream=None):
    rc = routing.c()
    _check("moe_top1_route", lib().moe_top1_route(_ptr(gate_logits, torch.float32), B, N_H, E, ctypes.byref(rc),
                                                  _ptr(ws), ws.numel(), _stream(stream)))


def moe_top1_route_noalloc(gate_logits: torch.Tensor, B: int, N_H: int, E: int, routing: Routing, stream=None):
    """Routing without a workspace, for callers that cannot allocate device memory:
    the routing scratch lives in a fixed 512 KiB device array inside the library
    (at most MOE_NOALLOC_MAX_TOKENS tokens). Calls that may overlap on the GPU
    share that array and must be ordered by the caller."""
    rc = routing.c()
    _check("moe_top1_route_noalloc", lib().moe_top1_route_noalloc(_ptr(gate_logits, torch.float32), B, N_H, E,
                                                                  ctypes.byref(rc), _stream(stream)))


def moe_top1_check_routing(routing: Routing, T: int, E: int, ws: torch.Tensor, stream=None):
    """Enqueues the check of a routing not produced by moe_top1_route; a malformed
    one sets MOE_FLAG_BAD_ROUTING in the workspace flag word (moe_top1_device_flags)."""
    rc = routing.c()
    _check("moe_top1_check_routing", lib().moe_top1_check_routing(ctypes.byref(rc), T, E, _ptr(ws), ws.numel(),
                                                                  _stream(stream)))


def moe_top1_fwd(x, W, bias, routing: Routing, B: int, N_H: int, E: int, H: int, math: int, routed,
                 ws: torch.Tensor, stream=None):
    rc = routing.c()
    f = torch.float32
    _check("moe_top1_fwd", lib().moe_top1_fwd(_ptr(x, f), _ptr(W, f), _ptr(bias, f), ctypes.byref(rc), B, N_H, E, H,
                                              math, _ptr(routed, f), _ptr(ws), ws.numel(), _stream(stream)))


def moe_top1_fwd_mean_collapse(x, W, bias, routing: Routing, B: int, N_H: int, E: int, H: int, math: int, ctx_mean,
                               ws: torch.Tensor, stream=None):
    """ctx_mean [B, H] = the horizon mean of moe_top1_fwd's [B * N_H, H] output."""
    rc = routing.c()
    f = torch.float32
    _check("moe_top1_fwd_mean_collapse",
           lib().moe_top1_fwd_mean_collapse(_ptr(x, f), _ptr(W, f), _ptr(bias, f), ctypes.byref(rc), B, N_H, E, H,
                                            math, _ptr(ctx_mean, f), _ptr(ws), ws.numel(), _stream(stream)))


def moe_top1_bwd(x, W, d_out, routing: Routing, B: int, N_H: int, E: int, H: int, math: int, d_x, dW, db,
                 accumulate_flags: int, ws: torch.Tensor, stream=None):
    rc = routing.c()
    f = torch.float32
    _check("moe_top1_bwd", lib().moe_top1_bwd(_ptr(x, f), _ptr(W, f), _ptr(d_out, f), ctypes.byref(rc), B, N_H, E,
                                              H, math, _ptr(d_x, f), _ptr(dW, f), _ptr(db, f),
                                              accumulate_flags, _ptr(ws), ws.numel(), _stream(stream)))


def moe_top1_bwd_mean_collapse(x, W, grad_ctx_mean, routing: Routing, B: int, N_H: int, E: int, H: int, math: int,
                               d_x, dW, db, accumulate_flags: int, ws: torch.Tensor, stream=None):
    """moe_top1_bwd with d_out[b * N_H + h] = grad_ctx_mean[b] / N_H (grad_ctx_mean is [B, H])."""
    rc = routing.c()
    f = torch.float32
    _check("moe_top1_bwd_mean_collapse",
           lib().moe_top1_bwd_mean_collapse(_ptr(x, f), _ptr(W, f), _ptr(grad_ctx_mean, f), ctypes.byref(rc), B, N_H,
                                            E, H, math, _ptr(d_x, f), _ptr(dW, f), _ptr(db, f), accumulate_flags,
                                            _ptr(ws), ws.numel(), _stream(stream)))


def moe_aux_loss_fwd_bwd(gate_logits, counts, B: int, N_H: int, E: int, lambda_eff, d_logits, loss_out, mean_p,
                         stats, ws: torch.Tensor, stream=None):
    f = torch.float32
    _check("moe_aux_loss_fwd_bwd",
           lib().moe_aux_loss_fwd_bwd(_ptr(gate_logits, f), _ptr(counts, torch.int32), B, N_H, E,
                                      _ptr(lambda_eff, f), _ptr(d_logits, f), _ptr(loss_out, f), _ptr(mean_p, f),
                                      _ptr(stats, f), _ptr(ws), ws.numel(), _stream(stream)))


def moe_aux_loss_fwd_bwd_lambda_update(gate_logits, counts, B: int, N_H: int, E: int, lambda_eff, d_logits,
                                      loss_out, mean_p, stats, ent_ema, lambda_floor: float,
                                      lambda_max_extra: float, ent_target: float, lambda_next, ws: torch.Tensor,
                                      stream=None):
    f = torch.float32
    _check("moe_aux_loss_fwd_bwd_lambda_update",
           lib().moe_aux_loss_fwd_bwd_lambda_update(
               _ptr(gate_logits, f), _ptr(counts, torch.int32), B, N_H, E, _ptr(lambda_eff, f), _ptr(d_logits, f),
               _ptr(loss_out, f), _ptr(mean_p, f), _ptr(stats, f), _ptr(ent_ema, f), lambda_floor,
               lambda_max_extra, ent_target, _ptr(lambda_next, f), _ptr(ws), ws.numel(), _stream(stream)))


def moe_lambda_eff_update(ent_ema, lambda_floor: float, lambda_max_extra: float, ent_target: float, lambda_eff,
                          stream=None):
    f = torch.float32
    _check("moe_lambda_eff_update",
           lib().moe_lambda_eff_update(_ptr(ent_ema, f), lambda_floor, lambda_max_extra, ent_target,
                                       _ptr(lambda_eff, f), _stream(stream)))


def moe_usage_entropy_ema_update(counts, T: int, E: int, alpha: float, reset: bool, usage_ema, ent_ema,
                                 ent_step=None, stream=None):
    """Gate-entropy producer for the lambda controller: updates usage_ema [E] and
    ent_ema [1] in place from this step's counts (or resets them to 1/E, ln E)."""
    f = torch.float32
    _check("moe_usage_entropy_ema_update",
           lib().moe_usage_entropy_ema_update(_ptr(counts, torch.int32), T, E, alpha, int(bool(reset)),
                                              _ptr(usage_ema, f), _ptr(ent_ema, f), _ptr(ent_step, f),
                                              _stream(stream)))


def moe_top1_selftest_wait_timeout(ws: torch.Tensor, limit_cycles: int, stream=None):
    """Runs one bounded wait that must time out (diagnostic of the failure path)."""
    _check("moe_top1_selftest_wait_timeout",
           lib().moe_top1_selftest_wait_timeout(_ptr(ws), ws.numel(), limit_cycles, _stream(stream)))


def moe_top1_device_flags(ws: torch.Tensor, stream=None) -> int:
    flags = ctypes.c_uint32(0)
    st = lib().moe_top1_device_flags(_ptr(ws), ws.numel(), _stream(stream), ctypes.byref(flags))
    if st not in (0, 7):
        raise MoeError("moe_top1_device_flags", st)
    return int(flags.value)
