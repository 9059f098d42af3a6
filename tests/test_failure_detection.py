"""Failure detection without a GPU fault.

A pipeline wait that never completes must give up after its bound, record
MOE_FLAG_WAIT_TIMEOUT in the workspace flag word, and return, leaving the CUDA
context usable; the host reads the flag with moe_top1_device_flags. The wait
here is a barrier nothing arrives on, with a ~1 ms limit (no trap, no fault).
"""
import numpy as np
import pytest
import torch

import oracle
from bwd_route_b200 import ops
from bwd_route_b200 import workloads as wl


@pytest.mark.gpu
def test_bounded_wait_times_out_and_reports_the_flag():
    ws = ops.new_workspace(1024, 4, 128, "cuda")
    assert ops.moe_top1_device_flags(ws) == 0
    ops.moe_top1_selftest_wait_timeout(ws, 2_000_000)  # ~1 ms of SM clock
    torch.cuda.synchronize()
    assert ops.moe_top1_device_flags(ws) == ops.MOE_FLAG_WAIT_TIMEOUT
    assert ops.moe_top1_device_flags(ws) == 0  # reading clears it
    # the context is still healthy: a normal call right after gives exact results
    inp = wl.generate(wl.WORKLOADS["small_b1024_e4_h128"], with_activations=False)
    r = ops.Routing.empty(inp.spec.T, 4, "cuda")
    ops.moe_top1_route(torch.from_numpy(inp.gate_logits).cuda(), inp.spec.B, inp.spec.N_H, 4, r, ws)
    np.testing.assert_array_equal(r.perm.cpu().numpy(), oracle.route(inp.gate_logits)[3])
    assert ops.moe_top1_device_flags(ws) == 0


def test_selftest_rejects_bad_limits_on_the_host():
    import ctypes
    L = ops.lib()
    ws = ctypes.c_void_p(0x7F0000000000)
    assert L.moe_top1_selftest_wait_timeout(ws, 4096, 0, None) == 1          # limit must be >= 1
    assert L.moe_top1_selftest_wait_timeout(ws, 4096, 10**12, None) == 1     # and bounded
    assert L.moe_top1_selftest_wait_timeout(None, 4096, 1000, None) == 1
    assert L.moe_top1_selftest_wait_timeout(ctypes.c_void_p(0x7F0000000010), 4096, 1000, None) == 3
    assert L.moe_top1_selftest_wait_timeout(ws, 16, 1000, None) == 5
