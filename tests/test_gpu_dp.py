"""The data-parallel gate on one GPU through NCCL (a one-rank job): the exchange
runs on the device and leaves every result bit-identical to the plain gate's,
since a one-rank sum is the identity."""
import datetime
import math
import socket

import pytest
import torch
import torch.distributed as dist

from bwd_route_b200 import ops
from bwd_route_b200 import workloads as wl
from bwd_route_b200.gate import MoETop1Gate
from gpu_harness import dev

pytestmark = pytest.mark.gpu


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _run(inp, data_parallel):
    s = inp.spec
    gate = MoETop1Gate(dev(inp.W), dev(inp.bias), s.B, s.N_H, ops.MOE_MATH_TF32, inp.lambda_floor,
                       inp.lambda_max_extra, inp.ent_target, inp.ent_ema)
    if data_parallel:
        gate.enable_data_parallel()
    logits, x, d_out = dev(inp.gate_logits), dev(inp.x), dev(inp.d_out)
    gate.update_controller(0.0, reset=True)
    for _ in range(3):
        gate.step(logits, x, d_out)
        gate.allreduce_gradients()
        gate.update_controller(0.5)
    torch.cuda.synchronize()
    assert ops.moe_top1_device_flags(gate.ws) == 0
    return {k: getattr(gate, k).clone() for k in ("dW", "db", "d_x", "usage_ema", "ent_ema", "lambda_eff")}


@pytest.mark.timeout(300)
def test_one_rank_nccl_job_matches_the_plain_gate_bitwise():
    inp = wl.generate(wl.WORKLOADS["skewed_b4096_e8_h128"])
    plain = _run(inp, False)
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{_free_port()}", rank=0, world_size=1,
                            timeout=datetime.timedelta(seconds=60), device_id=torch.device("cuda", 0))
    try:
        got = _run(inp, True)
    finally:
        dist.destroy_process_group()
    for k, v in plain.items():
        assert torch.equal(got[k], v), k
    # the skew keeps the usage entropy under its target: lambda above the floor
    assert float(got["lambda_eff"]) > inp.lambda_floor
    assert float(got["ent_ema"]) < 0.7 * math.log(inp.spec.E)
