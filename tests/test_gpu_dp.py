"""The data-parallel gate on the GPU.

1. Two ranks, each a process on the one GPU running the library's kernels on its
   half of the batch, exchanging over gloo (the group's collectives stage CUDA
   tensors through the host): after the exchange both ranks must hold the full
   batch's dW, db and expert counts -- checked against the oracle on the full
   batch -- and the same controller state. The two processes' kernels never wait
   on each other; only the host-side collectives do.
2. A one-rank NCCL job: the exchange runs on the device and leaves every result
   bit-identical to the plain gate's, since a one-rank sum is the identity.
"""
import datetime
import math
import os
import socket

import numpy as np
import torch.multiprocessing as mp

import pytest
import torch
import torch.distributed as dist

from bwd_route_b200 import ops
from bwd_route_b200 import workloads as wl
from bwd_route_b200.gate import MoETop1Gate
import oracle
from gpu_harness import TOL, assert_close, dev, tf32_mode

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


DP_SPEC = wl.make_spec("dp2_b2048_h5_e8_h256", 2048, 5, 8, 256, 42, skew_expert=4, skew_value=1.0)
DP_WORLD = 2


def _rank_gate(rank, port, out):
    torch.cuda.set_device(0)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=DP_WORLD, timeout=datetime.timedelta(seconds=120))
    try:
        inp = wl.generate(DP_SPEC)
        s = DP_SPEC
        half = s.B // DP_WORLD
        rows = slice(rank * half * s.N_H, (rank + 1) * half * s.N_H)
        gate = MoETop1Gate(dev(inp.W), dev(inp.bias), half, s.N_H, ops.MOE_MATH_TF32, inp.lambda_floor,
                           inp.lambda_max_extra, inp.ent_target, inp.ent_ema)
        gate.enable_data_parallel()
        gate.update_controller(0.0, reset=True)
        gate.step(dev(inp.gate_logits[rows]), dev(inp.x[rows]), dev(inp.d_out[rows]))
        gate.allreduce_gradients()
        gate.update_controller(0.5)
        torch.cuda.synchronize()
        out[rank] = {
            "flags": ops.moe_top1_device_flags(gate.ws),
            "dW": gate.dW.cpu().numpy().tobytes(), "db": gate.db.cpu().numpy().tobytes(),
            "d_x": gate.d_x.cpu().numpy().tobytes(),
            "counts": gate.routing.counts.cpu().numpy().tolist(),
            "counts_global": gate.counts_global.cpu().numpy().tolist(),
            "usage_ema": gate.usage_ema.cpu().numpy().tobytes(),
            "ent_ema": float(gate.ent_ema.item()), "lambda_eff": float(gate.lambda_eff.item()),
            "tokens": gate.dp_tokens,
        }
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(600)
def test_two_ranks_on_the_gpu_hold_the_full_batch_gradients_of_the_oracle():
    # every helper process is spawned: this process already holds a CUDA context
    out = mp.get_context("spawn").Manager().dict()
    mp.spawn(_rank_gate, args=(_free_port(), out), nprocs=DP_WORLD, join=True)
    s = DP_SPEC
    inp = wl.generate(s)
    E, H, T = s.E, s.H, s.T
    mode = tf32_mode(ops.MOE_MATH_TF32)
    atol, rtol = TOL[ops.MOE_MATH_TF32]
    idx, counts = oracle.route(inp.gate_logits)[:2]
    dW, db, sW, sb = oracle.bwd_dw(inp.x, inp.d_out, idx, E, mode)
    r0, r1 = out[0], out[1]
    for r in (r0, r1):
        assert r["flags"] == 0
        assert r["tokens"] == T
    # the exchanged results are the same bits on both ranks
    for k in ("dW", "db", "usage_ema"):
        assert r0[k] == r1[k], k
    assert r0["ent_ema"] == r1["ent_ema"] and r0["lambda_eff"] == r1["lambda_eff"]
    # and they are the full batch's
    assert_close("dW", np.frombuffer(r0["dW"], np.float32).reshape(E, H, H), dW, atol, rtol, scale=sW)
    assert_close("db", np.frombuffer(r0["db"], np.float32).reshape(E, H), db, atol, rtol, scale=sb)
    assert r0["counts_global"] == np.asarray(counts).tolist()
    # each rank's own routing and input gradient are those of its shard
    n = T // DP_WORLD
    for rank, r in ((0, r0), (1, r1)):
        rows = slice(rank * n, (rank + 1) * n)
        assert r["counts"] == np.asarray(oracle.route(inp.gate_logits[rows])[1]).tolist()
        d_x = np.frombuffer(r["d_x"], np.float32).reshape(n, H)
        assert_close(f"d_x rank {rank}", d_x, oracle.bwd_dx(inp.W, inp.d_out[rows], idx[rows], mode), atol, rtol)
    assert sum(r0["counts"][e] + r1["counts"][e] for e in range(E)) == T
    # the controller folded the global usage in: reset (1/E, ln E), then one step at weight 0.5
    u, ent, _ = oracle.usage_entropy_ema(counts, T, 0.5, False, np.full(E, 1.0 / E), math.log(E))
    assert abs(r0["ent_ema"] - ent) <= 1e-6 * max(1.0, abs(ent))
    np.testing.assert_allclose(np.frombuffer(r0["usage_ema"], np.float32), u, rtol=0, atol=1e-7)
    lam = oracle.lambda_eff(float(np.float32(r0["ent_ema"])), inp.lambda_floor, inp.lambda_max_extra,
                            float(np.float32(inp.ent_target)))
    assert abs(r0["lambda_eff"] - lam) <= 1e-6
