"""GPU parity of the gate-entropy producer (moe_usage_entropy_ema_update) and of
the closed lambda loop it feeds, against the CPU oracle."""
import math

import numpy as np
import pytest
import torch

import oracle
from bwd_route_b200 import ops
from bwd_route_b200 import workloads as wl
from bwd_route_b200.gate import MoETop1Gate
from gpu_harness import Guarded

pytestmark = pytest.mark.gpu

# The kernel computes in double and stores fp32: half an fp32 ulp plus slack.
RTOL, ATOL = 2e-7, 1e-7


def _close(name, got, want):
    got, want = np.asarray(got, np.float64), np.asarray(want, np.float64)
    bad = np.abs(got - want) > ATOL + RTOL * np.abs(want)
    assert not bad.any(), f"{name}: {got[bad][:4]} vs {want[bad][:4]}"


def _run(counts, T, alpha, reset, usage0, ent0, with_step=True):
    E = len(counts)
    c = torch.tensor(counts, dtype=torch.int32, device="cuda")
    u, e, h = Guarded(E), Guarded(1), Guarded(1)
    u.t.copy_(torch.tensor(usage0, dtype=torch.float32))
    e.t.fill_(ent0)
    ops.moe_usage_entropy_ema_update(c, T, E, alpha, reset, u.t, e.t, h.t if with_step else None)
    torch.cuda.synchronize()
    assert u.guards_intact() and e.guards_intact() and h.guards_intact()
    return u.t.cpu().numpy(), float(e.t.item()), float(h.t.item())


@pytest.mark.parametrize("E", [1, 2, 3, 8, 17, 32])
@pytest.mark.parametrize("alpha", [0.0, 0.05, 0.5, 1.0])
@pytest.mark.parametrize("reset", [False, True])
def test_producer_matches_oracle(E, alpha, reset):
    rng = np.random.default_rng(E * 100 + int(alpha * 20))
    counts = rng.integers(0, 5000, E).astype(np.int32)
    if E > 2:
        counts[rng.integers(0, E)] = 0
    T = int(counts.sum())
    usage0 = rng.dirichlet(np.ones(E)).astype(np.float32)
    ent0 = np.float32(rng.uniform(0.0, math.log(max(E, 2))))
    gu, ge, gh = _run(counts, T, alpha, reset, usage0, float(ent0))
    ou, oe, oh = oracle.usage_entropy_ema(counts, T, alpha, reset, usage0.astype(np.float64), float(ent0))
    _close("usage_ema", gu, ou)
    _close("ent_ema", ge, oe)
    _close("ent_step", gh, oh)


def test_producer_edge_cases():
    # no tokens: nothing observed, state unchanged bit for bit
    u0 = np.array([0.3, 0.7], np.float32)
    gu, ge, gh = _run([0, 0], 0, 0.5, False, u0, 0.25)
    assert gu.tobytes() == u0.tobytes() and ge == np.float32(0.25) and gh == 0.0
    # every token on one expert: entropy exactly 0; the optional output may be NULL
    gu, ge, _ = _run([0, 77, 0, 0], 77, 1.0, False, np.full(4, 0.25, np.float32), 1.0, with_step=False)
    assert ge == 0.0 and gu.tolist() == [0.0, 1.0, 0.0, 0.0]
    # reset: the cold-start state, and the next lambda is the floor
    gu, ge, _ = _run([1, 2, 3, 4, 5, 6, 7, 8], 36, 0.3, True, np.zeros(8, np.float32), 0.5)
    assert np.all(gu == np.float32(0.125)) and ge == np.float32(math.log(8))
    lam = torch.zeros(1, device="cuda")
    ops.moe_lambda_eff_update(torch.tensor([ge], device="cuda"), 0.01, 0.09, 0.7 * math.log(8), lam)
    assert float(lam.item()) == np.float32(0.01)


def test_closed_loop_follows_the_oracle_and_is_deterministic():
    """Route real logits each step, fold the usage into ent_ema, recompute lambda:
    the device state tracks the oracle's iteration step by step."""
    spec = wl.WORKLOADS["skewed_b4096_e8_h128"]
    inp = wl.generate(spec, with_activations=False)
    E, T = spec.E, spec.T
    W = torch.zeros(E, spec.H, spec.H, device="cuda")
    bias = torch.zeros(E, spec.H, device="cuda")
    target = 0.7 * math.log(E)
    runs = []
    for _ in range(2):
        gate = MoETop1Gate(W, bias, spec.B, spec.N_H, ops.MOE_MATH_FFMA, 0.01, 0.09, target, math.log(E))
        gate.update_controller(0.0, reset=True)
        torch.cuda.synchronize()
        # the oracle iterates on the device's fp32 state, as the device does
        prev_u, prev_e = gate.usage_ema.cpu().numpy().astype(np.float64), float(gate.ent_ema.item())
        rng = np.random.default_rng(7)
        trace = []
        for step in range(20):
            logits = inp.gate_logits + rng.normal(0, 0.5, inp.gate_logits.shape).astype(np.float32)
            gate.route(torch.from_numpy(logits).cuda())
            gate.update_controller(0.2)
            counts = oracle.route(logits)[1]
            ou, oe, _ = oracle.usage_entropy_ema(counts, T, 0.2, False, prev_u, prev_e)
            torch.cuda.synchronize()
            gu = gate.usage_ema.cpu().numpy()
            ge = float(gate.ent_ema.item())
            _close("usage_ema", gu, ou)
            _close("ent_ema", ge, oe)
            lam = float(gate.lambda_eff.item())
            want = oracle.lambda_eff(ge, 0.01, 0.09, target)
            assert abs(lam - want) <= 1e-6 * want, (step, lam, want)
            prev_u, prev_e = gu.astype(np.float64), ge
            trace.append((gu.tobytes(), ge, lam))
        runs.append(trace)
    assert runs[0] == runs[1]
    # the skew (+2 on expert 4, ~71 % of tokens) keeps the entropy below the target: lambda above the floor
    assert runs[0][-1][2] > 0.01


AUX_CASES = [wl.WORKLOADS["tiny_b8_e4_h128"], wl.WORKLOADS["skewed_b4096_e8_h128"],
             wl.make_spec("aux_b26215_h5_e5", 26215, 5, 5, 32, 405),  # 1024-token blocks, rows moved per float
             wl.make_spec("aux_empty_b0_e3", 0, 5, 3, 32, 406)]


@pytest.mark.parametrize("spec", AUX_CASES, ids=lambda s: s.name)
@pytest.mark.parametrize("target", ["separate", "lambda_eff", "ent_ema"])
def test_aux_with_lambda_update_is_the_two_calls(spec, target):
    """moe_aux_loss_fwd_bwd_lambda_update gives every bit of moe_aux_loss_fwd_bwd
    followed by moe_lambda_eff_update: the loss and d_logits with the weight the
    call began with, then the next weight, written into a buffer of its own, over
    lambda_eff, or over ent_ema. Twice in a row (the ticket is reset)."""
    inp = wl.generate(spec, with_activations=False)
    B, N_H, E, T = spec.B, spec.N_H, spec.E, spec.T
    logits = torch.from_numpy(np.ascontiguousarray(inp.gate_logits)).cuda() if T else None
    routing = ops.Routing.empty(T, E, "cuda")
    ws = ops.new_workspace(T, E, 32, "cuda")
    if T:
        ops.moe_top1_route(logits, B, N_H, E, routing, ws)
    else:
        routing.counts.zero_()
    lam0, ema0, floor, extra, tgt = 0.03, 0.2, 0.01, 0.09, 1.0

    def outs():
        return {"d": Guarded(T * E), "loss": Guarded(2), "mp": Guarded(E), "st": Guarded(3 * E + 4)}

    # the two calls
    ref = outs()
    lam = torch.tensor([lam0], device="cuda")
    ema = torch.tensor([ema0], device="cuda")
    ops.moe_aux_loss_fwd_bwd(logits, routing.counts, B, N_H, E, lam, ref["d"].t if T else None, ref["loss"].t,
                             ref["mp"].t, ref["st"].t, ws)
    ops.moe_lambda_eff_update(ema, floor, extra, tgt, lam)
    torch.cuda.synchronize()
    lam_next = float(lam.item())
    assert lam_next != np.float32(lam0)
    for rep in range(2):
        got = outs()
        lam = Guarded(1)
        lam.t.fill_(lam0)
        ema = Guarded(1)
        ema.t.fill_(ema0)
        nxt = Guarded(1)
        out_buf = {"separate": nxt, "lambda_eff": lam, "ent_ema": ema}[target]
        ops.moe_aux_loss_fwd_bwd_lambda_update(logits, routing.counts, B, N_H, E, lam.t,
                                               got["d"].t if T else None, got["loss"].t, got["mp"].t,
                                               got["st"].t, ema.t, floor, extra, tgt, out_buf.t, ws)
        torch.cuda.synchronize()
        assert ops.moe_top1_device_flags(ws) == 0
        for k in got:
            assert got[k].guards_intact(), k
            assert got[k].host().tobytes() == ref[k].host().tobytes(), k
        assert lam.guards_intact() and ema.guards_intact() and nxt.guards_intact()
        assert float(out_buf.t.item()) == lam_next
        if target != "lambda_eff":
            assert float(lam.t.item()) == np.float32(lam0)
        if target != "ent_ema":
            assert float(ema.t.item()) == np.float32(ema0)
