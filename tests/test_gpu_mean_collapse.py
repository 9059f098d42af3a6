"""GPU parity of the horizon mean [B, N_H, H] -> [B, H] folded into the gate,
against the oracle in both math modes: the backward (moe_top1_bwd_mean_collapse)
and the forward (moe_top1_fwd_mean_collapse)."""
import numpy as np
import pytest
import torch

import oracle
from bwd_route_b200 import ops
from bwd_route_b200 import workloads as wl
from gpu_harness import TOL, Guarded, assert_close, dev, tf32_mode

pytestmark = pytest.mark.gpu

MATHS = [ops.MOE_MATH_FFMA, ops.MOE_MATH_TF32]
MATH_ID = {ops.MOE_MATH_FFMA: "ffma", ops.MOE_MATH_TF32: "tf32"}

SPECS = [
    wl.make_spec("mc_b8_h5_e4_h128", 8, 5, 4, 128, 31),            # N_H not a power of two
    wl.make_spec("mc_b1024_h5_e4_h128", 1024, 5, 4, 128, 32),
    wl.make_spec("mc_b300_h1_e3_h128", 300, 1, 3, 128, 33),         # N_H = 1: the plain backward
    wl.make_spec("mc_b777_h3_e8_h256", 777, 3, 8, 256, 34),
    wl.make_spec("mc_b2048_h16_e8_h256", 2048, 16, 8, 256, 35),     # the throughput shape's N_H, 32k tokens
    wl.make_spec("mc_b700_h7_e32_h128", 700, 7, 32, 128, 36, skew_expert=3, skew_value=1.5),
]


def _run(inp, g_host, math, acc_flags=0, preset=None):
    s = inp.spec
    B, N_H, E, H, T = s.B, s.N_H, s.E, s.H, s.T
    out = {k: Guarded(n, shape=sh) for k, n, sh in
           [("d_x", T * H, (T, H)), ("dW", E * H * H, (E, H, H)), ("db", E * H, (E, H))]}
    if preset:
        for k, v in preset.items():
            out[k].t.copy_(dev(v).view_as(out[k].t))
    r = ops.Routing.empty(T, E, "cuda")
    ws = ops.new_workspace(T, E, H, "cuda")
    ops.moe_top1_route(dev(inp.gate_logits), B, N_H, E, r, ws)
    ops.moe_top1_bwd_mean_collapse(dev(inp.x), dev(inp.W), dev(g_host), r, B, N_H, E, H, math, out["d_x"].t,
                                   out["dW"].t, out["db"].t, acc_flags, ws)
    torch.cuda.synchronize()
    assert ops.moe_top1_device_flags(ws) == 0
    assert all(v.guards_intact() for v in out.values())
    return {k: v.host() for k, v in out.items()}


def _grad(spec):
    rng = np.random.default_rng(spec.seed + 1000)
    return rng.standard_normal((spec.B, spec.H)).astype(np.float32)


@pytest.mark.parametrize("math_mode", MATHS, ids=MATH_ID.get)
@pytest.mark.parametrize("spec", SPECS, ids=lambda s: s.name)
def test_mean_collapse_backward_parity(spec, math_mode):
    inp = wl.generate(spec)
    g = _grad(spec)
    got = _run(inp, g, math_mode)
    idx = oracle.route(inp.gate_logits)[0]
    want = oracle.bwd_mean_collapse(inp.x, inp.W, g, idx, spec.N_H, spec.E, tf32_mode(math_mode))
    atol, rtol = TOL[math_mode]
    assert_close("d_x", got["d_x"], want["d_x"], atol, rtol)
    assert_close("dW", got["dW"], want["dW"], atol, rtol, scale=want["dW_scale"])
    assert_close("db", got["db"], want["db"], atol, rtol, scale=want["db_scale"])


# FFMA also serves the widths TF32 does not (H a multiple of 32 up to 256).
FFMA_WIDTH_SPECS = [wl.make_spec(f"mc_ffma_b203_h5_e6_h{H}", 203, 5, 6, H, 400 + H) for H in (32, 96, 160, 224)]


@pytest.mark.parametrize("spec", FFMA_WIDTH_SPECS, ids=lambda s: s.name)
def test_mean_collapse_backward_parity_ffma_other_widths(spec):
    test_mean_collapse_backward_parity(spec, ops.MOE_MATH_FFMA)


@pytest.mark.parametrize("math_mode", MATHS, ids=MATH_ID.get)
def test_mean_collapse_matches_plain_backward_bitwise_for_power_of_two_horizons(math_mode):
    """With N_H = 16, g / N_H is exact, so the two entry points must agree bit for
    bit when they run the same kernels (only the gradient rows and the final scale
    differ): with TF32 at H = 256 the mean-collapse call takes the single pass by
    default, so the plain call is asked for it too."""
    spec = wl.make_spec("mc_eq_b512_h16_e8_h256", 512, 16, 8, 256, 37)
    inp = wl.generate(spec)
    g = _grad(spec)
    got = _run(inp, g, math_mode)
    d_out = np.repeat(g / np.float32(spec.N_H), spec.N_H, axis=0).astype(np.float32)
    s = spec
    r = ops.Routing.empty(s.T, s.E, "cuda")
    ws = ops.new_workspace(s.T, s.E, s.H, "cuda")
    ops.moe_top1_route(dev(inp.gate_logits), s.B, s.N_H, s.E, r, ws)
    d_x = torch.empty(s.T, s.H, device="cuda")
    dW = torch.empty(s.E, s.H, s.H, device="cuda")
    db = torch.empty(s.E, s.H, device="cuda")
    strategy = ops.MOE_BWD_SINGLE_PASS if math_mode == ops.MOE_MATH_TF32 else 0
    ops.moe_top1_bwd(dev(inp.x), dev(inp.W), dev(d_out), r, s.B, s.N_H, s.E, s.H, math_mode, d_x, dW, db, strategy, ws)
    torch.cuda.synchronize()
    assert got["d_x"].tobytes() == d_x.cpu().numpy().tobytes()
    assert got["dW"].tobytes() == dW.cpu().numpy().tobytes()
    assert got["db"].tobytes() == db.cpu().numpy().tobytes()


@pytest.mark.parametrize("math_mode", MATHS, ids=MATH_ID.get)
def test_mean_collapse_accumulate_flags(math_mode):
    spec = wl.make_spec("mc_acc_b200_h5_e4_h256", 200, 5, 4, 256, 38)
    inp = wl.generate(spec)
    g = _grad(spec)
    rng = np.random.default_rng(1)
    T, E, H = spec.T, spec.E, spec.H
    pre = {"d_x": rng.standard_normal((T, H)).astype(np.float32),
           "dW": rng.standard_normal((E, H, H)).astype(np.float32),
           "db": rng.standard_normal((E, H)).astype(np.float32)}
    plain = _run(inp, g, math_mode)
    acc = _run(inp, g, math_mode, acc_flags=ops.MOE_ACC_DX | ops.MOE_ACC_DW | ops.MOE_ACC_DB, preset=pre)
    for k in ("d_x", "dW", "db"):
        np.testing.assert_array_equal(acc[k], (pre[k] + plain[k]).astype(np.float32), err_msg=k)


# ---------------------------------------------------------------- forward through the horizon mean
FWD_SPECS = [
    wl.make_spec("mcf_b8_h5_e4_h128", 8, 5, 4, 128, 51),                # one partial tile
    wl.make_spec("mcf_b1024_h5_e4_h128", 1024, 5, 4, 128, 52),          # eight full tiles
    wl.make_spec("mcf_b777_h3_e8_h256", 777, 3, 8, 256, 53),            # ragged last tile, H = 256
    wl.make_spec("mcf_b2048_h16_e8_h256", 2048, 16, 8, 256, 54),        # the throughput shape's N_H, E, H
    wl.make_spec("mcf_b300_h32_e32_h128", 300, 32, 32, 128, 55),        # N_H and E at their maximum
    wl.make_spec("mcf_b257_h7_e4_h128", 257, 7, 4, 128, 56, skew_expert=2, skew_value=3.0),  # > 2 tokens per (b, e)
    wl.make_spec("mcf_b130_h5_e4_h128", 130, 5, 4, 128, 57, logits="binary"),               # frequent ties
    # the row-range split of the staged kernel (E <= 8, N_H <= 16): fewer rows than
    # SMs, ranges of several tiles with a partial last one, several tiles per CTA at
    # its largest horizon, an odd horizon (the swizzle phase of the staged rows moves
    # inside a row group), one expert; N_H = 32 at E = 8 takes the general kernel
    wl.make_spec("mcf_b100_h16_e8_h256", 100, 16, 8, 256, 62),
    wl.make_spec("mcf_b40000_h5_e8_h128", 40000, 5, 8, 128, 63),
    wl.make_spec("mcf_b20000_h16_e8_h128", 20000, 16, 8, 128, 66),
    wl.make_spec("mcf_b1500_h9_e6_h256", 1500, 9, 6, 256, 67),
    wl.make_spec("mcf_b3000_h32_e8_h256", 3000, 32, 8, 256, 64),
    wl.make_spec("mcf_b500_h7_e1_h256", 500, 7, 1, 256, 65),
]


def fwd_bound(spec, math):
    """A worst-case bound against the exact definition: |got - exact| <= c * mag,
    mag = (1/N_H) sum_h (sum_i |W x| + |bias|) from the oracle. fp32 sums: the
    horizon pre-sum (N_H terms), the K = E * H products and the epilogue's bias,
    scale and store (8 more roundings), each at most one unit 2^-24 of mag. TF32
    adds the rounding of both operands of every product, each below 2^-10
    relative."""
    c = (spec.E * spec.H + spec.N_H + 8) * 2.0 ** -24
    if math == ops.MOE_MATH_TF32:
        c += 2.0 ** -9
    return c


def fwd_reference(inp, idx, N_H, math):
    """The oracle the kernel is held to at the gate's own tolerances: FFMA against
    the exact definition (|g - o| <= 1e-5 + 1e-5 |o|); TF32 against the oracle's
    TF32 mode of the same mean, whose contraction operands are the per-(row,
    expert) horizon sums X_be (formed in fp32, ascending h) and W, rounded the way
    the tensor core rounds them (|g - o| <= 1e-4 + 2e-3 |o|)."""
    if math == ops.MOE_MATH_TF32:
        return oracle.fwd_mean_collapse_presum(inp.x, inp.W, inp.bias, idx, N_H, tf32_mode(math))
    return oracle.fwd_mean_collapse(inp.x, inp.W, inp.bias, idx, N_H)[0]


def fwd_outside(got, want, math):
    """Number of elements outside the tolerance of the math mode."""
    atol, rtol = TOL[math]
    err = np.abs(got.astype(np.float64) - want)
    return int((~(err <= atol + rtol * np.abs(want))).sum())


def _run_fwd(spec, inp, math):
    out = Guarded(spec.B * spec.H, shape=(spec.B, spec.H))
    r = ops.Routing.empty(spec.T, spec.E, "cuda")
    ws = ops.new_workspace(spec.T, spec.E, spec.H, "cuda")
    ops.moe_top1_route(dev(inp.gate_logits), spec.B, spec.N_H, spec.E, r, ws)
    ops.moe_top1_fwd_mean_collapse(dev(inp.x), dev(inp.W), dev(inp.bias), r, spec.B, spec.N_H, spec.E, spec.H,
                                   math, out.t, ws)
    torch.cuda.synchronize()
    assert ops.moe_top1_device_flags(ws) == 0
    assert out.guards_intact()
    return out.host(), r, ws


@pytest.mark.parametrize("math_mode", MATHS, ids=MATH_ID.get)
@pytest.mark.parametrize("spec", FWD_SPECS, ids=lambda s: s.name)
def test_fwd_mean_collapse_parity(spec, math_mode):
    inp = wl.generate(spec)
    got, _, _ = _run_fwd(spec, inp, math_mode)
    idx = oracle.route(inp.gate_logits)[0]
    assert np.isfinite(got).all()
    assert_close("ctx_mean", got, fwd_reference(inp, idx, spec.N_H, math_mode), *TOL[math_mode])
    # and the worst-case bound against the exact definition in both modes
    want, mag = oracle.fwd_mean_collapse(inp.x, inp.W, inp.bias, idx, spec.N_H)
    err = np.abs(got.astype(np.float64) - want)
    bound = fwd_bound(spec, math_mode) * mag
    assert (err <= bound).all(), f"max err/bound {np.max(err / bound):.3g}"


@pytest.mark.parametrize("spec", FFMA_WIDTH_SPECS, ids=lambda s: s.name)
def test_fwd_mean_collapse_parity_ffma_other_widths(spec):
    test_fwd_mean_collapse_parity(spec, ops.MOE_MATH_FFMA)


@pytest.mark.parametrize("math_mode", MATHS, ids=MATH_ID.get)
def test_fwd_mean_collapse_check_catches_one_token_on_the_wrong_expert(math_mode):
    """The parity check must be tight enough to see one horizon token of one row
    sent to another expert (its W and bias change): the kernel is handed a
    routing with that one index changed, and the result is compared with the
    oracle on the true routing."""
    spec = wl.make_spec("mcf_sens_b256_h16_e8_h256", 256, 16, 8, 256, 61)
    inp = wl.generate(spec)
    idx = oracle.route(inp.gate_logits)[0]
    want = fwd_reference(inp, idx, spec.N_H, math_mode)
    got, r, ws = _run_fwd(spec, inp, math_mode)
    assert fwd_outside(got, want, math_mode) == 0
    t = 5 * spec.N_H + 3  # row 5, horizon token 3
    r.expert_idx[t] = (int(idx[t]) + 1) % spec.E
    out = torch.empty(spec.B, spec.H, device="cuda")
    ops.moe_top1_fwd_mean_collapse(dev(inp.x), dev(inp.W), dev(inp.bias), r, spec.B, spec.N_H, spec.E, spec.H,
                                   math_mode, out, ws)
    torch.cuda.synchronize()
    bad = out.cpu().numpy()
    n_bad = fwd_outside(bad, want, math_mode)
    assert n_bad > spec.H // 2, n_bad   # row 5 is off almost everywhere
    assert fwd_outside(np.delete(bad, 5, axis=0), np.delete(want, 5, axis=0), math_mode) == 0  # other rows intact


@pytest.mark.parametrize("math_mode", MATHS, ids=MATH_ID.get)
@pytest.mark.parametrize("E", [5, 12])
def test_fwd_mean_collapse_ignores_expert_indices_out_of_range(math_mode, E):
    """The call reads only expert_idx; an index outside [0, E) contributes nothing
    (neither its W x nor a bias), as the oracle's reading of such a token."""
    spec = wl.make_spec(f"mcf_badidx_b300_h6_e{E}_h128", 300, 6, E, 128, 66)
    inp = wl.generate(spec)
    idx = oracle.route(inp.gate_logits)[0].copy()
    idx[::7] = E
    idx[3::11] = -1
    r = ops.Routing.empty(spec.T, E, "cuda")
    r.expert_idx.copy_(dev(idx))
    out = Guarded(spec.B * spec.H, shape=(spec.B, spec.H))
    ws = ops.new_workspace(spec.T, E, spec.H, "cuda")
    ops.moe_top1_fwd_mean_collapse(dev(inp.x), dev(inp.W), dev(inp.bias), r, spec.B, spec.N_H, E, spec.H, math_mode,
                                   out.t, ws)
    torch.cuda.synchronize()
    assert ops.moe_top1_device_flags(ws) == 0 and out.guards_intact()
    want = oracle.fwd_mean_collapse_presum(inp.x, inp.W, inp.bias, idx, spec.N_H, tf32_mode(math_mode))
    assert_close("ctx_mean", out.host(), want, *TOL[math_mode])


@pytest.mark.parametrize("math_mode", MATHS, ids=MATH_ID.get)
def test_fwd_mean_collapse_with_one_horizon_token_is_the_plain_forward_bitwise(math_mode):
    """N_H = 1: every (b, e) sum is one row or zero, the other experts add exact
    zeros, and the products run in the plain forward's k order, so the result
    must equal moe_top1_fwd bit for bit."""
    spec = wl.make_spec("mcf_b1000_h1_e8_h256", 1000, 1, 8, 256, 58)
    inp = wl.generate(spec)
    got, r, ws = _run_fwd(spec, inp, math_mode)
    routed = torch.empty(spec.T, spec.H, device="cuda")
    ops.moe_top1_fwd(dev(inp.x), dev(inp.W), dev(inp.bias), r, spec.B, 1, spec.E, spec.H, math_mode, routed, ws)
    torch.cuda.synchronize()
    assert got.tobytes() == routed.cpu().numpy().tobytes()


@pytest.mark.parametrize("math_mode", MATHS, ids=MATH_ID.get)
def test_fwd_mean_collapse_is_deterministic(math_mode):
    spec = FWD_SPECS[3]
    inp = wl.generate(spec)
    a, _, _ = _run_fwd(spec, inp, math_mode)
    b, _, _ = _run_fwd(spec, inp, math_mode)
    assert a.tobytes() == b.tobytes()


def test_fwd_mean_collapse_empty_batch_writes_nothing():
    spec = wl.make_spec("mcf_empty", 0, 5, 4, 128, 59)
    out = Guarded(0)
    r = ops.Routing.empty(0, 4, "cuda")
    ws = ops.new_workspace(0, 4, 128, "cuda")
    W = torch.zeros(4, 128, 128, device="cuda")
    b = torch.zeros(4, 128, device="cuda")
    ops.moe_top1_fwd_mean_collapse(torch.empty(0, 128, device="cuda"), W, b, r, 0, 5, 4, 128, ops.MOE_MATH_TF32,
                                   out.t, ws)
    torch.cuda.synchronize()
    assert out.guards_intact()


def test_fwd_mean_collapse_full_size_sampled_rows():
    """The 1,048,576-token workload (B 65536, N_H 16, E 8, H 256) through the gate,
    as the benchmark runs it; 64 sampled rows against the oracle."""
    from bwd_route_b200.gate import MoETop1Gate
    spec = wl.WORKLOADS[wl.THROUGHPUT_WORKLOAD]
    inp = wl.generate(spec)
    gate = MoETop1Gate(dev(inp.W), dev(inp.bias), spec.B, spec.N_H, ops.MOE_MATH_TF32)
    gate.route(dev(inp.gate_logits))
    gate.forward_mean_collapse(dev(inp.x))
    torch.cuda.synchronize()
    assert ops.moe_top1_device_flags(gate.ws) == 0
    rows = np.sort(np.random.default_rng(60).choice(spec.B, 64, replace=False))
    tok = (rows[:, None] * spec.N_H + np.arange(spec.N_H)).reshape(-1)
    idx = oracle.route(inp.gate_logits[tok])[0]
    got = gate.ctx_mean[torch.from_numpy(rows).cuda()].cpu().numpy()
    want = oracle.fwd_mean_collapse_presum(inp.x[tok], inp.W, inp.bias, idx, spec.N_H, tf32_mode(ops.MOE_MATH_TF32))
    assert_close("ctx_mean (sampled rows)", got, want, *TOL[ops.MOE_MATH_TF32])
