"""GPU parity: the CUDA library (through its C ABI) against the CPU oracle.

Integers (routing) must match bit for bit; floating point within the
tolerances of gpu_harness.TOL, element by element. Every output buffer is
surrounded by guard bands that must come back untouched, and the device flag
word must stay clear.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from bwd_route_b200 import ops
from bwd_route_b200 import workloads as wl
from gpu_harness import TOL, assert_close, dev, run_gpu, tf32_mode

pytestmark = pytest.mark.gpu

MATHS = [ops.MOE_MATH_FFMA, ops.MOE_MATH_TF32]
MATH_ID = {ops.MOE_MATH_FFMA: "ffma", ops.MOE_MATH_TF32: "tf32"}

# Workloads the oracle finishes in seconds (full comparison).
SMALL = ["tiny_b8_e4_h128", "tiny_uniform_b8_e4_h128", "tiny_identity_b8_e4_h128", "small_b1024_e4_h128",
         "skewed_b4096_e8_h128", "ties_b16384_e4_h128", "collapsed_b16384_e4_h128"]

# Ragged and degenerate shapes: token counts that are not tile multiples, one
# token, one expert, odd expert counts, the maximum expert count, H = 256.
EDGE = [
    wl.make_spec("one_token_e4_h128", 1, 1, 4, 128, 11),
    wl.make_spec("ragged_b1025_e4_h128", 1025, 5, 4, 128, 12),
    wl.make_spec("single_expert_b300_e1_h128", 300, 1, 1, 128, 13),
    wl.make_spec("odd_experts_b999_e5_h128", 999, 3, 5, 128, 14),
    wl.make_spec("max_experts_b2000_e32_h128", 2000, 3, 32, 128, 15),
    wl.make_spec("h256_b1500_e8_h256", 1500, 3, 8, 256, 16),
    wl.make_spec("h256_skewed_b777_e3_h256", 777, 1, 3, 256, 17, skew_expert=1, skew_value=3.0),
    # H = 256 with more 256-token tiles than CTA pairs: pairs run several tiles
    # and change expert inside their run (the expert weights are reloaded).
    wl.make_spec("h256_b4096_e8_h256", 4096, 8, 8, 256, 18),
    wl.make_spec("h256_max_experts_b4000_e32_h256", 4000, 5, 32, 256, 19),
]


# FFMA accepts every H that is a multiple of 32 up to 256 (TF32 only 128 and
# 256): ragged token counts with 5 and with 32 experts at each of the other widths.
FFMA_WIDTHS = [32, 64, 96, 160, 192, 224]
FFMA_SHAPES = ([wl.make_spec(f"ffma_b311_e5_h{H}", 311, 3, 5, H, 100 + H) for H in FFMA_WIDTHS] +
               [wl.make_spec(f"ffma_b700_e32_h{H}", 700, 3, 32, H, 300 + H) for H in FFMA_WIDTHS])


def lam_of(inp):
    return float(np.float32(oracle.lambda_eff(inp.ent_ema, inp.lambda_floor, inp.lambda_max_extra,
                                              inp.ent_target)))


def check_all(inp, math, full=True, acc_flags=0):
    lam = lam_of(inp)
    g = run_gpu(inp, math, lam, acc_flags=acc_flags)
    assert g["flags"] == 0
    assert g["guards_ok"], "a kernel wrote outside its output"
    idx, counts, offsets, perm = oracle.route(inp.gate_logits)
    np.testing.assert_array_equal(g["expert_idx"], idx)
    np.testing.assert_array_equal(g["counts"], counts)
    np.testing.assert_array_equal(g["offsets"], offsets)
    np.testing.assert_array_equal(g["perm"], perm)
    atol, rtol = TOL[math]
    mode = tf32_mode(math)
    assert_close("routed", g["routed"], oracle.fwd(inp.x, inp.W, inp.bias, idx, mode), atol, rtol)
    assert_close("d_x", g["d_x"], oracle.bwd_dx(inp.W, inp.d_out, idx, mode), atol, rtol)
    dW, db, sW, sb = oracle.bwd_dw(inp.x, inp.d_out, idx, inp.spec.E, mode)
    assert_close("dW", g["dW"], dW, atol, rtol, scale=sW)
    assert_close("db", g["db"], db, atol, rtol, scale=sb)
    for e in range(inp.spec.E):
        if counts[e] == 0:  # inactive experts: exactly zero
            assert np.all(g["dW"][e] == 0.0) and np.all(g["db"][e] == 0.0)
    check_aux(inp, g, counts, lam)
    return g


def check_aux(inp, g, counts, lam):
    T, E = inp.spec.T, inp.spec.E
    o = oracle.aux(inp.gate_logits, counts, lam)
    assert abs(g["loss"][0] - o["aux_raw"]) <= 1e-5 * abs(o["aux_raw"]) + 1e-7
    assert abs(g["loss"][1] - o["loss"]) <= 1e-5 * abs(o["loss"]) + 1e-9
    assert_close("mean_p", g["mean_p"], o["mean_p"], 1e-7, 1e-5)
    # d_logits is O(lambda E / T): compare it in units of lambda E / T
    unit = lam * E / T
    assert_close("d_logits/(lambda E/T)", g["d_logits"].astype(np.float64) / unit, o["d_logits_unscaled"],
                 1e-5, 1e-5)
    st = g["stats"]
    np.testing.assert_allclose(st[:E], counts / T, rtol=1e-6)
    np.testing.assert_array_equal(st[E:2 * E], g["mean_p"])
    np.testing.assert_array_equal(st[2 * E:3 * E], counts.astype(np.float32))
    assert st[3 * E] == g["loss"][0] and st[3 * E + 1] == np.float32(lam)
    f = counts / T
    hf = -sum(v * math.log(v) for v in f if v > 0)
    hm = -sum(v * math.log(v) for v in o["mean_p"] if v > 0)
    assert abs(st[3 * E + 2] - hf) <= 1e-5 * max(1.0, hf) and abs(st[3 * E + 3] - hm) <= 1e-5 * max(1.0, hm)


@pytest.mark.parametrize("math_mode", MATHS, ids=MATH_ID.get)
@pytest.mark.parametrize("name", SMALL)
def test_full_parity(name, math_mode):
    check_all(wl.generate(wl.WORKLOADS[name]), math_mode)


@pytest.mark.parametrize("math_mode", MATHS, ids=MATH_ID.get)
@pytest.mark.parametrize("spec", EDGE, ids=lambda s: s.name)
def test_edge_parity(spec, math_mode):
    check_all(wl.generate(spec), math_mode)


@pytest.mark.parametrize("spec", FFMA_SHAPES, ids=lambda s: s.name)
def test_ffma_parity_at_every_supported_width(spec):
    check_all(wl.generate(spec), ops.MOE_MATH_FFMA)


@pytest.mark.parametrize("math_mode", MATHS, ids=MATH_ID.get)
def test_straight_through_expert_path_gives_the_logits_no_gradient(math_mode):
    """STE: the top-1 choice is piecewise constant in the logits, so the expert
    path contributes nothing to their gradient. (1) The aux loss's logit
    gradient is bitwise the same before and after a backward of the expert path
    on the same tokens: the backward writes no logit gradient. (2) Changing the
    logits without changing any argmax (scaling by 2, exact in fp32) leaves the
    routing and every expert-path output bitwise unchanged, while the aux
    gradient does change."""
    spec = wl.make_spec("ste_b900_e8_h256", 900, 3, 8, 256, 71)
    inp = wl.generate(spec)
    B, N_H, E, H, T = spec.B, spec.N_H, spec.E, spec.H, spec.T
    logits, x, d_out = dev(inp.gate_logits), dev(inp.x), dev(inp.d_out)
    W, bias = dev(inp.W), dev(inp.bias)
    lam = torch.tensor([0.05], dtype=torch.float32, device="cuda")
    ws = ops.new_workspace(T, E, H, "cuda")

    def aux_grad(lg, r):
        d = torch.empty(T, E, device="cuda")
        ops.moe_aux_loss_fwd_bwd(lg, r.counts, B, N_H, E, lam, d, torch.empty(2, device="cuda"),
                                 torch.empty(E, device="cuda"), None, ws)
        return d

    def expert_path(lg):
        r = ops.Routing.empty(T, E, "cuda")
        ops.moe_top1_route(lg, B, N_H, E, r, ws)
        out = [torch.empty(T, H, device="cuda"), torch.empty(T, H, device="cuda"),
               torch.empty(E, H, H, device="cuda"), torch.empty(E, H, device="cuda")]
        ops.moe_top1_fwd(x, W, bias, r, B, N_H, E, H, math_mode, out[0], ws)
        ops.moe_top1_bwd(x, W, d_out, r, B, N_H, E, H, math_mode, out[1], out[2], out[3], 0, ws)
        return r, out

    r = ops.Routing.empty(T, E, "cuda")
    ops.moe_top1_route(logits, B, N_H, E, r, ws)
    before = aux_grad(logits, r).cpu().numpy()
    _, path = expert_path(logits)
    after = aux_grad(logits, r).cpu().numpy()
    torch.cuda.synchronize()
    assert ops.moe_top1_device_flags(ws) == 0
    assert before.tobytes() == after.tobytes()
    r2, path2 = expert_path(logits * 2.0)
    for name in ("expert_idx", "counts", "offsets", "perm"):
        assert torch.equal(getattr(r2, name), getattr(r, name)), name
    for a, b in zip(path, path2):
        assert torch.equal(a, b)
    assert not np.array_equal(aux_grad(logits * 2.0, r2).cpu().numpy(), before)


# The single-pass TF32 backward (MOE_BWD_SINGLE_PASS, or the horizon-mean gradient
# at H = 256) runs d_x and dW / db as one fused kernel: on CTA pairs at H = 256
# (256-token pair-tiles of one expert, 512 tokens per pair at least), on single
# CTAs at H = 128 (128-token tiles). Shapes that stress the tiling: a pair-tile the odd CTA has no token of, one it has a few of, one pair
# only, segments far shorter than a tile (32 experts), a range that crosses
# several expert boundaries at odd positions, more pairs than fit on the GPU at
# once; and the same kinds of shapes at H = 128.
FUSED_SHAPES = [
    wl.make_spec("fused_b90_e3_h128", 90, 1, 3, 128, 91),
    wl.make_spec("fused_b1000_h3_e32_h128", 1000, 3, 32, 128, 92, skew_expert=2, skew_value=1.0),
    wl.make_spec("fused_b30000_h3_e5_h128", 30000, 3, 5, 128, 93),
    wl.make_spec("fused_b100_e3_h256", 100, 1, 3, 256, 81),
    wl.make_spec("fused_b300_e1_h256", 300, 1, 1, 256, 82),
    wl.make_spec("fused_b333_h3_e2_h256", 333, 3, 2, 256, 83),
    wl.make_spec("fused_b2000_h2_e32_h256", 2000, 2, 32, 256, 84, skew_expert=7, skew_value=1.5),
    wl.make_spec("fused_b16384_h5_e5_h256", 16384, 5, 5, 256, 85),
    wl.make_spec("fused_b5000_h9_e8_h256", 5000, 9, 8, 256, 86, logits="binary"),
]


@pytest.mark.parametrize("spec", FUSED_SHAPES, ids=lambda s: s.name)
def test_fused_backward_parity(spec):
    check_all(wl.generate(spec), ops.MOE_MATH_TF32, acc_flags=ops.MOE_BWD_SINGLE_PASS)


@pytest.mark.parametrize("H", [128, 256])
def test_backward_strategies_agree_and_repeat(H):
    """The two TF32 strategies (two passes by default, one with the flag) agree
    within the TF32 tolerance (different MMA shapes for d_x, different fixed
    summation trees for dW / db), and each repeats bit for bit."""
    inp = wl.generate(wl.make_spec(f"strat_b3000_h3_e6_h{H}", 3000, 3, 6, H, 88))
    two = [run_gpu(inp, ops.MOE_MATH_TF32, 0.01, parts=("route", "bwd")) for _ in range(2)]
    one = [run_gpu(inp, ops.MOE_MATH_TF32, 0.01, parts=("route", "bwd"), acc_flags=ops.MOE_BWD_SINGLE_PASS)
           for _ in range(2)]
    for k in ("d_x", "dW", "db"):
        np.testing.assert_array_equal(two[0][k], two[1][k], err_msg=k)
        np.testing.assert_array_equal(one[0][k], one[1][k], err_msg=k)
    atol, rtol = TOL[ops.MOE_MATH_TF32]
    assert_close("d_x", one[0]["d_x"], two[0]["d_x"].astype(np.float64), atol, rtol)
    for k in ("dW", "db"):
        assert_close(k, one[0][k], two[0][k].astype(np.float64), atol, rtol, scale=np.abs(two[0][k]).max())


@pytest.mark.parametrize("math_mode", MATHS, ids=MATH_ID.get)
def test_backward_outputs_requested_separately(math_mode):
    """d_x alone, dW and db alone, db alone and all three by default (the separate
    contraction kernels), then d_x with db and all three in one pass (with TF32 the
    fused kernel): every combination against the oracle."""
    spec = wl.make_spec("bwd_parts_b1200_h3_e6_h256", 1200, 3, 6, 256, 87)
    inp = wl.generate(spec)
    B, N_H, E, H, T = spec.B, spec.N_H, spec.E, spec.H, spec.T
    mode = tf32_mode(math_mode)
    atol, rtol = TOL[math_mode]
    idx = oracle.route(inp.gate_logits)[0]
    want_dx = oracle.bwd_dx(inp.W, inp.d_out, idx, mode)
    want_dw, want_db, sW, sb = oracle.bwd_dw(inp.x, inp.d_out, idx, E, mode)
    x, W, d_out = dev(inp.x), dev(inp.W), dev(inp.d_out)
    r = ops.Routing.empty(T, E, "cuda")
    ws = ops.new_workspace(T, E, H, "cuda")
    ops.moe_top1_route(dev(inp.gate_logits), B, N_H, E, r, ws)
    for want, flags in ((("d_x",), 0), (("dW", "db"), 0), (("db",), 0), (("d_x", "dW", "db"), 0),
                        (("d_x", "db"), ops.MOE_BWD_SINGLE_PASS), (("d_x", "dW", "db"), ops.MOE_BWD_SINGLE_PASS)):
        out = {"d_x": torch.full((T, H), float("nan"), device="cuda"),
               "dW": torch.full((E, H, H), float("nan"), device="cuda"),
               "db": torch.full((E, H), float("nan"), device="cuda")}
        args = {k: (out[k] if k in want else None) for k in out}
        ops.moe_top1_bwd(x, W, d_out, r, B, N_H, E, H, math_mode, args["d_x"], args["dW"], args["db"], flags, ws)
        torch.cuda.synchronize()
        assert ops.moe_top1_device_flags(ws) == 0
        for k in ("d_x", "dW", "db"):
            g = out[k].cpu().numpy()
            if k not in want:
                assert np.isnan(g).all(), (want, k)  # not written
        if "d_x" in want:
            assert_close(f"d_x {want}", out["d_x"].cpu().numpy(), want_dx, atol, rtol)
        if "dW" in want:
            assert_close(f"dW {want}", out["dW"].cpu().numpy(), want_dw, atol, rtol, scale=sW)
        if "db" in want:
            assert_close(f"db {want}", out["db"].cpu().numpy(), want_db, atol, rtol, scale=sb)


def test_identity_experts_bit_exact():
    inp = wl.generate(wl.WORKLOADS["tiny_identity_b8_e4_h128"])
    g = run_gpu(inp, ops.MOE_MATH_FFMA, 0.01, parts=("route", "fwd"))
    np.testing.assert_array_equal(g["routed"], inp.x)
    g = run_gpu(inp, ops.MOE_MATH_TF32, 0.01, parts=("route", "fwd"))
    rnd = np.vectorize(lambda v: oracle.tf32_round(v, tf32_mode(ops.MOE_MATH_TF32)), otypes=[np.float32])
    np.testing.assert_array_equal(g["routed"], rnd(inp.x))


def test_tf32_operand_rounding_rule():
    """Black-box probe of how tcgen05 kind::tf32 reads an fp32 operand: with an
    identity expert the output is the rounded input itself, so inputs whose low
    13 mantissa bits sit just below, at and above half a TF32 ulp tell the rules
    apart. The parity tests use the rule that matches (gpu_harness.TF32_RULE)."""
    base = np.float32(1.0) + np.float32(2.0 ** -10) * np.arange(8, dtype=np.float32)
    low = np.array([0x0FFF, 0x1000, 0x1001, 0x1FFF, 0x0001, 0x0800], dtype=np.uint32)
    vals = []
    for b in base:
        for sgn in (1, -1):
            for lb in low:
                u = np.array([b * sgn], np.float32).view(np.uint32)[0] | lb
                vals.append(np.array([u], np.uint32).view(np.float32)[0])
    H, E = 128, 1
    T = (len(vals) + H - 1) // H
    x = np.zeros((T, H), np.float32)
    x.flat[:len(vals)] = vals
    spec = wl.make_spec("tf32_probe", T, 1, E, H, 1)
    inp = wl.Inputs(spec, np.zeros((T, E), np.float32), x, np.zeros((T, H), np.float32),
                    np.eye(H, dtype=np.float32)[None].copy(), np.zeros((E, H), np.float32))
    g = run_gpu(inp, ops.MOE_MATH_TF32, 0.01, parts=("route", "fwd"))
    got = g["routed"]
    matches = {}
    for mode in (oracle.TF32_RZ, oracle.TF32_RNA, oracle.TF32_RNE):
        want = np.vectorize(lambda v: oracle.tf32_round(v, mode), otypes=[np.float32])(x)
        matches[mode] = bool(np.array_equal(got, want))
    print("tf32 rounding rule matches (RZ, RNA, RNE):", matches)
    assert sum(matches.values()) == 1, matches
    assert matches[tf32_mode(ops.MOE_MATH_TF32)], matches


@pytest.mark.parametrize("name", ["skewed_b4096_e8_h128", "h256"])
@pytest.mark.parametrize("math_mode", MATHS, ids=MATH_ID.get)
def test_deterministic_bitwise(math_mode, name):
    spec = wl.make_spec("det_b4096_e8_h256", 4096, 4, 8, 256, 22) if name == "h256" else wl.WORKLOADS[name]
    inp = wl.generate(spec)
    a = run_gpu(inp, math_mode, 0.02)
    b = run_gpu(inp, math_mode, 0.02)
    for k in ["expert_idx", "perm", "routed", "d_x", "dW", "db", "d_logits", "loss", "mean_p", "stats"]:
        assert a[k].tobytes() == b[k].tobytes(), k


@pytest.mark.parametrize("B,N_H,E", [(32768, 4, 8), (26215, 5, 5), (26215, 5, 16), (26215, 5, 32)])
def test_aux_around_the_block_size_switch(B, N_H, E):
    """The aux kernel takes 256-token blocks up to 131,072 tokens and 1024-token
    blocks above. 131,072 tokens is the last count with the small blocks (512 of
    them); 131,075 is past the switch, and its last block holds three tokens.
    Routing and aux against the oracle, at every expert-row width (E = 5 moves
    rows one float at a time)."""
    inp = wl.generate(wl.make_spec(f"aux_b{B}_h{N_H}_e{E}", B, N_H, E, 32, 400 + E))
    lam = lam_of(inp)
    g = run_gpu(inp, ops.MOE_MATH_FFMA, lam, parts=("route", "aux"))
    assert g["flags"] == 0
    assert g["guards_ok"], "a kernel wrote outside its output"
    _, counts, _, _ = oracle.route(inp.gate_logits)
    np.testing.assert_array_equal(g["counts"], counts)
    check_aux(inp, g, counts, lam)


def test_uniform_logits_aux_is_exactly_one():
    inp = wl.generate(wl.WORKLOADS["tiny_uniform_b8_e4_h128"])
    g = run_gpu(inp, ops.MOE_MATH_FFMA, 0.03, parts=("route", "aux"))
    assert g["loss"][0] == 1.0
    assert np.all(g["mean_p"] == 0.25)
    T = inp.spec.T
    frac = g["counts"] / T
    expect = np.float32(0.03) * (frac[None, :] - 0.25) / T * np.ones((T, 1))
    np.testing.assert_allclose(g["d_logits"], expect, rtol=1e-6, atol=1e-12)
    # rows of the softmax gradient sum to zero
    assert np.all(np.abs(g["d_logits"].sum(axis=1)) <= 1e-6 * np.abs(g["d_logits"]).sum(axis=1) + 1e-12)


@pytest.mark.parametrize("H", [128, 256])
@pytest.mark.parametrize("math_mode", MATHS, ids=MATH_ID.get)
def test_accumulate_flags(math_mode, H):
    inp = wl.generate(wl.make_spec(f"acc_b600_e4_h{H}", 600, 2, 4, H, 21))
    rng = np.random.default_rng(0)
    T, E, H = inp.spec.T, inp.spec.E, inp.spec.H
    pre = {"d_x": rng.standard_normal((T, H)).astype(np.float32),
           "dW": rng.standard_normal((E, H, H)).astype(np.float32),
           "db": rng.standard_normal((E, H)).astype(np.float32)}
    for strategy in (0, ops.MOE_BWD_SINGLE_PASS):
        plain = run_gpu(inp, math_mode, 0.01, parts=("route", "bwd"), acc_flags=strategy)
        acc = run_gpu(inp, math_mode, 0.01, parts=("route", "bwd"), preset=pre,
                      acc_flags=strategy | ops.MOE_ACC_DX | ops.MOE_ACC_DW | ops.MOE_ACC_DB)
        for k in ("d_x", "dW", "db"):
            np.testing.assert_array_equal(acc[k], (pre[k] + plain[k]).astype(np.float32), err_msg=(strategy, k))


def test_empty_batch():
    spec = wl.make_spec("empty", 0, 5, 4, 128, 1)
    inp = wl.generate(spec)
    pre = {"dW": np.ones((4, 128, 128), np.float32), "db": np.ones((4, 128), np.float32),
           "counts": np.full(4, 7, np.int32), "offsets": np.full(5, 7, np.int32)}
    for m in MATHS:
        g = run_gpu(inp, m, 0.01, preset=pre)
        assert g["flags"] == 0 and g["guards_ok"]
        assert np.all(g["counts"] == 0) and np.all(g["offsets"] == 0)
        assert np.all(g["dW"] == 0) and np.all(g["db"] == 0)
        assert np.all(g["loss"] == 0) and np.all(g["mean_p"] == 0)


def test_route_special_values():
    nan, inf = np.nan, np.inf
    rows = [[nan, 1, 2, 0], [1, nan, 2, 0], [3, nan, 2, 0], [-0.0, 0.0, -1, 0], [-inf, -inf, -inf, -inf],
            [-inf, -5, -inf, -6], [inf, inf, 1, 0], [1, 1, 1, 1], [0, 0, 0, nan], [nan, nan, nan, nan]]
    lg = np.array(rows * 7, np.float32)
    T = lg.shape[0]
    spec = wl.make_spec("special", T, 1, 4, 128, 1)
    inp = wl.Inputs(spec, lg, np.zeros((T, 128), np.float32), np.zeros((T, 128), np.float32),
                    np.zeros((4, 128, 128), np.float32), np.zeros((4, 128), np.float32))
    g = run_gpu(inp, ops.MOE_MATH_FFMA, 0.01, parts=("route",))
    idx, counts, offsets, perm = oracle.route(lg)
    np.testing.assert_array_equal(g["expert_idx"], idx)
    np.testing.assert_array_equal(g["perm"], perm)
    np.testing.assert_array_equal(g["counts"], counts)


@pytest.mark.parametrize("E", [1, 2, 3, 7, 8, 9, 16, 17, 31, 32])
def test_route_expert_counts(E):
    T = 4099
    rng = np.random.default_rng(E)
    lg = rng.integers(0, 3, size=(T, E)).astype(np.float32)  # many ties
    spec = wl.make_spec(f"route_e{E}", T, 1, E, 128, 1)
    inp = wl.Inputs(spec, lg, np.zeros((0, 128), np.float32), np.zeros((0, 128), np.float32),
                    np.zeros((E, 128, 128), np.float32), np.zeros((E, 128), np.float32))
    g = run_gpu(inp, ops.MOE_MATH_FFMA, 0.01, parts=("route",))
    idx, counts, offsets, perm = oracle.route(lg)
    np.testing.assert_array_equal(g["expert_idx"], idx)
    np.testing.assert_array_equal(g["counts"], counts)
    np.testing.assert_array_equal(g["offsets"], offsets)
    np.testing.assert_array_equal(g["perm"], perm)


def test_lambda_eff_kernel():
    K = 8
    target = 0.7 * math.log(K)
    cases = [1.381, 0.746, target + 0.1, target, target / 2, 0.0, math.log(K), float("nan")]
    for ent in cases:
        e = torch.tensor([ent], dtype=torch.float32, device="cuda")
        lam = torch.zeros(1, dtype=torch.float32, device="cuda")
        ops.moe_lambda_eff_update(e, 0.01, 0.09, target, lam)
        ref = oracle.lambda_eff(float(np.float32(ent)), 0.01, 0.09, float(np.float32(target))) \
            if not math.isnan(ent) else 0.01
        assert abs(lam.item() - ref) <= 1e-6, (ent, lam.item(), ref)
    e = torch.tensor([1.381], dtype=torch.float32, device="cuda")
    lam = torch.zeros(1, dtype=torch.float32, device="cuda")
    ops.moe_lambda_eff_update(e, 0.01, 0.09, target, lam)
    assert abs(lam.item() - 0.0146) <= 5e-5  # the value printed on the controller page


@pytest.fixture(scope="module")
def large():
    return wl.generate(wl.WORKLOADS[wl.THROUGHPUT_WORKLOAD])


@pytest.mark.parametrize("math_mode", MATHS, ids=MATH_ID.get)
def test_large_workload_sampled(large, math_mode):
    """1,048,576 tokens, H = 256, in the launch configuration the benchmark times:
    routing and aux in full, the per-token outputs on sampled tokens, dW on
    sampled entries and db in full."""
    inp = large
    lam = lam_of(inp)
    g = run_gpu(inp, math_mode, lam)
    assert g["flags"] == 0 and g["guards_ok"]
    idx, counts, offsets, perm = oracle.route(inp.gate_logits)
    np.testing.assert_array_equal(g["expert_idx"], idx)
    np.testing.assert_array_equal(g["counts"], counts)
    np.testing.assert_array_equal(g["offsets"], offsets)
    np.testing.assert_array_equal(g["perm"], perm)
    atol, rtol = TOL[math_mode]
    mode = tf32_mode(math_mode)
    rng = np.random.default_rng(99)
    rows = np.sort(rng.choice(inp.spec.T, 512, replace=False))
    rows = np.concatenate([rows, [0, inp.spec.T - 1], perm[offsets[1:-1]]])  # ends and expert boundaries
    assert_close("routed", g["routed"][rows], oracle.fwd(inp.x[rows], inp.W, inp.bias, idx[rows], mode), atol, rtol)
    assert_close("d_x", g["d_x"][rows], oracle.bwd_dx(inp.W, inp.d_out[rows], idx[rows], mode), atol, rtol)
    n = 96
    e_l = rng.integers(0, inp.spec.E, n)
    o_l = rng.integers(0, inp.spec.H, n)
    i_l = rng.integers(0, inp.spec.H, n)
    vals, scales = oracle.bwd_dw_entries(inp.x, inp.d_out, idx, e_l, o_l, i_l, mode)
    assert_close("dW", g["dW"][e_l, o_l, i_l], vals, atol, rtol, scale=scales)
    db, sb = oracle.bwd_db(inp.d_out, idx, inp.spec.E)
    assert_close("db", g["db"], db, atol, rtol, scale=sb)
    check_aux(inp, g, counts, lam)


def test_large_workload_single_pass_backward(large):
    """The single-pass TF32 backward (MOE_BWD_SINGLE_PASS) at the full size, in the
    same sampled form: d_x on sampled tokens, the ends and the expert boundaries,
    dW on sampled entries, db in full."""
    inp = large
    g = run_gpu(inp, ops.MOE_MATH_TF32, lam_of(inp), parts=("route", "bwd"), acc_flags=ops.MOE_BWD_SINGLE_PASS)
    assert g["flags"] == 0 and g["guards_ok"]
    idx, counts, offsets, perm = oracle.route(inp.gate_logits)
    atol, rtol = TOL[ops.MOE_MATH_TF32]
    mode = tf32_mode(ops.MOE_MATH_TF32)
    rng = np.random.default_rng(98)
    rows = np.sort(rng.choice(inp.spec.T, 512, replace=False))
    rows = np.concatenate([rows, [0, inp.spec.T - 1], perm[offsets[1:-1]]])
    assert_close("d_x", g["d_x"][rows], oracle.bwd_dx(inp.W, inp.d_out[rows], idx[rows], mode), atol, rtol)
    n = 96
    e_l = rng.integers(0, inp.spec.E, n)
    o_l = rng.integers(0, inp.spec.H, n)
    i_l = rng.integers(0, inp.spec.H, n)
    vals, scales = oracle.bwd_dw_entries(inp.x, inp.d_out, idx, e_l, o_l, i_l, mode)
    assert_close("dW", g["dW"][e_l, o_l, i_l], vals, atol, rtol, scale=scales)
    db, sb = oracle.bwd_db(inp.d_out, idx, inp.spec.E)
    assert_close("db", g["db"], db, atol, rtol, scale=sb)
