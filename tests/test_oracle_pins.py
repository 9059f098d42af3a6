"""Pins of the CPU oracle to things other than itself (no GPU needed).

Each test ties one oracle function to a closed form, a value printed on the
pages, a finite difference, brute force with independent library routines
(numpy argmax / bincount / stable argsort, torch float64 autograd), or a
mathematical invariant -- chosen so that a dropped term, a wrong sign, a wrong
index or a transposed operand in the oracle fails at least one of them.
"""
import math
import os

import numpy as np
import pytest
import torch

import oracle
from bwd_route_b200 import workloads as wl

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def tiny(name="tiny_b8_e4_h128"):
    return wl.generate(wl.WORKLOADS[name])


# --------------------------------------------------------------------------- routing

def test_route_brute_force_tiny():
    inp = tiny()
    idx, counts, offsets, perm = oracle.route(inp.gate_logits)
    np.testing.assert_array_equal(idx, np.argmax(inp.gate_logits, axis=1))
    np.testing.assert_array_equal(counts, np.bincount(idx, minlength=4))
    np.testing.assert_array_equal(offsets, np.concatenate([[0], np.cumsum(counts)]))
    np.testing.assert_array_equal(perm, np.argsort(idx, kind="stable"))


@pytest.mark.parametrize("name", ["skewed_b4096_e8_h128", "ties_b16384_e4_h128", "small_b1024_e4_h128"])
def test_route_invariants_and_library(name):
    inp = wl.generate(wl.WORKLOADS[name], with_activations=False)
    idx, counts, offsets, perm = oracle.route(inp.gate_logits)
    T = inp.spec.T
    np.testing.assert_array_equal(np.sort(perm), np.arange(T))           # a permutation
    assert counts.sum() == T
    assert np.all(np.diff(idx[perm]) >= 0)                                # grouped by expert
    for e in range(inp.spec.E):
        seg = perm[offsets[e]:offsets[e + 1]]
        assert np.all(np.diff(seg) > 0)                                   # stable
        assert np.all(idx[seg] == e)
    # numpy's argmax returns the first maximum: the lowest-index tie-break.
    np.testing.assert_array_equal(idx, np.argmax(inp.gate_logits, axis=1))


def test_route_uniform_logits_all_to_expert0():
    inp = tiny("tiny_uniform_b8_e4_h128")
    idx, counts, _, perm = oracle.route(inp.gate_logits)
    assert np.all(idx == 0)
    np.testing.assert_array_equal(counts, [40, 0, 0, 0])
    np.testing.assert_array_equal(perm, np.arange(40))


def test_route_binary_logits_tie_fractions():
    # Logits iid uniform on {0, 1}: the lowest index among the maxima wins, so
    # P(e) = P(l_0..l_{e-1} all 0 and l_e = 1) (+ P(all 0) for e = 0):
    # (1/2 + 1/16, 1/4, 1/8, 1/16) for E = 4.
    inp = wl.generate(wl.WORKLOADS["ties_b16384_e4_h128"], with_activations=False)
    _, counts, _, _ = oracle.route(inp.gate_logits)
    T = inp.spec.T
    expect = np.array([9 / 16, 1 / 4, 1 / 8, 1 / 16])
    sigma = np.sqrt(expect * (1 - expect) / T)
    assert np.all(np.abs(counts / T - expect) < 5 * sigma), counts / T


def test_route_collapsed():
    inp = wl.generate(wl.WORKLOADS["collapsed_b16384_e4_h128"], with_activations=False)
    _, counts, _, _ = oracle.route(inp.gate_logits)
    np.testing.assert_array_equal(counts, [inp.spec.T, 0, 0, 0])


def test_route_special_values():
    nan, inf = np.float32(np.nan), np.float32(np.inf)
    lg = np.array([
        [nan, 1, 2],        # NaN at e=0: the scan never moves off e=0
        [1, nan, 2],        # NaN elsewhere never wins
        [3, nan, 2],
        [-0.0, 0.0, -1],    # -0 and +0 compare equal: lowest index
        [-inf, -inf, -inf],
        [-inf, -5, -inf],
        [inf, inf, 1],
        [1, 1, 1],
    ], dtype=np.float32)
    idx, _, _, _ = oracle.route(lg)
    np.testing.assert_array_equal(idx, [0, 2, 0, 0, 0, 1, 0, 0])


def test_route_empty():
    idx, counts, offsets, perm = oracle.route(np.zeros((0, 4), np.float32))
    assert idx.size == 0 and perm.size == 0
    np.testing.assert_array_equal(counts, [0, 0, 0, 0])
    np.testing.assert_array_equal(offsets, [0, 0, 0, 0, 0])


# --------------------------------------------------------------------------- tf32 rounding

def test_tf32_rounding_known_values():
    one = 1.0
    half_ulp = 2.0 ** -11   # tf32 keeps 10 mantissa bits: ulp(1) = 2^-10
    # exact tf32 values are fixed points of every mode
    for v in [1.0, -3.5, 1 + 2 ** -10, 2.0 ** -20, 65504.0]:
        for m in (1, 2, 3):
            assert oracle.tf32_round(v, m) == v
    # a tie at 1 + 2^-11
    assert oracle.tf32_round(one + half_ulp, oracle.TF32_RZ) == 1.0
    assert oracle.tf32_round(one + half_ulp, oracle.TF32_RNA) == 1 + 2 ** -10
    assert oracle.tf32_round(one + half_ulp, oracle.TF32_RNE) == 1.0          # 1.0 is even
    assert oracle.tf32_round(one + 3 * half_ulp, oracle.TF32_RNE) == 1 + 2 ** -9  # to even
    assert oracle.tf32_round(-(one + half_ulp), oracle.TF32_RNA) == -(1 + 2 ** -10)
    # just below a tie / just above
    assert oracle.tf32_round(one + half_ulp - 2 ** -23, oracle.TF32_RNA) == 1.0
    assert oracle.tf32_round(one + half_ulp + 2 ** -23, oracle.TF32_RNE) == 1 + 2 ** -10
    assert oracle.tf32_round(one + 2 ** -10 - 2 ** -23, oracle.TF32_RZ) == 1.0
    assert oracle.tf32_round(float(np.float32(1e-3)), oracle.TF32_NONE) == float(np.float32(1e-3))


def test_tf32_rounding_error_bounds():
    rng = np.random.default_rng(7)
    v = rng.standard_normal(2000).astype(np.float32) * 10.0 ** rng.integers(-8, 8, 2000)
    for x in v:
        x = float(x)
        ulp = 2.0 ** (math.frexp(abs(x))[1] - 11)     # tf32 ulp at |x|
        rz = oracle.tf32_round(x, oracle.TF32_RZ)
        rna = oracle.tf32_round(x, oracle.TF32_RNA)
        rne = oracle.tf32_round(x, oracle.TF32_RNE)
        assert abs(rz) <= abs(x) and abs(x - rz) < ulp
        assert abs(x - rna) <= ulp / 2 and abs(x - rne) <= ulp / 2
        for r in (rz, rna, rne):
            assert oracle.tf32_round(r, oracle.TF32_RZ) == r  # low 13 bits clear


# --------------------------------------------------------------------------- forward

def test_fwd_identity_weights_return_x():
    inp = tiny("tiny_identity_b8_e4_h128")
    idx, *_ = oracle.route(inp.gate_logits)
    np.testing.assert_array_equal(oracle.fwd(inp.x, inp.W, inp.bias, idx), inp.x.astype(np.float64))
    r = oracle.fwd(inp.x, inp.W, inp.bias, idx, oracle.TF32_RZ)
    expect = np.vectorize(lambda v: oracle.tf32_round(v, oracle.TF32_RZ))(inp.x)
    np.testing.assert_array_equal(r, expect)


def test_fwd_matches_torch_float64_gather_einsum():
    inp = tiny()
    idx, *_ = oracle.route(inp.gate_logits)
    x = torch.from_numpy(inp.x).double()
    W = torch.from_numpy(inp.W).double()
    b = torch.from_numpy(inp.bias).double()
    ix = torch.from_numpy(idx).long()
    ref = torch.einsum("toi,ti->to", W[ix], x) + b[ix]
    np.testing.assert_allclose(oracle.fwd(inp.x, inp.W, inp.bias, idx), ref.numpy(), rtol=1e-12, atol=1e-12)


def test_fwd_scaled_identity_closed_form():
    inp = tiny()
    E, H = inp.spec.E, inp.spec.H
    idx, *_ = oracle.route(inp.gate_logits)
    W = np.stack([np.eye(H, dtype=np.float32) * (e + 2) for e in range(E)])
    out = oracle.fwd(inp.x, W, inp.bias, idx)
    expect = inp.x.astype(np.float64) * (idx[:, None] + 2) + inp.bias[idx].astype(np.float64)
    np.testing.assert_allclose(out, expect, rtol=0, atol=1e-15)


# --------------------------------------------------------------------------- backward

def _loss_rows(inp, idx, x=None, W=None, bias=None, rows=None):
    x = inp.x if x is None else x
    W = inp.W if W is None else W
    bias = inp.bias if bias is None else bias
    if rows is not None:
        r = oracle.fwd(x[rows], W, bias, idx[rows])
        return float(np.sum(r * inp.d_out[rows].astype(np.float64)))
    r = oracle.fwd(x, W, bias, idx)
    return float(np.sum(r * inp.d_out.astype(np.float64)))


def test_dx_finite_difference():
    inp = tiny()
    idx, *_ = oracle.route(inp.gate_logits)
    dx = oracle.bwd_dx(inp.W, inp.d_out, idx)
    rng = np.random.default_rng(3)
    eps = 1e-3
    for _ in range(12):
        t, i = int(rng.integers(inp.spec.T)), int(rng.integers(inp.spec.H))
        xp, xm = inp.x.copy(), inp.x.copy()
        xp[t, i] = np.float32(inp.x[t, i] + eps)
        xm[t, i] = np.float32(inp.x[t, i] - eps)
        h = float(xp[t, i]) - float(xm[t, i])        # the perturbation fp32 really applied
        fd = (_loss_rows(inp, idx, x=xp, rows=[t]) - _loss_rows(inp, idx, x=xm, rows=[t])) / h
        assert abs(fd - dx[t, i]) <= 1e-9 * (1 + abs(dx[t, i])), (t, i, fd, dx[t, i])


def test_dx_identity_weights_return_d_out():
    inp = tiny("tiny_identity_b8_e4_h128")
    idx, *_ = oracle.route(inp.gate_logits)
    np.testing.assert_array_equal(oracle.bwd_dx(inp.W, inp.d_out, idx), inp.d_out.astype(np.float64))


def test_dw_db_finite_difference():
    inp = tiny()
    idx, *_ = oracle.route(inp.gate_logits)
    dW, db, _, _ = oracle.bwd_dw(inp.x, inp.d_out, idx, inp.spec.E)
    rng = np.random.default_rng(4)
    eps = 1e-3
    for _ in range(8):
        e, o, i = (int(rng.integers(inp.spec.E)), int(rng.integers(inp.spec.H)), int(rng.integers(inp.spec.H)))
        Wp, Wm = inp.W.copy(), inp.W.copy()
        Wp[e, o, i] = np.float32(inp.W[e, o, i] + eps)
        Wm[e, o, i] = np.float32(inp.W[e, o, i] - eps)
        h = float(Wp[e, o, i]) - float(Wm[e, o, i])
        fd = (_loss_rows(inp, idx, W=Wp) - _loss_rows(inp, idx, W=Wm)) / h
        assert abs(fd - dW[e, o, i]) <= 1e-8 * (1 + abs(dW[e, o, i])), (e, o, i, fd, dW[e, o, i])
        bp, bm = inp.bias.copy(), inp.bias.copy()
        bp[e, o] = np.float32(inp.bias[e, o] + eps)
        bm[e, o] = np.float32(inp.bias[e, o] - eps)
        h = float(bp[e, o]) - float(bm[e, o])
        fd = (_loss_rows(inp, idx, bias=bp) - _loss_rows(inp, idx, bias=bm)) / h
        assert abs(fd - db[e, o]) <= 1e-8 * (1 + abs(db[e, o]))


def test_bwd_matches_torch_autograd():
    inp = tiny()
    idx, *_ = oracle.route(inp.gate_logits)
    x = torch.from_numpy(inp.x).double().requires_grad_()
    W = torch.from_numpy(inp.W).double().requires_grad_()
    b = torch.from_numpy(inp.bias).double().requires_grad_()
    ix = torch.from_numpy(idx).long()
    y = torch.einsum("toi,ti->to", W[ix], x) + b[ix]
    (y * torch.from_numpy(inp.d_out).double()).sum().backward()
    dW, db, _, _ = oracle.bwd_dw(inp.x, inp.d_out, idx, inp.spec.E)
    np.testing.assert_allclose(oracle.bwd_dx(inp.W, inp.d_out, idx), x.grad.numpy(), rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(dW, W.grad.numpy(), rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(db, b.grad.numpy(), rtol=1e-12, atol=1e-12)


def test_dw_inactive_experts_exactly_zero_and_db_column_sums():
    for name in ["tiny_uniform_b8_e4_h128"]:
        inp = tiny(name)
        idx, counts, *_ = oracle.route(inp.gate_logits)
        dW, db, _, _ = oracle.bwd_dw(inp.x, inp.d_out, idx, inp.spec.E)
        for e in range(inp.spec.E):
            if counts[e] == 0:
                assert np.all(dW[e] == 0.0) and np.all(db[e] == 0.0)
            np.testing.assert_allclose(db[e], inp.d_out[idx == e].astype(np.float64).sum(axis=0),
                                       rtol=1e-12, atol=1e-12)
    inp = wl.generate(wl.make_spec("collapsed_small", 64, 5, 4, 32, 77, logits="binary",
                                   skew_expert=0, skew_value=10.0))
    idx, counts, *_ = oracle.route(inp.gate_logits)
    dW, db, _, _ = oracle.bwd_dw(inp.x, inp.d_out, idx, 4)
    assert np.all(dW[1:] == 0.0) and np.all(db[1:] == 0.0)


def test_dw_entries_match_full_and_scale_is_rss():
    inp = tiny()
    idx, *_ = oracle.route(inp.gate_logits)
    for mode in (oracle.TF32_NONE, oracle.TF32_RZ):
        dW, _, sW, _ = oracle.bwd_dw(inp.x, inp.d_out, idx, inp.spec.E, mode)
        rng = np.random.default_rng(5)
        e = rng.integers(0, 4, 50)
        o = rng.integers(0, 128, 50)
        i = rng.integers(0, 128, 50)
        v, s = oracle.bwd_dw_entries(inp.x, inp.d_out, idx, e, o, i, mode)
        np.testing.assert_allclose(v, dW[e, o, i], rtol=1e-13, atol=1e-13)
        np.testing.assert_allclose(s, sW[e, o, i], rtol=1e-13, atol=1e-13)
    # the scale is the root-sum-of-squares of the terms of the sum
    dW, _, sW, _ = oracle.bwd_dw(inp.x, inp.d_out, idx, inp.spec.E)
    k = 3
    e, o, ii = int(idx[k]), 5, 7
    terms = inp.d_out[idx == e, o].astype(np.float64) * inp.x[idx == e, ii].astype(np.float64)
    assert abs(sW[e, o, ii] - np.sqrt(np.sum(terms ** 2))) < 1e-12
    assert sW[e, o, ii] >= abs(dW[e, o, ii]) - 1e-12


def test_db_alone_matches_column_sums():
    inp = wl.generate(wl.WORKLOADS["skewed_b4096_e8_h128"])
    idx, *_ = oracle.route(inp.gate_logits)
    db, sb = oracle.bwd_db(inp.d_out, idx, 8)
    for e in range(8):
        sel = inp.d_out[idx == e].astype(np.float64)
        np.testing.assert_allclose(db[e], sel.sum(axis=0), rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(sb[e], np.sqrt((sel ** 2).sum(axis=0)), rtol=1e-12, atol=1e-12)


def test_tf32_mode_rounds_gemm_inputs_only():
    inp = tiny()
    idx, *_ = oracle.route(inp.gate_logits)
    r = np.vectorize(lambda v: oracle.tf32_round(v, oracle.TF32_RZ), otypes=[np.float32])
    x_t, W_t, g_t = r(inp.x), r(inp.W), r(inp.d_out)
    np.testing.assert_array_equal(oracle.fwd(inp.x, inp.W, inp.bias, idx, oracle.TF32_RZ),
                                  oracle.fwd(x_t, W_t, inp.bias, idx))
    np.testing.assert_array_equal(oracle.bwd_dx(inp.W, inp.d_out, idx, oracle.TF32_RZ),
                                  oracle.bwd_dx(W_t, g_t, idx))
    a = oracle.bwd_dw(inp.x, inp.d_out, idx, 4, oracle.TF32_RZ)
    b = oracle.bwd_dw(x_t, g_t, idx, 4)
    np.testing.assert_array_equal(a[0], b[0])
    np.testing.assert_array_equal(a[1], oracle.bwd_dw(inp.x, inp.d_out, idx, 4)[1])  # db unrounded


# --------------------------------------------------------------------------- aux loss

def test_aux_uniform_logits_closed_form():
    inp = tiny("tiny_uniform_b8_e4_h128")
    _, counts, *_ = oracle.route(inp.gate_logits)
    lam = 0.03
    res = oracle.aux(inp.gate_logits, counts, lam)
    T, E = inp.spec.T, inp.spec.E
    assert np.all(res["mean_p"] == 1.0 / E)
    assert res["aux_raw"] == 1.0
    frac = counts / T
    lam32 = float(np.float32(lam))
    expect = lam32 * (frac[None, :] - 1.0 / E) / T * np.ones((T, 1))
    np.testing.assert_allclose(res["d_logits"], expect, rtol=1e-14, atol=1e-18)


@pytest.mark.parametrize("counts", [[40, 0, 0, 0], [10, 10, 10, 10], [1, 2, 3, 34]])
def test_aux_uniform_logits_is_one_for_any_routing(counts):
    lg = np.zeros((40, 4), np.float32)
    assert oracle.aux(lg, np.array(counts, np.int32), 0.01)["aux_raw"] == 1.0


def test_aux_rows_sum_to_zero_and_sign():
    inp = wl.generate(wl.WORKLOADS["small_b1024_e4_h128"], with_activations=False)
    _, counts, *_ = oracle.route(inp.gate_logits)
    res = oracle.aux(inp.gate_logits, counts, 0.05)
    d = res["d_logits_unscaled"]
    # sum_j p_j (frac_j - g) = g - g sum_j p_j = 0: zero up to a few ulp of the terms
    # before cancellation, p_j * (frac_j + g).
    T = inp.spec.T
    p = np.exp(inp.gate_logits - inp.gate_logits.max(axis=1, keepdims=True).astype(np.float64))
    p /= p.sum(axis=1, keepdims=True)
    frac = counts / T
    g = (p * frac).sum(axis=1, keepdims=True)
    mag = (p * (frac + g)).sum(axis=1)
    assert np.all(np.abs(d.sum(axis=1)) <= 8 * 2.0 ** -52 * mag)
    assert np.max(np.abs(d.sum(axis=1))) < 1e-15
    # pushing a logit up raises aux when its expert is over-used relative to the token's mix
    assert np.all(res["mean_p"] > 0) and abs(res["mean_p"].sum() - 1.0) < 1e-12


def test_aux_finite_difference_with_frac_frozen():
    inp = wl.generate(wl.WORKLOADS["tiny_b8_e4_h128"], with_activations=False)
    _, counts, *_ = oracle.route(inp.gate_logits)
    lam = 0.05
    res = oracle.aux(inp.gate_logits, counts, lam)
    rng = np.random.default_rng(6)
    eps = 1e-3
    for _ in range(10):
        t, j = int(rng.integers(40)), int(rng.integers(4))
        lp, lm = inp.gate_logits.copy(), inp.gate_logits.copy()
        lp[t, j] = np.float32(lp[t, j] + eps)
        lm[t, j] = np.float32(lm[t, j] - eps)
        h = float(lp[t, j]) - float(lm[t, j])
        fd = (oracle.aux(lp, counts, lam)["loss"] - oracle.aux(lm, counts, lam)["loss"]) / h
        # central difference: O(eps^2) truncation error
        assert abs(fd - res["d_logits"][t, j]) <= 1e-6 * abs(res["d_logits"][t, j]) + 1e-12


def test_aux_matches_torch_autograd():
    inp = wl.generate(wl.WORKLOADS["skewed_b4096_e8_h128"], with_activations=False)
    _, counts, *_ = oracle.route(inp.gate_logits)
    lam = 0.02
    T, E = inp.spec.T, inp.spec.E
    lg = torch.from_numpy(inp.gate_logits).double().requires_grad_()
    frac = torch.from_numpy(counts).double() / T
    mean_p = torch.softmax(lg, dim=1).mean(dim=0)
    aux = E * (frac * mean_p).sum()
    (float(np.float32(lam)) * aux).backward()
    res = oracle.aux(inp.gate_logits, counts, lam)
    assert abs(res["aux_raw"] - aux.item()) <= 1e-12
    np.testing.assert_allclose(res["mean_p"], mean_p.detach().numpy(), rtol=1e-12)
    np.testing.assert_allclose(res["d_logits"], lg.grad.numpy(), rtol=1e-10, atol=1e-18)


def test_aux_empty_batch_is_zero():
    res = oracle.aux(np.zeros((0, 4), np.float32), np.zeros(4, np.int32), 0.01)
    assert res["aux_raw"] == 0.0 and res["loss"] == 0.0 and np.all(res["mean_p"] == 0)


# --------------------------------------------------------------------------- lambda_eff

def _read_rows(name):
    rows = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                rows.append(line.split())
    return rows


def test_lambda_eff_worked_example_from_page():
    rows = _read_rows("lambda_eff_worked_example.txt")
    assert len(rows) == 2
    for K, floor, extra, frac, ent, printed, dec in rows:
        target = float(frac) * math.log(int(K))
        lam = oracle.lambda_eff(float(ent), float(floor), float(extra), target)
        assert abs(lam - float(printed)) <= 0.5 * 10.0 ** -int(dec), (ent, lam, printed)
    # With 4 experts instead of 8 the printed values are not reproduced: the pin
    # really fixes the expert count and the target fraction.
    lam4 = oracle.lambda_eff(1.381, 0.01, 0.09, 0.7 * math.log(4))
    assert abs(lam4 - 0.0146) > 5e-5


def test_lambda_eff_five_regimes():
    K = 8
    target = 0.7 * math.log(K)
    env = {"target": target, "lnK": math.log(K)}
    for regime, expr, expected in _read_rows("lambda_eff_regimes.txt"):
        ent = eval(expr, {}, env)  # expressions of the fixture: target+0.1, target/2, lnK, 0
        lam = oracle.lambda_eff(ent, 0.01, 0.09, target)
        assert abs(lam - float(expected)) <= 1e-12, (regime, lam)


def test_lambda_eff_cold_start_is_floor():
    for K in (2, 4, 8, 32):
        assert oracle.lambda_eff(math.log(K), 0.01, 0.09, 0.7 * math.log(K)) == 0.01


# --------------------------------------------------------------------------- entropy producer

def _scipy_entropy(p):
    from scipy.stats import entropy
    return float(entropy(p))


def test_usage_entropy_matches_scipy_and_closed_forms():
    rng = np.random.default_rng(5)
    for E in (1, 2, 3, 8, 17, 32):
        counts = rng.integers(0, 1000, E).astype(np.int32)
        counts[rng.integers(0, E)] = 0                    # an inactive expert contributes 0 ln 0 = 0
        T = int(counts.sum())
        if T == 0:
            continue
        _, _, h = oracle.usage_entropy_ema(counts, T, 0.5, False, np.full(E, 1.0 / E), 0.0)
        assert abs(h - _scipy_entropy(counts / T)) <= 1e-12 * max(1.0, h)
    for E in (2, 4, 8, 32):                               # uniform usage: ln E
        _, _, h = oracle.usage_entropy_ema(np.full(E, 7, np.int32), 7 * E, 0.1, False, np.full(E, 1.0 / E), 0.0)
        assert abs(h - math.log(E)) <= 1e-14
    _, _, h = oracle.usage_entropy_ema(np.array([0, 0, 9, 0], np.int32), 9, 0.1, False, np.full(4, 0.25), 1.0)
    assert h == 0.0                                       # everything on one expert
    _, _, h = oracle.usage_entropy_ema(np.array([3, 0, 3, 0], np.int32), 6, 0.1, False, np.full(4, 0.25), 1.0)
    assert abs(h - math.log(2)) <= 1e-15                  # two equal halves


def test_usage_entropy_ema_weights_and_limits():
    counts = np.array([10, 30, 0, 60], np.int32)
    T = 100
    frac = counts / T
    h = _scipy_entropy(frac)
    u0, e0 = np.array([0.1, 0.2, 0.3, 0.4]), 0.9
    u, e, _ = oracle.usage_entropy_ema(counts, T, 1.0, False, u0, e0)      # weight 1: the step itself
    np.testing.assert_allclose(u, frac, rtol=0, atol=1e-15)
    assert abs(e - h) <= 1e-15
    u, e, _ = oracle.usage_entropy_ema(counts, T, 0.0, False, u0, e0)      # weight 0: unchanged
    np.testing.assert_array_equal(u, u0)
    assert e == e0
    u, e, _ = oracle.usage_entropy_ema(counts, T, 0.25, False, u0, e0)     # the weighted mean
    np.testing.assert_allclose(u, 0.75 * u0 + 0.25 * frac, rtol=0, atol=1e-15)
    assert abs(e - (0.75 * e0 + 0.25 * h)) <= 1e-15
    assert abs(u.sum() - 1.0) <= 1e-15                                      # still a distribution


def test_usage_entropy_ema_geometric_approach():
    """n updates with the same counts: ent_n = H + (ent_0 - H) (1 - alpha)^n."""
    counts = np.array([50, 25, 25], np.int32)
    alpha = 0.2
    h = _scipy_entropy(counts / 100)
    u, e = np.full(3, 1.0 / 3), math.log(3)
    for n in range(1, 40):
        u, e, _ = oracle.usage_entropy_ema(counts, 100, alpha, False, u, e)
        assert abs(e - (h + (math.log(3) - h) * (1 - alpha) ** n)) <= 1e-13
        np.testing.assert_allclose(u, counts / 100 + (1.0 / 3 - counts / 100) * (1 - alpha) ** n, rtol=0, atol=1e-14)


def test_usage_entropy_reset_is_the_cold_start_and_gives_the_floor():
    """The pages' bootstrap (usage 1/K, entropy ln K) and fold-boundary reset (lambda at its floor)."""
    for E in (2, 4, 8, 32):
        u, e, _ = oracle.usage_entropy_ema(np.arange(E, dtype=np.int32), E * (E - 1) // 2, 0.3, True,
                                           np.zeros(E), 0.123)
        np.testing.assert_array_equal(u, np.full(E, 1.0 / E))
        assert e == math.log(E)
        assert oracle.lambda_eff(e, 0.01, 0.09, 0.7 * math.log(E)) == 0.01


def test_usage_entropy_no_tokens_is_no_observation():
    u0 = np.array([0.5, 0.5])
    u, e, h = oracle.usage_entropy_ema(np.zeros(2, np.int32), 0, 0.5, False, u0, 0.3)
    np.testing.assert_array_equal(u, u0)
    assert e == 0.3 and h == 0.0


# --------------------------------------------------------------------------- backward through the horizon mean

def _collapse_case(B=3, N_H=4, E=3, H=32, seed=11):
    rng = np.random.default_rng(seed)
    T = B * N_H
    x = rng.standard_normal((T, H)).astype(np.float32)
    W = (rng.standard_normal((E, H, H)) / np.sqrt(H)).astype(np.float32)
    bias = (0.1 * rng.standard_normal((E, H))).astype(np.float32)
    logits = rng.standard_normal((T, E)).astype(np.float32)
    g = rng.standard_normal((B, H)).astype(np.float32)
    idx = oracle.route(logits)[0]
    return x, W, bias, g, idx, B, N_H, E, H


def _collapsed_loss(x, W, bias, g, idx, B, N_H):
    """L = sum_b g[b] . mean_h routed[b, h] in float64, straight from the definitions."""
    xd, Wd, bd = x.astype(np.float64), W.astype(np.float64), bias.astype(np.float64)
    routed = np.einsum("toi,ti->to", Wd[idx], xd) + bd[idx]
    ctx_mean = routed.reshape(B, N_H, -1).mean(axis=1)
    return float((g.astype(np.float64) * ctx_mean).sum())


def test_bwd_mean_collapse_finite_differences():
    x, W, bias, g, idx, B, N_H, E, H = _collapse_case()
    got = oracle.bwd_mean_collapse(x, W, g, idx, N_H, E)
    eps = 1e-3
    rng = np.random.default_rng(3)
    for _ in range(6):                                    # d_x entries
        t, i = rng.integers(0, B * N_H), rng.integers(0, H)
        xp, xm = x.astype(np.float64).copy(), x.astype(np.float64).copy()
        xp[t, i] += eps
        xm[t, i] -= eps
        fd = (_collapsed_loss(xp, W, bias, g, idx, B, N_H) - _collapsed_loss(xm, W, bias, g, idx, B, N_H)) / (2 * eps)
        assert abs(got["d_x"][t, i] - fd) <= 1e-8 * max(1.0, abs(fd)), (t, i)
    for _ in range(6):                                    # dW entries, including untouched experts
        e, o, i = rng.integers(0, E), rng.integers(0, H), rng.integers(0, H)
        Wp, Wm = W.astype(np.float64).copy(), W.astype(np.float64).copy()
        Wp[e, o, i] += eps
        Wm[e, o, i] -= eps
        fd = (_collapsed_loss(x, Wp, bias, g, idx, B, N_H) - _collapsed_loss(x, Wm, bias, g, idx, B, N_H)) / (2 * eps)
        assert abs(got["dW"][e, o, i] - fd) <= 1e-8 * max(1.0, abs(fd)), (e, o, i)
    for e in range(E):                                    # db: the mean of g over each expert's tokens' rows
        o = rng.integers(0, H)
        bp, bm = bias.astype(np.float64).copy(), bias.astype(np.float64).copy()
        bp[e, o] += eps
        bm[e, o] -= eps
        fd = (_collapsed_loss(x, W, bp, g, idx, B, N_H) - _collapsed_loss(x, W, bm, g, idx, B, N_H)) / (2 * eps)
        assert abs(got["db"][e, o] - fd) <= 1e-8 * max(1.0, abs(fd)), (e, o)


def test_bwd_mean_collapse_equals_plain_backward_on_the_broadcast_gradient():
    """With N_H a power of two, g / N_H is exact in fp32, so the collapsed backward
    must equal the (separately pinned) plain backward fed d_out = g[b] / N_H."""
    x, W, bias, g, idx, B, N_H, E, H = _collapse_case(N_H=8)
    d_out = np.repeat(g / np.float32(N_H), N_H, axis=0).astype(np.float32)
    for mode in (oracle.TF32_NONE, oracle.TF32_RZ):
        got = oracle.bwd_mean_collapse(x, W, g, idx, N_H, E, mode)
        np.testing.assert_allclose(got["d_x"], oracle.bwd_dx(W, d_out, idx, mode), rtol=1e-15, atol=1e-15)
        dW, db, _, _ = oracle.bwd_dw(x, d_out, idx, E, mode)
        np.testing.assert_allclose(got["dW"], dW, rtol=1e-15, atol=1e-15)
        np.testing.assert_allclose(got["db"], db, rtol=1e-15, atol=1e-15)


# ---------------------------------------------------------------- forward through the horizon mean
def test_fwd_mean_collapse_with_one_horizon_token_is_the_forward():
    x, W, bias, _, idx, B, N_H, E, H = _collapse_case(B=7, N_H=1)
    got, _ = oracle.fwd_mean_collapse(x, W, bias, idx, 1)
    np.testing.assert_array_equal(got, oracle.fwd(x, W, bias, idx))


def test_fwd_mean_collapse_is_the_horizon_mean_of_the_forward():
    x, W, bias, _, idx, B, N_H, E, H = _collapse_case(B=4, N_H=5)
    got, _ = oracle.fwd_mean_collapse(x, W, bias, idx, N_H)
    want = oracle.fwd(x, W, bias, idx).reshape(B, N_H, H).mean(axis=1)
    np.testing.assert_allclose(got, want, rtol=1e-13, atol=1e-14)


def test_fwd_mean_collapse_identity_experts_average_x():
    x, _, _, _, idx, B, N_H, E, H = _collapse_case(B=5, N_H=6)
    W = np.broadcast_to(np.eye(H, dtype=np.float32), (E, H, H)).copy()
    got, mag = oracle.fwd_mean_collapse(x, W, np.zeros((E, H), np.float32), idx, N_H)
    np.testing.assert_allclose(got, x.astype(np.float64).reshape(B, N_H, H).mean(axis=1), rtol=1e-15, atol=1e-15)
    np.testing.assert_allclose(mag, np.abs(x.astype(np.float64)).reshape(B, N_H, H).mean(axis=1), rtol=1e-15)


def test_fwd_mean_collapse_of_zero_input_averages_the_chosen_biases():
    x, W, bias, _, idx, B, N_H, E, H = _collapse_case(B=6, N_H=7, E=4)
    got, _ = oracle.fwd_mean_collapse(np.zeros_like(x), W, bias, idx, N_H)
    want = bias.astype(np.float64)[idx.reshape(B, N_H)].mean(axis=1)
    np.testing.assert_allclose(got, want, rtol=1e-15, atol=1e-17)


def test_fwd_mean_collapse_does_not_depend_on_the_horizon_order():
    x, W, bias, _, idx, B, N_H, E, H = _collapse_case(B=4, N_H=6)
    perm = np.random.default_rng(5).permutation(N_H)
    xs = x.reshape(B, N_H, H)[:, perm].reshape(B * N_H, H)
    ids = idx.reshape(B, N_H)[:, perm].reshape(-1)
    a, ma = oracle.fwd_mean_collapse(x, W, bias, idx, N_H)
    b, mb = oracle.fwd_mean_collapse(xs, W, bias, ids, N_H)
    np.testing.assert_allclose(a, b, rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(ma, mb, rtol=1e-13)


def test_fwd_mean_collapse_is_the_adjoint_of_the_pinned_backward():
    """ctx_mean is affine in x and its linear part is adjoint to the collapsed
    input gradient: sum_b g[b] . (ctx(x) - ctx(0)) = sum_t d_x[t] . x[t]."""
    x, W, bias, g, idx, B, N_H, E, H = _collapse_case(B=5, N_H=3, E=4)
    cx, _ = oracle.fwd_mean_collapse(x, W, bias, idx, N_H)
    c0, _ = oracle.fwd_mean_collapse(np.zeros_like(x), W, bias, idx, N_H)
    lhs = float((g.astype(np.float64) * (cx - c0)).sum())
    d_x = oracle.bwd_mean_collapse(x, W, g, idx, N_H, E, with_dw=False)["d_x"]
    rhs = float((d_x * x.astype(np.float64)).sum())
    assert abs(lhs - rhs) <= 1e-11 * max(1.0, abs(lhs)), (lhs, rhs)


def test_fwd_mean_collapse_magnitude_bounds_the_value_and_is_exact_for_positive_terms():
    x, W, bias, _, idx, B, N_H, E, H = _collapse_case(B=4, N_H=5)
    got, mag = oracle.fwd_mean_collapse(x, W, bias, idx, N_H)
    assert np.all(np.abs(got) <= mag * (1 + 1e-14))
    got, mag = oracle.fwd_mean_collapse(np.abs(x), np.abs(W), np.abs(bias), idx, N_H)
    np.testing.assert_allclose(mag, got, rtol=1e-14)


# ---------------------------------------------------------------- the same mean as a contraction over summed inputs
def _small_integer_case(B=5, N_H=6, E=4, H=32, seed=21):
    """Inputs whose fp32 horizon sums are exact (small integers), so the pre-summed
    form must agree with the definition to double rounding."""
    rng = np.random.default_rng(seed)
    x = rng.integers(-8, 9, size=(B * N_H, H)).astype(np.float32)
    W = (rng.integers(-4, 5, size=(E, H, H)) / 16.0).astype(np.float32)
    bias = (rng.integers(-4, 5, size=(E, H)) / 8.0).astype(np.float32)
    idx = oracle.route(rng.standard_normal((B * N_H, E)).astype(np.float32))[0]
    return x, W, bias, idx, B, N_H, E, H


def test_presum_horizon_mean_equals_the_definition_when_the_sums_are_exact():
    x, W, bias, idx, B, N_H, E, H = _small_integer_case()
    want, _ = oracle.fwd_mean_collapse(x, W, bias, idx, N_H)
    for mode in (oracle.TF32_NONE, oracle.TF32_RZ):  # integers and multiples of 1/16 are TF32 values
        got = oracle.fwd_mean_collapse_presum(x, W, bias, idx, N_H, mode)
        np.testing.assert_allclose(got, want, rtol=1e-14, atol=1e-14)


def test_presum_horizon_mean_with_one_horizon_token_is_the_tf32_forward():
    x, W, bias, _, idx, B, N_H, E, H = _collapse_case(B=9, N_H=1, E=4)
    for mode in (oracle.TF32_NONE, oracle.TF32_RZ, oracle.TF32_RNE):
        got = oracle.fwd_mean_collapse_presum(x, W, bias, idx, 1, mode)
        np.testing.assert_allclose(got, oracle.fwd(x, W, bias, idx, mode), rtol=1e-14, atol=1e-15)


def test_presum_horizon_mean_counts_each_expert_bias_once_per_token():
    # zero input: only the biases remain, n_be of expert e's bias per row
    x, W, bias, _, idx, B, N_H, E, H = _collapse_case(B=6, N_H=7, E=4)
    got = oracle.fwd_mean_collapse_presum(np.zeros_like(x), W, bias, idx, N_H, oracle.TF32_RZ)
    want = bias.astype(np.float64)[idx.reshape(B, N_H)].mean(axis=1)
    np.testing.assert_allclose(got, want, rtol=1e-15, atol=1e-17)
    # an expert index outside [0, E) contributes nothing (zero input, bias only)
    bad = idx.copy()
    bad[0] = E
    got = oracle.fwd_mean_collapse_presum(np.zeros_like(x), W, bias, bad, N_H, oracle.TF32_NONE)
    keep = idx.reshape(B, N_H).copy()
    want = bias.astype(np.float64)[keep]
    want[0, 0] = 0.0
    np.testing.assert_allclose(got, want.sum(axis=1) / N_H, rtol=1e-15, atol=1e-17)


def test_presum_horizon_mean_tf32_error_within_the_operand_rounding_bound():
    """Cutting X_be and W to 10 mantissa bits changes each product by less than
    2 * 2^-10 of its size; the fp32 horizon sums add at most N_H roundings of
    2^-24 each. So |tf32 - exact| <= (2^-9 + N_H 2^-24) * mag, and truncation
    (RZ) of positive operands can only lower the result."""
    x, W, bias, _, idx, B, N_H, E, H = _collapse_case(B=6, N_H=5, E=3, H=64)
    exact, mag = oracle.fwd_mean_collapse(x, W, bias, idx, N_H)
    got = oracle.fwd_mean_collapse_presum(x, W, bias, idx, N_H, oracle.TF32_RZ)
    assert np.all(np.abs(got - exact) <= (2.0 ** -9 + N_H * 2.0 ** -23) * mag)
    assert np.any(got != exact)  # the rounding does act
    xp, Wp, bp = np.abs(x), np.abs(W), np.abs(bias)
    exact, _ = oracle.fwd_mean_collapse(xp, Wp, bp, idx, N_H)
    none = oracle.fwd_mean_collapse_presum(xp, Wp, bp, idx, N_H, oracle.TF32_NONE)
    rz = oracle.fwd_mean_collapse_presum(xp, Wp, bp, idx, N_H, oracle.TF32_RZ)
    assert np.all(rz <= none)
    np.testing.assert_allclose(none, exact, rtol=N_H * 2.0 ** -23)


def test_presum_horizon_mean_sums_the_horizon_in_fp32_ascending():
    # one row, two horizon tokens on one expert: X = fl32(x0 + x1); with x0 = 1,
    # x1 = 2^-24 the fp32 sum rounds to 1 (the definition keeps 1 + 2^-24)
    H, E, N_H = 32, 1, 2
    x = np.zeros((N_H, H), np.float32)
    x[0, 0], x[1, 0] = 1.0, 2.0 ** -24
    W = np.zeros((E, H, H), np.float32)
    W[0, 0, 0] = 1.0
    idx = np.zeros(N_H, np.int32)
    got = oracle.fwd_mean_collapse_presum(x, W, np.zeros((E, H), np.float32), idx, N_H, oracle.TF32_NONE)
    assert got[0, 0] == 0.5
    exact, _ = oracle.fwd_mean_collapse(x, W, np.zeros((E, H), np.float32), idx, N_H)
    assert exact[0, 0] == (1.0 + 2.0 ** -24) / 2
