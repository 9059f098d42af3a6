"""Host-side pieces of bench.py (no GPU): the algorithmic bytes and flops the
roofline is computed from, the FP32 SIMT ceiling of the FFMA path, the L2 note
and the traffic record lookup."""
import json
import os

import bench
from bwd_route_b200 import workloads as wl

LARGE = wl.WORKLOADS["large_b65536_e8_h256"]


def test_algorithmic_bytes_and_flops_of_the_throughput_workload():
    T, E, H = LARGE.T, LARGE.E, LARGE.H
    step_bytes, step_flops, per = bench.algorithmic(LARGE)
    # x twice, d_out once, routed and d_x written: 5 H floats; logits twice and d_logits: 3 E floats;
    # expert_idx written, perm written and read: 16 bytes; W read and dW written per step
    assert step_bytes == T * (4 * (5 * H + 3 * E) + 16) + 2 * E * H * H * 4
    assert abs(step_bytes - 5.49e9) < 0.01e9
    assert step_flops == 6 * H * H * T
    assert per["fwd"] == T * (8 * H + 4) + E * H * H * 4 + E * H * 4
    # the backward call reads x and d_out once and writes d_x: 12 H bytes per token
    assert per["bwd"] == T * (12 * H + 4) + 2 * E * H * H * 4 + E * H * 4
    # the step's bytes are the two calls' plus the routing and aux traffic (logits read
    # twice, d_logits written, expert_idx written, perm written), less what the calls
    # count and the step does not (W read by both calls but counted once, bias and db)
    assert step_bytes - (per["fwd"] + per["bwd"]) == T * (4 * 3 * E + 8) - E * H * H * 4 - 2 * E * H * 4
    # the step roofline quoted in the docs: HBM-bound at the measured 6541 GB/s
    assert abs(step_bytes / 6541e9 * 1e6 - 839) < 1


def test_algorithmic_bytes_with_the_horizon_mean_gradient():
    T, E, H, B = LARGE.T, LARGE.E, LARGE.H, LARGE.B
    full, flops, per = bench.algorithmic(LARGE)
    coll, flops_c, per_c = bench.algorithmic(LARGE, "mean_collapse")
    assert flops_c == flops
    # d_out [T, H] is read once and routed [T, H] written once in the plain step;
    # the [B, H] gradient and the [B, H] mean replace them
    assert full - coll == 2 * (T * H * 4 - B * H * 4)
    assert per["bwd"] - per_c["bwd"] == T * H * 4 - B * H * 4
    assert per["fwd"] - per_c["fwd"] == T * H * 4 - B * H * 4


def test_fp32_simt_ceiling_and_l2_note():
    r = bench.simt_roofline(74.44992e12 * 1e-3, 1.0)  # exactly the peak for 1 ms
    assert abs(r["frac"] - 1.0) < 1e-9 and r["bound"] == "alu"
    assert "larger than L2" in bench.l2_note(LARGE, False, False)
    assert "fit in L2" in bench.l2_note(wl.WORKLOADS["tiny_b8_e4_h128"], False, False)
    assert "256 MB" in bench.l2_note(wl.WORKLOADS["tiny_b8_e4_h128"], False, True)


def test_traffic_record_is_well_formed_and_keyed_to_the_sources():
    text = open(bench.TRAFFIC_RECORD).read()
    data = json.loads(text.split("```json", 1)[1].split("```", 1)[0])
    recs = {(r["workload"], r["grad"]): r for r in data["records"]}
    assert set(recs) == {(LARGE.name, "token"), (LARGE.name, "mean_collapse")}
    for (_, grad), rec in recs.items():
        assert rec["math"] == "tf32"
        for f in rec["source_files"]:
            assert os.path.exists(os.path.join(bench.HERE, f)), f
        mid = wl.WORKLOADS[rec["measured_workload"]]
        assert (mid.E, mid.H, mid.N_H) == (LARGE.E, LARGE.H, LARGE.N_H) and rec["token_scale"] == LARGE.T / mid.T
        _, _, per = bench.algorithmic(LARGE, grad)
        assert set(rec["traffic_bytes_per_call"]) == {"fwd", "bwd"}
        for call, v in rec["traffic_bytes_per_call"].items():
            # the scaled figure is the stated rule applied to the stored measurement
            assert v == bench.scale_traffic(rec["measured_bytes_per_call"][call], rec["fixed_bytes_per_call"][call],
                                            rec["token_scale"])
            # the fixed part is W (and bias, or the partial-sum slots): far below the token part
            assert LARGE.E * LARGE.H * LARGE.H * 4 <= rec["fixed_bytes_per_call"][call] < 0.05 * v
            # the method's minimum bytes: d_out and x once; the two-pass backward reads d_out
            # once per pass (about 1.24 at this shape), the single pass once
            hi = 1.35 if (call == "bwd" and rec["bwd_passes"] == 2) else 1.1
            assert 0.85 < v / per[call] < hi, (grad, call, v / per[call])
        assert rec["bwd_passes"] == bench.bwd_passes("tf32", grad, LARGE.H, LARGE.T)
    # the lookup refuses other workloads, the FFMA path and a gradient mode with no record
    assert bench.recorded_traffic("fwd", "mid_b16384_e8_h256", "tf32") is None
    assert bench.recorded_traffic("fwd", LARGE.name, "ffma") is None
    assert bench.recorded_traffic("fwd", LARGE.name, "tf32", "other") is None


def test_traffic_scaling_rule():
    # fixed part kept, token part times the ratio
    assert bench.scale_traffic(1000, 100, 4) == 100 + 900 * 4
    assert bench.scale_traffic(100, 100, 4) == 100


def test_backward_strategy_rule_agrees_across_the_library_and_the_python_side():
    """The default TF32 backward strategy is decided in the library
    (bwd_single_pass_default in csrc/internal.h); the benchmark's pass count and
    the gate's launch count restate it. All three must agree: one pass for the
    horizon-mean gradient at H = 256 and at H = 128 above the library's threshold."""
    import re
    from bwd_route_b200 import ops
    from bwd_route_b200.gate import MoETop1Gate
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    src = open(os.path.join(root, "bwd_route_b200", "csrc", "internal.h")).read()
    limit = int(re.search(r"constexpr int64_t kBwdSinglePassMinT128 = (\d+);", src).group(1))
    assert "return (collapse && H == 256) || (H == 128 && T > kBwdSinglePassMinT128);" in src
    for H in (128, 256):
        for T in (1, limit - 1, limit, limit + 1, 4 * limit):
            for grad in ("token", "mean_collapse"):
                collapse = grad == "mean_collapse"
                lib = (collapse and H == 256) or (H == 128 and T > limit)
                assert bench.bwd_passes("tf32", grad, H, T) == (1 if lib else 2), (H, T, grad)
                assert bench.bwd_passes("ffma", grad, H, T) == 2
                n_tf32 = MoETop1Gate.launches_per_step(ops.MOE_MATH_TF32, H, T, 8, collapse)
                n_ffma = MoETop1Gate.launches_per_step(ops.MOE_MATH_FFMA, H, T, 8, collapse)
                assert n_ffma - n_tf32 == (1 if lib else 0), (H, T, grad)
