"""moe_top1_route_noalloc: routing for callers that cannot allocate device memory.

Such callers (a plug-in that only receives tensors from a host framework owning
all device memory, or a runtime that forbids allocation once running) cannot
hand the library a workspace, so this entry point keeps the routing scratch in a
fixed device array inside the library. Its results must be exactly those of
moe_top1_route, which takes a workspace, on two calls in a row -- the second call
finds the first call's contents still in the shared array.

The file sorts last so that a run stopping at the first failure has already run
every other test; it also passes alone in a fresh process.
"""
import numpy as np
import pytest
import torch

from bwd_route_b200 import ops
from bwd_route_b200 import workloads as wl

pytestmark = pytest.mark.gpu


def _route_both(spec):
    inp = wl.generate(spec, with_activations=False)
    B, N_H, E, T = spec.B, spec.N_H, spec.E, spec.T
    logits = torch.from_numpy(inp.gate_logits).cuda()
    ref = ops.Routing.empty(T, E, "cuda")
    ws = ops.new_workspace(T, E, spec.H, "cuda")
    ops.moe_top1_route(logits, B, N_H, E, ref, ws)
    got = ops.Routing.empty(T, E, "cuda")
    for t in (got.expert_idx, got.counts, got.offsets, got.perm):
        t.fill_(-7)  # stale values must be overwritten
    ops.moe_top1_route_noalloc(logits, B, N_H, E, got)
    torch.cuda.synchronize()
    return ref, got


def test_noalloc_route_equals_workspace_route_on_two_calls_in_a_row():
    # a larger call first, then a smaller one with other E: the second call sees
    # the first call's scratch contents, which must not leak into its results
    first = wl.WORKLOADS["skewed_b4096_e8_h128"]                      # 20,480 tokens, E 8
    second = wl.make_spec("noalloc_b1025_e5_h128", 1025, 3, 5, 128, 33)  # 3,075 tokens, E 5
    for spec in (first, second):
        ref, got = _route_both(spec)
        for name in ("expert_idx", "counts", "offsets", "perm"):
            a, b = getattr(ref, name).cpu().numpy(), getattr(got, name).cpu().numpy()
            np.testing.assert_array_equal(b, a, err_msg=f"{spec.name}: {name}")


def test_noalloc_route_rejects_more_tokens_than_its_scratch_holds():
    E = 4
    T = ops.MOE_NOALLOC_MAX_TOKENS + 1
    logits = torch.zeros(T, E, dtype=torch.float32, device="cuda")
    r = ops.Routing.empty(T, E, "cuda")
    with pytest.raises(ops.MoeError) as err:
        ops.moe_top1_route_noalloc(logits, T, 1, E, r)
    assert err.value.status_name == "MOE_ERR_UNSUPPORTED_SHAPE"
    # at the limit it runs
    T = ops.MOE_NOALLOC_MAX_TOKENS
    logits = torch.zeros(T, E, dtype=torch.float32, device="cuda")
    r = ops.Routing.empty(T, E, "cuda")
    ops.moe_top1_route_noalloc(logits, T, 1, E, r)
    torch.cuda.synchronize()
    assert r.counts.cpu().tolist() == [T, 0, 0, 0]


def test_noalloc_route_fills_the_whole_array_at_the_limit_with_32_experts():
    # T = MOE_NOALLOC_MAX_TOKENS and E = 32 use every entry of the fixed array
    # (2048 routing blocks x 32 experts, counts and bases): the result must still
    # be exactly moe_top1_route's
    E = 32
    T = ops.MOE_NOALLOC_MAX_TOKENS
    g = torch.Generator(device="cuda").manual_seed(7)
    logits = torch.randint(0, 4, (T, E), generator=g, device="cuda").to(torch.float32)  # many ties
    ref = ops.Routing.empty(T, E, "cuda")
    ws = ops.new_workspace(T, E, 0, "cuda")
    ops.moe_top1_route(logits, T, 1, E, ref, ws)
    got = ops.Routing.empty(T, E, "cuda")
    for t in (got.expert_idx, got.counts, got.offsets, got.perm):
        t.fill_(-7)
    ops.moe_top1_route_noalloc(logits, T, 1, E, got)
    torch.cuda.synchronize()
    for name in ("expert_idx", "counts", "offsets", "perm"):
        assert torch.equal(getattr(got, name), getattr(ref, name)), name


def test_noalloc_route_with_no_tokens_zeroes_counts_and_offsets():
    E = 6
    r = ops.Routing(torch.empty(0, dtype=torch.int32, device="cuda"),
                    torch.full((E,), 9, dtype=torch.int32, device="cuda"),
                    torch.full((E + 1,), 9, dtype=torch.int32, device="cuda"),
                    torch.empty(0, dtype=torch.int32, device="cuda"))
    ops.moe_top1_route_noalloc(torch.empty(0, E, device="cuda"), 0, 4, E, r)
    torch.cuda.synchronize()
    assert r.counts.cpu().tolist() == [0] * E
    assert r.offsets.cpu().tolist() == [0] * (E + 1)
