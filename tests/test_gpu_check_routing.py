"""moe_top1_check_routing on the GPU: routings written by moe_top1_route pass;
each kind of malformed routing, built on the host, sets MOE_FLAG_BAD_ROUTING.
The check reads only the routing arrays, so none of these cases can make a
kernel touch memory outside them."""
import numpy as np
import pytest
import torch

import oracle
from bwd_route_b200 import ops
from bwd_route_b200 import workloads as wl
from gpu_harness import dev

pytestmark = pytest.mark.gpu


def _flags(idx, counts, offsets, perm, T, E):
    r = ops.Routing(dev(np.asarray(idx, np.int32)), dev(np.asarray(counts, np.int32)),
                    dev(np.asarray(offsets, np.int32)), dev(np.asarray(perm, np.int32)))
    ws = ops.new_workspace(T, E, 0, "cuda")
    ops.moe_top1_check_routing(r, T, E, ws)
    return ops.moe_top1_device_flags(ws)


@pytest.mark.parametrize("name", ["tiny_b8_e4_h128", "skewed_b4096_e8_h128", "collapsed_b16384_e4_h128"])
def test_routing_from_the_library_passes(name):
    spec = wl.WORKLOADS[name]
    inp = wl.generate(spec, with_activations=False)
    r = ops.Routing.empty(spec.T, spec.E, "cuda")
    ws = ops.new_workspace(spec.T, spec.E, 0, "cuda")
    ops.moe_top1_route(dev(inp.gate_logits), spec.B, spec.N_H, spec.E, r, ws)
    ops.moe_top1_check_routing(r, spec.T, spec.E, ws)
    assert ops.moe_top1_device_flags(ws) == 0


def _good(T=5000, E=7, seed=3):
    lg = np.random.default_rng(seed).standard_normal((T, E)).astype(np.float32)
    return [np.array(a) for a in oracle.route(lg)], T, E


def _corrupt(kind):
    (idx, counts, offsets, perm), T, E = _good()
    if kind == "offsets not monotone":
        offsets[3], offsets[4] = offsets[4], offsets[3]
    elif kind == "offsets end short of T":
        offsets[E] = T - 1
    elif kind == "offsets start above 0":
        offsets[0] = 1
    elif kind == "counts disagree with offsets":
        counts[2] += 1
    elif kind == "perm entry past T":
        perm[1234] = T
    elif kind == "perm entry negative":
        perm[17] = -5
    elif kind == "perm out of order in a segment":
        k = offsets[2] + 10
        perm[k], perm[k + 1] = perm[k + 1], perm[k]
    elif kind == "token in another expert's segment":
        # swap one token of expert 1 with one of expert 2: each segment stays
        # sorted only by luck, but the expert of each moved token is wrong
        a, b = offsets[1], offsets[2]
        perm[a], perm[b] = perm[b], perm[a]
    elif kind == "duplicate token":
        k = offsets[4] + 3
        perm[k + 1] = perm[k]
    elif kind == "expert index out of range":
        idx[perm[offsets[5]]] = E
    elif kind == "routing of another batch":
        # this batch's expert indices with another batch's counts, offsets and perm
        (_, counts, offsets, perm), _, _ = _good(seed=4)
    else:
        raise ValueError(kind)
    return idx, counts, offsets, perm, T, E


KINDS = ["offsets not monotone", "offsets end short of T", "offsets start above 0", "counts disagree with offsets",
         "perm entry past T", "perm entry negative", "perm out of order in a segment",
         "token in another expert's segment", "duplicate token", "expert index out of range",
         "routing of another batch"]


def test_well_formed_host_routing_passes():
    (idx, counts, offsets, perm), T, E = _good()
    assert _flags(idx, counts, offsets, perm, T, E) == 0


@pytest.mark.parametrize("kind", KINDS)
def test_malformed_routing_is_flagged(kind):
    idx, counts, offsets, perm, T, E = _corrupt(kind)
    assert _flags(idx, counts, offsets, perm, T, E) == ops.MOE_FLAG_BAD_ROUTING


def test_empty_routing():
    E = 3
    assert _flags(np.zeros(1, np.int32), np.zeros(E), np.zeros(E + 1), np.zeros(1, np.int32), 0, E) == 0
    assert _flags(np.zeros(1, np.int32), np.zeros(E), [0, 0, 1, 0], np.zeros(1, np.int32), 0, E) == \
        ops.MOE_FLAG_BAD_ROUTING
