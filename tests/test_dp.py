"""The data-parallel exchange (bwd_route_b200.dp) on CPU with two gloo ranks:
each rank holds half of the batch and its oracle results; after the exchange
every rank must hold the full batch's dW, db and expert counts."""
import datetime
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from bwd_route_b200 import dp
from bwd_route_b200 import workloads as wl

SPEC = wl.make_spec("dp_b96_h5_e4_h128", 96, 5, 4, 128, 41, skew_expert=1, skew_value=0.5)
WORLD = 2


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _init(rank, port):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=WORLD, timeout=datetime.timedelta(seconds=30))


def _shard(a, rank):
    n = a.shape[0] // WORLD
    return a[rank * n:(rank + 1) * n]


def _rank_exchange(rank, port, out):
    _init(rank, port)
    try:
        inp = wl.generate(SPEC)
        E, H = SPEC.E, SPEC.H
        logits, x, d_out = (_shard(a, rank) for a in (inp.gate_logits, inp.x, inp.d_out))
        idx, counts = oracle.route(logits)[:2]
        dW, db, _, _ = oracle.bwd_dw(x, d_out, idx, E)
        grads = torch.from_numpy(np.concatenate([dW.ravel(), db.ravel()]).astype(np.float32))
        local = torch.from_numpy(np.asarray(counts, np.int32).copy())
        total = torch.zeros(E, dtype=torch.int32)
        out[("tokens", rank)] = dp.world_tokens(logits.shape[0], "cpu")
        dp.allreduce_gradients(grads)
        dp.global_counts(local, total)
        out[("grads", rank)] = grads.numpy().tobytes()
        out[("counts", rank)] = total.numpy().tolist()
        out[("local", rank)] = (local.numpy().tolist(), np.asarray(counts).tolist())
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(120)
def test_exchange_gives_every_rank_the_full_batch_results():
    out = mp.get_context("spawn").Manager().dict()
    mp.spawn(_rank_exchange, args=(_free_port(), out), nprocs=WORLD, join=True)
    inp = wl.generate(SPEC)
    E, H, T = SPEC.E, SPEC.H, SPEC.T
    idx, counts = oracle.route(inp.gate_logits)[:2]
    dW, db, sW, sb = oracle.bwd_dw(inp.x, inp.d_out, idx, E)
    # identical on every rank, bit for bit
    assert out[("grads", 0)] == out[("grads", 1)]
    got = np.frombuffer(out[("grads", 0)], np.float32).astype(np.float64)
    got_dW, got_db = got[:E * H * H].reshape(E, H, H), got[E * H * H:].reshape(E, H)
    # two fp32-rounded partials and one fp32 add: a few ulps of the sum's magnitude
    for name, g, o, s in (("dW", got_dW, dW, sW), ("db", got_db, db, sb)):
        err = np.abs(g - o) / np.maximum(np.maximum(np.abs(o), s), 1e-30)
        assert err.max() < 4e-7, (name, err.max())
    # counts: exact, the full batch's, on both ranks; the local counts untouched
    assert out[("counts", 0)] == out[("counts", 1)] == np.asarray(counts).tolist()
    for r in range(WORLD):
        assert out[("local", r)][0] == out[("local", r)][1]
        assert out[("tokens", r)] == T
    # and the controller signal built from them is the full batch's on every rank
    u0 = np.full(E, 1.0 / E)
    want = oracle.usage_entropy_ema(counts, T, 0.3, False, u0, 0.5)
    got_c = oracle.usage_entropy_ema(np.asarray(out[("counts", 1)], np.int32), out[("tokens", 1)], 0.3, False,
                                     u0, 0.5)
    np.testing.assert_array_equal(got_c[0], want[0])
    assert got_c[1:] == want[1:]


def _rank_unequal(rank, port, out):
    _init(rank, port)
    try:
        dp.world_tokens(100 + rank, "cpu")
        out[rank] = "accepted"
    except ValueError as e:
        out[rank] = str(e)
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(120)
def test_unequal_shards_are_rejected_on_every_rank():
    out = mp.get_context("spawn").Manager().dict()
    mp.spawn(_rank_unequal, args=(_free_port(), out), nprocs=WORLD, join=True)
    assert "differ in size" in out[0] and "differ in size" in out[1]


def test_argument_checks_need_no_process_group():
    with pytest.raises(ValueError):
        dp.allreduce_gradients(torch.zeros(4, dtype=torch.float64))
    with pytest.raises(ValueError):
        dp.allreduce_gradients(torch.zeros(4, 2).t())
    with pytest.raises(ValueError):
        dp.global_counts(torch.zeros(4, dtype=torch.int64), torch.zeros(4, dtype=torch.int32))
    with pytest.raises(ValueError):
        dp.global_counts(torch.zeros(4, dtype=torch.int32), torch.zeros(3, dtype=torch.int32))
