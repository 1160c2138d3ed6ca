"""Sequence sharding (nonlinear_rnn_paragru_b200.shard) on CPU: the exchange
logic of the sharded Newton solve on two gloo ranks, against one process.

The per-shard steps run in an fp64 CPU engine written here from the pages'
algorithm ("Параллельность RNN?", §1.2-§1.3: evaluate, solve the shard's
bidiagonal system by forward substitution from a zero incoming delta, then
add P_t ds_in), with the cell values and Jacobians of the oracle's step
functions.  What is under test is the driver: the exchange of maps, last
states and max|r|, the composition into each shard's incoming delta and next
initial state, and the global stopping rule.  The CUDA engine is checked on a
GPU in tests/test_shard_gpu.py.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from nonlinear_rnn_paragru_b200 import PARARNN_GRU, PARARNN_LSTM
from nonlinear_rnn_paragru_b200 import shard as sh
from nonlinear_rnn_paragru_b200.inputs import WORKLOADS, make_inputs

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
F64 = torch.float64


class Fp64Engine:
    """The three per-shard steps in float64 on the CPU."""

    def eval(self, s):
        B, Ts, D, S = s.B, s.Ts, s.D, s.S
        u = s.u.to(F64)
        a, bias = s.a.to(F64), s.bias.to(F64)
        G = u.shape[2]
        ug = u.permute(0, 1, 3, 2).reshape(-1, G).numpy()            # [(b,t,d), G]
        ag = a.t().repeat(B * Ts, 1).numpy()
        bg = bias.t().repeat(B * Ts, 1).numpy()
        hp = torch.cat([s.bound[S - 1][:, None], s.h[:, :-1]], 1)
        if S == 1:
            f, A, _, _ = oracle.gru_step(hp.reshape(-1).numpy(), ug, ag, bg)
            A = torch.from_numpy(A).reshape(B, Ts, D)
            r = s.h - torch.from_numpy(f).reshape(B, Ts, D)
            x, P = torch.zeros(B, D, dtype=F64), torch.ones(B, D, dtype=F64)
            xs, Ps = [], []
            for t in range(Ts):            # forward substitution from zero
                x = A[:, t] * x - r[:, t]
                P = A[:, t] * P
                xs.append(x)
                Ps.append(P)
            s._x, s._P = torch.stack(xs, 1), torch.stack(Ps, 1)
            s.agg[0], s.agg[1] = P, x
            s.last[0] = s.h[:, -1]
            res = r
        else:
            cp = torch.cat([s.bound[0][:, None], s.c[:, :-1]], 1)
            fc, fh, A, _, _ = oracle.lstm_step(cp.reshape(-1).numpy(), hp.reshape(-1).numpy(),
                                               ug, ag, bg)
            A = torch.from_numpy(A).reshape(B, Ts, D, 2, 2)
            rc = s.c - torch.from_numpy(fc).reshape(B, Ts, D)
            rh = s.h - torch.from_numpy(fh).reshape(B, Ts, D)
            x = torch.zeros(B, D, 2, dtype=F64)
            P = torch.eye(2, dtype=F64).expand(B, D, 2, 2).clone()
            xs, Ps = [], []
            for t in range(Ts):
                x = torch.einsum("bdij,bdj->bdi", A[:, t], x) - torch.stack([rc[:, t], rh[:, t]], -1)
                P = torch.einsum("bdij,bdjk->bdik", A[:, t], P)
                xs.append(x)
                Ps.append(P)
            s._x, s._P = torch.stack(xs, 1), torch.stack(Ps, 1)   # [B,Ts,D,2], [B,Ts,D,2,2]
            s.agg[0], s.agg[1], s.agg[2], s.agg[3] = P[..., 0, 0], P[..., 0, 1], P[..., 1, 0], P[..., 1, 1]
            s.agg[4], s.agg[5] = x[..., 0], x[..., 1]
            s.last[0], s.last[1] = s.c[:, -1], s.h[:, -1]
            res = torch.cat([rc, rh])
        s.rmax[0] = res.abs().max()      # NaN propagates

    def combine(self, s, aggs, lasts):
        x = torch.zeros(s.S, s.B, s.D, dtype=F64)
        for q in range(s.index):
            A = aggs[q]
            if s.S == 1:
                x = A[0:1] * x + A[1:2]
            else:
                x = torch.stack([A[0] * x[0] + A[1] * x[1] + A[4],
                                 A[2] * x[0] + A[3] * x[1] + A[5]])
        s.din.copy_(x)
        if s.index > 0:
            s.next_bound.copy_(lasts[s.index - 1] + x)

    def apply(self, s):
        if s.S == 1:
            s.h += s._x + s._P * s.din[0][:, None]
        else:
            d = s.din.permute(1, 2, 0)[:, None, :, :, None]                 # [B,1,D,2,1]
            ds = s._x + (s._P @ d)[..., 0]
            s.c += ds[..., 0]
            s.h += ds[..., 1]
        if s.index > 0:
            s.bound.copy_(s.next_bound)


def _inputs(cell, B, T, D):
    w = (WORKLOADS[2] if cell == "gru" else WORKLOADS[5]).scaled(B=B, T=T, D=D)
    x = make_inputs(w)
    g = torch.Generator().manual_seed(41)
    x["h0"] = torch.randn((B, D), generator=g) * 0.5
    if cell == "lstm":
        x["c0"] = torch.randn((B, D), generator=g) * 0.5
    return x


def _shards(cell, x, ranges):
    c = PARARNN_GRU if cell == "gru" else PARARNN_LSTM
    return [sh.Shard(r, c, x["u"][:, t0:t1].to(F64), x["a"], x["bias"], x.get("c0"), x["h0"],
                     dtype=F64) for r, (t0, t1) in enumerate(ranges)]


def _local(cell, x, world, **kw):
    T = x["u"].shape[1]
    shards = _shards(cell, x, sh.split_steps(T, world))
    st = sh.sharded_solve(shards, sh.LocalExchange(), Fp64Engine(), **kw)
    h = torch.cat([s.h for s in shards], 1).numpy()
    c = torch.cat([s.c for s in shards], 1).numpy() if cell == "lstm" else None
    return c, h, st


def test_split_steps():
    assert sh.split_steps(10, 3) == [(0, 4), (4, 7), (7, 10)]
    assert sh.split_steps(4, 4) == [(0, 1), (1, 2), (2, 3), (3, 4)]


@pytest.mark.parametrize("cell", ["gru", "lstm"])
def test_one_shard_is_the_oracle_newton(cell):
    # capped at n updates, the sharded driver with one shard gives the oracle's
    # n-th Newton iterate; converged, the sequential recurrence
    x = _inputs(cell, 2, 40, 8)
    for n in (1, 3):
        c, h, st = _local(cell, x, 1, tol=0.0, max_iters=n)
        if cell == "gru":
            r = oracle.gru_newton(x["u"], x["a"], x["bias"], x["h0"], tol=0.0, max_iters=n)
        else:
            r = oracle.lstm_newton(x["u"], x["a"], x["bias"], x["c0"], x["h0"], tol=0.0,
                                   max_iters=n)
            assert np.abs(c - r["c"]).max() < 1e-12
        assert np.abs(h - r["h"]).max() < 1e-12
        assert st["iters"] == n and st["status"] == "not_converged"
    c, h, st = _local(cell, x, 1, tol=1e-10, max_iters=40)
    ref = (oracle.gru_seq(x["u"], x["a"], x["bias"], x["h0"]) if cell == "gru"
           else oracle.lstm_seq(x["u"], x["a"], x["bias"], x["c0"], x["h0"])[1])
    assert st["status"] == "converged" and np.abs(h - ref).max() < 1e-9


@pytest.mark.parametrize("cell,world", [("gru", 3), ("lstm", 4)])
def test_shards_in_one_process_match_one_shard(cell, world):
    x = _inputs(cell, 2, 37, 8)
    c1, h1, s1 = _local(cell, x, 1, tol=1e-9, max_iters=37)
    cw, hw, sw = _local(cell, x, world, tol=1e-9, max_iters=37)
    assert np.abs(hw - h1).max() < 1e-10 and sw["iters"] == s1["iters"]
    if cell == "lstm":
        assert np.abs(cw - c1).max() < 1e-10


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, cell, q):
    import sys
    if ROOT not in sys.path:
        sys.path.insert(0, ROOT)
    import datetime
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        x = _inputs(cell, 2, 45, 16)
        t0, t1 = sh.split_steps(45, world)[rank]
        (s,) = [z for z in _shards(cell, x, sh.split_steps(45, world)) if z.index == rank]
        st = sh.sharded_solve([s], sh.ProcessGroupExchange(), Fp64Engine(), tol=1e-9,
                              max_iters=45)
        q.put((rank, t0, t1, s.h.numpy(), s.c.numpy() if s.c is not None else None, st))
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("cell", ["gru", "lstm"])
def test_two_gloo_ranks_match_one_process(cell):
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, cell, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted((q.get(timeout=180) for _ in range(world)), key=lambda z: z[0])
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    x = _inputs(cell, 2, 45, 16)
    c1, h1, s1 = _local(cell, x, 1, tol=1e-9, max_iters=45)
    for rank, t0, t1, h, c, st in res:
        assert np.abs(h - h1[:, t0:t1]).max() < 1e-6
        if cell == "lstm":
            assert np.abs(c - c1[:, t0:t1]).max() < 1e-6
        assert st["iters"] == s1["iters"] and st["status"] == "converged"
