"""Sequence sharding with the library's kernels (pararnn_shard_eval /
_combine / _apply) on one GPU: the shards of a sequence emulated in one
process (the exchange by indexing, nothing waits on another kernel), checked
against the fp64 oracle's Newton iterates and sequential recurrence."""
import numpy as np
import pytest
import torch

import oracle
import nonlinear_rnn_paragru_b200 as pr
from nonlinear_rnn_paragru_b200 import shard as sh
from nonlinear_rnn_paragru_b200.inputs import WORKLOADS, make_inputs

pytestmark = pytest.mark.gpu

TOL_STATE = 1e-4


def _run(cell, x, world, **kw):
    T = x["u"].shape[1]
    c = pr.PARARNN_GRU if cell == "gru" else pr.PARARNN_LSTM
    d = {k: v.cuda() for k, v in x.items()}
    shards = [sh.Shard(r, c, d["u"][:, t0:t1].contiguous(), d["a"], d["bias"], d.get("c0"),
                       d["h0"]) for r, (t0, t1) in enumerate(sh.split_steps(T, world))]
    st = sh.sharded_solve(shards, sh.LocalExchange(), **kw)
    torch.cuda.synchronize()
    h = torch.cat([s.h for s in shards], 1).cpu().numpy()
    cc = torch.cat([s.c for s in shards], 1).cpu().numpy() if cell == "lstm" else None
    return cc, h, st


def _x(cell, B, T, D, u_f32=False):
    w = (WORKLOADS[2] if cell == "gru" else WORKLOADS[3]).scaled(B=B, T=T, D=D)
    x = make_inputs(w)
    g = torch.Generator().manual_seed(43)
    x["h0"] = torch.randn((B, D), generator=g) * 0.5
    if cell == "lstm":
        x["c0"] = torch.randn((B, D), generator=g) * 0.5
    if u_f32:
        x["u"] = x["u"].float()
    return x


@pytest.mark.parametrize("cell,world", [("gru", 1), ("gru", 3), ("lstm", 4)])
def test_sharded_capped_iterates_match_oracle_newton(cuda_ok, cell, world):
    x = _x(cell, 2, 700, 64)
    for n in (1, 2):
        c, h, st = _run(cell, x, world, tol=0.0, max_iters=n)
        assert st["iters"] == n and st["status"] == "not_converged"
        if cell == "gru":
            r = oracle.gru_newton(x["u"], x["a"], x["bias"], x["h0"], tol=0.0, max_iters=n)
        else:
            r = oracle.lstm_newton(x["u"], x["a"], x["bias"], x["c0"], x["h0"], tol=0.0,
                                   max_iters=n)
            assert np.abs(c - r["c"]).max() < TOL_STATE
        assert np.abs(h - r["h"]).max() < TOL_STATE


@pytest.mark.parametrize("cell,world,u_f32", [("gru", 4, False), ("gru", 2, True),
                                              ("lstm", 3, False)])
def test_sharded_solve_matches_sequential(cuda_ok, cell, world, u_f32):
    x = _x(cell, 2, 1500, 96, u_f32)
    c, h, st = _run(cell, x, world, tol=1e-6, max_iters=64)
    assert st["status"] == "converged" and st["max_residual"] < 1e-6
    if cell == "gru":
        ref = oracle.gru_seq(x["u"], x["a"], x["bias"], x["h0"])
    else:
        rc, ref = oracle.lstm_seq(x["u"], x["a"], x["bias"], x["c0"], x["h0"])
        assert np.abs(c - rc).max() < TOL_STATE
    assert np.abs(h - ref).max() < TOL_STATE


def test_split_does_not_change_the_iterates(cuda_ok):
    x = _x("gru", 1, 900, 32)
    _, h1, s1 = _run("gru", x, 1, tol=1e-6, max_iters=64)
    _, h5, s5 = _run("gru", x, 5, tol=1e-6, max_iters=64)
    assert s1["iters"] == s5["iters"]
    assert np.abs(h1 - h5).max() < 1e-5
