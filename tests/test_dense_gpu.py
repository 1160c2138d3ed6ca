"""GPU parity of the dense-Jacobian Newton solve (the GRU with full recurrent
matrices) against the fp64 oracle: capped iterates against the oracle's dense
Newton, converged states against the sequential recurrence (max-abs 1e-4),
and the ParaGRU solve when the matrices are diagonal.

Marked gpu_pending: these have not yet run on a B200 (run -m gpu_pending)."""
import numpy as np
import pytest
import torch

import oracle
import nonlinear_rnn_paragru_b200 as pr
from nonlinear_rnn_paragru_b200.inputs import WORKLOADS, make_inputs

pytestmark = pytest.mark.gpu_pending

TOL_STATE = 1e-4
TOL_SOLVE = 1e-5   # global stopping: a decade above fp32 rounding of the states


def _inputs(B, T, D, f32=False, seed=5, w_scale=1.5):
    x = make_inputs(WORKLOADS[2].scaled(B=B, T=T, D=D))
    g = torch.Generator().manual_seed(seed)
    x["W"] = (torch.rand((3, D, D), generator=g) * 2 - 1) * (w_scale / D ** 0.5)
    x["h0"] = torch.randn((B, D), generator=g) * 0.5
    if f32:
        x["u"] = x["u"].float()  # the same values, read as fp32
    return x


def _run(x, **kw):
    d = "cuda"
    h, st = pr.dense_gru_solve(x["u"].to(d), x["W"].to(d), x["bias"].to(d), x["h0"].to(d), **kw)
    torch.cuda.synchronize()
    return h.cpu().numpy(), pr.read_stats(st)


@pytest.mark.parametrize("n", [1, 2])
def test_capped_iterates_match_oracle_dense_newton(cuda_ok, n):
    x = _inputs(2, 45, 40)   # three 16-step chunks, the last ragged; GEMM tiles ragged
    h, st = _run(x, tol=1e-30, max_iters=n)
    assert st["status"] == "not_converged" and st["iters"] == n and st["evals"] == n + 1
    r = oracle.dense_gru_newton(x["u"], x["W"], x["bias"], x["h0"], tol=0.0, max_iters=n)
    assert np.abs(h - r["h"]).max() < TOL_STATE


@pytest.mark.parametrize("B,T,D,f32", [(2, 300, 64, False), (1, 200, 64, True),
                                       (1, 70, 128, False), (3, 17, 8, False)])
def test_converges_to_the_sequential_recurrence(cuda_ok, B, T, D, f32):
    x = _inputs(B, T, D, f32=f32)
    h, st = _run(x, tol=TOL_SOLVE)
    assert st["status"] == "converged", st
    ref = oracle.dense_gru_seq(x["u"], x["W"], x["bias"], x["h0"])
    assert np.abs(h - ref).max() < TOL_STATE


def test_diagonal_matrices_give_the_paragru_solve(cuda_ok):
    x = _inputs(2, 256, 32)
    x["W"] = torch.stack([torch.diag(x["a"][g]) for g in range(3)])
    h, st = _run(x, tol=TOL_SOLVE)
    assert st["status"] == "converged"
    ref = oracle.gru_seq(x["u"], x["a"], x["bias"], x["h0"])
    assert np.abs(h - ref).max() < TOL_STATE
