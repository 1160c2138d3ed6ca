"""GPU parity of the dense-Jacobian Newton solve (the GRU with full recurrent
matrices) against the fp64 oracle.

- The tensor-core contraction (pararnn_dense_matmul, tf32 products with fp32
  sums) against fp64 matrix products: per-tensor error within the tf32 bound.
- CUDA-core path (PARARNN_FLAG_DENSE_SIMT, exact Newton steps): capped
  iterates against the oracle's dense Newton within max-abs 1e-4.
- Tensor-core path (the default): Newton steps are inexact by the tf32
  rounding of the chunk maps, so its capped iterates are compared within a
  bound derived from that rounding, and its converged states against the
  sequential recurrence within 1e-4, like every solve.
- Diagonal matrices give the ParaGRU solve.
"""
import numpy as np
import pytest
import torch

import oracle
import nonlinear_rnn_paragru_b200 as pr
from nonlinear_rnn_paragru_b200.inputs import WORKLOADS, make_inputs

pytestmark = pytest.mark.gpu

TOL_STATE = 1e-4
TOL_SOLVE = 1e-5   # global stopping: a decade above fp32 rounding of the states
# tf32 keeps 10 explicit mantissa bits: a product's inputs are rounded by up
# to 2^-11 relative, so a K-term sum carries at most about 2 * 2^-11 * K * max|a| max|b|
TF32_REL = 2.0 ** -10


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


@pytest.mark.parametrize("M,N,K,Z,mode", [(128, 128, 32, 1, 0), (200, 72, 96, 3, 0),
                                          (64, 64, 64, 6, 2), (512, 512, 512, 2, 1),
                                          (1000, 384, 128, 1, 0), (8, 8, 8, 4, 2)])
def test_tensor_core_matmul_matches_fp64(cuda_ok, M, N, K, Z, mode):
    g = torch.Generator().manual_seed(M + N + K + Z)
    A = torch.randn((Z, M, K), generator=g)
    Bm = torch.randn((Z, N, K), generator=g)
    C = torch.full((Z, M, N), float("nan"))
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    Cd = C.cuda()
    pr.pararnn_dense_matmul(A.cuda(), Bm.cuda(), Cd, mode, err)
    torch.cuda.synchronize()
    assert int(err[0]) == 0
    ref = torch.einsum("zmk,znk->zmn", A.double(), Bm.double())
    got = Cd.cpu().double()
    for z in range(Z):
        trans = mode == 1 or (mode == 2 and z % 2 == 0)
        gz = got[z].reshape(N, M).t() if trans else got[z]
        bound = 2 * TF32_REL * K * A[z].abs().max() * Bm[z].abs().max()
        assert (gz - ref[z]).abs().max() <= bound, (z, float((gz - ref[z]).abs().max()))
        # and far below that bound in practice (random signs): within 1e-3 relative
        rel = float((gz - ref[z]).abs().max() / ref[z].abs().max())
        assert rel < 1e-3, (z, rel)


# launches with at least one 128 x 256 tile per SM take the persistent form
# (one CTA per SM, double-buffered accumulators): all four store modes, ragged
# edges in M, N and K
@pytest.mark.parametrize("M,N,K,Z,mode", [(512, 512, 256, 40, 0), (300, 520, 96, 60, 2),
                                          (512, 512, 512, 20, 1), (256, 384, 64, 110, 3)])
def test_tensor_core_matmul_persistent_matches_fp64(cuda_ok, M, N, K, Z, mode):
    g = torch.Generator().manual_seed(M + N + K + Z + 1)
    A = torch.randn((Z, M, K), generator=g)
    Bm = torch.randn((Z, N, K), generator=g)
    C0 = torch.randn((Z, M, N), generator=g) if mode == 3 else torch.full((Z, M, N), float("nan"))
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    Cd = C0.cuda()
    pr.pararnn_dense_matmul(A.cuda(), Bm.cuda(), Cd, mode, err)
    torch.cuda.synchronize()
    assert int(err[0]) == 0
    ref = torch.einsum("zmk,znk->zmn", A.double(), Bm.double())
    if mode == 3:
        ref = ref + C0.double()
    got = Cd.cpu().double()
    for z in range(Z):
        trans = mode == 1 or (mode == 2 and z % 2 == 0)
        gz = got[z].reshape(N, M).t() if trans else got[z]
        bound = 2 * TF32_REL * K * A[z].abs().max() * Bm[z].abs().max()
        assert (gz - ref[z]).abs().max() <= bound, (z, float((gz - ref[z]).abs().max()))


@pytest.mark.parametrize("n", [1, 2])
def test_simt_capped_iterates_match_oracle_dense_newton(cuda_ok, n):
    x = _inputs(2, 45, 40)   # three 16-step chunks, the last ragged; GEMM tiles ragged
    h, st = _run(x, tol=1e-30, max_iters=n, flags=pr.PARARNN_FLAG_DENSE_SIMT)
    assert st["status"] == "not_converged" and st["iters"] == n and st["evals"] == n + 1
    r = oracle.dense_gru_newton(x["u"], x["W"], x["bias"], x["h0"], tol=0.0, max_iters=n)
    assert np.abs(h - r["h"]).max() < TOL_STATE


@pytest.mark.parametrize("n", [1, 2])
def test_tensor_core_capped_iterates_within_the_tf32_bound(cuda_ok, n):
    # one inexact Newton step: the chunk maps carry tf32 rounding (four levels
    # of products), so the iterate differs from the exact step by a few 1e-3
    # of the update at most
    x = _inputs(2, 45, 40)
    h, st = _run(x, tol=1e-30, max_iters=n)
    assert st["status"] == "not_converged" and st["iters"] == n and st["evals"] == n + 1
    r = oracle.dense_gru_newton(x["u"], x["W"], x["bias"], x["h0"], tol=0.0, max_iters=n)
    step = np.abs(r["h"]).max()
    assert np.abs(h - r["h"]).max() < 8 * 4 * TF32_REL * step


@pytest.mark.parametrize("B,T,D,f32,flags", [
    (2, 300, 64, False, 0), (1, 200, 64, True, 0), (1, 70, 128, False, 0), (3, 17, 8, False, 0),
    (1, 100, 256, False, 0), (1, 64, 512, True, 0), (1, 300, 512, False, 0),
    (2, 300, 64, False, 8), (1, 70, 128, False, 8)])   # 8 = PARARNN_FLAG_DENSE_SIMT
def test_converges_to_the_sequential_recurrence(cuda_ok, B, T, D, f32, flags):
    x = _inputs(B, T, D, f32=f32)
    h, st = _run(x, tol=TOL_SOLVE, flags=flags)
    assert st["status"] == "converged", st
    ref = oracle.dense_gru_seq(x["u"], x["W"], x["bias"], x["h0"])
    assert np.abs(h - ref).max() < TOL_STATE


@pytest.mark.parametrize("flags", [0, 8])
def test_diagonal_matrices_give_the_paragru_solve(cuda_ok, flags):
    x = _inputs(2, 256, 32)
    x["W"] = torch.stack([torch.diag(x["a"][g]) for g in range(3)])
    h, st = _run(x, tol=TOL_SOLVE, flags=flags)
    assert st["status"] == "converged"
    ref = oracle.gru_seq(x["u"], x["a"], x["bias"], x["h0"])
    assert np.abs(h - ref).max() < TOL_STATE
