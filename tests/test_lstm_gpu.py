"""GPU parity of the fused ParaLSTM Newton-scan solve against the fp64 oracle
(max-abs 1e-4 on both c and h)."""
import numpy as np
import pytest
import torch

import oracle
import nonlinear_rnn_paragru_b200 as pr
from nonlinear_rnn_paragru_b200.inputs import WORKLOADS, make_inputs

pytestmark = pytest.mark.gpu

TOL_STATE = 1e-4


def _solve(x, **kw):
    d = "cuda"
    c, h, st, hist = pr.lstm_solve(x["u"].to(d), x["a"].to(d), x["bias"].to(d),
                                   x["c0"].to(d), x["h0"].to(d), **kw)
    torch.cuda.synchronize()
    return (c.cpu().numpy(), h.cpu().numpy(), pr.read_stats(st),
            hist.cpu().numpy() if hist is not None else None)


def _ref(x):
    return oracle.lstm_seq(x["u"], x["a"], x["bias"], x["c0"], x["h0"])


def _check(x, **kw):
    c, h, st, hist = _solve(x, **kw)
    rc, rh = _ref(x)
    err = max(np.abs(c - rc).max(), np.abs(h - rh).max())
    assert err < TOL_STATE, (err, st)
    assert st["status"] == "converged", st
    return st, hist


@pytest.mark.parametrize("wl,D", [(3, 8), (3, 4736), (5, 4736)])
def test_certified_iterate_is_the_oracle_newton_result(cuda_ok, wl, D):
    # the oracle returns the first iterate whose residual is below tol.  The
    # solve checks the residual alone after an exact step from at most
    # sqrt(tol / 2) and returns that iterate when it is below tol / 2 (n
    # updates); otherwise the certifying evaluation forms its step too
    # (n + 1).  D = 8 is one tile on the whole-sequence kernel, D = 4736 is
    # 592 copies of it on the segment queue (one 128-step segment).  Exact
    # steps throughout.
    tol = 1e-6
    x = make_inputs(WORKLOADS[wl].scaled(B=1, T=128, D=8))
    r = oracle.lstm_newton(x["u"], x["a"], x["bias"], x["c0"], x["h0"], tol=tol,
                           max_iters=64)
    n, tr = r["iters"], r["trace"]
    spec = np.sqrt(0.5 * tol)
    # the oracle's residuals sit far from the thresholds the fp32 kernels test
    assert n >= 2 and tr[n] < 0.25 * tol and (tr[: n - 1] > 2 * spec).all()
    assert not 0.5 * spec < tr[n - 1] < 2 * spec
    expect = n if tr[n - 1] <= spec else n + 1
    xr = {k: v.repeat(*([1] * (v.dim() - 1)), D // 8) for k, v in x.items()}
    c, h, st, _ = _solve(xr, tol=tol, flags=pr.PARARNN_FLAG_EXACT_STEPS)
    assert st["status"] == "converged" and st["max_residual"] < tol, st
    assert st["iters"] == expect and st["evals"] == n + 1, (st, n, expect)
    assert np.abs(c - np.tile(r["c"], (1, 1, D // 8))).max() < TOL_STATE
    assert np.abs(h - np.tile(r["h"], (1, 1, D // 8))).max() < TOL_STATE


@pytest.mark.parametrize("B,T,D", [(2, 1000, 96), (1, 129, 64), (1, 1, 8),
                                   (3, 128, 32), (1, 2200, 40)])
def test_ragged_shapes_bf16(cuda_ok, B, T, D):
    _check(make_inputs(WORKLOADS[3].scaled(B=B, T=T, D=D)))


def test_fp32_inputs(cuda_ok):
    w = WORKLOADS[3].scaled(B=1, T=700, D=64)
    x = make_inputs(w)
    x["u"] = x["u"].float()
    _check(x)


def test_nonzero_initial_state(cuda_ok):
    x = make_inputs(WORKLOADS[3].scaled(B=2, T=600, D=64))
    g = torch.Generator().manual_seed(7)
    x["c0"] = torch.randn((2, 64), generator=g, dtype=torch.float32)
    x["h0"] = torch.randn((2, 64), generator=g, dtype=torch.float32) * 0.5
    _check(x)


def test_config5_shape_scaled(cuda_ok):
    st, _ = _check(make_inputs(WORKLOADS[5].scaled(B=2, T=2048, D=128)))


def test_config3_full_size(cuda_ok):
    st, _ = _check(make_inputs(WORKLOADS[3]))
    assert st["max_residual"] < 1e-6


def test_multi_cluster_chunks(cuda_ok):
    # T = 5000 spans several 16-CTA cluster chunks of 2048 steps
    st, hist = _check(make_inputs(WORKLOADS[3].scaled(B=1, T=5000, D=64)), hist=True)
    assert hist.sum() == 64 and hist[-1] == 0


@pytest.mark.parametrize("n", [1, 2])
def test_capped_iterates_match_oracle_newton(cuda_ok, n):
    x = make_inputs(WORKLOADS[3].scaled(B=1, T=900, D=64))
    c, h, st, _ = _solve(x, max_iters=n)
    r = oracle.lstm_newton(x["u"], x["a"], x["bias"], x["c0"], x["h0"], tol=0.0,
                           max_iters=n)
    assert st["status"] == "not_converged" and st["iters"] == n
    assert max(np.abs(c - r["c"]).max(), np.abs(h - r["h"]).max()) < TOL_STATE


@pytest.mark.parametrize("B,T,D", [(2, 500, 96), (1, 1000, 64), (1, 2049, 32), (1, 4096, 40),
                                   (3, 37, 24)])
def test_both_solvers_match_oracle(cuda_ok, B, T, D):
    # bf16 u with T <= 4096 runs the whole-sequence row kernel (clusters of
    # 1, 2, 4 and 8 CTAs above); the chunked solve is forced here so both stay
    # covered on short sequences
    x = make_inputs(WORKLOADS[3].scaled(B=B, T=T, D=D))
    rc, rh = _ref(x)
    for flags in (0, pr.PARARNN_FLAG_FORCE_CHUNKED):
        c, h, st, hist = _solve(x, flags=flags, hist=True)
        err = max(np.abs(c - rc).max(), np.abs(h - rh).max())
        assert err < TOL_STATE, (flags, err, st)
        assert st["status"] == "converged", (flags, st)
        assert hist.sum() == B * D


def test_seq_baseline_matches_oracle(cuda_ok):
    x = make_inputs(WORKLOADS[3].scaled(B=2, T=300, D=64))
    c, h = pr.seq_baseline(pr.PARARNN_LSTM, x["u"].cuda(), x["a"].cuda(),
                           x["bias"].cuda(), x["c0"].cuda(), x["h0"].cuda())
    torch.cuda.synchronize()
    rc, rh = _ref(x)
    assert max(np.abs(c.cpu().numpy() - rc).max(), np.abs(h.cpu().numpy() - rh).max()) < TOL_STATE


def test_absent_bias_with_nonzero_state_both_solvers(cuda_ok):
    x = make_inputs(WORKLOADS[3].scaled(B=2, T=1100, D=32))
    x["bias"] = torch.zeros_like(x["bias"])
    gen = torch.Generator().manual_seed(11)
    x["c0"] = torch.randn((2, 32), generator=gen) * 0.5
    x["h0"] = torch.randn((2, 32), generator=gen) * 0.5
    rc, rh = _ref(x)
    for flags in (0, pr.PARARNN_FLAG_FORCE_CHUNKED):
        c, h, st, _ = pr.lstm_solve(x["u"].cuda(), x["a"].cuda(), None, x["c0"].cuda(),
                                    x["h0"].cuda(), flags=flags)
        torch.cuda.synchronize()
        err = max(np.abs(c.cpu().numpy() - rc).max(), np.abs(h.cpu().numpy() - rh).max())
        assert err < TOL_STATE, (flags, err)
        assert pr.read_stats(st)["status"] == "converged"


@pytest.mark.parametrize("B,T,D", [(2, 3000, 160), (1, 4095, 320), (1, 2500, 640),
                                   (2, 3000, 600)])
def test_segmented_long_sequence_matches_oracle(cuda_ok, B, T, D):
    # with 40, 80 and 150 8-channel tiles, clusters of 4, 2 and 1 CTAs put a
    # CTA on each of 148 SMs: the row solve then runs in segments of 2048,
    # 1024 and 512 steps (ragged last segments here), each starting from the
    # (c, h) the one before converged to; a nonzero initial state checks the
    # first
    x = make_inputs(WORKLOADS[3].scaled(B=B, T=T, D=D))
    gen = torch.Generator().manual_seed(13)
    x["c0"] = torch.randn((B, D), generator=gen) * 0.5
    x["h0"] = torch.randn((B, D), generator=gen) * 0.5
    rc, rh = _ref(x)
    for flags in (0, pr.PARARNN_FLAG_FORCE_CHUNKED):
        c, h, st, hist = _solve(x, flags=flags, hist=True)
        err = max(np.abs(c - rc).max(), np.abs(h - rh).max())
        assert err < TOL_STATE, (flags, err, st)
        assert st["status"] == "converged", (flags, st)
        assert hist.sum() == B * D


@pytest.mark.parametrize("B,T,D,flags", [
    (1, 1500, 64, 0),                            # clusters of 4 over the whole sequence
    (2, 400, 48, 0),                             # one CTA per tile
    (1, 1500, 64, pr.PARARNN_FLAG_FORCE_CHUNKED)])
def test_channel_iteration_index_matches_oracle(cuda_ok, B, T, D, flags):
    # the per-channel index against the oracle's chan_k (within one; see the
    # ParaGRU test), for sequences solved in one launch
    x = make_inputs(WORKLOADS[3].scaled(B=B, T=T, D=D))
    ci = torch.full((B, D), -5, dtype=torch.int32, device="cuda")
    c, h, st, hist = _solve(x, hist=True, chan_iters=ci, flags=flags)
    k_gpu = ci.cpu().numpy()
    r = oracle.lstm_newton(x["u"], x["a"], x["bias"], x["c0"], x["h0"], tol=1e-6,
                           max_iters=64)
    diff = np.abs(k_gpu - r["chan_k"])
    assert diff.max() <= 1, (diff.max(), np.argwhere(diff > 1)[:5])
    assert (diff == 0).mean() > 0.9
    np.testing.assert_array_equal(hist, np.bincount(k_gpu.ravel(), minlength=66))


def _sensitivity(x, c, h):
    """Per (b, d) channel: max_t of the row-sum norm of sum_{s<=t} prod_{s<k<=t}
    A_k, from the oracle's fp64 2x2 Jacobians along the trajectory (c, h): a
    per-step residual of size r moves the state of a near-fixed point by at
    most r times this (to first order)."""
    u = x["u"].double().numpy()
    a, bias = x["a"].double().numpy(), x["bias"].double().numpy()
    B, T, _, D = u.shape
    n = B * D
    ag = np.tile(a.T, (B, 1))
    bg = np.tile(bias.T, (B, 1))
    S = np.zeros((n, 2, 2))
    best = np.zeros(n)
    cp = np.zeros(n)
    hp = np.zeros(n)
    eye = np.eye(2)
    for t in range(T):
        ut = u[:, t].transpose(0, 2, 1).reshape(n, 4)
        _, _, A, _, _ = oracle.lstm_step(cp, hp, ut, ag, bg)
        S = np.einsum("nij,njk->nik", A, S) + eye
        best = np.maximum(best, np.abs(S).sum(axis=2).max(axis=1))
        cp, hp = c[:, t].reshape(n), h[:, t].reshape(n)
    return best.reshape(B, D)


def test_config5_full_size(cuda_ok):
    # B=4, T=2048, D=4096, u ~ N(0, 4/sqrt(D)): 512-step segments on all SMs.
    # A few channels of this recurrence amplify a per-step perturbation by up
    # to about 2e5 (the sensitivity below): no fp32 trajectory matches the
    # fp64 one to 1e-4 there (the fp32 sequential loop misses it by 4.4e-4).
    # The solve guarantees its residual; the states are held to 1e-4 where
    # that bound allows and to the bound elsewhere.
    x = make_inputs(WORKLOADS[5])
    c, h, st, hist = _solve(x, hist=True)
    assert st["status"] == "converged" and st["max_residual"] < 1e-6, st
    assert hist.sum() == 4 * 4096 and hist[-1] == 0
    resc, resh = oracle.lstm_residual(x["u"], x["a"], x["bias"], x["c0"], x["h0"],
                                      c.astype(np.float64), h.astype(np.float64))
    assert max(np.abs(resc).max(), np.abs(resh).max()) < 1e-6
    rc, rh = _ref(x)
    err = np.maximum(np.abs(c - rc).max(axis=1), np.abs(h - rh).max(axis=1))   # [B, D]
    sens = _sensitivity(x, rc, rh)
    bound = np.maximum(TOL_STATE, 1e-6 * sens)
    assert (err <= bound).all(), (err.max(), float(np.argmax(err)), sens.max())
    assert (sens <= 100).mean() > 0.95          # most channels: the plain 1e-4
    assert (err[sens <= 100] < TOL_STATE).all()


def test_config5_fwd_then_adjoint_end_to_end(cuda_ok):
    # the GPU trajectory feeds the GPU adjoint; compared with BPTT on the exact
    # sequential trajectory (per-tensor relative error 1e-3)
    w = WORKLOADS[5]
    x = make_inputs(w)
    d = "cuda"
    xd = {k: v.to(d) for k, v in x.items()}
    c, h, st, _ = pr.lstm_solve(xd["u"], xd["a"], xd["bias"], xd["c0"], xd["h0"])
    g = pr.adjoint(pr.PARARNN_LSTM, xd["u"], xd["a"], xd["bias"], xd["h0"], h, xd["dLdh"],
                   c0=xd["c0"], c=c)
    torch.cuda.synchronize()
    assert pr.read_stats(st)["status"] == "converged"
    assert int(g["status"][0]) == 0
    rc, rh = _ref(x)
    ref = oracle.lstm_bptt(x["u"], x["a"], x["bias"], x["c0"], x["h0"], rc, rh, x["dLdh"])
    for k in ("du", "da", "dbias", "dh0", "dc0"):
        gk = g[k].cpu().numpy()
        rel = float(np.abs(gk - ref[k]).max() / max(np.abs(ref[k]).max(), 1e-30))
        assert rel <= 1e-3, (k, rel)


@pytest.mark.parametrize("flags", [0, pr.PARARNN_FLAG_FORCE_CHUNKED])
def test_nan_input_reports_nonfinite(cuda_ok, flags):
    x = make_inputs(WORKLOADS[3].scaled(B=1, T=900, D=32))
    x["u"][0, 300, 2, 9] = float("nan")
    _, _, st, _ = _solve(x, flags=flags, max_iters=8)
    assert st["status"] == "nonfinite", st
    _check(make_inputs(WORKLOADS[3].scaled(B=1, T=900, D=32)), flags=flags)


def test_row_kernel_withheld_mailbox_times_out(cuda_ok):
    # one tile of 1500 steps: a cluster of 4 CTAs of 512 steps; rank 1
    # withholds its exchange at the cap evaluation
    x = make_inputs(WORKLOADS[3].scaled(B=1, T=1500, D=8))
    opts = pr._opts(1e-6, 2, flags=pr.PARARNN_FLAG_INJECT_WITHHOLD, inject_chunk=1,
                    timeout_us=20000)
    _, _, st, _ = _solve(x, opts=opts, max_iters=2)
    assert st["status"] == "timeout", st
    _check(x)


# ---- the segment-queue solve (bf16 u, at least one 8-channel tile per
# resident CTA: 4 x 148 = 592 on a B200): every 128-step segment of every
# tile in one launch
@pytest.mark.parametrize("B,T,D,wl,nz", [(1, 1300, 4800, 3, True), (2, 700, 2400, 3, True),
                                         (1, 5000, 4800, 3, True), (2, 700, 2400, 5, False)])
def test_segment_queue_matches_oracle(cuda_ok, B, T, D, wl, nz):
    # configuration-3 inputs with a nonzero initial state, longer than one
    # whole-sequence solve (T > 4096: FORCE_ROW takes the chunked solve
    # there); and configuration-5 inputs from the zero state (with a random
    # initial state a few of those channels amplify rounding past 1e-4; see
    # the configuration-5 test)
    x = make_inputs(WORKLOADS[wl].scaled(B=B, T=T, D=D))
    if nz:
        g = torch.Generator().manual_seed(31)
        x["c0"] = torch.randn((B, D), generator=g)
        x["h0"] = torch.randn((B, D), generator=g) * 0.5
    rc, rh = _ref(x)
    for flags in (0, pr.PARARNN_FLAG_FORCE_ROW):
        c, h, st, hist = _solve(x, flags=flags, hist=True)
        err = max(np.abs(c - rc).max(), np.abs(h - rh).max())
        assert err < TOL_STATE, (flags, err, st)
        assert st["status"] == "converged", (flags, st)
        assert hist.sum() == B * D


def test_segment_queue_withheld_segment_times_out(cuda_ok):
    x = make_inputs(WORKLOADS[3].scaled(B=1, T=1024, D=4800))
    opts = pr._opts(1e-6, 64, flags=pr.PARARNN_FLAG_INJECT_WITHHOLD, inject_chunk=3,
                    timeout_us=20000)
    _, _, st, _ = _solve(x, opts=opts)
    assert st["status"] == "timeout", st
    _check(x)


def test_segment_queue_exact_capped_iterate_and_index(cuda_ok):
    # one 128-step segment per tile (T <= 128): with exact steps the capped
    # iterate is the oracle's first Newton iterate, and the per-channel index
    # the oracle's
    x = make_inputs(WORKLOADS[3].scaled(B=1, T=100, D=4800))
    c, h, st, _ = _solve(x, max_iters=1, flags=pr.PARARNN_FLAG_EXACT_STEPS)
    r = oracle.lstm_newton(x["u"], x["a"], x["bias"], x["c0"], x["h0"], tol=0.0, max_iters=1)
    assert st["status"] == "not_converged" and st["iters"] == 1 and st["evals"] == 2
    assert max(np.abs(c - r["c"]).max(), np.abs(h - r["h"]).max()) < TOL_STATE
    ci = torch.full((1, 4800), -5, dtype=torch.int32, device="cuda")
    c, h, st, hist = _solve(x, hist=True, chan_iters=ci, flags=pr.PARARNN_FLAG_EXACT_STEPS)
    k_gpu = ci.cpu().numpy()
    r = oracle.lstm_newton(x["u"], x["a"], x["bias"], x["c0"], x["h0"], tol=1e-6, max_iters=64)
    diff = np.abs(k_gpu - r["chan_k"])
    assert diff.max() <= 1 and (diff == 0).mean() > 0.9, diff.max()
    np.testing.assert_array_equal(hist, np.bincount(k_gpu.ravel(), minlength=66))


def _abs_sensitivity_at_zero(x):
    """Per (b, d) channel: max_t of the row-sum norm of
    sum_{s<=t} prod_{s<k<=t} |A_k|, with A_t the fp64 2x2 Jacobian of the cell
    at the zero state (the initial guess; c0 = h0 = 0 here): an error e_s
    added at each step of the linear scan moves the state by at most this
    times max |e_s|."""
    u = x["u"].double().numpy()
    a, bias = x["a"].double().numpy(), x["bias"].double().numpy()
    B, T, _, D = u.shape
    n = B * D
    ag, bg = np.tile(a.T, (B, 1)), np.tile(bias.T, (B, 1))
    S, best = np.zeros((n, 2, 2)), np.zeros(n)
    z = np.zeros(n)
    for t in range(T):
        ut = u[:, t].transpose(0, 2, 1).reshape(n, 4)
        _, _, A, _, _ = oracle.lstm_step(z, z, ut, ag, bg)
        S = np.einsum("nij,njk->nik", np.abs(A), S) + np.eye(2)
        best = np.maximum(best, S.sum(axis=2).max(axis=1))
    return best.reshape(B, D)


def test_segment_queue_inexact_first_iterate(cuda_ok):
    # Without PARARNN_FLAG_EXACT_STEPS the first evaluations use the
    # one-instruction tanh (gates within d = 2^-10 relative, with margin).
    # At the zero initial guess the cell's errors are |c~' - c'| <= 1.5 d,
    # |h~' - h'| <= 3 d, and the 2x2 Jacobian's row sums move by at most
    # 24 d (from the derivatives of c', h' and A in the gates), so per
    # channel the first iterate moves by at most S (3 d + 24 d max|s~|), S the
    # scan's row-sum sensitivity along the initial guess.
    x = make_inputs(WORKLOADS[3].scaled(B=1, T=128, D=4800))
    c, h, st, _ = _solve(x, max_iters=1)
    r = oracle.lstm_newton(x["u"], x["a"], x["bias"], x["c0"], x["h0"], tol=0.0, max_iters=1)
    assert st["status"] == "not_converged" and st["iters"] == 1
    err = np.maximum(np.abs(c - r["c"]).max(axis=1), np.abs(h - r["h"]).max(axis=1))  # [B, D]
    S = _abs_sensitivity_at_zero(x)
    d = 2.0 ** -10
    smax = np.maximum(np.abs(c).max(axis=1), np.abs(h).max(axis=1))
    bound = S * (3 * d + 24 * d * smax)
    assert (err <= bound).all(), (float((err / bound).max()), float(S.max()))
    assert err.max() > 1e-6            # the inexact evaluation was taken
    ce, he, ste, _ = _solve(x, flags=pr.PARARNN_FLAG_EXACT_STEPS)
    ci_, hi_, sti, _ = _solve(x)
    rc, rh = _ref(x)
    for cc, hh, ss in ((ce, he, ste), (ci_, hi_, sti)):
        assert ss["status"] == "converged" and ss["max_residual"] < 1e-6, ss
        assert max(np.abs(cc - rc).max(), np.abs(hh - rh).max()) < TOL_STATE
    assert sti["evals"] <= ste["evals"] + 1, (sti, ste)
