"""GPU parity of the fused ParaGRU Newton-scan solve against the fp64 oracle.

States must match the sequential fp64 recurrence within max-abs 1e-4
(fp32 state, fp32 or bf16 inputs).  Inputs are the seeded synthetic ones
both sides read (bf16 values widen exactly to fp64 for the oracle).
"""
import numpy as np
import pytest
import torch

import oracle
import nonlinear_rnn_paragru_b200 as pr
from nonlinear_rnn_paragru_b200.inputs import WORKLOADS, make_inputs

pytestmark = pytest.mark.gpu

TOL_STATE = 1e-4


def _solve(x, **kw):
    dev = "cuda"
    u = x["u"].to(dev)
    a = x["a"].to(dev)
    bias = x["bias"].to(dev)
    h0 = x["h0"].to(dev)
    h, stats, hist = pr.gru_solve(u, a, bias, h0, **kw)
    torch.cuda.synchronize()
    return h.cpu().numpy(), pr.read_stats(stats), (hist.cpu().numpy() if hist is not None else None)


def _ref(x):
    return oracle.gru_seq(x["u"], x["a"], x["bias"], x["h0"])


def test_config1_full(cuda_ok):
    w = WORKLOADS[1]
    x = make_inputs(w)
    h, st, _ = _solve(x, max_iters=w.T)
    err = np.abs(h - _ref(x)).max()
    assert err < TOL_STATE, err
    assert st["status"] == "converged" and st["max_residual"] < 1e-6
    assert 1 <= st["iters"] <= 12


@pytest.mark.parametrize("B,T,D", [(2, 1000, 96), (1, 257, 64), (3, 256, 32),
                                   (1, 1, 8), (2, 5, 40), (1, 2049, 128)])
def test_ragged_shapes_bf16(cuda_ok, B, T, D):
    x = make_inputs(WORKLOADS[2].scaled(B=B, T=T, D=D))
    h, st, _ = _solve(x)
    err = np.abs(h - _ref(x)).max()
    assert err < TOL_STATE, (err, st)
    assert st["status"] == "converged"


@pytest.mark.parametrize("B,T,D", [(1, 3000, 64), (2, 700, 48)])
def test_long_fp32(cuda_ok, B, T, D):
    x = make_inputs(WORKLOADS[4].scaled(B=B, T=T, D=D))
    h, st, hist = _solve(x, hist=True)
    err = np.abs(h - _ref(x)).max()
    assert err < TOL_STATE, (err, st)
    assert hist.sum() == B * D
    assert hist[-1] == 0   # every channel converged within the cap


def test_nonzero_h0(cuda_ok):
    x = make_inputs(WORKLOADS[2].scaled(B=2, T=600, D=64))
    x["h0"] = torch.randn((2, 64), generator=torch.Generator().manual_seed(5)) * 0.5
    h, st, _ = _solve(x)
    assert np.abs(h - _ref(x)).max() < TOL_STATE


def test_config2_full_size(cuda_ok):
    w = WORKLOADS[2]
    x = make_inputs(w)
    h, st, _ = _solve(x)
    err = np.abs(h - _ref(x)).max()
    assert err < TOL_STATE, (err, st)
    assert st["status"] == "converged"
    assert st["max_residual"] < 1e-6


def test_residual_of_result_is_small(cuda_ok):
    # property that holds at any size: the returned trajectory's residual
    x = make_inputs(WORKLOADS[2].scaled(B=1, T=4096, D=256))
    h, st, _ = _solve(x)
    res = oracle.gru_residual(x["u"], x["a"], x["bias"], x["h0"], h)
    assert np.abs(res).max() < 2e-6


def test_iteration_histogram_matches_oracle_counts(cuda_ok):
    x = make_inputs(WORKLOADS[4].scaled(B=1, T=2048, D=64))
    _, st, hist = _solve(x, hist=True, max_iters=32, flags=pr.PARARNN_FLAG_EXACT_STEPS)
    r = oracle.gru_newton(x["u"], x["a"], x["bias"], x["h0"], tol=1e-6, max_iters=32)
    # counts are reported, not asserted equal: fp32 vs fp64 may differ by one
    ks = np.nonzero(hist)[0]
    assert ks.max() <= r["chan_k"].max() + 1
    assert abs(st["evals"] - (r["iters"] + 1)) <= 1


@pytest.mark.parametrize("n", [1, 2, 3])
def test_capped_iterates_match_oracle_newton(cuda_ok, n):
    # with the cap at n updates the solver returns the n-th Newton iterate
    # (states after n updates of the page's scheme) and NOT_CONVERGED; exact
    # steps throughout
    x = make_inputs(WORKLOADS[2].scaled(B=1, T=1300, D=64))
    h, st, _ = _solve(x, max_iters=n, flags=pr.PARARNN_FLAG_EXACT_STEPS)
    r = oracle.gru_newton(x["u"], x["a"], x["bias"], x["h0"], tol=0.0, max_iters=n)
    assert st["status"] == "not_converged"
    assert st["iters"] == n and st["evals"] == n + 1
    assert np.abs(h - r["h"]).max() < TOL_STATE
    assert st["max_residual"] == pytest.approx(r["trace"][n], rel=1e-2)


def _tile_copies(x, n):
    # every 8-channel tile holds the same 8 channels (D is the last axis of
    # every input), so each tile stops as the whole problem does
    return {k: v.repeat(*([1] * (v.dim() - 1)), n) for k, v in x.items()}


@pytest.mark.parametrize("D", [8, 4736])
def test_certified_iterate_is_the_oracle_newton_result(cuda_ok, D):
    # the solve ends on the first iterate whose residual is below tol, the
    # oracle's rule.  After an exact step from a residual at most sqrt(tol)
    # the next evaluation is a residual-only check, and the solve returns the
    # oracle's iterate itself (n updates); otherwise the certifying
    # evaluation also forms its step (n + 1).  D = 8 is one tile on the
    # whole-sequence kernel, D = 4736 is 592 copies of it on the queue (one
    # 512-step segment).  Exact steps throughout.
    tol = 1e-6
    x = make_inputs(WORKLOADS[2].scaled(B=1, T=512, D=8))
    r = oracle.gru_newton(x["u"], x["a"], x["bias"], x["h0"], tol=tol, max_iters=64)
    n, tr = r["iters"], r["trace"]
    # the oracle's residuals sit far from the thresholds the fp32 kernels test
    assert n >= 2 and tr[n] < 0.5 * tol and (tr[: n - 1] > 2 * np.sqrt(tol)).all()
    assert not 0.5 * np.sqrt(tol) < tr[n - 1] < 2 * np.sqrt(tol)
    expect = n if tr[n - 1] <= np.sqrt(tol) else n + 1
    h, st, _ = _solve(_tile_copies(x, D // 8), tol=tol, flags=pr.PARARNN_FLAG_EXACT_STEPS)
    assert st["status"] == "converged" and st["max_residual"] < tol, st
    assert st["iters"] == expect and st["evals"] == n + 1, (st, n, expect)
    assert np.abs(h - np.tile(r["h"], (1, 1, D // 8))).max() < TOL_STATE


def test_withheld_record_times_out_without_hanging(cuda_ok):
    # host-injected fault: cluster chunk 0 of the first tile never publishes
    # (T = 5000 needs two 16-CTA cluster chunks), so its successor's bounded
    # wait expires and the solve reports TIMEOUT.
    x = make_inputs(WORKLOADS[2].scaled(B=1, T=5000, D=32))
    opts = pr._opts(1e-6, 16, flags=pr.PARARNN_FLAG_INJECT_WITHHOLD,
                    inject_chunk=0, timeout_us=20000)
    h, st, _ = _solve(x, max_iters=16, opts=opts)
    assert st["status"] == "timeout"
    # and the context is still usable
    h2, st2, _ = _solve(x, max_iters=16)
    assert st2["status"] == "converged"


def test_seq_baseline_matches_oracle(cuda_ok):
    x = make_inputs(WORKLOADS[2].scaled(B=2, T=512, D=64))
    _, h = pr.seq_baseline(pr.PARARNN_GRU, x["u"].cuda(), x["a"].cuda(),
                           x["bias"].cuda(), None, x["h0"].cuda())
    torch.cuda.synchronize()
    assert np.abs(h.cpu().numpy() - _ref(x)).max() < TOL_STATE


def test_repeat_calls_reuse_workspace(cuda_ok):
    x = make_inputs(WORKLOADS[2].scaled(B=1, T=1500, D=64))
    ws = pr.Workspace("cuda")
    outs = []
    for _ in range(3):
        h, st, _ = _solve(x, workspace=ws)
        outs.append(h)
    assert np.array_equal(outs[0], outs[1]) and np.array_equal(outs[1], outs[2])


def test_multi_cluster_lookback_fp32(cuda_ok):
    # T spans several 16-CTA cluster chunks: exercises the cross-cluster
    # decoupled look-back (plus a ragged tail chunk).
    x = make_inputs(WORKLOADS[4].scaled(B=1, T=20000, D=64))
    h, st, hist = _solve(x, hist=True)
    err = np.abs(h - _ref(x)).max()
    assert err < TOL_STATE, (err, st)
    assert st["status"] == "converged"


def test_binding_rejects_wrong_dtype(cuda_ok):
    x = make_inputs(WORKLOADS[2].scaled(B=1, T=64, D=32))
    with pytest.raises(TypeError):
        pr.gru_solve(x["u"].cuda(), x["a"].double().cuda(), None, None)


@pytest.mark.parametrize("B,T,D", [(2, 1000, 96), (1, 2049, 128), (1, 4096, 64),
                                   (3, 37, 24)])
def test_both_solvers_match_oracle(cuda_ok, B, T, D):
    # T <= 4096 runs whole sequences per CTA by default; the chunked cluster
    # solve is forced here so both stay covered on short sequences
    x = make_inputs(WORKLOADS[2].scaled(B=B, T=T, D=D))
    ref = _ref(x)
    for flags in (0, pr.PARARNN_FLAG_FORCE_CHUNKED):
        h, st, hist = _solve(x, flags=flags, hist=True)
        err = np.abs(h - ref).max()
        assert err < TOL_STATE, (flags, err, st)
        assert st["status"] == "converged", (flags, st)
        assert hist.sum() == B * D


def test_whole_sequence_fp32_inputs(cuda_ok):
    x = make_inputs(WORKLOADS[4].scaled(B=2, T=3000, D=40))
    h, st, _ = _solve(x)
    assert np.abs(h - _ref(x)).max() < TOL_STATE


def test_absent_bias_and_h0_read_as_zero(cuda_ok):
    # null bias and h0 on both solvers equal explicit zeros
    x = make_inputs(WORKLOADS[2].scaled(B=2, T=1500, D=40))
    x["bias"] = torch.zeros_like(x["bias"])
    ref = _ref(x)
    for flags in (0, pr.PARARNN_FLAG_FORCE_CHUNKED):
        h, st, _ = pr.gru_solve(x["u"].cuda(), x["a"].cuda(), None, None, flags=flags)
        torch.cuda.synchronize()
        assert np.abs(h.cpu().numpy() - ref).max() < TOL_STATE, flags
        assert pr.read_stats(st)["status"] == "converged"


def test_long_sequence_segments_match_oracle(cuda_ok):
    # T > 4096 with at least one 8-channel tile per SM (B * D / 8 = 150):
    # the sequence is solved 4096-step segment by segment, each starting from
    # the state the one before ended with; the look-back solve is forced for
    # comparison.  A nonzero h0 checks the first segment's start.
    x = make_inputs(WORKLOADS[2].scaled(B=1, T=9000, D=1200))
    x["h0"] = torch.randn((1, 1200), generator=torch.Generator().manual_seed(13)) * 0.5
    ref = _ref(x)
    for flags in (0, pr.PARARNN_FLAG_FORCE_CHUNKED):
        h, st, hist = _solve(x, flags=flags, hist=True)
        err = np.abs(h - ref).max()
        assert err < TOL_STATE, (flags, err, st)
        assert st["status"] == "converged", (flags, st)
        assert hist.sum() == 1200


def test_fp32_inputs_both_solvers(cuda_ok):
    x = make_inputs(WORKLOADS[4].scaled(B=3, T=2500, D=48))
    ref = _ref(x)
    for flags in (0, pr.PARARNN_FLAG_FORCE_CHUNKED):
        h, st, _ = _solve(x, flags=flags)
        assert np.abs(h - ref).max() < TOL_STATE, flags
        assert st["status"] == "converged", (flags, st)


@pytest.mark.parametrize("B,T,D,wl", [(1, 3000, 2400, 2), (2, 4000, 1200, 2),
                                      (1, 3500, 1600, 2), (1, 2500, 2400, 4)])
def test_short_segments_match_oracle(cuda_ok, B, T, D, wl):
    # 300 and 200 8-channel tiles: clusters of 1 and 2 CTAs already give two
    # CTAs per SM on 148 SMs, so sequences of up to 4096 steps are solved in
    # 1024- and 2048-step segments (ragged last segments here; the last case
    # has fp32 u), each from the state the one before converged to
    x = make_inputs(WORKLOADS[wl].scaled(B=B, T=T, D=D))
    x["h0"] = torch.randn((B, D), generator=torch.Generator().manual_seed(17)) * 0.5
    ref = _ref(x)
    for flags in (0, pr.PARARNN_FLAG_FORCE_CHUNKED):
        h, st, hist = _solve(x, flags=flags, hist=True)
        err = np.abs(h - ref).max()
        assert err < TOL_STATE, (flags, err, st)
        assert st["status"] == "converged", (flags, st)
        assert hist.sum() == B * D


@pytest.mark.parametrize("B,T,D,wl,flags", [
    (1, 2048, 64, 2, 0),                          # clusters of 2 over the whole sequence
    (2, 4000, 32, 4, 0),                          # fp32 u, clusters of 4
    (3, 900, 40, 2, 0),                           # one CTA per tile
    (1, 2048, 64, 2, pr.PARARNN_FLAG_FORCE_CHUNKED)])
def test_channel_iteration_index_matches_oracle(cuda_ok, B, T, D, wl, flags):
    # Per (b, d) channel: the updates applied before the first evaluation from
    # which the channel's own max_t |r_t| stays below tol.  Channels are
    # independent, so this is the oracle's per-channel chan_k of the joint
    # Newton solve, within one for fp32 against fp64 near the threshold.  The
    # sequences here are solved in one launch (no segments).
    x = make_inputs(WORKLOADS[wl].scaled(B=B, T=T, D=D))
    ci = torch.full((B, D), -5, dtype=torch.int32, device="cuda")
    h, st, hist = _solve(x, hist=True, chan_iters=ci, flags=flags | pr.PARARNN_FLAG_EXACT_STEPS)
    k_gpu = ci.cpu().numpy()
    r = oracle.gru_newton(x["u"], x["a"], x["bias"], x["h0"], tol=1e-6, max_iters=64)
    diff = np.abs(k_gpu - r["chan_k"])
    assert diff.max() <= 1, (diff.max(), np.argwhere(diff > 1)[:5])
    assert (diff == 0).mean() > 0.9
    assert len(np.unique(r["chan_k"])) >= 2        # the index varies by channel
    np.testing.assert_array_equal(hist, np.bincount(k_gpu.ravel(), minlength=66))
    assert k_gpu.max() + 1 <= st["evals"]


def test_config4_full_size_with_histogram(cuda_ok):
    # B=1, T=65536, D=2048, fp32 u: 4096-step segments, each from the state the
    # one before converged to; states against the fp64 sequential recurrence
    w = WORKLOADS[4]
    x = make_inputs(w)
    ci = torch.empty((w.B, w.D), dtype=torch.int32, device="cuda")
    h, st, hist = _solve(x, hist=True, chan_iters=ci)
    err = np.abs(h - _ref(x)).max()
    assert err < TOL_STATE, (err, st)
    assert st["status"] == "converged" and st["max_residual"] < 1e-6
    assert hist.sum() == w.D and hist[-1] == 0
    np.testing.assert_array_equal(hist, np.bincount(ci.cpu().numpy().ravel(), minlength=66))


@pytest.mark.parametrize("flags", [0, pr.PARARNN_FLAG_FORCE_CHUNKED])
def test_nan_input_reports_nonfinite(cuda_ok, flags):
    x = make_inputs(WORKLOADS[2].scaled(B=1, T=1500, D=32))
    x["u"][0, 700, 1, 5] = float("nan")
    _, st, _ = _solve(x, flags=flags, max_iters=8)
    assert st["status"] == "nonfinite", st
    # the context stays usable
    y = make_inputs(WORKLOADS[2].scaled(B=1, T=1500, D=32))
    h, st2, _ = _solve(y, flags=flags)
    assert st2["status"] == "converged"
    assert np.abs(h - _ref(y)).max() < TOL_STATE


# ---- the segment-queue solve (bf16 u, at least one 8-channel tile per
# resident CTA: 4 x 148 = 592 on a B200): every 512-step segment of every tile
# in one launch, each segment from the state its predecessor converged to
@pytest.mark.parametrize("B,T,D", [(1, 1300, 6000), (2, 2100, 3000), (3, 257, 2000)])
def test_segment_queue_matches_oracle(cuda_ok, B, T, D):
    x = make_inputs(WORKLOADS[2].scaled(B=B, T=T, D=D))
    x["h0"] = torch.randn((B, D), generator=torch.Generator().manual_seed(29)) * 0.5
    ref = _ref(x)
    for flags in (0, pr.PARARNN_FLAG_FORCE_ROW):
        h, st, hist = _solve(x, flags=flags, hist=True)
        err = np.abs(h - ref).max()
        assert err < TOL_STATE, (flags, err, st)
        assert st["status"] == "converged" and st["max_residual"] < 1e-6, (flags, st)
        assert hist.sum() == B * D and hist[-1] == 0


def test_segment_queue_channel_index_one_segment(cuda_ok):
    # T <= 512: one item per tile, so the per-channel index is the oracle's
    # (exact steps throughout: the oracle's index is that of exact Newton)
    x = make_inputs(WORKLOADS[2].scaled(B=1, T=250, D=6000))
    ci = torch.full((1, 6000), -5, dtype=torch.int32, device="cuda")
    h, st, hist = _solve(x, hist=True, chan_iters=ci, flags=pr.PARARNN_FLAG_EXACT_STEPS)
    k_gpu = ci.cpu().numpy()
    r = oracle.gru_newton(x["u"], x["a"], x["bias"], x["h0"], tol=1e-6, max_iters=64)
    diff = np.abs(k_gpu - r["chan_k"])
    assert diff.max() <= 1 and (diff == 0).mean() > 0.9, diff.max()
    np.testing.assert_array_equal(hist, np.bincount(k_gpu.ravel(), minlength=66))
    assert np.abs(h - _ref(x)).max() < TOL_STATE


def test_segment_queue_capped_iterates(cuda_ok):
    # with the cap at one update, every segment returns the first Newton
    # iterate from the state its predecessor ended with
    # (one segment: T <= 512; across segments the capped iterate of a
    # segment starts from its predecessor's, not from the whole-sequence
    # iterate)
    x = make_inputs(WORKLOADS[2].scaled(B=1, T=256, D=6000))
    h, st, _ = _solve(x, max_iters=1, flags=pr.PARARNN_FLAG_EXACT_STEPS)
    r = oracle.gru_newton(x["u"], x["a"], x["bias"], x["h0"], tol=0.0, max_iters=1)
    assert st["status"] == "not_converged" and st["iters"] == 1 and st["evals"] == 2
    assert np.abs(h - r["h"]).max() < TOL_STATE


def _scan_sensitivity(x, hprev):
    """Per channel: max_t sum_{s<=t} prod_{s<k<=t} |A_k|, with A_t the fp64
    Jacobian of the cell at (hprev_{t-1}, u_t): an error e_s added at each
    step of the linear scan h_t = f_t + A_t h_{t-1} moves h_t by at most
    this times max |e_s|."""
    u = x["u"].double().numpy()[0]            # [T, 3, D]
    a = x["a"].double().numpy().T             # [D, 3]
    bias = x["bias"].double().numpy().T
    T, _, D = u.shape
    s = np.zeros(D)
    best = np.zeros(D)
    hp = x["h0"].double().numpy()[0]
    for t in range(T):
        _, A, _, _ = oracle.gru_step(hp, u[t].T, a, bias)
        s = np.abs(A) * s + 1.0
        best = np.maximum(best, s)
        hp = hprev[t]
    return best


def test_segment_queue_inexact_first_iterate(cuda_ok):
    # Without PARARNN_FLAG_EXACT_STEPS the first evaluations of a segment use
    # the one-instruction tanh (gates within 2^-10 relative, with margin).
    # The first iterate is then h~_t = f~_t + A~_t h~_{t-1} instead of
    # h_t = f_t + A_t h_{t-1}, both evaluated at the initial guess.  With
    # |h| <= 1 the gate errors give |f~ - f| <= 1.5 d and |A~ - A| <= 8 d
    # (d = 2^-10, from the derivatives of f and A in the gates), so per channel
    # |h~ - h| <= S (1.5 d + 8 d max|h~|), S the scan's sensitivity.  A sign or
    # scaling slip in the inexact cell moves the iterate by O(S).
    x = make_inputs(WORKLOADS[2].scaled(B=1, T=256, D=6000))
    h, st, _ = _solve(x, max_iters=1)
    r = oracle.gru_newton(x["u"], x["a"], x["bias"], x["h0"], tol=0.0, max_iters=1)
    assert st["status"] == "not_converged" and st["iters"] == 1
    err = np.abs(h[0] - r["h"][0]).max(axis=0)                  # per channel
    S = _scan_sensitivity(x, np.zeros((256, 6000)))
    d = 2.0 ** -10
    bound = S * (1.5 * d + 8 * d * np.abs(h[0]).max(axis=0))
    assert (err <= bound).all(), (float((err / bound).max()), float(S.max()))
    assert err.max() > 1e-6            # the inexact evaluation was taken
    # and the solve converges to the same states in at most one more
    # evaluation than with exact steps throughout
    he, ste, _ = _solve(x, flags=pr.PARARNN_FLAG_EXACT_STEPS)
    hi, sti, _ = _solve(x)
    ref = _ref(x)
    for hh, ss in ((he, ste), (hi, sti)):
        assert ss["status"] == "converged" and ss["max_residual"] < 1e-6, ss
        assert np.abs(hh - ref).max() < TOL_STATE
    assert sti["evals"] <= ste["evals"] + 1, (sti, ste)


# ---- injected faults (host-set): a part of the exchange is withheld, the
# bounded waits for it run out, the call reports TIMEOUT, and the next call
# on the same device converges
def test_row_kernel_withheld_mailbox_times_out(cuda_ok):
    # one 8-channel tile of 3000 steps: a cluster of 4 CTAs exchanging maps
    # through mailboxes; rank 1 withholds its exchange at the cap evaluation
    x = make_inputs(WORKLOADS[2].scaled(B=1, T=3000, D=8))
    opts = pr._opts(1e-6, 2, flags=pr.PARARNN_FLAG_INJECT_WITHHOLD, inject_chunk=1,
                    timeout_us=20000)
    _, st, _ = _solve(x, opts=opts, max_iters=2)
    assert st["status"] == "timeout", st
    h, st2, _ = _solve(x)
    assert st2["status"] == "converged"
    assert np.abs(h - _ref(x)).max() < TOL_STATE


def test_segment_queue_withheld_segment_times_out(cuda_ok):
    # item 5 (segment 0 of tile 5) never publishes: segment 1 of tile 5
    # waits for it until its bounded wait runs out
    x = make_inputs(WORKLOADS[2].scaled(B=1, T=1024, D=6000))
    opts = pr._opts(1e-6, 64, flags=pr.PARARNN_FLAG_INJECT_WITHHOLD, inject_chunk=5,
                    timeout_us=20000)
    _, st, _ = _solve(x, opts=opts)
    assert st["status"] == "timeout", st
    h, st2, _ = _solve(x)
    assert st2["status"] == "converged"
    assert np.abs(h - _ref(x)).max() < TOL_STATE
