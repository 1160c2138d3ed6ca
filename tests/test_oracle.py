"""Pins of the fp64 CPU oracle against what the pages and the mathematics fix.

None of these compare the oracle with itself: each checks it against an
independent routine (torch's own GRU/LSTM cells and autograd, in float64),
central finite differences, closed forms, or the invariants the DEER
walkthrough states [Параллельность RNN?, §1.1-§1.3].
"""
import numpy as np
import pytest
import torch

import oracle
from nonlinear_rnn_paragru_b200.inputs import WORKLOADS, make_inputs



def _rand_gru(B, T, D, seed, a_range=1.0, bias_std=0.3):
    g = np.random.default_rng(seed)
    return dict(u=g.standard_normal((B, T, 3, D)),
                a=g.uniform(-a_range, a_range, (3, D)),
                bias=g.standard_normal((3, D)) * bias_std,
                h0=g.standard_normal((B, D)) * 0.5)


def _rand_lstm(B, T, D, seed, a_range=1.0, bias_std=0.3):
    g = np.random.default_rng(seed)
    return dict(u=g.standard_normal((B, T, 4, D)),
                a=g.uniform(-a_range, a_range, (4, D)),
                bias=g.standard_normal((4, D)) * bias_std,
                c0=g.standard_normal((B, D)) * 0.5,
                h0=g.standard_normal((B, D)) * 0.5)


# --------------------------------------------------------------------------
# torch float64 reference cells (library routines: nn.GRUCell / nn.LSTMCell)
# with the recurrent matrices set to diagonal blocks.
# --------------------------------------------------------------------------
def _torch_gru_cell(a, D):
    """nn.GRUCell computing h' = (1-z) h + z c with our z (torch's update
    gate is 1 - z, so its z-row carries -a_z and the input -(u_z + b_z))."""
    cell = torch.nn.GRUCell(3 * D, D, bias=False, dtype=torch.float64)
    with torch.no_grad():
        cell.weight_ih.copy_(torch.eye(3 * D, dtype=torch.float64))     # gate rows r, z, n
        whh = torch.zeros(3 * D, D, dtype=torch.float64)
        a = torch.as_tensor(a)
        whh[0:D] = torch.diag(a[1])        # r
        whh[D:2 * D] = torch.diag(-a[0])   # torch z = 1 - our z
        whh[2 * D:] = torch.diag(a[2])     # n: tanh(x_n + r * (W_hn h))
        cell.weight_hh.copy_(whh)
    return cell


def _torch_gru_x(u_t, bias):
    # u_t [B,3,D] (z,r,c) -> torch input (r, z, n) order
    b = torch.as_tensor(bias)
    u_t = torch.as_tensor(u_t)
    return torch.cat([u_t[:, 1] + b[1], -(u_t[:, 0] + b[0]), u_t[:, 2] + b[2]],
                     dim=1)


def _torch_gru_seq(u, a, bias, h0):
    B, T, _, D = u.shape
    cell = _torch_gru_cell(a, D)
    h = torch.as_tensor(h0).clone()
    out = []
    for t in range(T):
        h = cell(_torch_gru_x(u[:, t], bias), h)
        out.append(h)
    return torch.stack(out, 1)


def _torch_lstm_cell(a, D):
    cell = torch.nn.LSTMCell(4 * D, D, bias=False, dtype=torch.float64)
    with torch.no_grad():
        cell.weight_ih.copy_(torch.eye(4 * D, dtype=torch.float64))     # gate rows i, f, g, o
        whh = torch.zeros(4 * D, D, dtype=torch.float64)
        a = torch.as_tensor(a)
        for q in range(4):
            whh[q * D:(q + 1) * D] = torch.diag(a[q])
        cell.weight_hh.copy_(whh)
    return cell


def _torch_lstm_seq(u, a, bias, c0, h0):
    B, T, _, D = u.shape
    cell = _torch_lstm_cell(a, D)
    h, c = torch.as_tensor(h0).clone(), torch.as_tensor(c0).clone()
    b = torch.as_tensor(bias)
    hs, cs = [], []
    u = torch.as_tensor(u)
    for t in range(T):
        x = (u[:, t] + b).reshape(B, 4 * D)
        h, c = cell(x, (h, c))
        hs.append(h)
        cs.append(c)
    return torch.stack(cs, 1), torch.stack(hs, 1)


# ------------------------------------------------------------------ states --
def test_gru_seq_matches_torch_grucell():
    x = _rand_gru(2, 37, 5, seed=1)
    h = oracle.gru_seq(**x)
    with torch.no_grad():
        ht = _torch_gru_seq(x["u"], x["a"], x["bias"], x["h0"]).numpy()
    np.testing.assert_allclose(h, ht, rtol=0, atol=1e-13)


def test_lstm_seq_matches_torch_lstmcell():
    x = _rand_lstm(2, 37, 5, seed=2)
    c, h = oracle.lstm_seq(**x)
    with torch.no_grad():
        ct, ht = _torch_lstm_seq(x["u"], x["a"], x["bias"], x["c0"], x["h0"])
    np.testing.assert_allclose(c, ct.numpy(), rtol=0, atol=1e-12)
    np.testing.assert_allclose(h, ht.numpy(), rtol=0, atol=1e-13)


def test_seq_residual_is_exactly_zero():
    # The sequential trajectory satisfies every residual component exactly
    # [Параллельность RNN?, §1.1]; bitwise in fp64 (same step function).
    x = _rand_gru(2, 50, 7, seed=3)
    h = oracle.gru_seq(**x)
    res = oracle.gru_residual(x["u"], x["a"], x["bias"], x["h0"], h)
    assert np.all(res == 0.0)
    y = _rand_lstm(2, 50, 7, seed=4)
    c, h = oracle.lstm_seq(**y)
    rc, rh = oracle.lstm_residual(y["u"], y["a"], y["bias"], y["c0"], y["h0"],
                                  c, h)
    assert np.all(rc == 0.0) and np.all(rh == 0.0)


def test_residual_nonzero_off_trajectory():
    x = _rand_gru(1, 20, 3, seed=5)
    h = oracle.gru_seq(**x)
    h2 = h.copy()
    h2[0, 7, 1] += 1e-3
    res = oracle.gru_residual(x["u"], x["a"], x["bias"], x["h0"], h2)
    nz = np.argwhere(res != 0)
    # perturbing s_8 touches r_8 (directly) and r_9 (through f(s_8)) only
    assert {tuple(i) for i in nz} == {(0, 7, 1), (0, 8, 1)}
    assert res[0, 7, 1] == pytest.approx(1e-3, rel=1e-9)


# ------------------------------------------------------------- Jacobians --
def _fd(fun, x, eps=1e-6):
    return (fun(x + eps) - fun(x - eps)) / (2 * eps)


def test_gru_step_derivatives_vs_central_differences():
    g = np.random.default_rng(6)
    n = 64
    h = g.standard_normal(n)
    u = g.standard_normal((n, 3))
    a = g.uniform(-1, 1, (n, 3))
    b = g.standard_normal((n, 3)) * 0.3
    f, A, dfdu, dfda = oracle.gru_step(h, u, a, b)
    np.testing.assert_allclose(A, _fd(lambda hh: oracle.gru_step(hh, u, a, b)[0], h),
                               rtol=1e-7, atol=1e-9)
    for q in range(3):
        def fu(v, q=q):
            uu = u.copy(); uu[:, q] = v
            return oracle.gru_step(h, uu, a, b)[0]

        def fa(v, q=q):
            aa = a.copy(); aa[:, q] = v
            return oracle.gru_step(h, u, aa, b)[0]
        np.testing.assert_allclose(dfdu[:, q], _fd(fu, u[:, q]), rtol=1e-7, atol=1e-9)
        np.testing.assert_allclose(dfda[:, q], _fd(fa, a[:, q]), rtol=1e-7, atol=1e-9)


def test_gru_step_derivatives_vs_torch_autograd():
    g = np.random.default_rng(7)
    n = 16
    h = g.standard_normal(n)
    u = g.standard_normal((n, 3))
    a = g.uniform(-1, 1, (n, 3))
    b = g.standard_normal((n, 3)) * 0.3
    _, A, dfdu, dfda = oracle.gru_step(h, u, a, b)
    # torch cell per channel: D = n independent channels, B = 1
    ht = torch.tensor(h[None], requires_grad=True)
    ut = torch.tensor(u.T[None], requires_grad=True)          # [1,3,n]
    at = torch.tensor(a.T, requires_grad=True)                # [3,n]
    cell_out = _gru_functional(ht, ut, at, torch.tensor(b.T))
    gh, gu, ga = torch.autograd.grad(cell_out.sum(), (ht, ut, at))
    np.testing.assert_allclose(A, gh[0].numpy(), rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(dfdu, gu[0].T.numpy(), rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(dfda, ga.T.numpy(), rtol=1e-12, atol=1e-14)


def _gru_functional(h, u, a, b):
    # differentiable wrapper around nn.GRUCell's functional form
    D = h.shape[1]
    w_hh = torch.cat([torch.diag(a[1]), torch.diag(-a[0]), torch.diag(a[2])])
    x = torch.cat([u[:, 1] + b[1], -(u[:, 0] + b[0]), u[:, 2] + b[2]], dim=1)
    return torch._VF.gru_cell(x, h, torch.eye(3 * D, dtype=torch.float64), w_hh, None, None)


def test_lstm_step_derivatives_vs_central_differences():
    g = np.random.default_rng(8)
    n = 64
    c = g.standard_normal(n)
    h = g.standard_normal(n)
    u = g.standard_normal((n, 4))
    a = g.uniform(-1, 1, (n, 4))
    b = g.standard_normal((n, 4)) * 0.3
    fc, fh, A, dfdu, dfda = oracle.lstm_step(c, h, u, a, b)
    for p in range(2):  # output c', h'
        np.testing.assert_allclose(
            A[:, p, 0], _fd(lambda cc: oracle.lstm_step(cc, h, u, a, b)[p], c),
            rtol=1e-7, atol=1e-9)
        np.testing.assert_allclose(
            A[:, p, 1], _fd(lambda hh: oracle.lstm_step(c, hh, u, a, b)[p], h),
            rtol=1e-7, atol=1e-9)
        for q in range(4):
            def fu(v, q=q, p=p):
                uu = u.copy(); uu[:, q] = v
                return oracle.lstm_step(c, h, uu, a, b)[p]

            def fa(v, q=q, p=p):
                aa = a.copy(); aa[:, q] = v
                return oracle.lstm_step(c, h, u, aa, b)[p]
            np.testing.assert_allclose(dfdu[:, p, q], _fd(fu, u[:, q]), rtol=1e-7, atol=1e-9)
            np.testing.assert_allclose(dfda[:, p, q], _fd(fa, a[:, q]), rtol=1e-7, atol=1e-9)


# ------------------------------------------------------------------- BPTT --
def test_gru_bptt_vs_torch_autograd():
    x = _rand_gru(2, 23, 4, seed=9)
    g = np.random.default_rng(10).standard_normal((2, 23, 4))
    h = oracle.gru_seq(**x)
    out = oracle.gru_bptt(x["u"], x["a"], x["bias"], x["h0"], h, g)
    u = torch.tensor(x["u"], requires_grad=True)
    a = torch.tensor(x["a"], requires_grad=True)
    b = torch.tensor(x["bias"], requires_grad=True)
    h0 = torch.tensor(x["h0"], requires_grad=True)
    hh = h0
    hs = []
    for t in range(u.shape[1]):
        hh = _gru_functional(hh, u[:, t], a, b)
        hs.append(hh)
    L = (torch.stack(hs, 1) * torch.tensor(g)).sum()
    gu, ga, gb, gh0 = torch.autograd.grad(L, (u, a, b, h0))
    np.testing.assert_allclose(out["du"], gu.numpy(), rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(out["da"], ga.numpy(), rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(out["dbias"], gb.numpy(), rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(out["dh0"], gh0.numpy(), rtol=1e-10, atol=1e-12)


def test_lstm_bptt_vs_torch_autograd():
    x = _rand_lstm(2, 19, 3, seed=11)
    g = np.random.default_rng(12).standard_normal((2, 19, 3))
    c, h = oracle.lstm_seq(**x)
    out = oracle.lstm_bptt(x["u"], x["a"], x["bias"], x["c0"], x["h0"], c, h, g)
    u = torch.tensor(x["u"], requires_grad=True)
    a = torch.tensor(x["a"], requires_grad=True)
    b = torch.tensor(x["bias"], requires_grad=True)
    c0 = torch.tensor(x["c0"], requires_grad=True)
    h0 = torch.tensor(x["h0"], requires_grad=True)
    B, T, _, D = u.shape
    w_hh = torch.cat([torch.diag(a[q]) for q in range(4)])
    hh, cc = h0, c0
    hs = []
    for t in range(T):
        xt = (u[:, t] + b).reshape(B, 4 * D)
        hh, cc = torch._VF.lstm_cell(xt, (hh, cc), torch.eye(4 * D, dtype=torch.float64), w_hh, None, None)
        hs.append(hh)
    L = (torch.stack(hs, 1) * torch.tensor(g)).sum()
    gu, ga, gb, gc0, gh0 = torch.autograd.grad(L, (u, a, b, c0, h0))
    for k, ref in (("du", gu), ("da", ga), ("dbias", gb), ("dc0", gc0), ("dh0", gh0)):
        np.testing.assert_allclose(out[k], ref.numpy(), rtol=1e-10, atol=1e-12)


def test_gru_bptt_vs_finite_differences():
    x = _rand_gru(1, 6, 2, seed=13)
    g = np.random.default_rng(14).standard_normal((1, 6, 2))
    h = oracle.gru_seq(**x)
    out = oracle.gru_bptt(x["u"], x["a"], x["bias"], x["h0"], h, g)

    def loss(**kw):
        y = dict(x); y.update(kw)
        return float((oracle.gru_seq(**y) * g).sum())
    eps = 1e-6
    for idx in [(0, 0, 0, 0), (0, 3, 1, 1), (0, 5, 2, 0), (0, 2, 2, 1)]:
        up, um = x["u"].copy(), x["u"].copy()
        up[idx] += eps; um[idx] -= eps
        fd = (loss(u=up) - loss(u=um)) / (2 * eps)
        assert out["du"][idx] == pytest.approx(fd, rel=1e-6, abs=1e-9)
    for idx in [(0, 0), (1, 1), (2, 0)]:
        ap, am = x["a"].copy(), x["a"].copy()
        ap[idx] += eps; am[idx] -= eps
        fd = (loss(a=ap) - loss(a=am)) / (2 * eps)
        assert out["da"][idx] == pytest.approx(fd, rel=1e-6, abs=1e-9)


def test_lstm_bptt_vs_finite_differences():
    x = _rand_lstm(1, 6, 2, seed=15)
    g = np.random.default_rng(16).standard_normal((1, 6, 2))
    c, h = oracle.lstm_seq(**x)
    out = oracle.lstm_bptt(x["u"], x["a"], x["bias"], x["c0"], x["h0"], c, h, g)

    def loss(**kw):
        y = dict(x); y.update(kw)
        return float((oracle.lstm_seq(**y)[1] * g).sum())
    eps = 1e-6
    for idx in [(0, 0, 0, 0), (0, 3, 1, 1), (0, 5, 2, 0), (0, 2, 3, 1)]:
        up, um = x["u"].copy(), x["u"].copy()
        up[idx] += eps; um[idx] -= eps
        fd = (loss(u=up) - loss(u=um)) / (2 * eps)
        assert out["du"][idx] == pytest.approx(fd, rel=1e-6, abs=1e-9)
    for idx in [(0, 0), (1, 1), (2, 0), (3, 1)]:
        ap, am = x["a"].copy(), x["a"].copy()
        ap[idx] += eps; am[idx] -= eps
        fd = (loss(a=ap) - loss(a=am)) / (2 * eps)
        assert out["da"][idx] == pytest.approx(fd, rel=1e-6, abs=1e-9)


# ----------------------------------------------------------------- Newton --
@pytest.mark.parametrize("cell", ["gru", "lstm"])
def test_newton_prefix_exactness(cell):
    # ds_1 = -r_1 is exact [Параллельность RNN?, §1.3]; by induction over the
    # forward substitution, after k updates the first k states are the
    # sequential ones (brute force over every k for a tiny T).
    T = 12
    if cell == "gru":
        x = _rand_gru(1, T, 3, seed=17)
        ref = oracle.gru_seq(**x)
    else:
        x = _rand_lstm(1, T, 3, seed=18)
        ref_c, ref = oracle.lstm_seq(**x)
    for k in range(1, T + 1):
        if cell == "gru":
            r = oracle.gru_newton(**x, tol=0.0, max_iters=k)
            got = r["h"]
        else:
            r = oracle.lstm_newton(**x, tol=0.0, max_iters=k)
            got = r["h"]
            np.testing.assert_allclose(r["c"][:, :k], ref_c[:, :k], rtol=0, atol=1e-14)
        assert r["iters"] == k
        np.testing.assert_allclose(got[:, :k], ref[:, :k], rtol=0, atol=1e-14)
    # and T updates always suffice (exact in exact arithmetic)
    assert np.abs(got - ref).max() < 1e-13


def test_newton_affine_gru_converges_in_one_step():
    # a_z = a_c = 0 makes the ParaGRU step affine in h; Newton on an affine
    # residual is exact after one update [Параллельность RNN?, §1.2].
    x = _rand_gru(2, 64, 5, seed=19)
    x["a"][0] = 0.0
    x["a"][2] = 0.0
    r = oracle.gru_newton(**x, tol=1e-13, max_iters=10,
                          h_init=np.random.default_rng(20).standard_normal((2, 64, 5)))
    assert r["iters"] == 1
    assert r["trace"][1] < 1e-13
    np.testing.assert_allclose(r["h"], oracle.gru_seq(**x), rtol=0, atol=1e-13)


def test_newton_lstm_zero_weights_converges_in_two_steps():
    # a = 0: c is an affine recurrence independent of h; h' = o tanh(c') is
    # explicit given c, so the second update is exact.
    x = _rand_lstm(2, 64, 5, seed=21)
    x["a"][:] = 0.0
    r = oracle.lstm_newton(**x, tol=1e-13, max_iters=10)
    assert r["iters"] == 2
    assert r["trace"][1] > 1e-6 and r["trace"][2] < 1e-13


@pytest.mark.parametrize("cfg", [1, 2, 3, 4, 5])
def test_newton_reaches_sequential_root(cfg):
    w = WORKLOADS[cfg]
    ws = w.scaled(B=1, T=min(w.T, 512), D=32)
    x = make_inputs(ws)
    if w.cell == "gru":
        r = oracle.gru_newton(x["u"], x["a"], x["bias"], x["h0"], tol=1e-10,
                              max_iters=ws.T)
        ref = oracle.gru_seq(x["u"], x["a"], x["bias"], x["h0"])
        assert np.abs(r["h"] - ref).max() < 1e-9
    else:
        r = oracle.lstm_newton(x["u"], x["a"], x["bias"], x["c0"], x["h0"],
                               tol=1e-10, max_iters=ws.T)
        rc, ref = oracle.lstm_seq(x["u"], x["a"], x["bias"], x["c0"], x["h0"])
        assert np.abs(r["h"] - ref).max() < 1e-9
        assert np.abs(r["c"] - rc).max() < 1e-9
    assert r["trace"][-1] < 1e-10
    assert r["iters"] < ws.T


def _graded_inputs(cell, seed):
    # channel d gets recurrent weights scaled by 1.8 d / (D - 1) and inputs by
    # 0.3 .. 2: channel 0 is affine (a = 0), later ones need more iterations
    g = np.random.default_rng(seed)
    B, T, D = 2, 160, 8
    G = 3 if cell == "gru" else 4
    x = dict(u=g.standard_normal((B, T, G, D)) * np.linspace(0.3, 2.0, D),
             a=g.uniform(-1, 1, (G, D)) * np.linspace(0.0, 1.8, D),
             bias=g.standard_normal((G, D)) * 0.3,
             h0=g.standard_normal((B, D)) * 0.5)
    if cell == "lstm":
        x["c0"] = g.standard_normal((B, D)) * 0.5
    return x


@pytest.mark.parametrize("cell", ["gru", "lstm"])
def test_newton_chan_k_equals_solo_channel_runs(cell):
    # Channels of the diagonal cells are independent [Apple научила классические
    # RNN..., "Что именно сделали технически", item 3]: a channel's Newton
    # iterates inside the joint [B, T, D] system are those of the same channel
    # solved alone.  So its chan_k (the first iterate from which its own
    # max_t |r_t| stays below tol) must equal the update count of that solo run,
    # which stops at the first iterate below tol.  Recording the global maximum
    # (or any other channel's) instead fails: the counts below differ by channel.
    x = _graded_inputs(cell, 31)
    newton = oracle.gru_newton if cell == "gru" else oracle.lstm_newton
    r = newton(**x, tol=1e-6, max_iters=100)
    B, D = x["h0"].shape
    solo = np.zeros((B, D), dtype=np.int64)
    for b in range(B):
        for d in range(D):
            y = {k: np.ascontiguousarray(v[b:b + 1, ..., d:d + 1] if k in ("u", "h0", "c0")
                                         else v[:, d:d + 1]) for k, v in x.items()}
            solo[b, d] = newton(**y, tol=1e-6, max_iters=100)["iters"]
    assert len(np.unique(solo)) >= 3
    np.testing.assert_array_equal(r["chan_k"], solo)
    assert r["chan_k"].max() == r["iters"]
    # the affine channel (a = 0): one update for ParaGRU, two for ParaLSTM
    # [Параллельность RNN?, §1.2]
    assert (r["chan_k"][:, 0] == (1 if cell == "gru" else 2)).all()


# ------------------------------------------------------------------- scan --
def test_linrec_equals_closed_form_and_tree_order():
    # forward substitution == closed form (sum of products) == any
    # associative scan order [Параллельность RNN?, §1.3, Level 2]
    g = np.random.default_rng(23)
    n = 37
    A = g.uniform(-1.2, 1.2, n)
    b = g.standard_normal(n)
    x0 = 0.7
    xs = oracle.linrec(A, b, x0)
    # closed form: x_t = (prod_{s<=t} A_s) x0 + sum_j (prod_{j<s<=t} A_s) b_j
    closed = np.empty(n)
    for t in range(n):
        acc = np.prod(A[: t + 1]) * x0
        for j in range(t + 1):
            acc += np.prod(A[j + 1: t + 1]) * b[j]
        closed[t] = acc
    np.testing.assert_allclose(xs, closed, rtol=1e-12, atol=1e-12)
    # Hillis-Steele inclusive scan with the affine composition
    # (A2, b2) o (A1, b1) = (A2 A1, A2 b1 + b2)
    PA, Pb = A.copy(), b.copy()
    Pb[0] += A[0] * x0
    PA[0] = 0.0
    step = 1
    while step < n:
        nA, nb = PA.copy(), Pb.copy()
        for t in range(step, n):
            nA[t] = PA[t] * PA[t - step]
            nb[t] = PA[t] * Pb[t - step] + Pb[t]
        PA, Pb = nA, nb
        step *= 2
    np.testing.assert_allclose(xs, Pb, rtol=1e-12, atol=1e-12)


# ------------------------------------------- general cell (dense Jacobian) --
def _rand_dense(B, T, D, seed, w_scale=1.0):
    g = np.random.default_rng(seed)
    return dict(u=g.standard_normal((B, T, 3, D)),
                W=g.uniform(-1, 1, (3, D, D)) * w_scale / np.sqrt(D),
                bias=g.standard_normal((3, D)) * 0.3,
                h0=g.standard_normal((B, D)) * 0.5)


def _torch_dense_gru_cell(W, D):
    """nn.GRUCell with full recurrent matrices; our z is torch's 1 - z."""
    cell = torch.nn.GRUCell(3 * D, D, bias=False, dtype=torch.float64)
    W = torch.as_tensor(W)
    with torch.no_grad():
        cell.weight_ih.copy_(torch.eye(3 * D, dtype=torch.float64))     # gate rows r, z, n
        cell.weight_hh.copy_(torch.cat([W[1], -W[0], W[2]], 0))
    return cell


def test_dense_gru_seq_matches_torch_grucell():
    x = _rand_dense(2, 23, 7, seed=11)
    h = oracle.dense_gru_seq(**x)
    cell = _torch_dense_gru_cell(x["W"], 7)
    hh = torch.as_tensor(x["h0"]).clone()
    out = []
    with torch.no_grad():
        for t in range(23):
            hh = cell(_torch_gru_x(x["u"][:, t], x["bias"]), hh)
            out.append(hh)
    np.testing.assert_allclose(h, torch.stack(out, 1).numpy(), rtol=0, atol=1e-13)


def test_dense_gru_with_diagonal_matrices_is_paragru():
    x = _rand_gru(3, 40, 6, seed=12)
    W = np.stack([np.diag(x["a"][g]) for g in range(3)])
    hd = oracle.dense_gru_seq(x["u"], W, x["bias"], x["h0"])
    np.testing.assert_allclose(hd, oracle.gru_seq(**x), rtol=0, atol=1e-14)
    # one step: the dense Jacobian is diagonal with ParaGRU's A on it
    hp = x["h0"]
    f, J = oracle.dense_gru_step(hp, x["u"][:, 0], W, x["bias"])
    for b in range(3):
        f1, A1, _, _ = oracle.gru_step(hp[b], x["u"][b, 0].T, x["a"].T, x["bias"].T)
        np.testing.assert_allclose(f[b], f1, rtol=0, atol=1e-14)
        np.testing.assert_allclose(J[b], np.diag(A1), rtol=0, atol=1e-14)


def test_dense_gru_jacobian_vs_torch_autograd():
    D = 6
    x = _rand_dense(2, 1, D, seed=13, w_scale=2.0)
    _, J = oracle.dense_gru_step(x["h0"], x["u"][:, 0], x["W"], x["bias"])
    cell = _torch_dense_gru_cell(x["W"], D)
    for b in range(2):
        xt = _torch_gru_x(x["u"][b:b + 1, 0], x["bias"])
        Jt = torch.autograd.functional.jacobian(
            lambda h: cell(xt, h.unsqueeze(0))[0], torch.as_tensor(x["h0"][b]))
        np.testing.assert_allclose(J[b], Jt.numpy(), rtol=0, atol=1e-12)


def test_dense_gru_jacobian_vs_central_differences():
    D = 5
    x = _rand_dense(1, 1, D, seed=14, w_scale=2.0)
    h, u = x["h0"], x["u"][:, 0]
    _, J = oracle.dense_gru_step(h, u, x["W"], x["bias"])
    eps = 1e-6
    for j in range(D):
        e = np.zeros((1, D))
        e[0, j] = eps
        fp, _ = oracle.dense_gru_step(h + e, u, x["W"], x["bias"])
        fm, _ = oracle.dense_gru_step(h - e, u, x["W"], x["bias"])
        np.testing.assert_allclose(J[0][:, j], ((fp - fm) / (2 * eps))[0], rtol=0, atol=1e-8)


def test_dense_newton_prefix_exactness_and_root():
    # after k updates the first k states are exact [P4 §1.3: the first block
    # row of J ds = -r involves ds_1 alone, and so on down the bidiagonal]
    x = _rand_dense(2, 12, 5, seed=15, w_scale=1.5)
    ref = oracle.dense_gru_seq(**x)
    for k in range(1, 6):
        r = oracle.dense_gru_newton(**x, tol=0.0, max_iters=k)
        assert r["iters"] == k
        np.testing.assert_allclose(r["h"][:, :k], ref[:, :k], rtol=0, atol=1e-12)
        if k <= 2:   # (Newton converges quadratically, so only early on)
            assert np.abs(r["h"][:, k:] - ref[:, k:]).max() > 1e-6   # not exact further on
    r = oracle.dense_gru_newton(**x, tol=1e-12, max_iters=40)
    assert r["trace"][-1] < 1e-12
    np.testing.assert_allclose(r["h"], ref, rtol=0, atol=1e-12)


def test_dense_newton_with_diagonal_matrices_follows_paragru_newton():
    x = _rand_gru(2, 30, 4, seed=16)
    W = np.stack([np.diag(x["a"][g]) for g in range(3)])
    for n in (1, 2, 3):
        rd = oracle.dense_gru_newton(x["u"], W, x["bias"], x["h0"], tol=0.0, max_iters=n)
        rg = oracle.gru_newton(**x, tol=0.0, max_iters=n)
        np.testing.assert_allclose(rd["h"], rg["h"], rtol=0, atol=1e-13)


def test_dense_affine_maps_compose_in_any_grouping():
    # ds_t = J_t ds_{t-1} + b_t with full D x D blocks [P4 §1.3]: forward
    # substitution, 16-step chunks (chunk maps, carries, re-run) and a
    # Hillis-Steele tree of (J, b) maps give the same trajectory
    g = np.random.default_rng(17)
    T, D = 53, 6
    J = g.uniform(-1, 1, (T, D, D)) / np.sqrt(D)
    b = g.standard_normal((T, D))
    x, fs = np.zeros(D), []
    for t in range(T):
        x = J[t] @ x + b[t]
        fs.append(x)
    fs = np.array(fs)
    L = 16
    chunks = [(J[k:k + L], b[k:k + L]) for k in range(0, T, L)]
    maps = []
    for Jc, bc in chunks:
        P, dv = np.eye(D), np.zeros(D)
        for Jt, bt in zip(Jc, bc):
            P, dv = Jt @ P, Jt @ dv + bt
        maps.append((P, dv))
    carry, cs = np.zeros(D), []
    for P, dv in maps:
        cs.append(carry)
        carry = P @ carry + dv
    out = []
    for (Jc, bc), c0 in zip(chunks, cs):
        x = c0
        for Jt, bt in zip(Jc, bc):
            x = Jt @ x + bt
            out.append(x)
    np.testing.assert_allclose(np.array(out), fs, rtol=0, atol=1e-12)
    A, B_ = J.copy(), b.copy()          # inclusive prefix maps by doubling
    s = 1
    while s < T:
        A2, B2 = A.copy(), B_.copy()
        for t in range(s, T):
            A2[t] = A[t] @ A[t - s]
            B2[t] = A[t] @ B_[t - s] + B_[t]
        A, B_, s = A2, B2, 2 * s
    np.testing.assert_allclose(B_, fs, rtol=0, atol=1e-12)   # applied to x_0 = 0
