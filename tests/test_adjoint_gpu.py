"""GPU parity of the reverse adjoint scan against fp64 BPTT.

Gradients must match within 1e-3 relative per tensor:
max|g - g_ref| / max|g_ref| <= 1e-3.
"""
import numpy as np
import pytest
import torch

import oracle
import nonlinear_rnn_paragru_b200 as pr
from nonlinear_rnn_paragru_b200.inputs import WORKLOADS, make_inputs

pytestmark = pytest.mark.gpu

TOL_GRAD = 1e-3


def _rel(a, ref):
    return float(np.abs(a - ref).max() / max(np.abs(ref).max(), 1e-30))


def _gpu_adjoint(cell, x, h, c=None):
    d = "cuda"
    out = pr.adjoint(cell, x["u"].to(d), x["a"].to(d), x["bias"].to(d),
                     x["h0"].to(d), torch.as_tensor(h, dtype=torch.float32).to(d).contiguous(),
                     x["dLdh"].to(d),
                     c0=(x["c0"].to(d) if cell == pr.PARARNN_LSTM else None),
                     c=(torch.as_tensor(c, dtype=torch.float32).to(d).contiguous()
                        if c is not None else None))
    torch.cuda.synchronize()
    res = {k: (v.cpu().numpy() if v is not None else None) for k, v in out.items()}
    return res


def _check_gru(x, h):
    g = _gpu_adjoint(pr.PARARNN_GRU, x, h)
    assert int(g["status"][0]) == 0
    # the oracle differentiates the same (fp32-rounded) trajectory
    ref = oracle.gru_bptt(x["u"], x["a"], x["bias"], x["h0"],
                          h.astype(np.float32).astype(np.float64), x["dLdh"])
    for k in ("du", "da", "dbias", "dh0"):
        assert _rel(g[k], ref[k]) <= TOL_GRAD, (k, _rel(g[k], ref[k]))


def _check_lstm(x, c, h):
    g = _gpu_adjoint(pr.PARARNN_LSTM, x, h, c)
    assert int(g["status"][0]) == 0
    ref = oracle.lstm_bptt(x["u"], x["a"], x["bias"], x["c0"], x["h0"],
                           c.astype(np.float32).astype(np.float64),
                           h.astype(np.float32).astype(np.float64), x["dLdh"])
    for k in ("du", "da", "dbias", "dh0", "dc0"):
        assert _rel(g[k], ref[k]) <= TOL_GRAD, (k, _rel(g[k], ref[k]))


@pytest.mark.parametrize("B,T,D", [(2, 1000, 64), (1, 256, 32), (1, 1, 8),
                                   (3, 300, 40), (1, 3000, 32)])
def test_gru_adjoint_shapes(cuda_ok, B, T, D):
    x = make_inputs(WORKLOADS[2].scaled(B=B, T=T, D=D))
    h = oracle.gru_seq(x["u"], x["a"], x["bias"], x["h0"])
    _check_gru(x, h)


def test_gru_adjoint_lookback_path(cuda_ok):
    # fp32 projections and T > 4096 take the chunked look-back adjoint; bf16
    # with T <= 4096 (the shapes above) the whole-sequence one
    x = make_inputs(WORKLOADS[4].scaled(B=2, T=700, D=24), with_grad=True)
    _check_gru(x, oracle.gru_seq(x["u"], x["a"], x["bias"], x["h0"]))
    y = make_inputs(WORKLOADS[2].scaled(B=1, T=5000, D=16))
    _check_gru(y, oracle.gru_seq(y["u"], y["a"], y["bias"], y["h0"]))


@pytest.mark.parametrize("B,T,D", [(2, 700, 64), (1, 128, 32), (1, 3, 8), (1, 2500, 40)])
def test_lstm_adjoint_shapes(cuda_ok, B, T, D):
    x = make_inputs(WORKLOADS[5].scaled(B=B, T=T, D=D))
    c, h = oracle.lstm_seq(x["u"], x["a"], x["bias"], x["c0"], x["h0"])
    _check_lstm(x, c, h)


def test_gru_fwd_then_adjoint_end_to_end(cuda_ok):
    # the GPU trajectory feeds the GPU adjoint; compared with BPTT on the
    # exact sequential trajectory
    x = make_inputs(WORKLOADS[2].scaled(B=2, T=2048, D=128))
    d = "cuda"
    h, st, _ = pr.gru_solve(x["u"].to(d), x["a"].to(d), x["bias"].to(d), x["h0"].to(d))
    g = pr.adjoint(pr.PARARNN_GRU, x["u"].to(d), x["a"].to(d), x["bias"].to(d),
                   x["h0"].to(d), h, x["dLdh"].to(d))
    torch.cuda.synchronize()
    href = oracle.gru_seq(x["u"], x["a"], x["bias"], x["h0"])
    ref = oracle.gru_bptt(x["u"], x["a"], x["bias"], x["h0"], href, x["dLdh"])
    for k in ("du", "da", "dbias", "dh0"):
        assert _rel(g[k].cpu().numpy(), ref[k]) <= TOL_GRAD, k


def test_gru_adjoint_config2_full_size(cuda_ok):
    x = make_inputs(WORKLOADS[2])
    h = oracle.gru_seq(x["u"], x["a"], x["bias"], x["h0"])
    _check_gru(x, h)


def test_lstm_adjoint_config5_full_size(cuda_ok):
    x = make_inputs(WORKLOADS[5])
    c, h = oracle.lstm_seq(x["u"], x["a"], x["bias"], x["c0"], x["h0"])
    _check_lstm(x, c, h)


def test_adjoint_is_bitwise_reproducible(cuda_ok):
    x = make_inputs(WORKLOADS[2].scaled(B=2, T=1500, D=64))
    h = oracle.gru_seq(x["u"], x["a"], x["bias"], x["h0"])
    a = _gpu_adjoint(pr.PARARNN_GRU, x, h)
    b = _gpu_adjoint(pr.PARARNN_GRU, x, h)
    for k in ("du", "da", "dbias", "dh0"):
        assert np.array_equal(a[k], b[k]), k


@pytest.mark.parametrize("T", [1500, 4500])
def test_gru_adjoint_nonzero_h0_without_bias(cuda_ok, T):
    # the state before the first step is h0, not the zero fill of a load that
    # starts before the sequence; an absent bias reads as zero.  T = 1500
    # takes the whole-sequence adjoint, T = 4500 the look-back one.
    x = make_inputs(WORKLOADS[2].scaled(B=2, T=T, D=24))
    x["h0"] = torch.randn((2, 24), generator=torch.Generator().manual_seed(7)) * 0.5
    x["bias"] = torch.zeros_like(x["bias"])
    h = oracle.gru_seq(x["u"], x["a"], x["bias"], x["h0"])
    d = "cuda"
    out = pr.adjoint(pr.PARARNN_GRU, x["u"].to(d), x["a"].to(d), None, x["h0"].to(d),
                     torch.as_tensor(h, dtype=torch.float32).to(d).contiguous(),
                     x["dLdh"].to(d))
    torch.cuda.synchronize()
    g = {k: (v.cpu().numpy() if v is not None else None) for k, v in out.items()}
    assert int(g["status"][0]) == 0
    ref = oracle.gru_bptt(x["u"], x["a"], x["bias"], x["h0"],
                          h.astype(np.float32).astype(np.float64), x["dLdh"])
    for k in ("du", "da", "dbias", "dh0"):
        assert _rel(g[k], ref[k]) <= TOL_GRAD, (k, _rel(g[k], ref[k]))


def test_lstm_adjoint_nonzero_initial_state(cuda_ok):
    x = make_inputs(WORKLOADS[5].scaled(B=2, T=700, D=32))
    gen = torch.Generator().manual_seed(9)
    x["c0"] = torch.randn((2, 32), generator=gen) * 0.5
    x["h0"] = torch.randn((2, 32), generator=gen) * 0.5
    c, h = oracle.lstm_seq(x["u"], x["a"], x["bias"], x["c0"], x["h0"])
    _check_lstm(x, c, h)


def test_lstm_adjoint_lookback_path(cuda_ok):
    # fp32 projections and T > 4096 take the chunked look-back adjoint; bf16
    # with T <= 4096 (the shapes above) the whole-sequence one
    x = make_inputs(WORKLOADS[5].scaled(B=2, T=500, D=24))
    x["u"] = x["u"].float()  # the same values, read as fp32
    c, h = oracle.lstm_seq(x["u"], x["a"], x["bias"], x["c0"], x["h0"])
    _check_lstm(x, c, h)
    y = make_inputs(WORKLOADS[5].scaled(B=1, T=4500, D=16))
    c, h = oracle.lstm_seq(y["u"], y["a"], y["bias"], y["c0"], y["h0"])
    _check_lstm(y, c, h)


def test_lstm_adjoint_is_bitwise_reproducible(cuda_ok):
    x = make_inputs(WORKLOADS[5].scaled(B=2, T=1500, D=32))
    c, h = oracle.lstm_seq(x["u"], x["a"], x["bias"], x["c0"], x["h0"])
    g1 = _gpu_adjoint(pr.PARARNN_LSTM, x, h, c)
    g2 = _gpu_adjoint(pr.PARARNN_LSTM, x, h, c)
    for k in ("du", "da", "dbias", "dh0", "dc0"):
        assert np.array_equal(g1[k], g2[k]), k


@pytest.mark.parametrize("cell", ["gru", "lstm"])
def test_adjoint_clusters_with_many_tiles(cuda_ok, cell):
    # T = 1000 takes clusters of 2 CTAs; 1024 tiles of 8 channels give each
    # cluster about seven, so the mailbox ring turns over many times while the
    # last rank (which receives nothing) runs ahead of the first
    w = WORKLOADS[2 if cell == "gru" else 5].scaled(B=8, T=1000, D=1024)
    x = make_inputs(w)
    if cell == "gru":
        h = oracle.gru_seq(x["u"], x["a"], x["bias"], x["h0"])
        _check_gru(x, h)
    else:
        c, h = oracle.lstm_seq(x["u"], x["a"], x["bias"], x["c0"], x["h0"])
        _check_lstm(x, c, h)


@pytest.mark.parametrize("cell,wl", [(pr.PARARNN_GRU, 2), (pr.PARARNN_GRU, 4),
                                     (pr.PARARNN_LSTM, 5)])
def test_nan_input_reports_nonfinite(cuda_ok, cell, wl):
    # bf16 u: the whole-sequence adjoint; fp32 u (workload 4): the look-back one
    x = make_inputs(WORKLOADS[wl].scaled(B=1, T=600, D=32), with_grad=True)
    if cell == pr.PARARNN_GRU:
        h = oracle.gru_seq(x["u"], x["a"], x["bias"], x["h0"])
        c = None
    else:
        c, h = oracle.lstm_seq(x["u"], x["a"], x["bias"], x["c0"], x["h0"])
    x["u"][0, 200, 0, 3] = float("nan")
    g = _gpu_adjoint(cell, x, h, c)
    assert int(g["status"][0]) == 2          # PARARNN_STATUS_NONFINITE


@pytest.mark.parametrize("cell,wl,T,inject", [
    (pr.PARARNN_GRU, 4, 700, 0),     # fp32 u: look-back; ticket 0 (the last chunk) withholds
    (pr.PARARNN_GRU, 2, 1500, 2),    # bf16 u: whole sequence, cluster rank 2 withholds
    (pr.PARARNN_LSTM, 5, 1500, 1)])
def test_withheld_exchange_times_out(cuda_ok, cell, wl, T, inject):
    x = make_inputs(WORKLOADS[wl].scaled(B=1, T=T, D=8 if wl != 4 else 32), with_grad=True)
    if cell == pr.PARARNN_GRU:
        h = oracle.gru_seq(x["u"], x["a"], x["bias"], x["h0"])
        c = None
    else:
        c, h = oracle.lstm_seq(x["u"], x["a"], x["bias"], x["c0"], x["h0"])
    d = "cuda"
    opts = pr._opts(flags=pr.PARARNN_FLAG_INJECT_WITHHOLD, inject_chunk=inject,
                    timeout_us=20000)
    out = pr.adjoint(cell, x["u"].to(d), x["a"].to(d), x["bias"].to(d), x["h0"].to(d),
                     torch.as_tensor(h, dtype=torch.float32).to(d).contiguous(), x["dLdh"].to(d),
                     c0=(x["c0"].to(d) if c is not None else None),
                     c=(torch.as_tensor(c, dtype=torch.float32).to(d).contiguous()
                        if c is not None else None), opts=opts)
    torch.cuda.synchronize()
    assert int(out["status"][0]) == 3          # PARARNN_STATUS_TIMEOUT
    # the next call on the same device is clean
    if cell == pr.PARARNN_GRU:
        _check_gru(x, h)
    else:
        _check_lstm(x, c, h)


# ---- the ParaGRU queue adjoint (bf16 u, at least one 32-channel tile per
# resident CTA: 148 on a B200): every 128-step segment in one
# launch, last segments first, each segment's carry from the one after it
@pytest.mark.parametrize("B,T,D", [(1, 700, 6000), (2, 1300, 3000), (1, 256, 6000),
                                   (1, 130, 4736), (1, 1, 6000), (1, 128, 4800)])
def test_queue_adjoint_matches_bptt(cuda_ok, B, T, D):
    x = make_inputs(WORKLOADS[2].scaled(B=B, T=T, D=D))
    x["h0"] = torch.randn((B, D), generator=torch.Generator().manual_seed(37)) * 0.5
    h = oracle.gru_seq(x["u"], x["a"], x["bias"], x["h0"])
    _check_gru(x, h)
    # and the whole-sequence kernel on the same inputs
    d = "cuda"
    hh = torch.as_tensor(h, dtype=torch.float32).to(d).contiguous()
    q = pr.adjoint(pr.PARARNN_GRU, x["u"].to(d), x["a"].to(d), x["bias"].to(d), x["h0"].to(d),
                   hh, x["dLdh"].to(d))
    r = pr.adjoint(pr.PARARNN_GRU, x["u"].to(d), x["a"].to(d), x["bias"].to(d), x["h0"].to(d),
                   hh, x["dLdh"].to(d), opts=pr._opts(flags=pr.PARARNN_FLAG_FORCE_ROW))
    torch.cuda.synchronize()
    for k in ("du", "da", "dbias", "dh0"):
        assert _rel(q[k].cpu().numpy(), r[k].cpu().numpy()) <= TOL_GRAD, k


def test_queue_adjoint_is_bitwise_reproducible(cuda_ok):
    x = make_inputs(WORKLOADS[2].scaled(B=1, T=900, D=6000))
    h = oracle.gru_seq(x["u"], x["a"], x["bias"], x["h0"])
    a = _gpu_adjoint(pr.PARARNN_GRU, x, h)
    b = _gpu_adjoint(pr.PARARNN_GRU, x, h)
    for k in ("du", "da", "dbias", "dh0"):
        assert np.array_equal(a[k], b[k]), k


def test_queue_adjoint_withheld_carry_times_out(cuda_ok):
    # item 5 (the last segment of tile 5) never publishes its carry: the
    # segment before it waits until its bounded wait runs out
    x = make_inputs(WORKLOADS[2].scaled(B=1, T=600, D=6000))
    h = oracle.gru_seq(x["u"], x["a"], x["bias"], x["h0"])
    d = "cuda"
    opts = pr._opts(flags=pr.PARARNN_FLAG_INJECT_WITHHOLD, inject_chunk=5, timeout_us=20000)
    out = pr.adjoint(pr.PARARNN_GRU, x["u"].to(d), x["a"].to(d), x["bias"].to(d), x["h0"].to(d),
                     torch.as_tensor(h, dtype=torch.float32).to(d).contiguous(), x["dLdh"].to(d),
                     opts=opts)
    torch.cuda.synchronize()
    assert int(out["status"][0]) == 3
    _check_gru(x, h)


def _offset_view(t, d="cuda"):
    # the same values one float past a 16-byte boundary (4-byte aligned only)
    buf = torch.empty(t.numel() + 4, dtype=t.dtype, device=d)
    v = buf[1:1 + t.numel()].view(t.shape)
    v.copy_(t.to(d))
    assert v.data_ptr() % 16 == 4
    return v


@pytest.mark.parametrize("cell,B,T,D", [(pr.PARARNN_GRU, 1, 700, 6000),
                                        (pr.PARARNN_GRU, 2, 1000, 64),
                                        (pr.PARARNN_LSTM, 1, 700, 4800)])
def test_adjoint_rows_4byte_aligned(cuda_ok, cell, B, T, D):
    # rows of a, bias, h0 (c0) that are 4-byte but not 16-byte aligned cannot
    # be staged by bulk copies: the call takes the look-back adjoint, whose
    # gradients match BPTT and the aligned call's
    lstm = cell == pr.PARARNN_LSTM
    x = make_inputs(WORKLOADS[3 if lstm else 2].scaled(B=B, T=T, D=D), with_grad=True)
    d = "cuda"
    if lstm:
        c, h = oracle.lstm_seq(x["u"], x["a"], x["bias"], x["c0"], x["h0"])
        ref = oracle.lstm_bptt(x["u"], x["a"], x["bias"], x["c0"], x["h0"],
                               c.astype(np.float32).astype(np.float64),
                               h.astype(np.float32).astype(np.float64), x["dLdh"])
        keys = ("du", "da", "dbias", "dh0", "dc0")
    else:
        c, h = None, oracle.gru_seq(x["u"], x["a"], x["bias"], x["h0"])
        ref = oracle.gru_bptt(x["u"], x["a"], x["bias"], x["h0"],
                              h.astype(np.float32).astype(np.float64), x["dLdh"])
        keys = ("du", "da", "dbias", "dh0")
    hh = torch.as_tensor(h, dtype=torch.float32).to(d).contiguous()
    cc = torch.as_tensor(c, dtype=torch.float32).to(d).contiguous() if lstm else None
    outs = []
    for shift in (False, True):
        prep = _offset_view if shift else (lambda t: t.to(d))
        outs.append(pr.adjoint(cell, x["u"].to(d), prep(x["a"]), prep(x["bias"]),
                               prep(x["h0"]), hh, x["dLdh"].to(d),
                               c0=prep(x["c0"]) if lstm else None, c=cc))
    torch.cuda.synchronize()
    for o in outs:
        assert int(o["status"][0]) == 0
        for k in keys:
            assert _rel(o[k].cpu().numpy(), ref[k]) <= TOL_GRAD, k
    for k in keys:
        assert _rel(outs[1][k].cpu().numpy(), outs[0][k].cpu().numpy()) <= TOL_GRAD, k


# ---- the ParaLSTM queue adjoint (bf16 u, at least one 32-channel tile per
# resident CTA: 148 on a B200)
def _lstm_queue_inputs(B, T, D):
    x = make_inputs(WORKLOADS[3].scaled(B=B, T=T, D=D), with_grad=True)
    g = torch.Generator().manual_seed(41)
    x["c0"] = torch.randn((B, D), generator=g) * 0.5
    x["h0"] = torch.randn((B, D), generator=g) * 0.5
    c, h = oracle.lstm_seq(x["u"], x["a"], x["bias"], x["c0"], x["h0"])
    return x, c, h


@pytest.mark.parametrize("B,T,D", [(1, 700, 4800), (2, 1300, 2400), (1, 256, 4800),
                                   (1, 1, 4736), (1, 130, 4808)])
def test_lstm_queue_adjoint_matches_bptt(cuda_ok, B, T, D):
    x, c, h = _lstm_queue_inputs(B, T, D)
    _check_lstm(x, c, h)
    # and the whole-sequence kernel on the same inputs
    d = "cuda"
    hh = torch.as_tensor(h, dtype=torch.float32).to(d).contiguous()
    cc = torch.as_tensor(c, dtype=torch.float32).to(d).contiguous()
    args = (pr.PARARNN_LSTM, x["u"].to(d), x["a"].to(d), x["bias"].to(d), x["h0"].to(d), hh,
            x["dLdh"].to(d))
    q = pr.adjoint(*args, c0=x["c0"].to(d), c=cc)
    r = pr.adjoint(*args, c0=x["c0"].to(d), c=cc, opts=pr._opts(flags=pr.PARARNN_FLAG_FORCE_ROW))
    torch.cuda.synchronize()
    for k in ("du", "da", "dbias", "dh0", "dc0"):
        assert _rel(q[k].cpu().numpy(), r[k].cpu().numpy()) <= TOL_GRAD, k


def test_lstm_queue_adjoint_is_bitwise_reproducible(cuda_ok):
    x, c, h = _lstm_queue_inputs(1, 900, 4800)
    a = _gpu_adjoint(pr.PARARNN_LSTM, x, h, c)
    b = _gpu_adjoint(pr.PARARNN_LSTM, x, h, c)
    for k in ("du", "da", "dbias", "dh0", "dc0"):
        assert np.array_equal(a[k], b[k]), k


def test_lstm_queue_adjoint_withheld_carry_times_out(cuda_ok):
    # item 5 (the last segment of tile 5) never publishes its carry
    x, c, h = _lstm_queue_inputs(1, 600, 4800)
    d = "cuda"
    opts = pr._opts(flags=pr.PARARNN_FLAG_INJECT_WITHHOLD, inject_chunk=5, timeout_us=20000)
    out = pr.adjoint(pr.PARARNN_LSTM, x["u"].to(d), x["a"].to(d), x["bias"].to(d),
                     x["h0"].to(d), torch.as_tensor(h, dtype=torch.float32).to(d).contiguous(),
                     x["dLdh"].to(d), c0=x["c0"].to(d),
                     c=torch.as_tensor(c, dtype=torch.float32).to(d).contiguous(), opts=opts)
    torch.cuda.synchronize()
    assert int(out["status"][0]) == 3
    _check_lstm(x, c, h)
