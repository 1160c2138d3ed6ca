"""GPU parity of the single-step decode entry points against the fp64 oracle's
sequential recurrence (max-abs 1e-4 on the states, as for the solves)."""
import numpy as np
import pytest
import torch

import oracle
import nonlinear_rnn_paragru_b200 as pr
from nonlinear_rnn_paragru_b200.inputs import WORKLOADS, make_inputs

pytestmark = pytest.mark.gpu

TOL_STATE = 1e-4


@pytest.mark.parametrize("wl", [2, 4])   # bf16 and fp32 projections
def test_gru_steps_continue_the_solve(cuda_ok, wl):
    # solve the first T0 steps in parallel, then decode the rest one step at a
    # time from the last solved state (in place); the whole trajectory must
    # match the sequential recurrence
    B, T, D, T0 = 3, 300, 40, 256
    x = make_inputs(WORKLOADS[wl].scaled(B=B, T=T, D=D))
    x["h0"] = torch.randn((B, D), generator=torch.Generator().manual_seed(3)) * 0.5
    ref = oracle.gru_seq(x["u"], x["a"], x["bias"], x["h0"])
    d = "cuda"
    u, a, bias = x["u"].to(d), x["a"].to(d), x["bias"].to(d)
    h, st, _ = pr.gru_solve(u[:, :T0].contiguous(), a, bias, x["h0"].to(d))
    state = h[:, -1].contiguous()
    steps = []
    for t in range(T0, T):
        pr.gru_step(u[:, t].contiguous(), a, bias, state, out=state)
        steps.append(state.clone())
    torch.cuda.synchronize()
    got = np.concatenate([h.cpu().numpy(), torch.stack(steps, 1).cpu().numpy()], axis=1)
    assert np.abs(got - ref).max() < TOL_STATE


def test_gru_step_from_zero_state_without_bias(cuda_ok):
    x = make_inputs(WORKLOADS[2].scaled(B=4, T=1, D=64))
    x["bias"] = torch.zeros_like(x["bias"])
    ref = oracle.gru_seq(x["u"], x["a"], x["bias"], torch.zeros((4, 64)))[:, 0]
    d = "cuda"
    h = pr.gru_step(x["u"][:, 0].contiguous().to(d), x["a"].to(d))
    torch.cuda.synchronize()
    assert np.abs(h.cpu().numpy() - ref).max() < TOL_STATE


@pytest.mark.parametrize("f32", [False, True])
def test_lstm_steps_continue_the_solve(cuda_ok, f32):
    B, T, D, T0 = 2, 200, 48, 150
    x = make_inputs(WORKLOADS[3].scaled(B=B, T=T, D=D))
    if f32:
        x["u"] = x["u"].float()  # the same values, read as fp32
    gen = torch.Generator().manual_seed(4)
    x["c0"] = torch.randn((B, D), generator=gen) * 0.5
    x["h0"] = torch.randn((B, D), generator=gen) * 0.5
    rc, rh = oracle.lstm_seq(x["u"], x["a"], x["bias"], x["c0"], x["h0"])
    d = "cuda"
    u, a, bias = x["u"].to(d), x["a"].to(d), x["bias"].to(d)
    c, h, st, _ = pr.lstm_solve(u[:, :T0].contiguous(), a, bias, x["c0"].to(d), x["h0"].to(d))
    cs, hs = c[:, -1].contiguous(), h[:, -1].contiguous()
    out_c, out_h = [], []
    for t in range(T0, T):
        pr.lstm_step(u[:, t].contiguous(), a, bias, cs, hs, out=(cs, hs))
        out_c.append(cs.clone())
        out_h.append(hs.clone())
    torch.cuda.synchronize()
    gc = np.concatenate([c.cpu().numpy(), torch.stack(out_c, 1).cpu().numpy()], axis=1)
    gh = np.concatenate([h.cpu().numpy(), torch.stack(out_h, 1).cpu().numpy()], axis=1)
    assert max(np.abs(gc - rc).max(), np.abs(gh - rh).max()) < TOL_STATE


def test_step_in_place_equals_out_of_place(cuda_ok):
    x = make_inputs(WORKLOADS[3].scaled(B=2, T=1, D=64))
    d = "cuda"
    gen = torch.Generator().manual_seed(6)
    c0 = (torch.randn((2, 64), generator=gen) * 0.5).to(d)
    h0 = (torch.randn((2, 64), generator=gen) * 0.5).to(d)
    u_t, a, bias = x["u"][:, 0].contiguous().to(d), x["a"].to(d), x["bias"].to(d)
    c1, h1 = pr.lstm_step(u_t, a, bias, c0, h0)
    c2, h2 = c0.clone(), h0.clone()
    pr.lstm_step(u_t, a, bias, c2, h2, out=(c2, h2))
    torch.cuda.synchronize()
    assert torch.equal(c1, c2) and torch.equal(h1, h2)
