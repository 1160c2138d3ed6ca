"""pararnn_adjoint_noalloc: the adjoint for callers that cannot provide
device scratch memory (the library uses a fixed array of its own instead).

Such callers run under an allocator they do not control, or on a path where a
cudaMalloc and its implicit synchronisation cannot be afforded.  Each call is
checked through the C ABI against the workspace-based pararnn_adjoint on the
same inputs and against the fp64 BPTT of the oracle, on two calls in a row
(the second call finds the first call's leftovers in the shared array):
- the first call in the process runs on a side stream (torch streams are
  non-blocking), so the array's first-use clear must be ordered on it;
- whole-sequence (bf16 u, T <= 4096) and look-back (fp32 u) calls alternate,
  and the two kinds use the shared array differently.
This file is collected last on purpose; it also passes run alone.
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


def _case(w):
    x = make_inputs(w, with_grad=True)
    h = oracle.gru_seq(x["u"], x["a"], x["bias"], x["h0"]).astype(np.float32)
    ref = oracle.gru_bptt(x["u"], x["a"], x["bias"], x["h0"], h.astype(np.float64), x["dLdh"])
    xd = {k: v.to("cuda") for k, v in x.items()}
    xd["h"] = torch.as_tensor(h).to("cuda").contiguous()
    return xd, ref


def _noalloc(xd, stream=None):
    B, T, _, D = xd["u"].shape
    dev = "cuda"
    o = dict(du=torch.empty((B, T, 3, D), dtype=torch.float32, device=dev),
             da=torch.empty((3, D), dtype=torch.float32, device=dev),
             dbias=torch.empty((3, D), dtype=torch.float32, device=dev),
             dh0=torch.empty((B, D), dtype=torch.float32, device=dev),
             status=torch.full((1,), -7, dtype=torch.int32, device=dev))
    pr.pararnn_adjoint_noalloc(pr.PARARNN_GRU, xd["u"], xd["a"], xd["bias"], None,
                               xd["h0"], None, xd["h"], xd["dLdh"], o["du"], o["da"],
                               o["dbias"], None, o["dh0"], o["status"], stream)
    return o


def _check(o, ws_ref, ref, what):
    torch.cuda.synchronize()
    assert int(o["status"][0]) == 0, what
    for k in ("du", "da", "dbias", "dh0"):
        g = o[k].cpu().numpy()
        r1 = _rel(g, ws_ref[k].cpu().numpy())
        r2 = _rel(g, ref[k])
        assert r1 <= TOL_GRAD and r2 <= TOL_GRAD, (what, k, r1, r2)


def test_noalloc_first_call_on_a_side_stream(cuda_ok):
    xd, ref = _case(WORKLOADS[2].scaled(B=2, T=1000, D=96))
    ws_ref = pr.adjoint(pr.PARARNN_GRU, xd["u"], xd["a"], xd["bias"], xd["h0"], xd["h"],
                        xd["dLdh"])
    torch.cuda.synchronize()
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        for call in range(2):
            o = _noalloc(xd, s)
            s.synchronize()
            _check(o, ws_ref, ref, ("side stream", call))


@pytest.mark.parametrize("shape", [(8, 4096, 1024), (2, 1000, 96)])
def test_noalloc_adjoint_matches_workspace_adjoint_twice(cuda_ok, shape):
    B, T, D = shape
    xd, ref = _case(WORKLOADS[2].scaled(B=B, T=T, D=D))
    ws_ref = pr.adjoint(pr.PARARNN_GRU, xd["u"], xd["a"], xd["bias"], xd["h0"], xd["h"],
                        xd["dLdh"])
    torch.cuda.synchronize()
    for call in range(2):
        _check(_noalloc(xd), ws_ref, ref, (shape, call))


def test_noalloc_alternates_whole_sequence_and_lookback_calls(cuda_ok):
    # bf16 u, T = 1000: the whole-sequence adjoint (partial sums in the array);
    # fp32 u: the look-back adjoint (header, flags and records in the array)
    row, ref_row = _case(WORKLOADS[2].scaled(B=2, T=1000, D=64))
    lb, ref_lb = _case(WORKLOADS[4].scaled(B=2, T=700, D=48))
    ws_row = pr.adjoint(pr.PARARNN_GRU, row["u"], row["a"], row["bias"], row["h0"], row["h"],
                        row["dLdh"])
    ws_lb = pr.adjoint(pr.PARARNN_GRU, lb["u"], lb["a"], lb["bias"], lb["h0"], lb["h"],
                       lb["dLdh"])
    torch.cuda.synchronize()
    for call in range(2):
        _check(_noalloc(row), ws_row, ref_row, ("whole sequence", call))
        _check(_noalloc(lb), ws_lb, ref_lb, ("look-back", call))
