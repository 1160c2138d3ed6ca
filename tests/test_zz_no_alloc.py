"""pararnn_adjoint_noalloc: the adjoint for callers that cannot provide
device scratch memory (the library uses a fixed array of its own instead).

Checked through the C ABI against the workspace-based pararnn_adjoint on the
same inputs, on two calls in a row (the second call finds the first call's
leftovers in the shared array).  This file is collected last on purpose.
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


def _bufs(B, T, D, G, dev):
    return dict(du=torch.empty((B, T, G, D), dtype=torch.float32, device=dev),
                da=torch.empty((G, D), dtype=torch.float32, device=dev),
                dbias=torch.empty((G, D), dtype=torch.float32, device=dev),
                dh0=torch.empty((B, D), dtype=torch.float32, device=dev),
                status=torch.zeros(1, dtype=torch.int32, device=dev))


@pytest.mark.parametrize("shape", [(8, 4096, 1024), (2, 1000, 96)])
def test_noalloc_adjoint_matches_workspace_adjoint_twice(cuda_ok, shape):
    B, T, D = shape
    dev = "cuda"
    w = WORKLOADS[2].scaled(B=B, T=T, D=D)
    x = make_inputs(w)
    xd = {k: v.to(dev) for k, v in x.items()}
    h = torch.as_tensor(oracle.gru_seq(x["u"], x["a"], x["bias"], x["h0"]),
                        dtype=torch.float32).to(dev).contiguous()
    ref = pr.adjoint(pr.PARARNN_GRU, xd["u"], xd["a"], xd["bias"], xd["h0"], h, xd["dLdh"])
    torch.cuda.synchronize()
    for call in range(2):
        o = _bufs(B, T, D, 3, dev)
        pr.pararnn_adjoint_noalloc(pr.PARARNN_GRU, xd["u"], xd["a"], xd["bias"], None,
                                   xd["h0"], None, h, xd["dLdh"], o["du"], o["da"],
                                   o["dbias"], None, o["dh0"], o["status"])
        torch.cuda.synchronize()
        assert int(o["status"][0]) == 0, call
        for k in ("du", "da", "dbias", "dh0"):
            r = _rel(o[k].cpu().numpy(), ref[k].cpu().numpy())
            assert r <= TOL_GRAD, (call, k, r)


def test_noalloc_refuses_problems_beyond_its_scratch(cuda_ok):
    # ParaLSTM B=4, T=2048, D=4096 needs about 40 MiB of scratch: refused
    # with PARARNN_ERR_WORKSPACE_TOO_SMALL before anything is launched
    B, T, D = 4, 2048, 4096
    assert pr.pararnn_workspace_size(pr.PARARNN_LSTM, B, T, D, 0, 1) > (16 << 20)
    lib = pr.load_library()
    rc = lib.pararnn_adjoint_noalloc(pr.PARARNN_LSTM, 16, pr.PARARNN_BF16, 16, None, None,
                                     None, 16, 16, 16, 16, 16, None, None, None, B, T, D,
                                     16, None)
    assert rc == -3
