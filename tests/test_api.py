"""Host-side checks of the C ABI: the library loads, exports every entry
point include/pararnn.h declares, sizes workspaces, and rejects bad
arguments before touching the GPU (these run without one)."""
import ctypes
import os
import re

import pytest
import torch

import nonlinear_rnn_paragru_b200 as pr

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    src = open(os.path.join(ROOT, "include", "pararnn.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)   # drop comments
    decl = r"^\s*(?:const\s+)?(?:int|size_t|void|char)\s*\*?\s*(pararnn_[a-z_0-9]+)\s*\("
    return sorted(set(re.findall(decl, src, flags=re.M)))


def test_library_exports_every_declared_symbol():
    lib = pr.load_library()
    names = _declared()
    assert "pararnn_gru_solve" in names and "pararnn_adjoint" in names
    for n in names:
        assert hasattr(lib, n), n


def test_header_declares_the_boundary_calls():
    names = _declared()
    for n in ("pararnn_gru_solve", "pararnn_lstm_solve", "pararnn_adjoint",
              "pararnn_workspace_size", "pararnn_workspace_init",
              "pararnn_seq_baseline", "pararnn_gru_step", "pararnn_lstm_step",
              "pararnn_strerror"):
        assert n in names


def test_workspace_sizes():
    s1 = pr.pararnn_workspace_size(pr.PARARNN_GRU, 8, 4096, 1024, 64, 0)
    s2 = pr.pararnn_workspace_size(pr.PARARNN_GRU, 8, 4096, 1024, 16, 0)
    assert s1 > s2 > 0 and s1 % 256 == 0
    assert pr.pararnn_workspace_size(pr.PARARNN_LSTM, 4, 2048, 4096, 0, 1) > 0
    assert pr.pararnn_workspace_size(pr.PARARNN_GRU, 1, 256, 63, 0, 0) == 0   # D % 8
    assert pr.pararnn_workspace_size(7, 1, 256, 64, 0, 0) == 0                 # cell
    assert pr.pararnn_workspace_size(pr.PARARNN_GRU, 0, 256, 64, 0, 0) == 0


def test_strerror_covers_codes():
    for code in (0, -1, -2, -3, -4, -5, -6):
        assert pr.pararnn_strerror(code)
    assert "unknown" in pr.pararnn_strerror(-99)


def _call_gru(**over):
    lib = pr.load_library()
    args = dict(u=0x1000, dt=pr.PARARNN_BF16, a=0x2000, bias=None, h0=None,
                h=0x3000, B=1, T=8, D=32, opts=None, stats=0x4000, hist=None,
                ws=0x10000, wsb=1 << 20, stream=None)
    args.update(over)
    o = pr._opts() if args["opts"] is None else args["opts"]
    return lib.pararnn_gru_solve(args["u"], args["dt"], args["a"], args["bias"],
                                 args["h0"], args["h"], args["B"], args["T"],
                                 args["D"], ctypes.byref(o), args["stats"],
                                 args["hist"], args["ws"], args["wsb"],
                                 args["stream"])


@pytest.mark.parametrize("over,code", [
    (dict(u=None), -1), (dict(h=None), -1), (dict(stats=None), -1),
    (dict(ws=None), -1), (dict(D=12), -1), (dict(B=0), -1), (dict(T=0), -1),
    (dict(dt=5), -2), (dict(u=0x1008), -5), (dict(h=0x3004), -5),
    (dict(ws=0x10010), -5),
])
def test_gru_solve_rejects_bad_arguments_on_host(over, code):
    assert _call_gru(**over) == code


def test_lstm_requires_c_output():
    lib = pr.load_library()
    rc = lib.pararnn_lstm_solve(0x1000, pr.PARARNN_BF16, 0x2000, None, None, None,
                                None, 0x3000, 1, 8, 32, None, 0x4000, None, 0x10000,
                                1 << 20, None)
    assert rc == -1


def test_adjoint_argument_checks():
    lib = pr.load_library()
    base = [pr.PARARNN_GRU, 0x1000, pr.PARARNN_BF16, 0x2000, None, None, None,
            None, 0x3000, 0x5000, 0x6000, 0x7000, None, None, None, 1, 8, 32,
            0x4000, 0x10000, 1 << 20, None]
    a = list(base); a[0] = 9
    assert lib.pararnn_adjoint(*a) == -1           # bad cell
    a = list(base); a[5] = 0x8000                  # c0 given for GRU
    assert lib.pararnn_adjoint(*a) == -1
    a = list(base); a[9] = None                    # no dL/dh
    assert lib.pararnn_adjoint(*a) == -1
    a = list(base); a[10] = 0x6004                 # misaligned du
    assert lib.pararnn_adjoint(*a) == -5
    a = list(base); a[20] = 16                     # workspace too small
    assert lib.pararnn_adjoint(*a) == -3


def test_binding_rejects_host_tensors():
    u = torch.zeros((1, 8, 3, 32), dtype=torch.bfloat16)
    a = torch.zeros((3, 32))
    with pytest.raises(ValueError):
        pr._ptr(a)
    with pytest.raises(ValueError):
        pr._uptr(u)


@pytest.mark.parametrize("over,code", [
    (dict(u=None), -1), (dict(a=None), -1), (dict(hn=None), -1), (dict(D=12), -1),
    (dict(B=0), -1), (dict(dt=5), -2), (dict(u=0x1001), -5), (dict(hn=0x3002), -5),
    (dict(hp=0x5002), -5), (dict(bias=0x6001), -5),
])
def test_step_rejects_bad_arguments_on_host(over, code):
    lib = pr.load_library()
    g = dict(u=0x1000, dt=pr.PARARNN_BF16, a=0x2000, bias=None, hp=None, hn=0x3000,
             B=2, D=32)
    g.update(over)
    assert lib.pararnn_gru_step(g["u"], g["dt"], g["a"], g["bias"], g["hp"], g["hn"],
                                g["B"], g["D"], None) == code


def test_lstm_step_needs_distinct_outputs():
    lib = pr.load_library()
    ok = [0x1000, pr.PARARNN_F32, 0x2000, None, None, None, 0x3000, 0x4000, 2, 32, None]
    a = list(ok); a[6] = None
    assert lib.pararnn_lstm_step(*a) == -1         # no c output
    a = list(ok); a[7] = 0x3000
    assert lib.pararnn_lstm_step(*a) == -1         # c and h the same array
    a = list(ok); a[0] = 0x1002
    assert lib.pararnn_lstm_step(*a) == -5         # fp32 u_t needs 4-byte alignment


def test_unfused_workspace_and_argument_checks():
    lib = pr.load_library()
    g = pr.pararnn_unfused_workspace_size(pr.PARARNN_GRU, 8, 4096, 1024)
    l = pr.pararnn_unfused_workspace_size(pr.PARARNN_LSTM, 8, 4096, 1024)
    n = 8 * 4096 * 1024
    assert g >= 8 * n and l >= 24 * n and g % 256 == 0 and l % 256 == 0
    assert pr.pararnn_unfused_workspace_size(pr.PARARNN_GRU, 1, 16, 12) == 0   # D % 8
    assert pr.pararnn_unfused_workspace_size(5, 1, 16, 16) == 0                # cell
    o = pr._opts()
    base = [pr.PARARNN_GRU, 0x1000, pr.PARARNN_BF16, 0x2000, None, None, None, None,
            0x3000, 1, 8, 16, ctypes.byref(o), 0x4000, 0x10000, 1 << 20, None]
    a = list(base); a[0] = 7
    assert lib.pararnn_solve_unfused(*a) == -1      # bad cell
    a = list(base); a[7] = 0x5000
    assert lib.pararnn_solve_unfused(*a) == -1      # c given for ParaGRU
    a = list(base); a[8] = None
    assert lib.pararnn_solve_unfused(*a) == -1      # no h
    a = list(base); a[2] = 4
    assert lib.pararnn_solve_unfused(*a) == -2      # dtype
    a = list(base); a[14] = 0x10010
    assert lib.pararnn_solve_unfused(*a) == -5      # workspace alignment
    a = list(base); a[15] = 64
    assert lib.pararnn_solve_unfused(*a) == -3      # workspace too small
    a = list(base); a[0] = pr.PARARNN_LSTM
    assert lib.pararnn_solve_unfused(*a) == -1      # ParaLSTM without c


def test_bench_plan_follows_the_library_dispatch_rules():
    # bench.py counts launches and cell evaluations per segment from its own
    # statement of the library's dispatch (csrc/api.cu); on 148 SMs:
    import bench
    from nonlinear_rnn_paragru_b200.inputs import WORKLOADS
    plan = {k: bench.fwd_plan(w, sms=148) for k, w in WORKLOADS.items()}
    assert plan[1] == ("gru_newton_row", 4, 256)      # 8 tiles: one launch
    assert plan[2] == ("gru_newton_row", 4, 1024)     # 1024 tiles: 2 CTAs/SM at k = 1
    assert plan[3] == ("lstm_newton_row", 6.5, 512)   # 1024 tiles: 1 CTA/SM at k = 1
    assert plan[4] == ("gru_newton_row", 4, 4096)     # T > 4096, 256 tiles >= 148
    assert plan[5] == ("lstm_newton_row", 6.5, 512)   # 2048 tiles
    assert len(bench.fwd_segments(WORKLOADS[4], sms=148)) == 16
    # few tiles keep one launch over the whole sequence
    assert bench.fwd_plan(WORKLOADS[2].scaled(B=1, D=64), sms=148)[2] == 4096
    assert bench.fwd_plan(WORKLOADS[3].scaled(B=1, D=64), sms=148)[2] == 4096
    # fp32 ParaLSTM and long sequences with few tiles take the chunked kernels
    import dataclasses
    lstm_f32 = dataclasses.replace(WORKLOADS[3], u_dtype="f32")
    assert bench.fwd_plan(lstm_f32, sms=148)[0] == "lstm_newton_fused"
    assert bench.fwd_plan(WORKLOADS[2].scaled(B=1, T=9000, D=64), sms=148)[0] == "gru_newton_fused"


def test_dense_workspace_and_argument_checks():
    lib = pr.load_library()
    assert pr.pararnn_dense_workspace_size(2, 300, 64) >= 2 * 300 * 64 * 64 * 4
    assert pr.pararnn_dense_workspace_size(2, 300, 136) == 0     # D above 128
    assert pr.pararnn_dense_workspace_size(2, 300, 60) == 0      # D % 8
    o = pr._opts()
    base = [0x1000, pr.PARARNN_BF16, 0x2000, None, None, 0x3000, 2, 16, 64,
            ctypes.byref(o), 0x4000, 0x10000, 1 << 30, None]
    a = list(base); a[8] = 136
    assert lib.pararnn_dense_gru_solve(*a) == -1    # D above 128
    a = list(base); a[2] = None
    assert lib.pararnn_dense_gru_solve(*a) == -1    # no W
    a = list(base); a[1] = 9
    assert lib.pararnn_dense_gru_solve(*a) == -2    # dtype
    a = list(base); a[2] = 0x2002
    assert lib.pararnn_dense_gru_solve(*a) == -5    # W alignment
    a = list(base); a[12] = 1024
    assert lib.pararnn_dense_gru_solve(*a) == -3    # workspace too small
