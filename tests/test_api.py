"""Host-side checks of the C ABI: the library loads, exports every entry
point include/pararnn.h declares, sizes workspaces, and rejects bad
arguments before touching the GPU.  No test here calls an entry point with a
made-up address in a process that can see a GPU: those calls run in a child
process with CUDA_VISIBLE_DEVICES="" (tests/host_abi_checks.py)."""
import json
import os
import re
import subprocess
import sys

import pytest
import torch

import nonlinear_rnn_paragru_b200 as pr
import host_abi_checks  # tests/ is on sys.path (pytest rootdir-relative import)

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


# ---- argument checks, run in a child process that sees no GPU (the calls
# pass made-up device addresses; see tests/host_abi_checks.py)
@pytest.fixture(scope="module")
def host_rcs():
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "tests", "host_abi_checks.py")],
                       env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    return json.loads(r.stdout.strip().splitlines()[-1])


@pytest.mark.parametrize("case", host_abi_checks.case_names())
def test_entry_points_reject_bad_arguments_on_host(host_rcs, case):
    got, want = host_rcs[case]
    assert got == want, (case, got, want)


def test_host_checks_refuse_to_run_with_a_device_visible():
    env = dict(os.environ)
    env.pop("CUDA_VISIBLE_DEVICES", None)
    r = subprocess.run([sys.executable, os.path.join(ROOT, "tests", "host_abi_checks.py")],
                       env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 2 and "refusing" in r.stderr


def test_binding_rejects_host_tensors():
    u = torch.zeros((1, 8, 3, 32), dtype=torch.bfloat16)
    a = torch.zeros((3, 32))
    with pytest.raises(ValueError):
        pr._ptr(a)
    with pytest.raises(ValueError):
        pr._uptr(u)


def test_unfused_workspace_sizes():
    g = pr.pararnn_unfused_workspace_size(pr.PARARNN_GRU, 8, 4096, 1024)
    l = pr.pararnn_unfused_workspace_size(pr.PARARNN_LSTM, 8, 4096, 1024)
    n = 8 * 4096 * 1024
    assert g >= 8 * n and l >= 24 * n and g % 256 == 0 and l % 256 == 0
    assert pr.pararnn_unfused_workspace_size(pr.PARARNN_GRU, 1, 16, 12) == 0   # D % 8
    assert pr.pararnn_unfused_workspace_size(5, 1, 16, 16) == 0                # cell


def test_bench_plan_follows_the_library_dispatch_rules():
    # bench.py counts launches and cell evaluations per segment from its own
    # statement of the library's dispatch (csrc/api.cu); on 148 SMs:
    import bench
    from nonlinear_rnn_paragru_b200.inputs import WORKLOADS
    plan = {k: bench.fwd_plan(w, sms=148) for k, w in WORKLOADS.items()}
    assert plan[1] == ("gru_newton_row", 3.75, 256)      # 8 tiles: one launch
    assert plan[2] == ("gru_newton_queue", 3.75, 512)    # 1024 tiles >= 4 x 148 resident CTAs
    assert bench.fwd_launches(WORKLOADS[2], sms=148) == 1
    # fewer tiles than resident queue CTAs: the row kernel, launch by segment
    assert bench.fwd_plan(WORKLOADS[2].scaled(B=2), sms=148) == ("gru_newton_row", 3.75, 2048)
    assert bench.fwd_launches(WORKLOADS[2].scaled(B=2), sms=148) == 2
    assert plan[3] == ("lstm_newton_queue", 10.0, 128)  # 1024 tiles >= 4 x 148
    assert plan[4] == ("gru_newton_row", 3.75, 4096)     # T > 4096, 256 tiles >= 148
    assert plan[5] == ("lstm_newton_queue", 10.0, 128)  # 2048 tiles
    assert bench.fwd_launches(WORKLOADS[3], sms=148) == 1
    assert bench.fwd_plan(WORKLOADS[3].scaled(B=1, D=512), sms=148) == ("lstm_newton_row", 6.5, 2048)
    assert len(bench.fwd_segments(WORKLOADS[4], sms=148)) == 16
    # few tiles keep one launch over the whole sequence
    assert bench.fwd_plan(WORKLOADS[2].scaled(B=1, D=64), sms=148)[2] == 4096
    assert bench.fwd_plan(WORKLOADS[3].scaled(B=1, D=64), sms=148)[2] == 4096
    # fp32 ParaLSTM and long sequences with few tiles take the chunked kernels
    import dataclasses
    lstm_f32 = dataclasses.replace(WORKLOADS[3], u_dtype="f32")
    assert bench.fwd_plan(lstm_f32, sms=148)[0] == "lstm_newton_fused"
    assert bench.fwd_plan(WORKLOADS[2].scaled(B=1, T=9000, D=64), sms=148)[0] == "gru_newton_fused"


def test_dense_workspace_sizes():
    assert pr.pararnn_dense_workspace_size(2, 300, 64) >= 2 * 300 * 64 * 64 * 4
    assert pr.pararnn_dense_workspace_size(2, 300, 520) == 0     # D above the maximum
    assert pr.pararnn_dense_workspace_size(2, 300, 60) == 0      # D % 8


def test_flag_constants_match_header():
    src = open(os.path.join(ROOT, "include", "pararnn.h")).read()
    flags = dict(re.findall(r"#define (PARARNN_FLAG_\w+) (\d+)u", src))
    assert len(flags) >= 5
    for name, val in flags.items():
        assert getattr(pr, name) == int(val), name
