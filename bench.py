#!/usr/bin/env python
"""Benchmark of the ParaGRU / ParaLSTM Newton-scan hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload 1..5]
                    [--impl ours|reference]

One step = one pass of the whole hot path over one batch of the workload:
the fused Newton-scan forward solve and, for workloads with a backward pass,
the reverse adjoint scan.  The default workload is ParaGRU B=8, T=4096,
D=1024 with bf16 input projections (forward + adjoint), the layer shape the
throughput metric is quoted on.  Inputs are seeded synthetic tensors of that
shape; u alone (201 MB) is larger than the 126 MB L2, so no flush is needed
between timed steps.

Under torchrun (N > 1) every rank solves its own independent problem of the
same size (weak scaling, no data-path collective); the time is the max over
ranks and `value` counts the token-channels of all ranks.  `--impl reference`
times the fp64 CPU oracle (sequential recurrence + BPTT) on a bounded sample
of the same workload.  Rank 0 prints one JSON line.
"""
import argparse
import json
import os
import statistics
import sys
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from nonlinear_rnn_paragru_b200.inputs import WORKLOADS, make_inputs  # noqa: E402

METRIC = "Newton-solved token*channels/s (fwd+bwd)"
UNIT = "tokch/s"
# DRAM bytes (read + write) of one launch of the dominant kernel, taken with
# ncu on this build for the workload in the key.  None when not captured for
# the kernel as it stands.
NCU_TRAFFIC_BYTES = {
    # one launch (the whole solve), profiles/gru_newton_queue_b8_t4096_d1024.md
    ("gru_newton_queue", "gru_b8_t4096_d1024_bf16"): 201_853_696 + 103_506_432,
}
# Special-function (MUFU) work per element and cell evaluation.  The roofline
# counts the cell in its plain form, the algorithmic figure: ParaGRU 3 exp + 3
# reciprocals, ParaLSTM 5 exp + 5 reciprocals.  Most kernels issue fewer, and
# the second element of fwd_plan() is the issued count for an exact
# evaluation:
#   gru_newton_queue (ParaGRU with bf16 u and at least one 8-channel tile per
#     resident CTA, four CTAs per SM: every 512-step segment of every tile in
#     one launch): the cell pass of gru_newton_row, 3 ex2 + 0.75 rcp for an
#     exact evaluation; the inexact early evaluations issue 3 tanh;
#   gru_newton_row (ParaGRU with T <= 4096, or longer with at least one
#     8-channel tile per SM, then in 4096-step segments): 3 ex2 + 0.75 rcp (one
#     reciprocal serves the four sigmoids of a step pair, one the four tanh of
#     two pairs);
#   gru_newton_fused (ParaGRU otherwise): 3 ex2 + 2 rcp;
#   lstm_newton_queue (ParaLSTM, bf16 u, at least one 8-channel tile per
#     resident CTA, four CTAs per SM: every 128-step segment in one launch):
#     5 ex2 + 5 rcp for an exact evaluation (one reciprocal per gate and per
#     tanh(c')); the inexact early evaluations issue 5 tanh;
#   lstm_newton_row (ParaLSTM, bf16 u, T <= 4096, in segments where
#     smaller clusters fill the SMs): 5 ex2 + 1.5 rcp (one
#     reciprocal per step pair for the six sigmoids, one for the two tanh(g),
#     one for the two tanh(c'));
#   lstm_newton_fused (ParaLSTM otherwise): 5 ex2 + 3 rcp.
MUFU_ALGORITHMIC = {"gru": 6, "lstm": 10}
QUEUE_CTAS_PER_SM = 4   # residency of gru_newton_queue and lstm_newton_queue (128 registers)


# --force-row: the bf16 problems take the whole-sequence (row) kernels where
# the segment queues would (PARARNN_FLAG_FORCE_ROW on the solve and adjoint)
FORCE_ROW = False


def fwd_plan(w, sms=None):
    """(kernel, MUFU ops per evaluation, segment length) of the forward solve
    as the library dispatches it: the segment-queue kernels solve every
    512-step (ParaGRU) or 128-step (ParaLSTM) segment of a problem with bf16 u
    and at least one 8-channel tile per resident CTA in one launch; otherwise the row kernels
    solve a sequence in segments of k x 1024 (ParaGRU, two CTAs per SM) or
    k x 512 steps (ParaLSTM, one CTA per SM), one launch each, k the smallest
    cluster size below the one the whole sequence needs at which its
    8-channel tiles fill the SMs, and a ParaGRU sequence longer than 4096
    steps in 4096-step segments."""
    if sms is None:
        sms = torch.cuda.get_device_properties(0).multi_processor_count
    tiles8 = w.B * ((w.D + 7) // 8)
    if (w.cell == "gru" and w.u_dtype == "bf16" and tiles8 >= QUEUE_CTAS_PER_SM * sms
            and not FORCE_ROW):
        return "gru_newton_queue", 3.75, 512
    if w.cell == "lstm":
        if w.u_dtype == "bf16" and tiles8 >= QUEUE_CTAS_PER_SM * sms and not FORCE_ROW:
            return "lstm_newton_queue", 10.0, 128
        if w.u_dtype == "bf16" and w.T <= 4096:
            cls, seg = 1, w.T
            while cls * 512 < w.T:
                cls *= 2
            k = 1
            while k < cls:
                if k * tiles8 >= sms:
                    seg = k * 512
                    break
                k *= 2
            return "lstm_newton_row", 6.5, seg
        return "lstm_newton_fused", 8, w.T
    if w.T <= 4096:
        cls, seg = 1, w.T
        while cls * 1024 < w.T:
            cls *= 2
        k = 1
        while k < cls:
            if k * tiles8 >= 2 * sms:
                seg = k * 1024
                break
            k *= 2
        return "gru_newton_row", 3.75, seg
    if tiles8 >= sms:
        return "gru_newton_row", 3.75, 4096
    return "gru_newton_fused", 5, w.T


def fwd_kernel(w, sms=None):
    return fwd_plan(w, sms)[:2]


def fwd_segments(w, sms=None):
    seg = fwd_plan(w, sms)[2]
    return [(s0, min(seg, w.T - s0)) for s0 in range(0, w.T, seg)]


def fwd_launches(w, sms=None):
    """Launches of the forward kernel per solve."""
    queue = fwd_plan(w, sms)[0] in ("gru_newton_queue", "lstm_newton_queue")
    return 1 if queue else len(fwd_segments(w, sms))
# algorithmic HBM bytes per token-channel: inputs read once, outputs written once
def fwd_bytes(w):
    ue = 2 if w.u_dtype == "bf16" else 4
    return w.G * ue + (4 if w.cell == "gru" else 8)


def adj_bytes(w):
    ue = 2 if w.u_dtype == "bf16" else 4
    states = 4 if w.cell == "gru" else 8
    return w.G * ue + states + 4 + 4 * w.G   # u, states, dL/dh in; du out


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", type=int, default=2, choices=sorted(WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extra", action="store_true",
                    help="skip the unfused-tier and decode-step measurements")
    ap.add_argument("--e2e-steps", type=int, default=8)
    ap.add_argument("--force-row", action="store_true",
                    help="bf16 problems: the whole-sequence kernels instead of the segment queues")
    return ap.parse_args()


# ----------------------------------------------------------- distributed --
def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x, world, device="cuda"):
    """Max of a per-rank scalar over all ranks (timing is the slowest rank)."""
    if world == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def weak_value(world, units_per_rank, ms_max):
    """Whole-job throughput: every rank's units over the slowest rank's time."""
    return world * units_per_rank / (ms_max * 1e-3)


def rank_seed(rank):
    """Each rank solves its own independent problem."""
    return 1000 * rank


# ---------------------------------------------------------------- clocks --
_SAMPLER_CHILD = r"""
import select, sys, time
import pynvml
pynvml.nvmlInit()
bus = sys.argv[1]
h = (pynvml.nvmlDeviceGetHandleByPciBusId(bus) if bus
     else pynvml.nvmlDeviceGetHandleByIndex(int(sys.argv[2])))
for _ in range(5):  # the first queries are slow: take them before the timed region
    pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM)
    pynvml.nvmlDeviceGetCurrentClocksEventReasons(h)
print("ready", pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM), flush=True)
period = float(sys.argv[3])
rows = []
# sample until the parent closes stdin, then write every sample at once
while not select.select([sys.stdin], [], [], 0)[0]:
    t = time.monotonic()
    rows.append("%.6f %d %d" % (t, pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM),
                                pynvml.nvmlDeviceGetCurrentClocksEventReasons(h)))
    time.sleep(period)
sys.stdout.write("\n".join(rows) + "\n")
"""


class ClockSampler:
    """Samples SM clock and throttle reasons through NVML while running.

    The sampling loop runs in a child process (its own interpreter, so the
    timed loop's Python thread cannot starve it), stamping each sample with
    the system's monotonic clock; the samples kept are those inside the
    host-time bracket of the `with` block, which encloses the synchronised
    timed region.  The device is found by its PCI bus id (NVML does not
    follow CUDA_VISIBLE_DEVICES)."""

    REASONS = {
        "gpu_idle": 0x1, "applications_clocks_setting": 0x2, "sw_power_cap": 0x4,
        "hw_slowdown": 0x8, "sync_boost": 0x10, "sw_thermal_slowdown": 0x20,
        "hw_thermal_slowdown": 0x40, "hw_power_brake_slowdown": 0x80,
        "display_clock_setting": 0x100,
    }

    def __init__(self, index, period=0.0002):
        import subprocess
        self.mhz, self.reasons = [], set()
        self.max_mhz = None
        self.proc = None
        self.t0 = self.t1 = None
        try:
            pr_ = torch.cuda.get_device_properties(index)
            bus = "%08x:%02x:%02x.0" % (pr_.pci_domain_id, pr_.pci_bus_id, pr_.pci_device_id)
        except Exception:
            bus = ""
        try:
            self.proc = subprocess.Popen(
                [sys.executable, "-c", _SAMPLER_CHILD, bus, str(index), str(period)],
                stdin=subprocess.PIPE, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL,
                text=True)
            line = self.proc.stdout.readline().split()
            if len(line) != 2 or line[0] != "ready":
                raise RuntimeError("clock sampler did not start")
            self.max_mhz = int(line[1])
        except Exception:  # no NVML: clocks stay unreported
            self._stop_child()

    def _stop_child(self):
        """Closes the child's stdin (its signal to stop) -> its samples."""
        out = ""
        if self.proc is not None:
            try:
                out = self.proc.communicate(input="", timeout=30)[0] or ""
            except Exception:
                self.proc.kill()
                self.proc.communicate()
            self.proc = None
        return out

    def __enter__(self):
        self.t0 = time.monotonic()
        return self

    def __exit__(self, *a):
        self.t1 = time.monotonic()
        for ln in self._stop_child().splitlines():
            f = ln.split()
            if len(f) != 3:
                continue
            t, mhz, r = float(f[0]), int(f[1]), int(f[2])
            if self.t0 <= t <= self.t1:
                self.mhz.append(mhz)
                for name, bit in self.REASONS.items():
                    if r & bit and name != "gpu_idle":
                        self.reasons.add(name)

    def summary(self):
        if not self.mhz:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [],
                    "samples": 0}
        return {"sm_mhz": statistics.median(self.mhz), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.mhz)}


def measured_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return json.load(f), "measured"
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0}, "fallback"


# ------------------------------------------------------------- our path --
class Path:
    """Device buffers and the step (forward solve + adjoint) of one workload."""

    def __init__(self, w, x, pr):
        self.w, self.x, self.pr = w, x, pr
        d = "cuda"
        B, T, D, G = w.B, w.T, w.D, w.G
        self.lstm = w.cell == "lstm"
        self.h = torch.empty((B, T, D), dtype=torch.float32, device=d)
        self.c = torch.empty((B, T, D), dtype=torch.float32, device=d) if self.lstm else None
        self.stats = torch.zeros(4, dtype=torch.int32, device=d)
        self.hist = (torch.empty(66, dtype=torch.int32, device=d) if w.histogram else None)
        self.ws = pr.Workspace(d)
        self.wsa = pr.Workspace(d)
        self.opts = pr._opts(1e-6, 64, flags=pr.PARARNN_FLAG_FORCE_ROW if FORCE_ROW else 0)
        cell = pr.PARARNN_LSTM if self.lstm else pr.PARARNN_GRU
        self.fbuf = self.ws.get(pr.pararnn_workspace_size(cell, B, T, D, 64, 0))
        if w.adjoint:
            self.du = torch.empty((B, T, G, D), dtype=torch.float32, device=d)
            self.da = torch.empty((G, D), dtype=torch.float32, device=d)
            self.db = torch.empty((G, D), dtype=torch.float32, device=d)
            self.dh0 = torch.empty((B, D), dtype=torch.float32, device=d)
            self.dc0 = torch.empty((B, D), dtype=torch.float32, device=d) if self.lstm else None
            self.status = torch.zeros(1, dtype=torch.int32, device=d)
            self.abuf = self.wsa.get(pr.pararnn_workspace_size(cell, B, T, D, 0, 1))

    def launches_per_step(self):
        n = 1 + fwd_launches(self.w) + (1 if self.hist is not None else 0)  # init, solves, [hist]
        return n + (3 if self.w.adjoint else 0)            # init, adjoint, reduce

    def forward(self, x=None):
        x = x or self.x
        pr = self.pr
        if self.lstm:
            pr.pararnn_lstm_solve(x["u"], x["a"], x["bias"], x["c0"], x["h0"], self.c,
                                  self.h, self.opts, self.stats, self.hist, self.fbuf)
        else:
            pr.pararnn_gru_solve(x["u"], x["a"], x["bias"], x["h0"], self.h, self.opts,
                                 self.stats, self.hist, self.fbuf)

    def element_evaluations(self, x=None):
        """Cell evaluations performed by one solve, summed over (b, t, d).

        Every tile stops on its own, after the first evaluation at which all
        its channels are below tol, so a tile of channels d0..d0+w-1 was
        evaluated 1 + max over its channels of the per-channel iteration index
        (opts.chan_iters) times, and each of its channels that often.  Tiles
        are 8 channels for the row and segment-queue kernels, whose tiles hold
        a whole sequence or segment: this is exact there.  A sequence the
        library solves segment by segment is solved here one segment per call,
        each from the state the one before ended in, which is the arithmetic
        the segmented solve does.  For the chunked kernels (32-channel tiles)
        a channel reports its slowest chunk, so this is an upper bound there.
        Untimed.
        """
        x = x or self.x
        pr = self.pr
        kern = fwd_kernel(self.w)[0]
        width = 32 if kern.endswith("_fused") else 8
        B, D = self.w.B, self.w.D
        evals = 0
        c_in, h_in = x.get("c0"), x["h0"]
        ci = torch.zeros((B, D), dtype=torch.int32, device="cuda")
        opts = self.pr._opts(1e-6, 64, flags=self.opts.flags, chan_iters=ci)
        for s0, n in fwd_segments(self.w):
            u = x["u"][:, s0:s0 + n].contiguous()
            h = torch.empty((B, n, D), dtype=torch.float32, device="cuda")
            if self.lstm:
                c = torch.empty_like(h)
                pr.pararnn_lstm_solve(u, x["a"], x["bias"], c_in, h_in, c, h, opts,
                                      self.stats, None, self.fbuf)
                c_in = c[:, -1].contiguous()
            else:
                pr.pararnn_gru_solve(u, x["a"], x["bias"], h_in, h, opts, self.stats,
                                     None, self.fbuf)
            h_in = h[:, -1].contiguous()
            k = ci.cpu().long()
            pad = (-D) % width
            if pad:
                k = torch.nn.functional.pad(k, (0, pad))
            tile_k = k.view(B, -1, width).amax(dim=2)          # [B, tiles]
            per_ch = tile_k.repeat_interleave(width, dim=1)[:, :D]
            evals += n * int((per_ch + 1).sum())
        return evals

    def backward(self, x=None):
        x = x or self.x
        pr = self.pr
        cell = pr.PARARNN_LSTM if self.lstm else pr.PARARNN_GRU
        if FORCE_ROW:
            pr.pararnn_adjoint_ex(cell, x["u"], x["a"], x["bias"], x.get("c0"), x["h0"], self.c,
                                  self.h, x["dLdh"], self.du, self.da, self.db, self.dc0,
                                  self.dh0, self.status, self.abuf, self.opts)
        else:
            pr.pararnn_adjoint(cell, x["u"], x["a"], x["bias"], x.get("c0"), x["h0"], self.c,
                               self.h, x["dLdh"], self.du, self.da, self.db, self.dc0, self.dh0,
                               self.status, self.abuf)

    def step(self, x=None):
        self.forward(x)
        if self.w.adjoint:
            self.backward(x)


def time_events(fn, n):
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    e0.record()
    for _ in range(n):
        fn()
    e1.record()
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / n  # ms


def extra_measurements(w, x, pr, fwd_ms):
    """Measurements outside the timed step, each guarded so that a failure is
    reported in the JSON line instead of ending the run:
      unfused: the same forward solve by the unfused tier (Jacobians and
        residuals through HBM, a separate scan, the host checking the
        residual each iteration), against the fused solve's fwd_ms;
      decode: one decode step for the workload's batch of states, replayed
        from a captured CUDA graph of 64 steps (kernel time, not the
        Python call rate), with its algorithmic bytes per step."""
    lstm = w.cell == "lstm"
    cell = pr.PARARNN_LSTM if lstm else pr.PARARNN_GRU
    res = {}
    try:
        ws = pr.Workspace("cuda")

        def unfused():
            return pr.solve_unfused(cell, x["u"], x["a"], x["bias"],
                                    x["c0"] if lstm else None, x["h0"], workspace=ws)
        _, _, st = unfused()
        ms = time_events(unfused, 3)
        s = pr.read_stats(st)
        res["unfused"] = {"fwd_ms": round(ms, 4), "fused_fwd_ms": round(fwd_ms, 4),
                          "unfused_over_fused": round(ms / fwd_ms, 2),
                          "status": s["status"], "iters": s["iters"]}
    except Exception as e:  # reported, not fatal
        res["unfused"] = {"error": str(e)[:300]}
    try:
        G = w.G
        u_t = x["u"][:, 0].contiguous()
        h = x["h0"].clone()
        c = x["c0"].clone() if lstm else None

        def step():
            if lstm:
                pr.lstm_step(u_t, x["a"], x["bias"], c, h, out=(c, h))
            else:
                pr.gru_step(u_t, x["a"], x["bias"], h, out=h)
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            for _ in range(3):
                step()
        torch.cuda.current_stream().wait_stream(side)
        torch.cuda.synchronize()
        n = 64
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            for _ in range(n):
                step()
        graph.replay()
        ms = time_events(graph.replay, 10) / n
        ue = 2 if w.u_dtype == "bf16" else 4
        nbytes = w.B * w.D * (G * ue + (16 if lstm else 8))
        res["decode"] = {"us_per_step": round(ms * 1e3, 3), "B": w.B, "D": w.D,
                         "bytes_per_step": nbytes,
                         "achieved_gbs": round(nbytes / (ms * 1e-3) / 1e9, 1)}
    except Exception as e:
        res["decode"] = {"error": str(e)[:300]}
    if w.name == WORKLOADS[2].name:  # once, with the default workload's line
        try:
            res["dense"] = dense_measurement(pr)
        except Exception as e:
            res["dense"] = {"error": str(e)[:300]}
    return res


def dense_measurement(pr, B=1, T=1024, D=512):
    """Dense-Jacobian DEER (the GRU with full recurrent matrices) at one size:
    time per solve (CUDA events around whole solves, which synchronise on the
    host every iteration) and the tensor-core contractions' algorithmic
    FLOPs per Newton iteration: the chunk maps' tree, B*Tp*(1/2+1/4+1/8+1/16)
    products of 2 D^3, and the pre-activations, 2 B T D 3D.  `frac` divides
    their rate over the whole solve (a lower bound for the GEMM kernel alone)
    by a tf32 peak: the measured bf16 GEMM peak times the nominal tf32/bf16
    ratio (1.1 / 2.25)."""
    import math
    w = WORKLOADS[2].scaled(B=B, T=T, D=D)
    x = make_inputs(w, device="cuda")
    g = torch.Generator().manual_seed(5)
    W = ((torch.rand((3, D, D), generator=g) * 2 - 1) * (1.5 / math.sqrt(D))).cuda()
    ws = pr.Workspace("cuda")
    h, st = pr.dense_gru_solve(x["u"], W, x["bias"], x["h0"], workspace=ws)
    s = pr.read_stats(st)
    ms = time_events(lambda: pr.dense_gru_solve(x["u"], W, x["bias"], x["h0"], workspace=ws), 3)
    Tp = -(-T // 16) * 16
    tree = B * Tp * (15 / 16) * 2 * D ** 3
    pre = 2 * B * T * D * 3 * D
    # the pre-activations run at every evaluation, the tree at every update
    flops = s["iters"] * tree + s["evals"] * pre
    peaks, src = measured_peaks()
    tf32_peak = peaks["bf16_tflops"] * (1.1 / 2.25)
    achieved = flops / (ms * 1e-3) / 1e12
    return {"workload": f"dense GRU B={B} T={T} D={D} fp32 u(bf16 values)", "ms_per_solve": round(ms, 3),
            "iters": s["iters"], "evals": s["evals"], "status": s["status"],
            "tensor_tflop_per_solve": round(flops / 1e12, 4),
            "roofline": {"bound": "tensor", "achieved": round(achieved, 2),
                         "peak": round(tf32_peak, 1), "unit": "TFLOP/s (tf32)",
                         "frac": round(achieved / tf32_peak, 4),
                         "peak_source": f"bf16 {peaks['bf16_tflops']} ({src}) x 1.1/2.25"}}


def cpu_baseline(w, seconds_hint=10.0):
    """The fp64 oracle (sequential recurrence + BPTT) on a bounded sample of
    the workload: all of T, a slice of the channels."""
    import oracle
    Dk = 64
    ws = w.scaled(B=1, D=Dk)
    x = make_inputs(ws, with_grad=True)
    reps, t_total, n = 0, 0.0, 0
    t0 = time.perf_counter()
    while True:
        t1 = time.perf_counter()
        if w.cell == "gru":
            h = oracle.gru_seq(x["u"], x["a"], x["bias"], x["h0"])
            if w.adjoint:
                oracle.gru_bptt(x["u"], x["a"], x["bias"], x["h0"], h, x["dLdh"])
        else:
            c, h = oracle.lstm_seq(x["u"], x["a"], x["bias"], x["c0"], x["h0"])
            if w.adjoint:
                oracle.lstm_bptt(x["u"], x["a"], x["bias"], x["c0"], x["h0"], c, h, x["dLdh"])
        t_total += time.perf_counter() - t1
        n += ws.tokch
        reps += 1
        if time.perf_counter() - t0 > seconds_hint or reps >= 2000:
            break
    res = {"value": n / t_total, "unit": UNIT, "cores": oracle.get_threads(),
           "kind": "oracle",
           "sample": f"B=1, T={w.T}, D={Dk} slice of {w.name}, fp64 sequential "
                     f"{'recurrence + BPTT' if w.adjoint else 'recurrence'}, "
                     f"{reps} repetition(s), {t_total:.1f} s"}
    # the fp64 reference Newton on the same slice (global stopping at the
    # same tol): updates it applies before its residual is below tol
    try:
        if w.cell == "gru":
            r = oracle.gru_newton(x["u"], x["a"], x["bias"], x["h0"], tol=1e-6, max_iters=64)
        else:
            r = oracle.lstm_newton(x["u"], x["a"], x["bias"], x["c0"], x["h0"], tol=1e-6,
                                   max_iters=64)
        res["oracle_newton_updates"] = int(r["iters"])
    except Exception as e:  # reported, not fatal
        res["oracle_newton_updates"] = f"error: {str(e)[:120]}"
    return res


def run_ours(args, world, rank):
    import nonlinear_rnn_paragru_b200 as pr
    pr.load_library()  # fails loudly when the CUDA library is missing
    w = WORKLOADS[args.workload]
    x = make_inputs(w, seed=rank_seed(rank), device="cuda", with_grad=w.adjoint)
    path = Path(w, x, pr)
    for _ in range(max(args.warmup, 3)):
        path.step()
    torch.cuda.synchronize()
    barrier(world)
    sampler = ClockSampler(torch.cuda.current_device())
    with sampler:
        ms = time_events(path.step, args.steps)
        barrier(world)
    ms_max = max_over_ranks(ms, world)
    st = pr.read_stats(path.stats)
    value = weak_value(world, w.tokch, ms_max)

    # per-kernel timing (same stream, CUDA events) for the roofline
    fwd_ms = time_events(path.forward, max(3, args.steps // 2))
    adj_ms = time_events(path.backward, max(3, args.steps // 2)) if w.adjoint else 0.0
    clk = sampler.summary()
    peaks, src = measured_peaks()
    f_mhz = clk["sm_mhz"] or peaks.get("sm_max_mhz", 1965.0)
    mufu_peak = 148 * 16 * f_mhz * 1e6 / 1e12          # Tops/s
    kern, issued_per_eval = fwd_kernel(w)
    mufu_per_eval = MUFU_ALGORITHMIC[w.cell]
    elem_evals = path.element_evaluations()
    mufu_done = elem_evals * mufu_per_eval / (fwd_ms * 1e-3) / 1e12
    hbm_ach = w.tokch * fwd_bytes(w) / (fwd_ms * 1e-3) / 1e9
    traffic = NCU_TRAFFIC_BYTES.get((kern, w.name))
    roofline = {"bound": "alu", "kernel": kern, "achieved": round(mufu_done, 3),
                "peak": round(mufu_peak, 3),
                "unit": "Tops/s (MUFU; algorithmic %d ops per element evaluation)" % mufu_per_eval,
                "frac": round(mufu_done / mufu_peak, 4), "traffic": traffic,
                "peak_source": f"148 SMs x 16 MUFU/clk x {f_mhz:.0f} MHz sampled",
                "ops_per_launch": elem_evals * mufu_per_eval / fwd_launches(w),
                "launches_per_solve": fwd_launches(w),
                "mean_evals": round(elem_evals / w.tokch, 3),
                "issued_per_exact_eval": issued_per_eval}
    hbm = {"fwd_achieved_gbs": round(hbm_ach, 1), "peak_gbs": peaks["hbm_gbs"],
           "frac": round(hbm_ach / peaks["hbm_gbs"], 4), "peak_kind": src,
           "fwd_bytes_per_tokch": fwd_bytes(w)}
    if w.adjoint:
        adj_gbs = w.tokch * adj_bytes(w) / (adj_ms * 1e-3) / 1e9
        hbm.update({"adj_achieved_gbs": round(adj_gbs, 1),
                    "adj_frac": round(adj_gbs / peaks["hbm_gbs"], 4),
                    "adj_bytes_per_tokch": adj_bytes(w)})

    # naive step-by-step GPU loop (forward only), same inputs
    cell = pr.PARARNN_LSTM if path.lstm else pr.PARARNN_GRU
    seq_ms = time_events(lambda: pr.pararnn_seq_baseline(cell, x["u"], x["a"], x["bias"],
                                                        x.get("c0"), x["h0"], path.c, path.h),
                         2)

    # end to end through the public API with host buffers: every step copies
    # its inputs in from pinned host memory, runs the library's solve and
    # adjoint, and copies all its outputs back.  Steps are double-buffered
    # over three streams (copy in, compute, copy out), as a caller streaming
    # batches runs them: the copy in of step k+1 and the copy out of step k-1
    # overlap step k (PCIe is full duplex).  Timed from the first copy in to
    # the last copy out, on the device.
    host = {k: v.cpu().pin_memory() for k, v in x.items()}
    paths = [path, Path(w, x, pr)]  # the second buffer set: outputs and workspaces
    devs = [{k: torch.empty_like(v) for k, v in x.items()} for _ in paths]

    def outs_of(pth):
        o = [pth.h] + ([pth.c] if pth.lstm else [])
        if w.adjoint:
            o += [pth.du, pth.da, pth.db, pth.dh0] + ([pth.dc0] if pth.lstm else [])
        return o

    host_outs = [[torch.empty(o.shape, dtype=o.dtype, pin_memory=True) for o in outs_of(pth)]
                 for pth in paths]
    s_in, s_cmp, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    ev_in = [torch.cuda.Event() for _ in paths]
    ev_cmp = [torch.cuda.Event() for _ in paths]
    ev_out = [torch.cuda.Event() for _ in paths]

    def e2e_run(n):
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(s_in)
        s_out.wait_event(e0)
        for k in range(n):
            j = k & 1
            with torch.cuda.stream(s_in):
                if k >= 2:
                    s_in.wait_event(ev_cmp[j])     # step k-2 has read these inputs
                for key in devs[j]:
                    devs[j][key].copy_(host[key], non_blocking=True)
                ev_in[j].record(s_in)
            with torch.cuda.stream(s_cmp):
                s_cmp.wait_event(ev_in[j])
                if k >= 2:
                    s_cmp.wait_event(ev_out[j])    # step k-2's outputs are copied out
                paths[j].step(devs[j])
                ev_cmp[j].record(s_cmp)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev_cmp[j])
                for ho, o in zip(host_outs[j], outs_of(paths[j])):
                    ho.copy_(o, non_blocking=True)
                ev_out[j].record(s_out)
        e1.record(s_out)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / n

    e2e_run(2)
    barrier(world)
    e2e_ms = max_over_ranks(e2e_run(args.e2e_steps), world)
    outs = outs_of(path)
    h2d = sum(v.numel() * v.element_size() for v in host.values())
    d2h = sum(o.numel() * o.element_size() for o in outs)

    out = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": max(args.warmup, 3), "ms_per_step": ms_max,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f32", "data": "synthetic",
        "config": {"workload": w.name + (" fwd+adjoint" if w.adjoint else " fwd"),
                   "kernels": "whole-sequence (--force-row)" if FORCE_ROW else "library default",
                   "cell": w.cell, "B": w.B, "T": w.T, "D": w.D, "u_dtype": w.u_dtype,
                   "tol": 1e-6, "l2": "inputs larger than L2 (u alone exceeds 126 MB)",
                   "parallelism": f"{world} independent replica(s)"},
        "newton": {"iters": st["iters"], "evals": st["evals"],
                   "max_residual": st["max_residual"], "status": st["status"]},
        "fwd_ms": round(fwd_ms, 4), "adj_ms": round(adj_ms, 4),
        "fwd_tokch_per_s": w.tokch / (fwd_ms * 1e-3),
        "roofline": roofline, "hbm_roofline": hbm,
        "seq_gpu_baseline": {"fwd_ms": round(seq_ms, 3),
                             "speedup_fused_fwd": round(seq_ms / fwd_ms, 2),
                             "pages_claim": "up to 665x over sequential (hardware not stated)"},
        "e2e": {"value": weak_value(world, w.tokch, e2e_ms), "unit": UNIT,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "ms_per_step": round(e2e_ms, 3), "steps": args.e2e_steps,
                "schedule": "double-buffered over copy-in, compute and copy-out streams"},
        "clocks": clk,
        "gpu_launches": path.launches_per_step() * args.steps,
    }
    if rank == 0 and not args.no_extra:
        out.update(extra_measurements(w, x, pr, fwd_ms))
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline(w)
    return out


def run_reference(args, world, rank):
    w = WORKLOADS[args.workload]
    cb = cpu_baseline(w, seconds_hint=10.0)
    t = w.tokch / cb["value"]
    return {"impl": "reference", "metric": METRIC, "value": cb["value"], "unit": UNIT,
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": t * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": w.name + (" fwd+adjoint" if w.adjoint else " fwd"),
                       "cell": w.cell, "B": w.B, "T": w.T, "D": w.D},
            "cpu_baseline": cb,
            "e2e": {"value": cb["value"], "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


def main():
    global FORCE_ROW
    args = parse()
    FORCE_ROW = args.force_row
    if args.impl == "reference":
        rank = int(os.environ.get("RANK", "0"))
        if rank != 0:
            return 0
        print(json.dumps(run_reference(args, int(os.environ.get("WORLD_SIZE", "1")), 0)),
              flush=True)
        return 0
    world, rank, _ = dist_setup()
    out = run_ours(args, world, rank)
    if rank == 0:
        print(json.dumps(out), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
