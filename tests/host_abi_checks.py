"""Argument checks of the C ABI that must reject a call on the host, before
anything is enqueued.

These calls pass addresses that no allocator handed out (0x1000, 0x2000,
...): the point is that the library refuses them by size, alignment or
missing-argument checks alone.  So that a regressed check can never launch a
kernel on such an address, the calls run only in a process that sees no GPU:
``tests/test_api.py`` starts this file as ``python tests/host_abi_checks.py``
with ``CUDA_VISIBLE_DEVICES=""`` and reads the JSON it prints
({case: [returned code, expected code]}).  Run directly with a device
visible, it refuses to make the calls.
"""
import ctypes
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def _gru(lib, pr, **over):
    g = dict(u=0x1000, dt=pr.PARARNN_BF16, a=0x2000, bias=None, h0=None,
             h=0x3000, B=1, T=8, D=32, opts=None, stats=0x4000, hist=None,
             ws=0x10000, wsb=1 << 20)
    g.update(over)
    o = pr._opts() if g["opts"] is None else g["opts"]
    return lib.pararnn_gru_solve(g["u"], g["dt"], g["a"], g["bias"], g["h0"], g["h"],
                                 g["B"], g["T"], g["D"], ctypes.byref(o), g["stats"],
                                 g["hist"], g["ws"], g["wsb"], None)


def _adj(lib, pr, fn="pararnn_adjoint", **over):
    a = [pr.PARARNN_GRU, 0x1000, pr.PARARNN_BF16, 0x2000, None, None, None,
         None, 0x3000, 0x5000, 0x6000, 0x7000, None, None, None, 1, 8, 32,
         0x4000, 0x10000, 1 << 20, None]
    for i, v in over.items():
        a[int(i[1:])] = v
    if fn == "pararnn_adjoint_noalloc":
        del a[19:21]  # no workspace arguments
    return getattr(lib, fn)(*a)


def _step(lib, pr, **over):
    g = dict(u=0x1000, dt=pr.PARARNN_BF16, a=0x2000, bias=None, hp=None, hn=0x3000,
             B=2, D=32)
    g.update(over)
    return lib.pararnn_gru_step(g["u"], g["dt"], g["a"], g["bias"], g["hp"], g["hn"],
                                g["B"], g["D"], None)


def _lstm_step(lib, pr, **over):
    a = [0x1000, pr.PARARNN_F32, 0x2000, None, None, None, 0x3000, 0x4000, 2, 32, None]
    for i, v in over.items():
        a[int(i[1:])] = v
    return lib.pararnn_lstm_step(*a)


def _unfused(lib, pr, **over):
    o = pr._opts()
    a = [pr.PARARNN_GRU, 0x1000, pr.PARARNN_BF16, 0x2000, None, None, None, None,
         0x3000, 1, 8, 16, ctypes.byref(o), 0x4000, 0x10000, 1 << 20, None]
    for i, v in over.items():
        a[int(i[1:])] = v
    return lib.pararnn_solve_unfused(*a)


def _dense(lib, pr, **over):
    o = pr._opts()
    a = [0x1000, pr.PARARNN_BF16, 0x2000, None, None, 0x3000, 2, 16, 64,
         ctypes.byref(o), 0x4000, 0x10000, 1 << 30, None]
    for i, v in over.items():
        a[int(i[1:])] = v
    return lib.pararnn_dense_gru_solve(*a)


def _cases(pr):
    """name -> (call(lib), expected return code)."""
    C = {}
    for name, over, code in [
            ("u_null", dict(u=None), -1), ("h_null", dict(h=None), -1),
            ("stats_null", dict(stats=None), -1), ("ws_null", dict(ws=None), -1),
            ("D12", dict(D=12), -1), ("B0", dict(B=0), -1), ("T0", dict(T=0), -1),
            ("dtype", dict(dt=5), -2), ("u_misaligned", dict(u=0x1008), -5),
            ("h_misaligned", dict(h=0x3004), -5), ("ws_misaligned", dict(ws=0x10010), -5),
            ("chan_iters_misaligned", dict(opts=pr._opts(chan_iters=0x5002)), -5)]:
        C["gru_solve_" + name] = ((lambda o: lambda lib: _gru(lib, pr, **o))(over), code)
    C["lstm_solve_needs_c"] = (lambda lib: lib.pararnn_lstm_solve(
        0x1000, pr.PARARNN_BF16, 0x2000, None, None, None, None, 0x3000, 1, 8, 32, None,
        0x4000, None, 0x10000, 1 << 20, None), -1)
    for name, over, code in [
            ("bad_cell", dict(a0=9), -1), ("c0_for_gru", dict(a5=0x8000), -1),
            ("no_dLdh", dict(a9=None), -1), ("du_misaligned", dict(a10=0x6004), -5),
            ("ws_too_small", dict(a20=16), -3)]:
        C["adjoint_" + name] = ((lambda o: lambda lib: _adj(lib, pr, **o))(over), code)
    # ParaLSTM B=4, T=2048, D=4096 needs about 40 MiB of scratch: more than the
    # no-allocation adjoint's built-in array
    C["adjoint_noalloc_beyond_scratch"] = (lambda lib: _adj(
        lib, pr, "pararnn_adjoint_noalloc", a0=pr.PARARNN_LSTM, a5=0x8000, a7=0x9000,
        a15=4, a16=2048, a17=4096), -3)
    C["adjoint_noalloc_bad_cell"] = (lambda lib: _adj(lib, pr, "pararnn_adjoint_noalloc",
                                                      a0=9), -1)
    for name, over, code in [
            ("u_null", dict(u=None), -1), ("a_null", dict(a=None), -1),
            ("out_null", dict(hn=None), -1), ("D12", dict(D=12), -1), ("B0", dict(B=0), -1),
            ("dtype", dict(dt=5), -2), ("u_misaligned", dict(u=0x1001), -5),
            ("out_misaligned", dict(hn=0x3002), -5), ("prev_misaligned", dict(hp=0x5002), -5),
            ("bias_misaligned", dict(bias=0x6001), -5)]:
        C["gru_step_" + name] = ((lambda o: lambda lib: _step(lib, pr, **o))(over), code)
    for name, over, code in [("no_c", dict(a6=None), -1), ("c_is_h", dict(a7=0x3000), -1),
                             ("f32_u_misaligned", dict(a0=0x1002), -5)]:
        C["lstm_step_" + name] = ((lambda o: lambda lib: _lstm_step(lib, pr, **o))(over), code)
    for name, over, code in [
            ("bad_cell", dict(a0=7), -1), ("c_for_gru", dict(a7=0x5000), -1),
            ("no_h", dict(a8=None), -1), ("dtype", dict(a2=4), -2),
            ("ws_misaligned", dict(a14=0x10010), -5), ("ws_too_small", dict(a15=64), -3),
            ("lstm_without_c", dict(a0=pr.PARARNN_LSTM), -1)]:
        C["unfused_" + name] = ((lambda o: lambda lib: _unfused(lib, pr, **o))(over), code)
    for name, over, code in [
            ("D_above_max", dict(a8=520), -1), ("no_W", dict(a2=None), -1),
            ("dtype", dict(a1=9), -2), ("W_misaligned", dict(a2=0x2002), -5),
            ("W_not_16_aligned", dict(a2=0x2004), -5), ("h_not_16_aligned", dict(a5=0x3008), -5),
            ("ws_too_small", dict(a12=1024), -3)]:
        C["dense_" + name] = ((lambda o: lambda lib: _dense(lib, pr, **o))(over), code)
    for name, args, code in [
            ("K_not_multiple_of_4", (0x1000, 0x2000, 0x3000, 8, 8, 6, 1, 0, 0x4000, None), -1),
            ("bad_store_mode", (0x1000, 0x2000, 0x3000, 8, 8, 8, 1, 4, 0x4000, None), -1),
            ("no_err", (0x1000, 0x2000, 0x3000, 8, 8, 8, 1, 0, None, None), -1),
            ("A_misaligned", (0x1004, 0x2000, 0x3000, 8, 8, 8, 1, 0, 0x4000, None), -5)]:
        C["dense_matmul_" + name] = ((lambda a_: lambda lib: lib.pararnn_dense_matmul(*a_))(args),
                                     code)
    # sequence sharding: ParaGRU shard B=1, Ts=8, D=32
    def _seval(lib, **over):
        a = [pr.PARARNN_GRU, 0x1000, pr.PARARNN_BF16, 0x2000, None, None, None, None, 0x3000,
             1, 8, 32, 0x4000, 0x5000, 0x6000, 0x10000, 1 << 20, None]
        for i, v in over.items():
            a[int(i[1:])] = v
        return lib.pararnn_shard_eval(*a)
    for name, over, code in [("bad_cell", dict(a0=5), -1), ("c_for_gru", dict(a7=0x7000), -1),
                             ("no_h", dict(a8=None), -1), ("no_agg", dict(a12=None), -1),
                             ("dtype", dict(a2=3), -2), ("D12", dict(a11=12), -1),
                             ("agg_misaligned", dict(a12=0x4002), -5),
                             ("ws_too_small", dict(a16=64), -3)]:
        C["shard_eval_" + name] = ((lambda o: lambda lib: _seval(lib, **o))(over), code)
    C["shard_combine_rank_out_of_range"] = (lambda lib: lib.pararnn_shard_combine(
        pr.PARARNN_GRU, 0x1000, 0x2000, 2, 2, 1, 32, 0x3000, 0x4000, None), -1)
    C["shard_combine_needs_bound"] = (lambda lib: lib.pararnn_shard_combine(
        pr.PARARNN_GRU, 0x1000, 0x2000, 2, 1, 1, 32, 0x3000, None, None), -1)
    C["shard_apply_lstm_needs_c"] = (lambda lib: lib.pararnn_shard_apply(
        pr.PARARNN_LSTM, 0x1000, None, 0x3000, 1, 8, 32, 0x10000, 1 << 20, None), -1)
    return C


def case_names():
    import nonlinear_rnn_paragru_b200 as pr
    return sorted(_cases(pr))


def main():
    if os.environ.get("CUDA_VISIBLE_DEVICES", None) != "":
        print("refusing: run with CUDA_VISIBLE_DEVICES=\"\" (these calls pass made-up "
              "device addresses)", file=sys.stderr)
        return 2
    import nonlinear_rnn_paragru_b200 as pr
    lib = pr.load_library()
    out = {name: [int(call(lib)), code] for name, (call, code) in _cases(pr).items()}
    print(json.dumps(out))
    return 0


if __name__ == "__main__":
    sys.exit(main())
