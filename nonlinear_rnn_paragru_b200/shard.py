"""Sequence sharding: the Newton solve with the time axis split over GPUs.

Shard r of W holds steps [T_r, T_{r+1}) of every (b, d) channel.  In the
page's block-bidiagonal system of a Newton iteration ("Параллельность RNN?",
§1.3) a shard couples to the shards before it only through the delta entering
its first step, and the scan's operator is associative ("Уровень 2"), so each
iteration is (include/pararnn.h, "Sequence sharding"):

  1. every shard evaluates its residual and Jacobians at the iterate and
     solves its part from a zero incoming delta (pararnn_shard_eval), giving
     its map ds_out = P ds_in + d, its last state(s) and its max|r|;
  2. one exchange: all-gather of the maps and last states (2 or 6 plus 1 or 2
     D-wide planes per batch row and shard) and an all-reduce of max|r|;
  3. every shard composes the maps of the shards before it into its incoming
     delta and its next initial state (pararnn_shard_combine) and adds the
     update to its iterate (pararnn_shard_apply).

The iterates are those of Newton on the whole sequence, and the stopping rule
is global (the update of the first iteration whose max|r| over all shards is
below tol is applied; the cap ends with a residual-only evaluation), so the
result does not depend on the split.  Every step of the arithmetic runs in
the library's kernels; this module only orders the calls and the exchange.
The exchange is an all-gather and an all-reduce through torch.distributed
(NCCL between GPUs) or, with every shard in one process, plain indexing.

`engine` is the object that runs the per-shard steps: :class:`CudaShardEngine`
(the library's kernels) for use; tests substitute an fp64 CPU engine to check
the exchange logic on gloo ranks without a GPU.
"""
import torch
import torch.distributed as dist

from . import (PARARNN_GRU, PARARNN_LSTM, STATUS_NAMES, Workspace, load_library,
               pararnn_shard_apply, pararnn_shard_combine, pararnn_shard_eval,
               pararnn_shard_workspace_size)


class Shard:
    """One shard's inputs, iterate and exchange buffers."""

    def __init__(self, index, cell, u, a, bias, c0=None, h0=None, dtype=torch.float32):
        """u [B, Ts, G, D] the shard's slice of the projections; c0, h0 [B, D]
        the sequence's initial state (used by shard 0 only).  The library's
        kernels take float32 states; `dtype` is for substitute engines."""
        self.index, self.cell = index, cell
        self.u, self.a, self.bias = u, a, bias
        B, Ts, G, D = u.shape
        self.B, self.Ts, self.D = B, Ts, D
        self.S = 2 if cell == PARARNN_LSTM else 1        # state planes (c, h) or (h)
        self.NA = 6 if cell == PARARNN_LSTM else 2       # map planes
        dev, f32 = u.device, dtype
        self.h = torch.zeros((B, Ts, D), dtype=f32, device=dev)
        self.c = torch.zeros((B, Ts, D), dtype=f32, device=dev) if self.S == 2 else None
        # initial state: the true one for shard 0, the previous shard's
        # (initially zero) last state otherwise
        self.bound = torch.zeros((self.S, B, D), dtype=f32, device=dev)
        if index == 0:
            if h0 is not None:
                self.bound[self.S - 1].copy_(h0)
            if self.S == 2 and c0 is not None:
                self.bound[0].copy_(c0)
        self.agg = torch.empty((self.NA, B, D), dtype=f32, device=dev)
        self.last = torch.empty((self.S, B, D), dtype=f32, device=dev)
        self.rmax = torch.zeros(1, dtype=f32, device=dev)
        self.din = torch.empty((self.S, B, D), dtype=f32, device=dev)
        self.next_bound = torch.empty((self.S, B, D), dtype=f32, device=dev)


class CudaShardEngine:
    """The per-shard steps on the shard's GPU, through the C ABI."""

    def __init__(self):
        load_library()  # fails loudly when the CUDA library is missing
        self._ws = {}

    def _workspace(self, s):
        ws = self._ws.setdefault(s.index, Workspace(s.u.device))
        return ws.get(pararnn_shard_workspace_size(s.cell, s.B, s.Ts, s.D))

    def eval(self, s):
        lstm = s.cell == PARARNN_LSTM
        pararnn_shard_eval(s.cell, s.u, s.a, s.bias, s.bound[0] if lstm else None,
                           s.bound[s.S - 1], s.c, s.h, s.agg, s.last, s.rmax,
                           self._workspace(s))

    def combine(self, s, aggs, lasts):
        pararnn_shard_combine(s.cell, aggs, lasts, s.index, s.din,
                              s.next_bound if s.index > 0 else None)

    def apply(self, s):
        pararnn_shard_apply(s.cell, s.din, s.c, s.h, self._workspace(s))
        if s.index > 0:
            s.bound.copy_(s.next_bound)


class ProcessGroupExchange:
    """One shard per process: shard index = rank in `group`."""

    def __init__(self, group=None):
        self.group = group
        self.world = dist.get_world_size(group)
        self.rank = dist.get_rank(group)

    def gather(self, tensors):
        (t,) = tensors
        out = torch.empty((self.world,) + tuple(t.shape), dtype=t.dtype, device=t.device)
        dist.all_gather(list(out.unbind(0)), t.contiguous(), group=self.group)
        return out

    def max(self, tensors):
        (t,) = tensors
        # a NaN residual travels as +inf: a max reduction need not keep NaN
        m = torch.nan_to_num(t, nan=float("inf"))
        dist.all_reduce(m, op=dist.ReduceOp.MAX, group=self.group)
        return float(m.item())


class LocalExchange:
    """Every shard in this process (one GPU, or emulated shards in a test)."""

    def gather(self, tensors):
        return torch.stack(list(tensors), 0)

    def max(self, tensors):
        m = torch.stack([t.reshape(()) for t in tensors]).max()
        return float(m.item())


def sharded_solve(shards, exchange, engine=None, tol=1e-6, max_iters=64):
    """Newton solve of the shards this process holds (one for a process
    group, all of them for a LocalExchange).  Returns the stats shared by
    every shard: iters (updates applied), evals, max_residual, status."""
    engine = engine or CudaShardEngine()
    st = {"iters": 0, "evals": 0, "max_residual": 0.0, "status": STATUS_NAMES[0]}
    for k in range(max_iters + 1):
        for s in shards:
            engine.eval(s)
        aggs = exchange.gather([s.agg for s in shards])
        lasts = exchange.gather([s.last for s in shards])
        r = exchange.max([s.rmax for s in shards])  # NaN-propagating (host decision)
        st["evals"], st["max_residual"] = k + 1, r
        if r != r or r == float("inf"):
            st["status"] = STATUS_NAMES[2]
            break
        if k == max_iters:              # residual-only evaluation at the cap
            if not r < tol:
                st["status"] = STATUS_NAMES[1]
            break
        for s in shards:
            engine.combine(s, aggs, lasts)
            engine.apply(s)
        st["iters"] = k + 1
        if r < tol:                     # the certified iteration's update is applied
            break
    return st


def split_steps(T, world):
    """[T_r, T_{r+1}) of each of `world` shards: equal lengths, the first
    T % world shards one step longer."""
    q, rem = divmod(T, world)
    out, t0 = [], 0
    for r in range(world):
        n = q + (1 if r < rem else 0)
        out.append((t0, t0 + n))
        t0 += n
    return out
