"""One layer quantized across the ranks of a process group: the calibration
tokens and the rows of W are split between ranks.

Two facts of the method make this split exact ([GPTQ-tool] "GPTQ" How it
works, Steps 3 and 5):
  * H = (2/n) X^T X is a sum over tokens, so every rank can accumulate the
    part of its own tokens (scaled by 2 / n_total) and one all-reduce (sum)
    of the k x k fp32 matrix gives the layer's H;
  * every row of W is quantized from its own weights and the shared H, so,
    once all ranks hold the same inverse factor, any block of rows can be
    swept on any rank with no exchange during the sweep.

So per layer: partial H -> all-reduce -> the inverse factor on every rank
(replicated: cheaper than moving it) -> each rank sweeps its contiguous block
of rows -> codes, scales, zeros and the per-row losses are all-gathered.
The collectives are plain torch.distributed calls (NCCL between GPUs); the
kernels are the library's.

``plan_factory`` builds the per-rank plan; it defaults to ``GptqPlan`` and
exists so that the orchestration can run with another implementation of the
same interface.
"""

from __future__ import annotations

import torch
import torch.distributed as dist

from .api import GptqPlan, QuantConfig


def even_split(n: int, parts: int) -> list[tuple[int, int]]:
    """Contiguous [start, stop) ranges of n items over ``parts`` owners, the
    first n % parts owners taking one extra item."""
    if parts <= 0:
        raise ValueError("parts must be positive")
    base, extra = divmod(int(n), parts)
    out, s = [], 0
    for p in range(parts):
        e = s + base + (1 if p < extra else 0)
        out.append((s, e))
        s = e
    return out


def _gather_rows(t: torch.Tensor, counts: list[int], group) -> torch.Tensor:
    """All-gather row blocks of different heights (padded to the largest)."""
    rmax = max(counts)
    pad = torch.zeros((rmax,) + tuple(t.shape[1:]), dtype=t.dtype, device=t.device)
    pad[: t.shape[0]] = t
    outs = [torch.empty_like(pad) for _ in counts]
    dist.all_gather(outs, pad, group=group)
    return torch.cat([o[:c] for o, c in zip(outs, counts)], dim=0)


class ShardedLayer:
    """A layer of r x k weights whose tokens and rows are split over ``group``."""

    def __init__(self, r: int, k: int, cfg: QuantConfig, device, group=None, plan_factory=None,
                 **plan_kw):
        self.group = group
        self.world = dist.get_world_size(group)
        self.rank = dist.get_rank(group)
        self.r, self.k, self.cfg = int(r), int(k), cfg
        self.rows = even_split(self.r, self.world)
        self.r0, self.r1 = self.rows[self.rank]
        if self.r1 <= self.r0:
            raise ValueError(f"rank {self.rank} has no rows (r={r}, world={self.world})")
        factory = plan_factory or GptqPlan
        self.plan = factory(self.r1 - self.r0, self.k, cfg, device, **plan_kw)

    def token_range(self, n: int) -> tuple[int, int]:
        """This rank's share [start, stop) of n calibration tokens."""
        return even_split(n, self.world)[self.rank]

    def hessian_add(self, X_local: torch.Tensor, n_total: int, stream=None):
        """Accumulate (2 / n_total) X_local^T X_local into this rank's partial H."""
        self.plan.hessian_add(X_local, n_total, stream)

    def reduce_hessian(self):
        """Sum the partial Hessians of all ranks (in place, on every rank)."""
        dist.all_reduce(self.plan.H, op=dist.ReduceOp.SUM, group=self.group)

    def prepare(self, stream=None):
        self.plan.prepare(stream)

    def quantize(self, W: torch.Tensor, stream=None):
        """Sweep this rank's rows; W is the full (r, k) matrix or this rank's
        (r1 - r0, k) block."""
        if W.shape[0] == self.r:
            W = W[self.r0:self.r1]
        elif W.shape[0] != self.r1 - self.r0:
            raise ValueError(f"W has {W.shape[0]} rows; expected {self.r} or {self.r1 - self.r0}")
        self.plan.quantize(W, stream)

    def run(self, X_local, n_total: int, W: torch.Tensor) -> dict:
        """Partial H of this rank's tokens, all-reduce, factor, sweep, gather."""
        chunks = [X_local] if isinstance(X_local, torch.Tensor) else X_local
        for X in chunks:
            self.hessian_add(X, n_total)
        self.reduce_hessian()
        self.prepare()
        self.quantize(W)
        self.plan.check()
        return self.gather()

    def gather(self) -> dict:
        """The whole layer's codes, scales, zeros and per-row losses on every rank."""
        counts = [e - s for s, e in self.rows]
        p = self.plan
        out = dict(codes=_gather_rows(p.codes, counts, self.group),
                   scales=_gather_rows(p.scales, counts, self.group),
                   zeros=_gather_rows(p.zeros, counts, self.group),
                   g_idx=p.g_idx, perm=p.perm)
        if getattr(p, "loss", None) is not None:
            rows = _gather_rows(p.loss[:-1].reshape(-1, 1), counts, self.group).reshape(-1)
            out["loss_rows"] = rows
            out["loss"] = rows.sum()
        return out
