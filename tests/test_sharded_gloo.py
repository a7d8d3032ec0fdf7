"""The N > 1 path on CPU ranks (gloo, world size 2): token-sharded Hessian with
an all-reduce, replicated factor, row-sharded sweep and the final gather
(post_weight_quantization_23_b200.sharded), plus the bench's cross-rank
helpers.

The per-rank compute is a CPU stand-in with the plan's interface, built on
the oracle (test infrastructure), so what these tests check is the
orchestration: the shards, the collectives and the assembly.  Its result
must equal the single-process oracle on the whole layer.
"""

import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle as O
import synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


class OraclePlan:
    """CPU stand-in for GptqPlan (same attributes and calls), backed by the oracle."""

    def __init__(self, r, k, cfg, device, want_loss=True):
        self.r, self.k, self.cfg = r, k, cfg
        self.H = torch.zeros(k, k, dtype=torch.float64)
        self.want_loss = want_loss

    def hessian_add(self, X, n_total, stream=None):
        self.H += torch.from_numpy(O.hessian(X.numpy(), n_total=n_total))

    def prepare(self, stream=None):
        pass  # the oracle factors inside gptq()

    def quantize(self, W, stream=None):
        c = self.cfg
        res = O.gptq(W.numpy(), self.H.numpy(), c.bits, c.group_size, c.block_size, c.percdamp,
                     c.act_order, sym=c.sym, static_groups=c.static_groups)
        self.codes = torch.from_numpy(res["codes"].astype(np.uint8))
        self.scales = torch.from_numpy(np.ascontiguousarray(res["scales"], dtype=np.float32))
        self.zeros = torch.from_numpy(np.ascontiguousarray(res["zeros"], dtype=np.int32))
        self.g_idx = torch.from_numpy(res["g_idx"].astype(np.int32))
        self.perm = torch.from_numpy(res["perm"].astype(np.int32))
        rows = np.asarray(res["loss_rows"], dtype=np.float64)
        self.loss = torch.from_numpy(np.concatenate([rows, [rows.sum()]]))

    def check(self):
        pass


def _spec():
    return synth.CONFIGS["tiny"].scaled(r=37, k=96, n=1536, group_size=32, block_size=32)


def _sharded_worker(rank, world, port, tag):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from post_weight_quantization_23_b200 import QuantConfig
        from post_weight_quantization_23_b200.sharded import ShardedLayer

        spec = _spec()
        cfg = QuantConfig(spec.bits, spec.group_size, spec.block_size, spec.percdamp,
                          act_order=(tag in ("act", "static", "sym_static")),
                          sym=(tag == "sym_static"), static_groups=(tag in ("static", "sym_static")))
        W = synth.make_w(spec, 3).float()
        X = synth.make_x(spec, 3).float()
        layer = ShardedLayer(spec.r, spec.k, cfg, "cpu", plan_factory=OraclePlan)
        t0, t1 = layer.token_range(spec.n)
        out = layer.run(X[t0:t1], spec.n, W)
        # every rank holds the same H after the all-reduce, and the whole layer after the gather
        ref = O.gptq(W.numpy(), O.hessian(X.numpy()), cfg.bits, cfg.group_size, cfg.block_size,
                     cfg.percdamp, cfg.act_order, sym=cfg.sym, static_groups=cfg.static_groups)
        assert np.allclose(layer.plan.H.numpy(), O.hessian(X.numpy()), rtol=1e-12, atol=1e-14)
        assert out["codes"].shape == (spec.r, spec.k)
        assert np.array_equal(out["codes"].numpy().astype(np.int64), ref["codes"])
        assert np.allclose(out["scales"].numpy(), ref["scales"], rtol=1e-6)
        assert np.array_equal(out["zeros"].numpy(), ref["zeros"])
        assert np.array_equal(out["g_idx"].numpy(), ref["g_idx"])
        assert abs(float(out["loss"]) - ref["loss"]) <= 1e-9 * abs(ref["loss"])
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("tag", ["plain", "act", "static", "sym_static"])
def test_sharded_layer_two_ranks_matches_single_process(tag):
    mp.spawn(_sharded_worker, args=(2, _free_port(), tag), nprocs=2, join=True)


def _bench_worker(rank, world, port):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    sys.path.insert(0, ROOT)
    import bench

    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # the slowest rank's time is the step time every rank reports
        assert bench.max_over_ranks(10.0 + rank, world) == 10.0 + world - 1
        # the reference arm runs on rank 0 only; the others return at once
        if rank != 0:
            class A:
                pass
            assert bench.reference_arm(A(), None, world, rank) == 0
    finally:
        dist.destroy_process_group()


def test_bench_rank_helpers_two_ranks():
    mp.spawn(_bench_worker, args=(2, _free_port()), nprocs=2, join=True)


def test_even_split_covers_and_balances():
    from post_weight_quantization_23_b200.sharded import even_split
    for n in (0, 1, 7, 64, 4097):
        for p in (1, 2, 3, 8):
            parts = even_split(n, p)
            assert parts[0][0] == 0 and parts[-1][1] == n
            assert all(a[1] == b[0] for a, b in zip(parts, parts[1:]))
            sizes = [e - s for s, e in parts]
            assert max(sizes) - min(sizes) <= 1
