"""The one-layer-over-ranks orchestration (post_weight_quantization_23_b200.
sharded) on the real plan: ShardedLayer with GptqPlan on a one-rank NCCL
group on one GPU.  Its all-reduce and all-gathers run for real (trivially, on
one rank) and the result must match the oracle on the whole layer, like the
single-process plan.  (The two-rank orchestration itself is covered on CPU
ranks in test_sharded_gloo.py.)"""

import datetime
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist

import synth
from _parity import compare, layer_inputs

pytestmark = pytest.mark.gpu


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.mark.parametrize("act_order", [False, True])
def test_sharded_layer_one_rank_matches_oracle(act_order):
    from post_weight_quantization_23_b200 import QuantConfig
    from post_weight_quantization_23_b200.sharded import ShardedLayer
    spec = synth.CONFIGS["q_proj"].scaled(r=256, k=1024, n=16384, act_order=act_order)
    W, X, Wd, Xd = layer_inputs(spec, seed=9)
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{_free_port()}", rank=0,
                            world_size=1, timeout=datetime.timedelta(seconds=60),
                            device_id=torch.device("cuda", 0))
    try:
        cfg = QuantConfig(4, 128, 128, 0.01, act_order)
        layer = ShardedLayer(spec.r, spec.k, cfg, "cuda", hessian_tokens_hint=spec.n)
        t0, t1 = layer.token_range(spec.n)
        assert (t0, t1) == (0, spec.n)
        out = layer.run(Xd[t0:t1], spec.n, Wd)
        torch.cuda.synchronize()
        gpu = {"H": layer.plan.H.cpu(), "U": layer.plan.U.cpu(), "perm": out["perm"].cpu(),
               "codes": out["codes"].cpu(), "scales": out["scales"].cpu(),
               "zeros": out["zeros"].cpu(), "g_idx": out["g_idx"].cpu(),
               "loss_rows": out["loss_rows"].cpu()}
    finally:
        dist.destroy_process_group()
    a = compare(gpu, W.numpy(), X.numpy(), cfg)
    print("sharded one rank", a)
    a.assert_ok()
    assert np.isclose(float(out["loss"]), float(gpu["loss_rows"].sum()))
