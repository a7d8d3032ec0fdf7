"""Shared helpers of the GPU parity tests: run the CUDA path and the oracle
on the same seeded inputs and measure the agreement the acceptance criteria
name (H relative Frobenius, code match rate with a tie-aware replay, scale /
zero agreement, g_idx, pack, loss)."""

from __future__ import annotations

import dataclasses

import numpy as np
import torch

import oracle as O
import synth

# acceptance tolerances
TOL_H_REL_FRO = 1e-5
TOL_CODE_MATCH = 0.999
TOL_SCALE_REL = 1e-4
TOL_LOSS_REL = 1e-3
TIE_TAU = 1e-3


def gpu_quantize(W, X, cfg, chunk_tokens=8192, deq_dtype=torch.float32):
    from post_weight_quantization_23_b200 import GptqPlan
    r, k = W.shape
    plan = GptqPlan(r, k, cfg, W.device, want_loss=True, deq_dtype=deq_dtype,
                    hessian_tokens_hint=chunk_tokens)
    n = X.shape[0]
    for a in range(0, n, chunk_tokens):
        plan.hessian_add(X[a:a + chunk_tokens], n)
    plan.prepare()
    plan.quantize(W)
    if k % 32 == 0:
        plan.pack()
        plan.dequant()
    plan.check()
    res = {key: v.detach().cpu() for key, v in plan.result().items() if torch.is_tensor(v)}
    if k % 32 != 0:
        res.pop("qweight", None)
        res.pop("deq", None)
    return res


@dataclasses.dataclass
class Agreement:
    h_rel_fro: float
    u_rel_max: float
    u_row_rel: float
    code_match: float
    n_forced: int
    replay_mismatch: int
    zero_mismatch_replay: int
    scale_rel_replay: float
    loss_rel: float
    loss_rel_replay: float
    gidx_equal: bool
    perm_equal: bool
    perm_tie_swaps: int

    def assert_ok(self, strict_match=True):
        assert self.h_rel_fro <= TOL_H_REL_FRO, self
        assert self.perm_equal and self.gidx_equal, self
        assert self.replay_mismatch == 0, self
        assert self.zero_mismatch_replay == 0, self
        assert self.scale_rel_replay <= TOL_SCALE_REL, self
        if strict_match:
            assert self.code_match >= TOL_CODE_MATCH, self
        assert self.loss_rel <= TOL_LOSS_REL, self


def compare(gpu, W_np, X_np, cfg, rows=None, H=None):
    """Oracle on the same inputs; ``rows`` restricts the sweep comparison to a
    sample of rows (rows are independent given U).  ``H`` may carry the
    oracle's own Hessian of X when it was computed in chunks beforehand."""
    if H is None:
        H = O.hessian(X_np)
    Hg = gpu["H"].double().numpy()
    h_rel = float(np.linalg.norm(Hg - H) / np.linalg.norm(H))
    Wc = W_np if rows is None else W_np[rows]
    gperm = gpu["perm"].numpy().astype(np.int64)
    sym = bool(getattr(cfg, "sym", False))
    stat = bool(getattr(cfg, "static_groups", False))
    # the oracle's own act-order (before accepting the GPU's tie-equivalent one)
    Hf = O.fix_dead_columns(H, Wc[:1])[0]
    own_perm = O.act_order_perm(Hf) if cfg.act_order else np.arange(H.shape[0])
    perm_diff = int((own_perm != gperm).sum())
    # the act-order permutation is decided from floating-point diag(H): the
    # oracle takes the GPU's order where (and only where) it is a valid order
    # within the Hessian tolerance; everything downstream is then compared
    fp = gperm if cfg.act_order else None
    ref = O.gptq(Wc, H, cfg.bits, cfg.group_size, cfg.block_size, cfg.percdamp, cfg.act_order,
                 force_perm=fp, tau_perm=TOL_H_REL_FRO, sym=sym, static_groups=stat)
    sel = slice(None) if rows is None else rows
    codes = gpu["codes"].numpy().astype(np.int64)[sel]
    zeros = gpu["zeros"].numpy().astype(np.int64)[sel]
    scales = gpu["scales"].numpy()[sel]
    rep = O.gptq(Wc, H, cfg.bits, cfg.group_size, cfg.block_size, cfg.percdamp, cfg.act_order,
                 force_codes=codes, force_zeros=zeros, tau=TIE_TAU, force_perm=fp,
                 tau_perm=TOL_H_REL_FRO, sym=sym, static_groups=stat)
    perm_equal = bool(np.array_equal(gperm, ref["perm"]))
    U = gpu["U"].double().numpy()
    u_rel = float(np.abs(U - ref["U"]).max() / np.abs(ref["U"]).max())
    # per row of U relative to that row (the sweep uses U[i, j] / U[i, i])
    u_row = float(np.max(np.linalg.norm(U - ref["U"], axis=1) / np.linalg.norm(ref["U"], axis=1)))
    loss_g = gpu["loss_rows"].numpy()[sel].sum()
    return Agreement(
        h_rel_fro=h_rel,
        u_rel_max=u_rel,
        u_row_rel=u_row,
        code_match=float((codes == ref["codes"]).mean()),
        n_forced=int(rep["n_forced"]),
        replay_mismatch=int((codes != rep["codes"]).sum()),
        zero_mismatch_replay=int((zeros != rep["zeros"].astype(np.int64)).sum()),
        scale_rel_replay=float(np.max(np.abs(scales - rep["scales"]) / np.abs(rep["scales"]))),
        loss_rel=float(abs(loss_g - ref["loss_rows"].sum()) / ref["loss_rows"].sum()),
        loss_rel_replay=float(abs(loss_g - rep["loss_rows"].sum()) / rep["loss_rows"].sum()),
        gidx_equal=bool(np.array_equal(gpu["g_idx"].numpy(), ref["g_idx"])),
        perm_equal=perm_equal,
        perm_tie_swaps=perm_diff,
    )


def layer_inputs(spec, seed, device="cuda"):
    W = synth.make_w(spec, seed)
    X = synth.make_x(spec, seed)
    return W, X, W.to(device), X.to(device)
