"""Python front end of libgptq_b200: device buffers and call sequencing.

``GptqPlan`` owns every device buffer one layer needs (allocated once with
torch, the library itself allocates nothing) and issues the C ABI calls of the
hot path in order on one stream:

    hessian_add (per X chunk)  ->  prepare  ->  quantize  ->  pack  ->  dequant

``check()`` synchronises and turns the device status words into exceptions.
All arithmetic happens in the CUDA library; this module only sequences calls.
"""

from __future__ import annotations

import dataclasses

import torch

from . import _lib
from ._lib import GptqError, NotPositiveDefinite, make_config  # noqa: F401


@dataclasses.dataclass
class QuantConfig:
    bits: int = 4
    group_size: int = 128
    block_size: int = 128
    percdamp: float = 0.01
    act_order: bool = False

    def c(self):
        return make_config(self.bits, self.group_size, self.block_size, self.percdamp,
                           self.act_order)

    def ngroups(self, k: int) -> int:
        G = k if self.group_size == -1 else self.group_size
        return (k + G - 1) // G


class GptqPlan:
    """Preallocated buffers and the call sequence for one (r, k) layer."""

    def __init__(self, r: int, k: int, cfg: QuantConfig, device="cuda", want_loss=True,
                 deq_dtype=torch.float16, hessian_tokens_hint: int = 0):
        if not torch.cuda.is_available():
            raise GptqError(_lib.GPTQ_ERR_CUDA, "GptqPlan", "no CUDA device")
        _lib.load()
        self.r, self.k, self.cfg = int(r), int(k), cfg
        self.ccfg = cfg.c()
        dev = torch.device(device)
        self.device = dev
        ng = cfg.ngroups(k)
        f32, i32 = torch.float32, torch.int32
        self.H = torch.zeros(k, k, dtype=f32, device=dev)
        self.U = torch.empty(k, k, dtype=f32, device=dev)
        self.perm = torch.empty(k, dtype=i32, device=dev)
        self.invperm = torch.empty(k, dtype=i32, device=dev)
        self.dead = torch.empty(k, dtype=torch.uint8, device=dev)
        self.d_info = torch.zeros(1, dtype=i32, device=dev)
        self.d_status = torch.zeros(1, dtype=i32, device=dev)
        self.codes = torch.empty(r, k, dtype=torch.uint8, device=dev)
        self.scales = torch.empty(r, ng, dtype=f32, device=dev)
        self.zeros = torch.empty(r, ng, dtype=i32, device=dev)
        self.g_idx = torch.empty(k, dtype=i32, device=dev)
        self.loss = torch.zeros(r + 1, dtype=torch.float64, device=dev) if want_loss else None
        self.qweight = torch.empty(r, k * cfg.bits // 32, dtype=i32, device=dev)
        self.deq = torch.empty(r, k, dtype=deq_dtype, device=dev) if deq_dtype is not None else None

        def ws(op, n=0):
            nbytes = _lib.workspace_size(op, r, k, n, self.ccfg)
            return torch.empty(max(nbytes, 1), dtype=torch.uint8, device=dev) if nbytes else None

        self.ws_h = ws(_lib.OP_HESSIAN, hessian_tokens_hint)
        self.ws_p = ws(_lib.OP_PREPARE_HINV)
        self.ws_q = ws(_lib.OP_QUANTIZE)
        self.n_seen = 0

    # -- stages -----------------------------------------------------------
    def hessian_reset(self):
        self.H.zero_()
        self.n_seen = 0

    def hessian_add(self, X: torch.Tensor, n_total: int, stream=None):
        """H += (2 / n_total) X^T X for one chunk of calibration tokens."""
        _lib.hessian_accumulate(X, self.H, 2.0 / float(n_total), self.ws_h, stream)
        self.n_seen += X.shape[0]

    def prepare(self, stream=None):
        _lib.prepare_hinv(self.H, self.ccfg, self.U, self.perm, self.invperm, self.dead,
                          self.d_info, self.ws_p, stream)

    def quantize(self, W: torch.Tensor, stream=None):
        _lib.quantize_layer(W, self.U, self.perm, self.dead, self.H if self.loss is not None else None,
                            self.ccfg, self.codes, self.scales, self.zeros, self.g_idx, self.loss,
                            self.d_status, self.ws_q, stream)

    def pack(self, stream=None):
        _lib.pack(self.codes, self.cfg.bits, self.qweight, stream)

    def dequant(self, stream=None):
        if self.deq is not None:
            _lib.dequant(self.qweight, self.scales, self.zeros, self.g_idx, self.k, self.cfg.bits,
                         self.deq, stream)

    def run_after_hessian(self, W: torch.Tensor, stream=None):
        """prepare -> quantize -> pack -> dequant, no synchronisation."""
        self.prepare(stream)
        self.quantize(W, stream)
        self.pack(stream)
        self.dequant(stream)

    def check(self):
        """Synchronise and raise on a device-reported failure."""
        torch.cuda.synchronize(self.device)
        info = int(self.d_info.item())
        if info != 0:
            raise NotPositiveDefinite(_lib.GPTQ_ERR_NOT_PD, "gptq_prepare_hinv",
                                      f"pivot {info - 1} (processing order) not positive")
        st = int(self.d_status.item())
        if st != 0:
            raise GptqError(st, "gptq_quantize_layer")

    def result(self) -> dict:
        out = dict(codes=self.codes, scales=self.scales, zeros=self.zeros, g_idx=self.g_idx,
                   qweight=self.qweight, perm=self.perm, invperm=self.invperm, dead=self.dead,
                   U=self.U, H=self.H)
        if self.loss is not None:
            out["loss_rows"] = self.loss[:-1]
            out["loss"] = self.loss[-1]
        if self.deq is not None:
            out["deq"] = self.deq
        return out


def quantize_layer(W: torch.Tensor, X=None, cfg: QuantConfig | None = None, H=None,
                   chunk_tokens: int = 65536, want_loss=True, deq_dtype=torch.float16) -> dict:
    """Quantize one layer on the GPU: W (r, k) and either calibration inputs X
    (n, k) (a tensor or an iterable of chunks, on the device) or a ready
    Hessian H (k, k) fp32.  Returns the plan's result dict (device tensors)."""
    cfg = cfg or QuantConfig()
    r, k = W.shape
    plan = GptqPlan(r, k, cfg, W.device, want_loss=want_loss, deq_dtype=deq_dtype,
                    hessian_tokens_hint=chunk_tokens)
    if H is not None:
        plan.H.copy_(H)
    else:
        chunks = [X[i:i + chunk_tokens] for i in range(0, X.shape[0], chunk_tokens)] \
            if isinstance(X, torch.Tensor) else list(X)
        n_total = sum(c.shape[0] for c in chunks)
        for c in chunks:
            plan.hessian_add(c, n_total)
    plan.run_after_hessian(W)
    plan.check()
    return plan.result()
