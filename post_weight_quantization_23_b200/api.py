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
    sym: bool = False  # symmetric grid (zero point at the middle code)
    static_groups: bool = False  # grids fitted before the sweep, original column groups

    def c(self):
        return make_config(self.bits, self.group_size, self.block_size, self.percdamp,
                           self.act_order, self.sym, self.static_groups)

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
        if self.ws_h is not None:
            self.ws_h.zero_()
        self.ws_p = ws(_lib.OP_PREPARE_HINV)
        self.ws_q = ws(_lib.OP_QUANTIZE)
        self.n_seen = 0

    # -- stages -----------------------------------------------------------
    def hessian_reset(self):
        """Zero H and the Hessian workspace (whose second int32 is the sticky
        device status word of gptq_hessian_accumulate)."""
        self.H.zero_()
        if self.ws_h is not None:
            self.ws_h.zero_()
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

    def matmul(self, X: torch.Tensor, out: torch.Tensor | None = None, stream=None):
        """Y = X W_hat^T with this plan's packed weights (after pack()).  The
        groups are runs of group_size columns unless act-order reordered them
        with dynamic groups; only then is g_idx passed to the kernel."""
        g_idx = self.g_idx if (self.cfg.act_order and not self.cfg.static_groups) else None
        return quant_matmul(X, self.qweight, self.scales, self.zeros, self.cfg.bits,
                            self.cfg.group_size, g_idx, out, stream)

    def run_after_hessian(self, W: torch.Tensor, stream=None):
        """prepare -> quantize -> pack -> dequant, no synchronisation."""
        self.prepare(stream)
        self.quantize(W, stream)
        self.pack(stream)
        self.dequant(stream)

    def capture(self, fn) -> "torch.cuda.CUDAGraph":
        """Record the library calls that ``fn()`` issues (with this plan's
        fixed buffers) into a CUDA graph; ``graph.replay()`` then re-runs them
        without per-kernel launch cost.  Inputs must stay at the same
        addresses between replays (copy new data into them)."""
        dev = self.device
        s = torch.cuda.Stream(dev)
        s.wait_stream(torch.cuda.current_stream(dev))
        with torch.cuda.stream(s):
            fn()  # first calls on a stream outside capture: lazy set-up happens here
        torch.cuda.current_stream(dev).wait_stream(s)
        torch.cuda.synchronize(dev)
        try:
            g = torch.cuda.CUDAGraph(keep_graph=True)
        except TypeError:
            g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=s):
            fn()
        return g

    def status(self) -> dict:
        """Synchronise and read the device status words of the three stages:
        the Hessian workspace's status, d_info of the factor and d_status of
        the sweep."""
        torch.cuda.synchronize(self.device)
        hs = int(self.ws_h[4:8].view(torch.int32).item()) if self.ws_h is not None else 0
        return {"hessian": hs, "d_info": int(self.d_info.item()),
                "d_status": int(self.d_status.item())}

    def check(self):
        """Synchronise and raise on a device-reported failure (the earliest
        stage first: a Hessian that gave up also poisons the factor)."""
        st = self.status()
        if st["hessian"] != 0:
            raise GptqError(st["hessian"], "gptq_hessian_accumulate", "bounded wait gave up")
        info = st["d_info"]
        if info == self.k + 1:
            raise GptqError(_lib.GPTQ_ERR_TIMEOUT, "gptq_prepare_hinv", "bounded wait gave up")
        if info != 0:
            raise NotPositiveDefinite(_lib.GPTQ_ERR_NOT_PD, "gptq_prepare_hinv",
                                      f"pivot {info - 1} (processing order) not positive")
        if st["d_status"] != 0:
            raise GptqError(st["d_status"], "gptq_quantize_layer")

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


def quant_matmul(X: torch.Tensor, qweight: torch.Tensor, scales: torch.Tensor,
                 zeros: torch.Tensor, bits: int, group_size: int, g_idx=None,
                 out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """The inference product Y = X W_hat^T read straight from packed weights
    (gptq_gemm): X (m, k) f16/bf16 on the device, qweight (n, k*bits/32),
    scales / zeros (n, ngroups), g_idx (k,) or None for runs of group_size
    columns.  Returns Y (m, n) in X's dtype (``out`` if given)."""
    m = X.shape[0]
    n = qweight.shape[0]
    if out is None:
        out = torch.empty(m, n, dtype=X.dtype, device=X.device)
    _lib.gemm(X, qweight, scales, zeros, g_idx, bits, group_size, out, stream)
    return out


def hadamard_block(k: int, largest: int = 8192) -> int:
    """The largest power of two that divides k, at most ``largest`` (0 if
    below 256, which gptq_rotate does not take)."""
    b = k & -k if k > 0 else 0
    b = min(b, largest)
    return b if b >= 256 else 0


def rotation_signs(k: int, seed: int, device="cuda") -> torch.Tensor:
    """Seeded random signs (int8, +1 / -1) for rotate()."""
    g = torch.Generator().manual_seed(int(seed))
    s = torch.randint(0, 2, (k,), generator=g, dtype=torch.int8) * 2 - 1
    return s.to(device)


def rotate(x: torch.Tensor, signs: torch.Tensor, block: int | None = None, inverse=False,
           out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Rotation preprocessing (gptq_rotate): each row of x becomes
    x diag(s) H_b / sqrt(b) (or its inverse).  Apply the same signs and block
    to W and X before quantizing; ``out`` may be x itself (in place)."""
    block = block or hadamard_block(x.shape[1])
    if out is None:
        out = torch.empty_like(x)
    _lib.rotate(x, signs, block, out, inverse, stream)
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


class HostPipeline:
    """End-to-end layer quantization from HOST buffers (pinned memory):
    X is streamed to the device in chunks on a copy stream while the Hessian
    accumulates the previous chunk on the compute stream (two device staging
    buffers, event-ordered), W is copied once, and the packed result (qweight,
    scales, zeros, g_idx) plus the layer loss are copied back to pinned host
    buffers.  ``run`` enqueues everything and returns; ``wait`` synchronises."""

    def __init__(self, plan: GptqPlan, chunk_tokens: int, x_dtype: torch.dtype,
                 w_dtype: torch.dtype):
        self.plan = plan
        self.chunk = int(chunk_tokens)
        dev = plan.device
        self.stage = [torch.empty(self.chunk, plan.k, dtype=x_dtype, device=dev) for _ in range(2)]
        self.Wd = torch.empty(plan.r, plan.k, dtype=w_dtype, device=dev)
        self.copy_stream = torch.cuda.Stream(dev)
        self.compute_stream = torch.cuda.Stream(dev)
        self.copied = [torch.cuda.Event() for _ in range(2)]
        self.consumed = [torch.cuda.Event() for _ in range(2)]
        pin = dict(pin_memory=True)
        self.out_qweight = torch.empty(plan.qweight.shape, dtype=plan.qweight.dtype, **pin)
        self.out_scales = torch.empty(plan.scales.shape, dtype=plan.scales.dtype, **pin)
        self.out_zeros = torch.empty(plan.zeros.shape, dtype=plan.zeros.dtype, **pin)
        self.out_gidx = torch.empty(plan.g_idx.shape, dtype=plan.g_idx.dtype, **pin)
        self.out_loss = torch.empty(1, dtype=torch.float64, **pin)
        self.out_status = torch.empty(3, dtype=torch.int32, **pin)

    def h2d_bytes(self, X_host, W_host) -> int:
        return X_host.numel() * X_host.element_size() + W_host.numel() * W_host.element_size()

    def d2h_bytes(self) -> int:
        return sum(t.numel() * t.element_size() for t in (
            self.out_qweight, self.out_scales, self.out_zeros, self.out_gidx, self.out_loss,
            self.out_status))

    def run(self, X_host: torch.Tensor, W_host: torch.Tensor):
        plan, cs, ks = self.plan, self.copy_stream, self.compute_stream
        n = X_host.shape[0]
        ks.wait_stream(torch.cuda.current_stream(plan.device))
        cs.wait_stream(ks)  # staging buffers and Wd are free once the last run's compute is done
        with torch.cuda.stream(ks):
            plan.hessian_reset()
        with torch.cuda.stream(cs):
            self.Wd.copy_(W_host, non_blocking=True)
        for i, a in enumerate(range(0, n, self.chunk)):
            b = i % 2
            rows = min(self.chunk, n - a)
            with torch.cuda.stream(cs):
                if i >= 2:
                    cs.wait_event(self.consumed[b])
                self.stage[b][:rows].copy_(X_host[a:a + rows], non_blocking=True)
                self.copied[b].record(cs)
            ks.wait_event(self.copied[b])
            plan.hessian_add(self.stage[b][:rows], n, stream=ks)
            self.consumed[b].record(ks)
        ks.wait_stream(cs)
        plan.run_after_hessian(self.Wd, stream=ks)
        with torch.cuda.stream(ks):
            self.out_qweight.copy_(plan.qweight, non_blocking=True)
            self.out_scales.copy_(plan.scales, non_blocking=True)
            self.out_zeros.copy_(plan.zeros, non_blocking=True)
            self.out_gidx.copy_(plan.g_idx, non_blocking=True)
            if plan.loss is not None:
                self.out_loss.copy_(plan.loss[-1:], non_blocking=True)
            self.out_status[0:1].copy_(plan.d_info, non_blocking=True)
            self.out_status[1:2].copy_(plan.d_status, non_blocking=True)
            if plan.ws_h is not None:
                self.out_status[2:3].copy_(plan.ws_h[4:8].view(torch.int32), non_blocking=True)
        torch.cuda.current_stream(plan.device).wait_stream(ks)

    def wait(self):
        self.compute_stream.synchronize()
        if self.plan.ws_h is not None and int(self.out_status[2]) != 0:
            raise GptqError(int(self.out_status[2]), "gptq_hessian_accumulate")
        if int(self.out_status[0]) == self.plan.k + 1:
            raise GptqError(_lib.GPTQ_ERR_TIMEOUT, "gptq_prepare_hinv")
        if int(self.out_status[0]) != 0:
            raise NotPositiveDefinite(_lib.GPTQ_ERR_NOT_PD, "gptq_prepare_hinv")
        if int(self.out_status[1]) != 0:
            raise GptqError(int(self.out_status[1]), "gptq_quantize_layer")
