"""Seeded synthetic layers for GPTQ: weights W (out, in) and calibration
activations X (tokens, in).

This module only draws random numbers; it holds none of the quantization
method's arithmetic.  Both the CUDA library's tests/bench and the CPU oracle
consume its tensors, so "the same inputs" means the same bytes.  Everything is
generated on the CPU with ``torch.Generator`` (never relying on CPU/GPU RNG
agreement); X is produced in fixed generation chunks of ``GEN_CHUNK`` tokens,
each with its own derived seed, so any token range can be regenerated alone
and the bytes do not depend on how a consumer splits X.

The layer shapes follow the workloads the GPTQ pages quantize (Llama-7B
projections, an OPT-175B-width layer, a 7B decoder stack); their calibration
sets (WikiText-2 / C4 text through real checkpoints) are not available, so
these seeded distributions stand in for them:

* ``mixed``     X = Z L, Z ~ N(0, 1), L = I + strictly-lower N(0, 1/k)
                (correlated channels with a well-conditioned mixing).
* ``lognormal`` X = Z diag(c), Z ~ N(0, 1), c_j ~ lognormal(0, 1), a seeded
                fraction of channels multiplied by an outlier factor.
* ``silu``      X = silu(a) * b, a, b ~ N(0, 1) (heavy-tailed gated MLP input).
"""

from __future__ import annotations

import dataclasses
import math

import torch

GEN_CHUNK = 8192  # tokens per independently seeded generation chunk

_DT = {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}


@dataclasses.dataclass(frozen=True)
class LayerSpec:
    name: str
    r: int                 # out-features (rows of W)
    k: int                 # in-features (columns of W, channels of X)
    n: int                 # calibration tokens
    w_std: float
    w_dtype: str           # "f32" | "f16" | "bf16"
    x_dtype: str
    x_kind: str            # "mixed" | "lognormal" | "silu"
    outlier_frac: float = 0.0
    outlier_mult: float = 1.0
    bits: int = 4
    group_size: int = 128
    block_size: int = 128
    percdamp: float = 0.01
    act_order: bool = False
    sym: bool = False            # symmetric grid
    static_groups: bool = False  # grids fixed before the sweep

    def scaled(self, r=None, k=None, n=None, **kw):
        """Same distributions at other sizes (for parity runs the oracle can finish)."""
        return dataclasses.replace(self, r=r or self.r, k=k or self.k, n=n or self.n, **kw)


CONFIGS = {
    "tiny": LayerSpec("tiny", 64, 128, 2048, 0.02, "f32", "f32", "mixed",
                      bits=4, group_size=32, block_size=32),
    "q_proj": LayerSpec("q_proj", 4096, 4096, 262144, 0.02, "f16", "f16", "lognormal",
                        outlier_frac=0.01, outlier_mult=20.0),
    "down_proj": LayerSpec("down_proj", 4096, 11008, 262144, 0.015, "f16", "f16", "silu",
                           act_order=True),
    "opt175_width": LayerSpec("opt175_width", 12288, 12288, 131072, 0.01, "f16", "f16",
                              "lognormal", outlier_frac=0.005, outlier_mult=50.0,
                              bits=3, group_size=-1),
}

# One decoder layer of the 7B-shaped stack: (name, rows, in-features, X stream).
STACK_LAYER = (
    ("qkv", 12288, 4096, "attn_in"),
    ("o", 4096, 4096, "attn_out"),
    ("gate_up", 22016, 4096, "mlp_in"),
    ("down", 4096, 11008, "down_in"),
)
STACK_LAYERS = 32
STACK_TOKENS = 65536


def stack_spec(sublayer, tokens=STACK_TOKENS):
    """LayerSpec of one sub-layer of the 7B-shaped stack (int4, g128, act-order)."""
    for name, r, k, stream in STACK_LAYER:
        if name == sublayer:
            kind = "silu" if stream == "down_in" else "lognormal"
            return LayerSpec(f"stack_{name}", r, k, tokens, 0.02, "f16", "f16", kind,
                             outlier_frac=0.0 if kind == "silu" else 0.01,
                             outlier_mult=1.0 if kind == "silu" else 20.0,
                             act_order=True)
    raise KeyError(sublayer)


for _name, _r, _k, _stream in STACK_LAYER:
    CONFIGS[f"stack_{_name}"] = stack_spec(_name)


def tensor_seed(seed, layer, tensor_id):
    """Per-tensor seed: seed*1000 + layer*10 + tensor_id."""
    return int(seed) * 1000 + int(layer) * 10 + int(tensor_id)


def _gen(seed):
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed) & ((1 << 63) - 1))
    return g


def make_w(spec: LayerSpec, seed: int, layer: int = 0) -> torch.Tensor:
    """W (r, k) ~ N(0, w_std^2) in spec.w_dtype, on the CPU."""
    g = _gen(tensor_seed(seed, layer, 1))
    w = torch.randn(spec.r, spec.k, generator=g, dtype=torch.float32) * spec.w_std
    return w.to(_DT[spec.w_dtype])


def channel_scales(spec: LayerSpec, seed: int, layer: int = 0) -> torch.Tensor:
    """Per-channel scales c (k,) for the lognormal kind: lognormal(0, 1) with a
    seeded set of round(outlier_frac*k) channels multiplied by outlier_mult."""
    g = _gen(tensor_seed(seed, layer, 2))
    c = torch.exp(torch.randn(spec.k, generator=g, dtype=torch.float64))
    n_out = int(round(spec.outlier_frac * spec.k))
    if n_out:
        idx = torch.randperm(spec.k, generator=g)[:n_out]
        c[idx] *= spec.outlier_mult
    return c


def mixing_matrix(spec: LayerSpec, seed: int, layer: int = 0) -> torch.Tensor:
    """L = I + strictly-lower N(0, 1/k) entries (k, k), fp64."""
    g = _gen(tensor_seed(seed, layer, 3))
    M = torch.randn(spec.k, spec.k, generator=g, dtype=torch.float64) / math.sqrt(spec.k)
    return torch.eye(spec.k, dtype=torch.float64) + torch.tril(M, diagonal=-1)


def _x_chunk(spec, seed, layer, c, rows, aux):
    g = _gen(tensor_seed(seed, layer, 4) * 100003 + c)
    if spec.x_kind == "mixed":
        z = torch.randn(rows, spec.k, generator=g, dtype=torch.float64)
        return (z @ aux).to(_DT[spec.x_dtype])
    if spec.x_kind == "lognormal":
        z = torch.randn(rows, spec.k, generator=g, dtype=torch.float32)
        return (z * aux).to(_DT[spec.x_dtype])
    if spec.x_kind == "silu":
        a = torch.randn(rows, spec.k, generator=g, dtype=torch.float32)
        b = torch.randn(rows, spec.k, generator=g, dtype=torch.float32)
        return (torch.nn.functional.silu(a) * b).to(_DT[spec.x_dtype])
    raise ValueError(spec.x_kind)


def make_x(spec: LayerSpec, seed: int, layer: int = 0, t0: int = 0, t1: int | None = None,
           out: torch.Tensor | None = None) -> torch.Tensor:
    """Rows [t0, t1) of X (n, k) in spec.x_dtype, on the CPU.  ``out`` may be a
    preallocated (t1-t0, k) tensor (pinned host memory, say)."""
    t1 = spec.n if t1 is None else t1
    if not (0 <= t0 <= t1 <= spec.n):
        raise ValueError("token range out of bounds")
    if out is None:
        out = torch.empty(t1 - t0, spec.k, dtype=_DT[spec.x_dtype])
    aux = None
    if spec.x_kind == "mixed":
        aux = mixing_matrix(spec, seed, layer)
    elif spec.x_kind == "lognormal":
        aux = channel_scales(spec, seed, layer).to(torch.float32)
    c0 = t0 // GEN_CHUNK
    c1 = (t1 + GEN_CHUNK - 1) // GEN_CHUNK
    for c in range(c0, c1):
        a = c * GEN_CHUNK
        rows = min(GEN_CHUNK, spec.n - a)
        xc = _x_chunk(spec, seed, layer, c, rows, aux)
        lo, hi = max(a, t0), min(a + rows, t1)
        out[lo - t0:hi - t0] = xc[lo - a:hi - a]
    return out


def dtype_of(name: str) -> torch.dtype:
    return _DT[name]


def make_x_device(spec: LayerSpec, seed: int, device, layer: int = 0) -> torch.Tensor:
    """X (n, k) of the same distribution as ``make_x``, drawn on the device with
    the device's generator (fast; the bytes differ from ``make_x``, so this is
    for timing runs only, never for a comparison with the oracle)."""
    g = torch.Generator(device=device)
    g.manual_seed(tensor_seed(seed, layer, 5))
    dt = _DT[spec.x_dtype]
    out = torch.empty(spec.n, spec.k, dtype=dt, device=device)
    if spec.x_kind == "lognormal":
        c = channel_scales(spec, seed, layer).to(device=device, dtype=torch.float32)
    elif spec.x_kind == "mixed":
        L = mixing_matrix(spec, seed, layer).to(device=device, dtype=torch.float32)
    step = 16384
    for a in range(0, spec.n, step):
        rows = min(step, spec.n - a)
        if spec.x_kind == "lognormal":
            z = torch.randn(rows, spec.k, generator=g, device=device) * c
        elif spec.x_kind == "silu":
            z = torch.nn.functional.silu(torch.randn(rows, spec.k, generator=g, device=device))
            z *= torch.randn(rows, spec.k, generator=g, device=device)
        else:
            z = torch.randn(rows, spec.k, generator=g, device=device) @ L
        out[a:a + rows] = z.to(dt)
    return out


def make_w_device(spec: LayerSpec, seed: int, device, layer: int = 0) -> torch.Tensor:
    """W (r, k) ~ N(0, w_std^2) drawn on the device (timing runs only)."""
    g = torch.Generator(device=device)
    g.manual_seed(tensor_seed(seed, layer, 6))
    w = torch.randn(spec.r, spec.k, generator=g, device=device) * spec.w_std
    return w.to(_DT[spec.w_dtype])
