"""GPTQ oracle: a plain, slow, obviously-correct fp64 CPU implementation of GPTQ
layer-wise quantization.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path imports this package:
only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline / reference
arm of ``bench.py`` may import, call or execute anything under ``oracle/``.
It shares no code with the CUDA library (``post_weight_quantization_23_b200``)
and never imports it; the only module both sides use is the seeded input
generator ``synth``, which holds none of the method's arithmetic.

Every function cites the web page passage it follows, by page title and
section.  The pages are:

* "GPTQ" (ozercemkelahmet.com/tools/gptq): *How it works* Steps 1-9,
  *Optional refinements*, *A worked example*, *A minimal Python sketch*,
  *Memory arithmetic*, *Glossary*.  Called [GPTQ-tool] below.
* "GPTQ Quantization: Complete Technical Guide" (notes.jayaprakash.net):
  *Quantization Equation*, *Detailed Algorithm*, *Example: Quantizing a Single
  Weight*, *Computing the Hessian*, *Configuration Deep Dive*.  [GPTQ-guide].
* "GPTQ" paper breakdown (ai360xpert.com/papers/gptq): *How It Works*.
  [GPTQ-breakdown].
* "What Is GPTQ? Classic 4-Bit LLM Quantization" (ai-tldr.dev): *How it
  works*, Step 3 (grouping and scales).  [What-is-GPTQ].

Parity status: every function here is pinned by a ``-m "not gpu"`` test
against worked numbers printed on the pages, closed forms, invariants or
brute force, except where its docstring says "parity unpinned".
"""

from .gptq_oracle import (  # noqa: F401
    NotPositiveDefinite,
    hessian,
    fix_dead_columns,
    act_order_perm,
    damp,
    hinv_upper_factor,
    grid_params,
    static_grids,
    quantize_codes,
    sweep_unblocked,
    sweep_blocked,
    sweep_obs,
    sweep_replay,
    rtn,
    layer_loss,
    gptq,
    pack,
    unpack,
    dequant,
    dequant_matmul,
    rotation_matrix,
    rotate,
    storage_bits_per_weight,
    group_count,
)
