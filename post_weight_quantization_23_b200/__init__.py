"""GPTQ layer-wise weight quantization on B200 (sm_100a).

The compute path is the C ABI library ``libgptq_b200.so`` (include/gptq.h),
built in-tree by ``python -m post_weight_quantization_23_b200.build``.  This
package is its thin Python front end: ``_lib`` (ctypes marshalling) and
``api`` (device buffers and call order).  Importing it does not need a GPU;
every call into the library does, and raises if the library is missing.
"""

from ._lib import (  # noqa: F401
    EXPORTED,
    GptqError,
    NotPositiveDefinite,
    LIB_PATH,
    load,
)
from .api import (GptqPlan, QuantConfig, hadamard_block, quant_matmul,  # noqa: F401
                  quantize_layer, rotate, rotation_signs)
