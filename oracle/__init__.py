"""Plain, slow, obviously correct CPU oracle for BitDelta compress and multi-tenant apply.

TEST INFRASTRUCTURE ONLY. Nothing on the product path may import, call or link this
package: only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` use it. It shares no code with the CUDA
library under ``tenant_serving_b200/`` and never imports it.

Every function works in float64 on exactly decoded inputs (bf16 / fp16 / fp32 bit
patterns are widened without rounding) and follows the method step by step as the
source pages state it:

* "bitdelta — BitDelta (ZIP-7) Per-User Personalization Without LoRA", section
  "How BitDelta Works" (1. Delta Computation, 2. Group Quantization, 3. 1-bit
  Quantization, 4. Reconstruction, 5. Serving) and "Safety Benefits: 1. Outlier
  Clipping".
* "BitDelta Guide: 1-Bit Delta Quantization for LLM Serving", "1. Mathematical
  Formulation: Sign Bits and Scalar Scaling", "2. Optimal L2 Norm Initialization" and
  "Systems Mechanics: 1. Decoupled Forward Pass".
* "Per-Axis Weight Deltas for Frequent Model Updates", "Key Contributions" item 1
  (row / column scale vectors, mask packed along the input axis).
* ``oracle.fp8``: an e4m3 base with per-row scales under the same delta path ("BitDelta
  Guide", "3. Quantized Base Model Compatibility"; "Per-Axis Weight Deltas", Future
  Directions, FP8 co-design).

Every function here is pinned by ``tests/test_oracle.py`` against the pages' worked
examples, closed forms, invariants or brute force; none is "parity unpinned".
"""

from .bitdelta import (  # noqa: F401
    MODE_GROUP,
    MODE_ROW,
    MODE_COL,
    MODE_TENSOR,
    MODE_BLOCK,
    decode,
    delta,
    clip_stats,
    clip,
    abs_mean_scales,
    sign_bits,
    pack_bits,
    unpack_bits,
    compress,
    expand_scales,
    reconstruct,
    apply_multi,
    apply_rows,
)
from .fp8 import (  # noqa: F401
    E4M3_MAX,
    e4m3_value,
    e4m3_round,
    quantize_base,
    dequantize_base,
    apply_multi_fp8,
)
