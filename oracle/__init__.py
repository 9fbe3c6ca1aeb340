"""fp64 CPU oracle for CalibQuant's decode hot path (TEST INFRASTRUCTURE ONLY).

This package is the slow, obviously-correct reference that the CUDA library is
checked against. Only the test-suite, ``__graft_entry__.smoke()`` and the CPU
baseline leg of ``bench.py`` may import it; the product path never does, and the
library has no CPU fallback.

It shares no code with the CUDA path: every step is written here from the
method's definitions in plain numpy float64 (library primitives only: min/max,
rint, matmul, exp).

Citations name the CalibQuant article (QbitAI's Chinese write-up of
"CalibQuant: 1-Bit KV Cache Quantization for Multimodal LLMs", arXiv
2502.14882) and its sections:

* "Method 1"  -- channel-wise KV cache quantization (uniform b-bit integer
  quantization with per-channel min/max statistics);
* "Method 2"  -- post-scaling of the dequantization into the vector products;
* "Method 3"  -- post-quantization calibration of the attention scores;
* "Runtime analysis" -- the decode-throughput measurement.

The formulas of that page were lost when it was converted to text; where a step
is open, the reading taken is stated in the function's docstring.

Parity status: every public function here is pinned by ``tests/test_oracle_*``
against closed forms, exact rational arithmetic on small inputs, a library
attention routine, invariants of the method, or hand-derived bit positions.
"""

from .calibquant import (  # noqa: F401
    levels,
    channel_stats,
    quantize_codes,
    stored_stats,
    dequantize,
    scores_dequantized,
    scores_post_scaled,
    calibrate,
    softmax,
    attend_dequantized,
    attend_post_scaled,
    quantize_cache,
    decode_attention,
    decode_attention_mixed,
)
from .layouts import (  # noqa: F401
    LAYOUT_CANONICAL,
    LAYOUT_OCTET_K,
    LAYOUT_OCTET_V,
    padded_tokens,
    codes_nbytes,
    pack_codes,
    unpack_codes,
    bit_position,
)
