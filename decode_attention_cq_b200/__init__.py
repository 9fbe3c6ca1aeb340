"""libcalibq -- CalibQuant 1-bit visual-KV-cache quantization and decode
attention for NVIDIA B200 (sm_100a).

The compute lives in ``lib/libcalibq.so`` (hand-written CUDA behind a C ABI,
``include/calibq.h``); ``calibq`` is its ctypes binding and ``synth`` draws the
seeded synthetic workloads. Build with ``python -m decode_attention_cq_b200.build_lib``.
"""

from .calibq import (  # noqa: F401
    CQ_F16,
    CQ_F32,
    LAYOUT_CANONICAL,
    LAYOUT_OCTET_K,
    LAYOUT_OCTET_V,
    KERNEL_AUTO,
    KERNEL_CLUSTER,
    KERNEL_ENV,
    KERNEL_PIPE,
    KERNEL_ROW,
    KERNEL_TCGEN05,
    DEVICE_WAIT_TIMEOUT,
    CalibqError,
    QuantizedCache,
    cq_codes_bytes,
    cq_decode_attn,
    cq_decode_attn_ex,
    cq_decode_attn_mixed,
    cq_decode_attn_mixed_workspace_size,
    cq_decode_attn_workspace_size,
    cq_decode_kernel_name,
    cq_decode_launch_count,
    cq_set_decode_kernel,
    cq_dequant,
    cq_quantize_kv,
    cq_quantize_kv_workspace_size,
    cq_version,
)
