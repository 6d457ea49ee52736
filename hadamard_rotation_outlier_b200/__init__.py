"""B200-native fused Hadamard rotate + quantise (QuaRot-style online rotation).

The computation lives in ``libhadq.so`` (CUDA kernels for sm_100a behind the C
ABI declared in ``include/hadq.h``).  This package holds the ctypes binding
(same names as the C entry points), the in-tree build step and the seeded
synthetic input generators.
"""

from .binding import (  # noqa: F401
    HADQ_ERR_CUDA,
    HADQ_ERR_INVALID_ARG,
    HADQ_ERR_MISALIGNED,
    HADQ_ERR_UNSUPPORTED,
    HADQ_OK,
    MAX_DIM,
    HadqError,
    hadq_dequant_rotate_inv,
    hadq_dequant_rotate_inv_asym,
    hadq_dequant_rotate_inv_kron,
    hadq_dequant_rotate_inv_kron_pm1,
    hadq_dequant_rotate_inv_keep,
    hadq_kv_decode_attention,
    hadq_kv_decode_attention_noalloc,
    hadq_kv_decode_workspace_size,
    hadq_last_error,
    hadq_launch_count,
    hadq_kron_plan,
    hadq_plan,
    hadq_rotate_quantize,
    hadq_rotate_quantize_asym,
    hadq_rotate_quantize_kron,
    hadq_rotate_quantize_kron_pm1,
    hadq_rotate_quantize_keep,
    hyquant_keep_slots,
    hadq_status_str,
    hadq_version,
    load_library,
)
