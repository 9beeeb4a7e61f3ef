"""any4 on B200: Python binding of libany4 (the sm_100a CUDA library).

This module only marshals arguments: every step of the any4 path (quantize,
pack, dequant, matmul) runs in the CUDA kernels of libany4.so, reached through its
C ABI (include/any4.h).  PyTorch provides device memory and the current
stream.  There is no CPU fallback: if the library is missing or the device is
not an sm_100 GPU, the calls raise.

Paper: "any4: Learned 4-bit Numeric Representation for LLMs" (arXiv 2507.04610).
"""
from ._native import (  # noqa: F401
    ANY4_ERR_ALIGN,
    ANY4_ERR_CUDA,
    ANY4_ERR_NULL,
    ANY4_ERR_RANGE,
    ANY4_ERR_SHAPE,
    ANY4_ERR_TIMEOUT,
    ANY4_ERR_UNSUPPORTED,
    ANY4_ERR_WORKSPACE,
    ANY4_GROUP_MAX,
    ANY4_QUANTIZE_MAX_ITER,
    ANY4_QUANTIZE_MAX_K,
    ANY4_STATIC_SCRATCH_BYTES,
    PATHS,
    Any4Error,
    Any4Prepared,
    any4_bits_per_weight,
    any4_dequant,
    any4_dequant_bits,
    any4_group_sums,
    any4_read_probe,
    any4_matmul,
    any4_matmul_bits,
    any4_matmul_bits_workspace_size,
    any4_matmul_choose_path,
    any4_matmul_grouped,
    any4_matmul_static_scratch,
    any4_matmul_workspace_size,
    any4_pack,
    any4_pack_bits,
    any4_prepare,
    any4_repack,
    any4_quantize,
    any4_quantize_bits,
    any4_status_string,
    any4_version,
    library,
    library_path,
)
