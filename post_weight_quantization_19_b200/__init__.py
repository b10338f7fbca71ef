"""B200-native (sm_100a) GPTQ per-layer solve behind a C ABI.

The compute lives in libgptq_b200.so (hand-written CUDA kernels): the
tcgen05/TMA Hessian on CTA pairs; a blocked Cholesky of the damped Hessian
taken from the bottom-right corner (fp32 128 x 128 diagonal blocks on one CTA,
3xTF32 tensor-core products, outer 1024-column blocks for wide layers) with the
inverse factor U assembled over a merge tree; the column sweep with a row of
each 128-column block held by 8 lanes in registers and lazy trailing updates
as tensor-core GEMMs; fused unpermute/loss/pack.  This package holds the nvcc
build step, a ctypes view of include/gptq.h and a thin torch binding with the
same entry-point names.
"""

from .gptq import (  # noqa: F401
    GPTQError,
    gptq_check_device_status,
    gptq_hessian_accumulate,
    gptq_last_phase_ms,
    gptq_launch_count,
    gptq_layer_host_workspace_bytes,
    gptq_dequant_fp16,
    gptq_dequant_gemv,
    gptq_factor,
    gptq_factor_plan,
    gptq_gemm_pair_form,
    gptq_linear_fp16,
    gptq_pack,
    gptq_quantize_layer,
    gptq_quantize_with_factor,
    gptq_quantize_workspace_bytes,
    gptq_set_gemm_pair,
    gptq_set_phase_timing,
    gptq_solve_layer_host,
)
from .sharded import row_shard, shard_range, solve_layer_sharded, token_shard  # noqa: F401
from .chain import quantize_chain  # noqa: F401
