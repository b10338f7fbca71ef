"""Plain float64 CPU oracle for the GPTQ per-layer solve.

TEST INFRASTRUCTURE ONLY: the tests, the smoke check and the benchmark's CPU
baseline leg import this package.  The library under
``post_weight_quantization_19_b200`` never imports it and has no CPU path.
"""

from .gptq_ref import (  # noqa: F401
    act_order_perm,
    brute_force_min_loss,
    dampen,
    dequant_gemv,
    dequantize,
    gptq_quantize_layer,
    gptq_quantize_rows_lowmem,
    gptq_sweep,
    hessian,
    hessian_rows,
    inverse_upper_cholesky,
    inverse_upper_cholesky_lowmem,
    layer_loss,
    layer_loss_direct,
    pack_rows,
    quant_params,
    quantize,
    quantize_chain,
    rtn,
    unpack_rows,
)
