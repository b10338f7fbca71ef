"""ctypes view of the C ABI declared in include/gptq.h (no marshalling here)."""

from __future__ import annotations

import ctypes
import os

from . import build as _build

_LIB = None

STATUS = {
    0: "GPTQ_OK",
    1: "GPTQ_ERR_INVALID_ARG",
    2: "GPTQ_ERR_NOT_PD",
    3: "GPTQ_ERR_CUDA",
    4: "GPTQ_ERR_NO_MEMORY",
    5: "GPTQ_ERR_TIMEOUT",
}

c_void_p, c_int, c_int64, c_float, c_size_t = (ctypes.c_void_p, ctypes.c_int, ctypes.c_int64,
                                              ctypes.c_float, ctypes.c_size_t)

# name -> (restype, argtypes); mirrors include/gptq.h one to one.
SIGNATURES = {
    "gptq_status_string": (ctypes.c_char_p, [c_int]),
    "gptq_hessian_accumulate": (c_int, [c_void_p, c_int64, c_int64, c_int64, c_void_p, c_void_p]),
    "gptq_quantize_workspace_bytes": (c_size_t, [c_int64, c_int64, c_int, c_int, c_int, c_int]),
    "gptq_quantize_layer": (c_int, [c_void_p, c_int64, c_int64, c_void_p, c_int, c_int, c_int,
                                    c_float, c_int, c_void_p, c_void_p, c_void_p, c_void_p,
                                    c_void_p, c_void_p, c_void_p, c_void_p, c_size_t, c_void_p]),
    "gptq_factor_workspace_bytes": (c_size_t, [c_int64, c_int]),
    "gptq_factor": (c_int, [c_void_p, c_int64, c_float, c_int, c_void_p, c_void_p, c_void_p,
                            c_size_t, c_void_p]),
    "gptq_quantize_with_factor_workspace_bytes": (c_size_t, [c_int64, c_int64, c_int, c_int,
                                                             c_int]),
    "gptq_quantize_with_factor": (c_int, [c_void_p, c_int64, c_int64, c_void_p, c_void_p,
                                          c_void_p, c_int, c_int, c_int, c_int, c_void_p,
                                          c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                                          c_void_p, c_void_p, c_size_t, c_void_p]),
    "gptq_pack": (c_int, [c_void_p, c_int64, c_int64, c_int, c_void_p, c_void_p]),
    "gptq_dequant_gemv": (c_int, [c_void_p, c_void_p, c_void_p, c_void_p, c_int64, c_int64, c_int,
                                  c_int, c_void_p, c_int64, c_void_p, c_void_p]),
    "gptq_dequant_fp16": (c_int, [c_void_p, c_void_p, c_void_p, c_void_p, c_int64, c_int64, c_int,
                                  c_int, c_void_p, c_void_p]),
    "gptq_linear_fp16": (c_int, [c_void_p, c_int64, c_int64, c_void_p, c_int64, c_void_p, c_void_p]),
    "gptq_quantize_layer_noalloc": (c_int, [c_void_p, c_int64, c_int64, c_void_p, c_int, c_int,
                                            c_int, c_float, c_int, c_void_p, c_void_p, c_void_p,
                                            c_void_p, c_void_p, c_void_p, c_void_p, c_void_p]),
    "gptq_layer_host_workspace_bytes": (c_size_t, [c_int64, c_int64, c_int64, c_int, c_int, c_int,
                                                   c_int]),
    "gptq_solve_layer_host": (c_int, [c_void_p, c_int64, c_void_p, c_int64, c_int64, c_int, c_int,
                                      c_int, c_float, c_int, c_void_p, c_void_p, c_void_p,
                                      c_void_p, c_void_p, c_void_p, c_size_t, c_void_p]),
    "gptq_check_device_status": (c_int, [c_void_p]),
    "gptq_launch_count": (ctypes.c_uint64, []),
    "gptq_last_error": (ctypes.c_char_p, []),
    "gptq_set_phase_timing": (c_int, [c_int]),
    "gptq_last_phase_ms": (c_int, [c_void_p, c_int]),
    "gptq_factor_plan": (c_size_t, [c_int64, c_int64, c_int, c_void_p, c_size_t]),
    "gptq_selftest_timeout": (c_int, [c_void_p, c_void_p]),
    "gptq_gemm_pair_form": (c_int, [c_void_p, c_size_t]),
    "gptq_set_gemm_pair": (c_int, [c_int]),
}


def library_path() -> str:
    return _build.LIB


def load(build_if_missing: bool = True) -> ctypes.CDLL:
    """Load libgptq_b200.so from the package directory (building it if absent).

    There is no fallback: without the compiled library every entry point of
    this package raises.
    """
    global _LIB
    if _LIB is not None:
        return _LIB
    path = library_path()
    if not os.path.exists(path):
        if not build_if_missing:
            raise RuntimeError(f"GPTQ CUDA library missing: {path}")
        _build.build()
    lib = ctypes.CDLL(path)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _LIB = lib
    return lib
