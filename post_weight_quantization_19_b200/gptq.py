"""Python binding of the C ABI: the same entry points, taking torch CUDA tensors.

Argument marshalling only -- dtype/shape/device checks and pointer extraction.
Every step of the solve runs in the CUDA kernels of libgptq_b200.so; there is
no CPU path.  PyTorch provides device memory and streams.
"""

from __future__ import annotations

import ctypes

import torch

from . import _abi


class GPTQError(RuntimeError):
    def __init__(self, status: int, where: str):
        lib = _abi.load()
        msg = lib.gptq_status_string(status).decode()
        detail = lib.gptq_last_error().decode() if status == 3 else ""
        super().__init__(f"{where}: {_abi.STATUS.get(status, status)} ({msg})"
                         + (f": {detail}" if detail else ""))
        self.status = status


def _check(status: int, where: str) -> None:
    if status != 0:
        raise GPTQError(status, where)


def _stream(stream) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream


# Option bits of the layer solve (include/gptq.h).
ACT_ORDER, SYMMETRIC, STATIC_GROUPS = 1, 2, 4


def _options(act_order: bool, sym: bool, static_groups: bool) -> int:
    return ((ACT_ORDER if act_order else 0) | (SYMMETRIC if sym else 0)
            | (STATIC_GROUPS if static_groups else 0))


def _ptr(t: torch.Tensor | None, dtype: torch.dtype | None = None, name: str = "") -> int | None:
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t.data_ptr()


def gptq_hessian_accumulate(X: torch.Tensor, H: torch.Tensor, stream=None) -> None:
    """H += 2 X^T X on the GPU (X fp16 [n, d] row-major, H fp32 [d, d])."""
    lib = _abi.load()
    n, d = X.shape
    if H.shape != (d, d):
        raise ValueError("H must be [d, d]")
    _check(lib.gptq_hessian_accumulate(_ptr(X, torch.float16, "X"), n, d, d,
                                       _ptr(H, torch.float32, "H"), _stream(stream)),
           "gptq_hessian_accumulate")


def gptq_quantize_workspace_bytes(r: int, d: int, bits: int, group: int, block: int = 128,
                                  act_order: bool = False, sym: bool = False,
                                  static_groups: bool = False) -> int:
    return int(_abi.load().gptq_quantize_workspace_bytes(
        r, d, bits, group, block, _options(act_order, sym, static_groups)))


def gptq_quantize_layer(W: torch.Tensor, H: torch.Tensor, *, bits: int, group: int,
                        block: int = 128, damp: float = 0.01, act_order: bool = False,
                        sym: bool = False, static_groups: bool = False,
                        W_hat: torch.Tensor | None = None, codes: torch.Tensor | None = None,
                        g_idx: torch.Tensor | None = None, workspace: torch.Tensor | None = None,
                        outputs: dict | None = None, stream=None) -> dict:
    """GPTQ solve of one layer.  H is consumed.  Returns qweight/scales/zeros/loss (+ optional).

    ``sym`` selects the symmetric quantiser and ``static_groups`` fixes every
    group's parameters from the original W before the sweep (GPTQ_SYMMETRIC and
    GPTQ_STATIC_GROUPS of the C header).  ``outputs`` may hold preallocated
    ``qweight``, ``scales`` and ``zeros`` tensors.
    """
    options = _options(act_order, sym, static_groups)
    lib = _abi.load()
    r, d = W.shape
    G = 1 if group == -1 else d // max(group, 1)
    dev = W.device
    out = dict(outputs or {})
    qweight = out.get("qweight")
    if qweight is None:
        qweight = torch.empty((r, d * bits // 32), dtype=torch.int32, device=dev)
    scales = out.get("scales")
    if scales is None:
        scales = torch.empty((r, G), dtype=torch.float32, device=dev)
    zeros = out.get("zeros")
    if zeros is None:
        zeros = torch.empty((r, G), dtype=torch.int32, device=dev)
    need = lib.gptq_quantize_workspace_bytes(r, d, bits, group, block, options)
    if need == 0 and r > 0:
        raise GPTQError(1, "gptq_quantize_workspace_bytes")
    if workspace is None:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=dev)
    loss = ctypes.c_double(0.0)
    _check(lib.gptq_quantize_layer(
        _ptr(W, torch.float32, "W"), r, d, _ptr(H, torch.float32, "H"), bits, group, block,
        float(damp), options, _ptr(W_hat, torch.float32, "W_hat"),
        _ptr(qweight, torch.int32, "qweight"), _ptr(scales, torch.float32, "scales"),
        _ptr(zeros, torch.int32, "zeros"), _ptr(g_idx, torch.int32, "g_idx"),
        _ptr(codes, torch.uint8, "codes"), ctypes.byref(loss), _ptr(workspace, None, "workspace"),
        workspace.numel() * workspace.element_size(), _stream(stream)), "gptq_quantize_layer")
    res = {"qweight": qweight, "scales": scales, "zeros": zeros, "loss": loss.value}
    if W_hat is not None:
        res["W_hat"] = W_hat
    if codes is not None:
        res["codes"] = codes
    if g_idx is not None:
        res["g_idx"] = g_idx
    return res


def gptq_dequant_gemv(qweight: torch.Tensor, scales: torch.Tensor, zeros: torch.Tensor,
                      x: torch.Tensor, bits: int, group: int, g_idx: torch.Tensor | None = None,
                      y: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """y [m, r] = x [m, d] W^^T from the packed layer (x fp32, m <= GPTQ_GEMV_MAX_M)."""
    lib = _abi.load()
    if x.dim() == 1:
        x = x.unsqueeze(0)
    m, d = x.shape
    r = qweight.shape[0]
    if y is None:
        y = torch.empty((m, r), dtype=torch.float32, device=x.device)
    _check(lib.gptq_dequant_gemv(
        _ptr(qweight, torch.int32, "qweight"), _ptr(scales, torch.float32, "scales"),
        _ptr(zeros, torch.int32, "zeros"), _ptr(g_idx, torch.int32, "g_idx"), r, d, bits, group,
        _ptr(x, torch.float32, "x"), m, _ptr(y, torch.float32, "y"), _stream(stream)),
        "gptq_dequant_gemv")
    return y


def gptq_factor(H: torch.Tensor, *, damp: float = 0.01, act_order: bool = False,
                workspace: torch.Tensor | None = None, stream=None) -> dict:
    """Damp, order and factor H in place: returns {"U": H, "perm", "lambda"} for
    ``gptq_quantize_with_factor`` (perm is None without act-order)."""
    lib = _abi.load()
    d = H.shape[0]
    if H.shape != (d, d):
        raise ValueError("H must be [d, d]")
    options = ACT_ORDER if act_order else 0
    need = lib.gptq_factor_workspace_bytes(d, options)
    if need == 0:
        raise GPTQError(1, "gptq_factor_workspace_bytes")
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=H.device)
    perm = torch.empty(d, dtype=torch.int32, device=H.device) if act_order else None
    lam = torch.empty(1, dtype=torch.float32, device=H.device)
    _check(lib.gptq_factor(_ptr(H, torch.float32, "H"), d, float(damp), options,
                           _ptr(perm, torch.int32, "perm"), _ptr(lam, torch.float32, "lambda"),
                           _ptr(workspace, None, "workspace"),
                           workspace.numel() * workspace.element_size(), _stream(stream)),
           "gptq_factor")
    return {"U": H, "perm": perm, "lambda": lam}


def gptq_quantize_with_factor(W: torch.Tensor, factor: dict, *, bits: int, group: int,
                              block: int = 128, sym: bool = False, static_groups: bool = False,
                              W_hat: torch.Tensor | None = None, codes: torch.Tensor | None = None,
                              g_idx: torch.Tensor | None = None,
                              workspace: torch.Tensor | None = None, outputs: dict | None = None,
                              stream=None) -> dict:
    """The sweep half of the solve from ``gptq_factor``'s result (U, perm, lambda are
    only read).  Returns qweight/scales/zeros/loss like ``gptq_quantize_layer``."""
    lib = _abi.load()
    r, d = W.shape
    U, perm, lam = factor["U"], factor["perm"], factor["lambda"]
    options = _options(perm is not None, sym, static_groups)
    G = 1 if group == -1 else d // max(group, 1)
    dev = W.device
    out = dict(outputs or {})
    qweight = out.get("qweight")
    if qweight is None:
        qweight = torch.empty((r, d * bits // 32), dtype=torch.int32, device=dev)
    scales = out.get("scales")
    if scales is None:
        scales = torch.empty((r, G), dtype=torch.float32, device=dev)
    zeros = out.get("zeros")
    if zeros is None:
        zeros = torch.empty((r, G), dtype=torch.int32, device=dev)
    need = lib.gptq_quantize_with_factor_workspace_bytes(r, d, bits, group, block)
    if need == 0 and r > 0:
        raise GPTQError(1, "gptq_quantize_with_factor_workspace_bytes")
    if workspace is None:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=dev)
    loss = ctypes.c_double(0.0)
    _check(lib.gptq_quantize_with_factor(
        _ptr(W, torch.float32, "W"), r, d, _ptr(U, torch.float32, "U"),
        _ptr(perm, torch.int32, "perm"), _ptr(lam, torch.float32, "lambda"), bits, group, block,
        options, _ptr(W_hat, torch.float32, "W_hat"), _ptr(qweight, torch.int32, "qweight"),
        _ptr(scales, torch.float32, "scales"), _ptr(zeros, torch.int32, "zeros"),
        _ptr(g_idx, torch.int32, "g_idx"), _ptr(codes, torch.uint8, "codes"), ctypes.byref(loss),
        _ptr(workspace, None, "workspace"), workspace.numel() * workspace.element_size(),
        _stream(stream)), "gptq_quantize_with_factor")
    res = {"qweight": qweight, "scales": scales, "zeros": zeros, "loss": loss.value}
    if W_hat is not None:
        res["W_hat"] = W_hat
    if codes is not None:
        res["codes"] = codes
    if g_idx is not None:
        res["g_idx"] = g_idx
    return res


def gptq_dequant_fp16(qweight: torch.Tensor, scales: torch.Tensor, zeros: torch.Tensor, d: int,
                      bits: int, group: int, g_idx: torch.Tensor | None = None,
                      W16: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """W16 [r, d] fp16 = s (q - z) from the packed layer."""
    lib = _abi.load()
    r = qweight.shape[0]
    if W16 is None:
        W16 = torch.empty((r, d), dtype=torch.float16, device=qweight.device)
    _check(lib.gptq_dequant_fp16(
        _ptr(qweight, torch.int32, "qweight"), _ptr(scales, torch.float32, "scales"),
        _ptr(zeros, torch.int32, "zeros"), _ptr(g_idx, torch.int32, "g_idx"), r, d, bits, group,
        _ptr(W16, torch.float16, "W16"), _stream(stream)), "gptq_dequant_fp16")
    return W16


def gptq_linear_fp16(X: torch.Tensor, W16: torch.Tensor, Y: torch.Tensor | None = None,
                     stream=None) -> torch.Tensor:
    """Y [n, r] = fp16(X [n, d] W16 [r, d]^T), fp32 accumulation on the tensor cores."""
    lib = _abi.load()
    n, d = X.shape
    r = W16.shape[0]
    if W16.shape[1] != d:
        raise ValueError("W16 must be [r, d]")
    if Y is None:
        Y = torch.empty((n, r), dtype=torch.float16, device=X.device)
    _check(lib.gptq_linear_fp16(_ptr(X, torch.float16, "X"), n, d, _ptr(W16, torch.float16, "W16"),
                                r, _ptr(Y, torch.float16, "Y"), _stream(stream)),
           "gptq_linear_fp16")
    return Y


def gptq_pack(codes: torch.Tensor, bits: int, qweight: torch.Tensor | None = None,
              stream=None) -> torch.Tensor:
    lib = _abi.load()
    r, d = codes.shape
    if qweight is None:
        qweight = torch.empty((r, d * bits // 32), dtype=torch.int32, device=codes.device)
    _check(lib.gptq_pack(_ptr(codes, torch.uint8, "codes"), r, d, bits,
                         _ptr(qweight, torch.int32, "qweight"), _stream(stream)), "gptq_pack")
    return qweight


def gptq_layer_host_workspace_bytes(r: int, d: int, n: int, bits: int, group: int,
                                    block: int = 128, act_order: bool = False,
                                    sym: bool = False, static_groups: bool = False) -> int:
    return int(_abi.load().gptq_layer_host_workspace_bytes(
        r, d, n, bits, group, block, _options(act_order, sym, static_groups)))


def gptq_solve_layer_host(X: torch.Tensor, W: torch.Tensor, *, bits: int, group: int,
                          block: int = 128, damp: float = 0.01, act_order: bool = False,
                          sym: bool = False, static_groups: bool = False,
                          dev_workspace: torch.Tensor, outputs: dict, stream=None) -> float:
    """Whole layer from host (CPU, ideally pinned) tensors; fills ``outputs`` host tensors."""
    lib = _abi.load()
    n, d = X.shape
    r = W.shape[0]
    for t, name in ((X, "X"), (W, "W")):
        if t.is_cuda or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous host tensor")
    if X.dtype != torch.float16 or W.dtype != torch.float32:
        raise ValueError("X must be float16 and W float32")
    loss = ctypes.c_double(0.0)
    gi = outputs.get("g_idx")
    _check(lib.gptq_solve_layer_host(
        X.data_ptr(), n, W.data_ptr(), r, d, bits, group, block, float(damp),
        _options(act_order, sym, static_groups),
        outputs["qweight"].data_ptr(), outputs["scales"].data_ptr(), outputs["zeros"].data_ptr(),
        gi.data_ptr() if gi is not None else None, ctypes.byref(loss),
        _ptr(dev_workspace, None, "dev_workspace"),
        dev_workspace.numel() * dev_workspace.element_size(), _stream(stream)),
        "gptq_solve_layer_host")
    return loss.value


def gptq_check_device_status(stream=None) -> int:
    return int(_abi.load().gptq_check_device_status(_stream(stream)))


def gptq_launch_count() -> int:
    return int(_abi.load().gptq_launch_count())


def gptq_set_phase_timing(enable: bool) -> None:
    _abi.load().gptq_set_phase_timing(int(enable))


def gptq_last_phase_ms() -> list[float]:
    buf = (ctypes.c_float * 4)()
    n = _abi.load().gptq_last_phase_ms(buf, 4)
    return [float(buf[i]) for i in range(n)]


def gptq_factor_plan(d: int, outer_cols: int = 0, side_streams: bool = True) -> str:
    """The factorisation's launches and stream events for a d x d H_d (no GPU used)."""
    lib = _abi.load()
    n = lib.gptq_factor_plan(d, outer_cols, int(side_streams), None, 0)
    if n == 0:
        raise GPTQError(1, "gptq_factor_plan: invalid arguments")
    buf = ctypes.create_string_buffer(n)
    lib.gptq_factor_plan(d, outer_cols, int(side_streams), buf, n)
    return buf.value.decode()


def gptq_gemm_pair_form() -> tuple[int, str]:
    """(form, probe record) of the two-CTA product on the current device: 0-5 a
    cluster launch form, 6 the one-CTA fallback, -1 not probed yet."""
    lib = _abi.load()
    buf = ctypes.create_string_buffer(512)
    form = lib.gptq_gemm_pair_form(buf, 512)
    return int(form), buf.value.decode()


def gptq_set_gemm_pair(enable: bool) -> bool:
    """Run products with two or more row tiles on CTA pairs (True) or one CTA per
    tile (False, the default); returns the previous setting."""
    return bool(_abi.load().gptq_set_gemm_pair(int(bool(enable))))
