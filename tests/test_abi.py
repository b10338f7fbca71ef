"""The C-ABI library loads on a machine without a GPU and exports the header.

Only host-side logic is exercised here: symbol presence, status strings,
workspace size queries and argument validation (which returns before any CUDA
call).  Compute is covered by the GPU tests.
"""

import ctypes
import os
import re

import pytest

from post_weight_quantization_19_b200 import _abi

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _header_functions():
    with open(os.path.join(ROOT, "include", "gptq.h")) as f:
        text = f.read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(gptq_[a-z_0-9]+)\s*\(", text)))


def test_every_declared_symbol_is_exported(lib):
    names = _header_functions()
    assert len(names) >= 11
    for name in names:
        assert hasattr(lib, name), name
    assert sorted(_abi.SIGNATURES) == names


def test_status_strings(lib):
    for code in range(6):
        assert lib.gptq_status_string(code)
    assert lib.gptq_status_string(999) == b"unknown status"


def test_workspace_query(lib):
    ws = lib.gptq_quantize_workspace_bytes
    base = ws(4096, 4096, 4, 128, 128, 0)
    # working copy of W, superblock errors and codes (every merge-tree node of a
    # 4096-wide factor is square, so the factorisation needs no extra scratch)
    assert base >= 4096 * 4096 * 4 + 4096 * 1024 * 4 + 4096 * 4096
    # wide layers also hold a copy of the outer panel (d x 1024 floats)
    assert ws(64, 49152, 3, 128, 128, 0) >= 64 * 49152 * 5 + 49152 * 1024 * 4
    assert ws(4096, 4096, 4, 128, 128, 1) >= base + 4096 * 4096 * 4   # permuted H
    assert base % 256 == 0
    for bad in [(16, 100, 4, -1, 128, 0),      # d % 32
                (16, 256, 5, -1, 128, 0),      # bits
                (16, 256, 4, 48, 128, 0),      # group not a divisor of the block
                (16, 256, 4, 96, 128, 0),
                (16, 256, 4, -1, 96, 0),       # block
                (-1, 256, 4, -1, 128, 0),
                (16, 256, 4, -1, 128, 8)]:     # unknown option bit
        assert ws(*bad) == 0, bad
    # the option bits GPTQ_SYMMETRIC and GPTQ_STATIC_GROUPS need no extra workspace
    assert ws(4096, 4096, 4, 128, 128, 2 | 4) == base
    hw = lib.gptq_layer_host_workspace_bytes(128, 256, 2048, 4, -1, 128, 0)
    assert hw >= 2048 * 256 * 2 + 256 * 256 * 4 + 128 * 256 * 4


def test_validation_returns_before_cuda(lib):
    p = ctypes.c_void_p(4096)   # never dereferenced: validation fails first
    loss = ctypes.c_double(-1)
    q = lib.gptq_quantize_layer
    # bits
    assert q(p, 8, 256, p, 5, -1, 128, 0.01, 0, None, p, p, p, None, None,
             ctypes.byref(loss), p, 1 << 30, None) == 1
    # damp negative / NaN
    assert q(p, 8, 256, p, 4, -1, 128, -1.0, 0, None, p, p, p, None, None,
             ctypes.byref(loss), p, 1 << 30, None) == 1
    assert q(p, 8, 256, p, 4, -1, 128, float("nan"), 0, None, p, p, p, None, None,
             ctypes.byref(loss), p, 1 << 30, None) == 1
    # unknown option bit
    assert q(p, 8, 256, p, 4, -1, 128, 0.01, 8, None, p, p, p, None, None,
             ctypes.byref(loss), p, 1 << 30, None) == 1
    # missing output pointer
    assert q(p, 8, 256, p, 4, -1, 128, 0.01, 0, None, None, p, p, None, None,
             ctypes.byref(loss), p, 1 << 30, None) == 1
    # workspace too small
    ws = ctypes.c_void_p(1 << 20)
    assert q(p, 8, 256, p, 4, -1, 128, 0.01, 0, None, p, p, p, None, None,
             ctypes.byref(loss), ws, 1024, None) == 4
    # empty layer: OK, loss 0, nothing enqueued
    assert q(p, 0, 256, p, 4, -1, 128, 0.01, 0, None, p, p, p, None, None,
             ctypes.byref(loss), p, 0, None) == 0
    assert loss.value == 0.0
    h = lib.gptq_hessian_accumulate
    assert h(p, 10, 100, 100, p, None) == 1          # d % 32
    assert h(p, 10, 128, 100, p, None) == 1          # ldx < d
    assert h(ctypes.c_void_p(4098), 10, 128, 128, p, None) == 1   # X not 16-byte aligned
    assert h(p, -1, 128, 128, p, None) == 1
    assert h(p, 0, 128, 128, p, None) == 0           # no tokens: nothing to do
    assert lib.gptq_pack(p, 4, 100, 4, p, None) == 1
    assert lib.gptq_pack(p, 4, 128, 6, p, None) == 1
    gv = lib.gptq_dequant_gemv
    assert gv(p, p, p, None, 8, 100, 4, -1, p, 1, p, None) == 1     # d % 32
    assert gv(p, p, p, None, 8, 128, 5, -1, p, 1, p, None) == 1     # bits
    assert gv(p, p, p, None, 8, 128, 4, 48, p, 1, p, None) == 1     # group not a multiple of 32
    assert gv(p, p, p, None, 8, 128, 4, -1, p, 9, p, None) == 1     # m > GPTQ_GEMV_MAX_M
    assert gv(p, p, p, None, 8, 128, 4, -1, ctypes.c_void_p(4100), 1, p, None) == 1  # x alignment
    assert gv(p, p, p, None, 8, 128, 4, -1, None, 1, p, None) == 1  # missing x
    assert gv(p, p, p, None, 0, 128, 4, -1, p, 1, p, None) == 0     # no rows: nothing to do
    assert gv(p, p, p, None, 8, 128, 4, -1, p, 0, p, None) == 0     # no vectors
    fw = lib.gptq_factor_workspace_bytes
    assert fw(100, 0) == 0 and fw(256, 8) == 0 and fw(256, 1) > fw(256, 0) > 0
    f = lib.gptq_factor
    assert f(p, 100, 0.01, 0, None, p, p, 1 << 30, None) == 1     # d % 32
    assert f(p, 256, 0.01, 1, None, p, p, 1 << 30, None) == 1     # act-order without perm
    assert f(p, 256, -1.0, 0, None, p, p, 1 << 30, None) == 1     # damp
    assert f(p, 256, 0.01, 0, None, p, ctypes.c_void_p(1 << 20), 64, None) == 4   # workspace
    qf = lib.gptq_quantize_with_factor
    assert lib.gptq_quantize_with_factor_workspace_bytes(8, 256, 4, 128, 128) > 0
    assert qf(p, 8, 256, p, None, p, 4, 128, 128, 1, None, p, p, p, None, None,
              ctypes.byref(loss), p, 1 << 30, None) == 1             # act-order without perm
    assert qf(p, 8, 256, p, None, p, 5, 128, 128, 0, None, p, p, p, None, None,
              ctypes.byref(loss), p, 1 << 30, None) == 1             # bits
    assert qf(p, 0, 256, p, None, p, 4, 128, 128, 0, None, p, p, p, None, None,
              ctypes.byref(loss), p, 0, None) == 0                   # no rows
    df = lib.gptq_dequant_fp16
    assert df(p, p, p, None, 8, 100, 4, -1, p, None) == 1           # d % 32
    assert df(p, p, p, None, 8, 128, 6, -1, p, None) == 1           # bits
    assert df(p, p, p, None, 8, 128, 4, -1, ctypes.c_void_p(4104), None) == 1   # W16 alignment
    assert df(p, p, p, None, 0, 128, 4, -1, p, None) == 0           # no rows
    lf = lib.gptq_linear_fp16
    assert lf(p, 16, 100, p, 64, p, None) == 1                      # d % 32
    assert lf(p, 16, 128, p, 40, p, None) == 1                      # r % 32
    assert lf(ctypes.c_void_p(4104), 16, 128, p, 64, p, None) == 1  # X alignment
    assert lf(p, 0, 128, p, 64, p, None) == 0                       # no tokens
    assert lf(p, 16, 128, p, 0, p, None) == 0                       # no outputs
    st = lib.gptq_selftest_timeout
    assert st(None, None) == 1 and st(ctypes.c_void_p(4100), None) == 1
    na = lib.gptq_quantize_layer_noalloc
    # a bad argument is reported as such even for a layer beyond the fixed scratch
    assert na(p, 4096, 4096, p, 4, 128, 128, -1.0, 0, None, p, p, p, None, None,
              ctypes.byref(loss), None) == 1
    assert na(p, 4096, 4096, p, 4, 128, 128, 0.01, 0, None, None, p, p, None, None,
              ctypes.byref(loss), None) == 1
    assert na(p, 4096, 4096, p, 4, 128, 128, 0.01, 0, None, p, p, p, None, None,
              ctypes.byref(loss), None) == 4


def test_no_kernels_launched_on_cpu(lib):
    assert lib.gptq_launch_count() == 0


def test_library_is_in_tree():
    path = _abi.library_path()
    assert path.startswith(os.path.join(ROOT, "post_weight_quantization_19_b200"))
    assert os.path.exists(path)
