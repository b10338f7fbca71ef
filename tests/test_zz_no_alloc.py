"""gptq_quantize_layer_noalloc through the C ABI (needs a GPU).

Some callers cannot allocate device memory (a pool that forbids side
allocations, a runtime that reserved the device up front, a host that passes
only inputs and outputs), so the library offers a variant of the layer solve
whose scratch is a fixed array inside the library.  These tests call that
entry point twice in a row, on two different layers, and check each result
against the ordinary entry point with a caller workspace, with the tolerances
of the parity tests.  The file is named so that pytest collects it last.
"""

import ctypes

import numpy as np
import pytest

from parity_util import LOSS_REL, assert_codes_close
from synth import make_problem

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def g():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import post_weight_quantization_19_b200 as mod
    return mod


def _buffers(r, d, bits, group):
    G = 1 if group == -1 else d // group
    return {
        "qweight": torch.empty((r, d * bits // 32), dtype=torch.int32, device="cuda"),
        "scales": torch.empty((r, G), dtype=torch.float32, device="cuda"),
        "zeros": torch.empty((r, G), dtype=torch.int32, device="cuda"),
        "codes": torch.empty((r, d), dtype=torch.uint8, device="cuda"),
        "W_hat": torch.empty((r, d), dtype=torch.float32, device="cuda"),
        "g_idx": torch.empty((d,), dtype=torch.int32, device="cuda"),
    }


def _noalloc(lib, W, H, bits, group, block, act_order, out):
    r, d = W.shape
    loss = ctypes.c_double(-1.0)
    st = lib.gptq_quantize_layer_noalloc(
        W.data_ptr(), r, d, H.data_ptr(), bits, group, block, 0.01, int(act_order),
        out["W_hat"].data_ptr(), out["qweight"].data_ptr(), out["scales"].data_ptr(),
        out["zeros"].data_ptr(), out["g_idx"].data_ptr(), out["codes"].data_ptr(),
        ctypes.byref(loss), torch.cuda.current_stream().cuda_stream)
    return st, loss.value


def test_noalloc_matches_workspace_entry_point_on_two_calls(g):
    from post_weight_quantization_19_b200 import _abi

    lib = _abi.load()
    # two different layers back to back: the second must not see the first's leftovers
    cases = [(64, 512, 4096, 4, 128, 128, False, 31), (48, 384, 3000, 3, -1, 64, True, 32)]
    for r, d, n, bits, group, block, act, seed in cases:
        X, W = make_problem(r, d, n, seed=seed)
        Wd = torch.from_numpy(W).cuda()
        H = torch.zeros((d, d), dtype=torch.float32, device="cuda")
        g.gptq_hessian_accumulate(torch.from_numpy(X).cuda(), H)
        ref_out = _buffers(r, d, bits, group)
        ref = g.gptq_quantize_layer(Wd, H.clone(), bits=bits, group=group, block=block,
                                    act_order=act, W_hat=ref_out["W_hat"],
                                    codes=ref_out["codes"], g_idx=ref_out["g_idx"],
                                    outputs=ref_out)
        out = _buffers(r, d, bits, group)
        st, loss = _noalloc(lib, Wd, H.clone(), bits, group, block, act, out)
        assert st == 0, lib.gptq_status_string(st)
        torch.cuda.synchronize()
        assert_codes_close(out["codes"].cpu().numpy(), ref_out["codes"].cpu().numpy())
        assert abs(loss - ref["loss"]) <= LOSS_REL * ref["loss"]
        np.testing.assert_allclose(out["scales"].cpu().numpy(), ref_out["scales"].cpu().numpy(),
                                   rtol=1e-4)
        np.testing.assert_array_equal(out["g_idx"].cpu().numpy(), ref_out["g_idx"].cpu().numpy())


def test_noalloc_rejects_a_layer_beyond_its_scratch(g):
    from post_weight_quantization_19_b200 import _abi

    lib = _abi.load()
    r = d = 4096   # needs more than the fixed scratch
    assert lib.gptq_quantize_workspace_bytes(r, d, 4, 128, 128, 0) > (64 << 20)
    W = torch.zeros((r, d), device="cuda")
    H = torch.eye(d, device="cuda")
    out = _buffers(r, d, 4, 128)
    st, _ = _noalloc(lib, W, H, 4, 128, 128, False, out)
    assert st == 4   # GPTQ_ERR_NO_MEMORY, nothing enqueued
    assert b"GPTQ_NOALLOC_SCRATCH_BYTES" in lib.gptq_last_error()
