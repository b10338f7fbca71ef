"""Full-size layers on the GPU, checked on sampled rows against the float64 oracle.

The GPU runs the whole layer in the launch configuration the benchmark times;
the oracle computes the full float64 Hessian and U (rows are independent once
U is fixed) and sweeps a seeded sample of rows.
"""

import numpy as np
import pytest

import oracle
from parity_util import H_REL_FRO, LOSS_REL, assert_codes_close, gpu_layer, rel_fro
from synth import workload, workload_inputs

torch = pytest.importorskip("torch")
pytestmark = [pytest.mark.gpu, pytest.mark.slow]


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def _check_sampled(name: str, nrows: int = 64):
    wl = workload(name)
    X, W = workload_inputs(wl)
    got = gpu_layer(X, W, bits=wl.bits, group=wl.group, block=wl.block, damp=wl.damp,
                    act_order=wl.act_order)
    H = oracle.hessian(X)
    err = rel_fro(got["H"], H)
    assert err <= H_REL_FRO, err
    rows = np.sort(np.random.default_rng(wl.seed).choice(wl.r, nrows, replace=False))
    ref = oracle.gptq_quantize_layer(W, H, bits=wl.bits, group=wl.group, block=wl.block,
                                     damp=wl.damp, act_order=wl.act_order, rows=rows)
    match = assert_codes_close(got["codes"][rows], ref["codes"])
    gl = oracle.layer_loss(W[rows], got["W_hat"][rows], H)
    assert abs(gl - ref["loss"]) <= LOSS_REL * ref["loss"], (gl, ref["loss"])
    total = oracle.layer_loss(W, got["W_hat"], H)
    assert abs(got["loss"] - total) <= LOSS_REL * total, (got["loss"], total)
    np.testing.assert_array_equal(got["qweight"][rows], oracle.pack_rows(got["codes"][rows],
                                                                         wl.bits))
    print(f"{name}: H rel {err:.2e}, codes {match:.6f}, sampled loss rel "
          f"{abs(gl - ref['loss']) / ref['loss']:.2e}")


def test_llama7b_q_proj_4096x4096():
    _check_sampled("llama7b_q_proj_4096x4096")
