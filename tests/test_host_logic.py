"""Host-side orchestration in the package, run on the CPU with the device entry
points played by the oracle (same arguments and outputs as the binding's)."""

import numpy as np
import pytest

import oracle
from synth import make_activations, make_weights

torch = pytest.importorskip("torch")


def test_chain_driver_feeds_each_layer_the_quantised_outputs(monkeypatch):
    # quantize_chain must call the Hessian on the current inputs, solve, dequantise
    # the packed result to fp16 and run it forward; with the entry points played
    # by the oracle the result is the oracle's chain exactly.
    from post_weight_quantization_19_b200 import chain

    exact = {}   # the driver's fp32 H buffer -> the float64 Hessian it stands for

    def hessian(X, H, stream=None):
        exact[H.data_ptr()] = oracle.hessian(X.numpy())

    def quantize_layer(W, H, *, bits, group, block, damp, act_order, sym, static_groups,
                       g_idx, stream=None):
        o = oracle.gptq_quantize_layer(W.numpy(), exact.pop(H.data_ptr()), bits=bits, group=group,
                                       block=block, damp=damp, act_order=act_order, sym=sym,
                                       static_groups=static_groups)
        g_idx.copy_(torch.from_numpy(o["g_idx"]))
        return {"qweight": torch.from_numpy(oracle.pack_rows(o["codes"], bits)),
                "scales": torch.from_numpy(o["scales"]), "zeros": torch.from_numpy(o["zeros"]),
                "loss": o["loss"], "g_idx": g_idx}

    def dequant_fp16(qweight, scales, zeros, d, bits, group, g_idx=None, stream=None):
        y = oracle.dequant_gemv(qweight.numpy(), scales.numpy(), zeros.numpy(), bits, group,
                                np.eye(d), g_idx=g_idx.numpy())
        return torch.from_numpy(y.T.astype(np.float16))

    def linear_fp16(X, W16, stream=None):
        Y = X.numpy().astype(np.float64) @ W16.numpy().astype(np.float64).T
        return torch.from_numpy(Y.astype(np.float16))

    monkeypatch.setattr(chain, "gptq_hessian_accumulate", hessian)
    monkeypatch.setattr(chain, "gptq_quantize_layer", quantize_layer)
    monkeypatch.setattr(chain, "gptq_dequant_fp16", dequant_fp16)
    monkeypatch.setattr(chain, "gptq_linear_fp16", linear_fp16)

    X0 = make_activations(600, 64, seed=5)
    Ws = [make_weights(96, 64, seed=6), make_weights(32, 96, seed=7)]
    for act in (False, True):
        got = chain.quantize_chain(torch.from_numpy(X0), [torch.from_numpy(W) for W in Ws],
                                   bits=4, group=32, act_order=act, keep_inputs=True)
        ref = oracle.quantize_chain(X0, Ws, bits=4, group=32, act_order=act)
        assert len(got) == 2
        for g_, r_ in zip(got, ref):
            np.testing.assert_array_equal(g_["inputs"].numpy(), r_["inputs"])
            np.testing.assert_array_equal(g_["qweight"].numpy(), oracle.pack_rows(r_["codes"], 4))
            assert g_["loss"] == r_["loss"]
        last = (ref[-1]["inputs"].astype(np.float64)
                @ ref[-1]["What"].astype(np.float16).astype(np.float64).T).astype(np.float16)
        np.testing.assert_array_equal(got[-1]["outputs"].numpy(), last)


def test_chain_driver_rejects_mismatched_layers():
    from post_weight_quantization_19_b200 import chain
    X0 = torch.zeros((8, 64), dtype=torch.float16)
    with pytest.raises(ValueError):
        chain.quantize_chain(X0, [torch.zeros((32, 96))], bits=4, group=32)
