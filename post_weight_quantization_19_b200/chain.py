"""A chain of linear layers quantised in order, each calibrated on the outputs
of the quantised layers before it.

GPTQ reading card, §计算设置: the reference implementation loads one block at a
time, accumulates the layer Hessians, quantises the block, then runs the
quantised block to produce the next block's inputs.  Here the chain is a
sequence of linear layers with no nonlinearity between them: layer k is solved
on H_k = 2 X_k^T X_k, and X_{k+1} = fp16(X_k fp16(W^_k)^T) is computed from its
packed output (dequantised to FP16 and multiplied in floating point, as the
"GPTQ" concept page describes inference, §3 技術原理).  Every step runs in the
library's kernels: the Hessian, the solve, the FP16 dequantisation and the
forward product.
"""

from __future__ import annotations

import torch

from .gptq import (gptq_dequant_fp16, gptq_hessian_accumulate, gptq_linear_fp16,
                   gptq_quantize_layer)


def quantize_chain(X0: torch.Tensor, Ws: list, *, bits: int, group: int, block: int = 128,
                   damp: float = 0.01, act_order: bool = False, sym: bool = False,
                   static_groups: bool = False, keep_inputs: bool = False,
                   stream=None) -> list[dict]:
    """Quantise W_0, W_1, ... (fp32 [r_k, d_k], d_{k+1} = r_k) on calibration
    tokens X0 (fp16 [n, d_0]).

    Returns one ``gptq_quantize_layer`` result per layer (with ``g_idx``), plus
    ``inputs`` = X_k when ``keep_inputs``, and ``outputs`` = X_{k+1} for the last
    layer.  The tensors stay on the device; nothing is synchronised except by
    the solve itself, which reads its loss back.
    """
    X = X0
    outs = []
    for k, W in enumerate(Ws):
        r, d = W.shape
        if X.shape[1] != d:
            raise ValueError(f"layer {k}: W has {d} inputs, the previous layer gives {X.shape[1]}")
        H = torch.zeros((d, d), dtype=torch.float32, device=W.device)
        gptq_hessian_accumulate(X, H, stream=stream)
        g_idx = torch.empty(d, dtype=torch.int32, device=W.device)
        res = gptq_quantize_layer(W, H, bits=bits, group=group, block=block, damp=damp,
                                  act_order=act_order, sym=sym, static_groups=static_groups,
                                  g_idx=g_idx, stream=stream)
        W16 = gptq_dequant_fp16(res["qweight"], res["scales"], res["zeros"], d, bits, group,
                                g_idx=g_idx, stream=stream)
        if keep_inputs:
            res["inputs"] = X
        X = gptq_linear_fp16(X, W16, stream=stream)
        outs.append(res)
    if outs:
        outs[-1]["outputs"] = X
    return outs
