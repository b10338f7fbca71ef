"""Write the oracle's result for sampled rows of the OPT-175B fc2 layer.

    python tests/golden/make_opt175b_fc2_rows.py

The layer (W 12288 x 49152, X 65536 x 49152 fp16, 3-bit, group 128) is too
large for the oracle to solve inside a GPU test: its float64 H is 19.3 GB and
the factorisation alone takes minutes of host time.  This script runs only the
oracle (``oracle.gptq_quantize_rows_lowmem``) on the seeded synthetic inputs of
``synth`` and stores, for 16 seeded rows, the codes, scales, zeros and per-row
objective, with a fingerprint of the inputs so that a changed generator is
detected instead of compared against.  About 20-30 minutes and 32 GB of host
memory on 8 cores.
"""

from __future__ import annotations

import os
import sys
import time

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(os.path.dirname(HERE))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
from synth import workload, workload_inputs  # noqa: E402

NAME = "opt175b_fc2_12288x49152"
OUT = os.path.join(HERE, "opt175b_fc2_rows.npz")
NROWS = 16


def sample_rows(r: int, seed: int) -> np.ndarray:
    return np.sort(np.random.default_rng(seed).choice(r, NROWS, replace=False))


def fingerprint(X: np.ndarray, W: np.ndarray, rows: np.ndarray) -> np.ndarray:
    """A few float64 sums that any change of the seeded inputs moves."""
    return np.array([
        float(np.sum(X[:, :256], dtype=np.float64)),
        float(np.sum(X[-4096:, -512:], dtype=np.float64)),
        float(np.sum(X[::997, ::13], dtype=np.float64)),
        float(np.sum(W[rows], dtype=np.float64)),
        float(np.sum(W[::101], dtype=np.float64)),
    ])


def main() -> None:
    wl = workload(NAME)
    t0 = time.time()
    X, W = workload_inputs(wl)
    rows = sample_rows(wl.r, wl.seed)
    print(f"inputs {time.time() - t0:.1f} s", flush=True)
    res = oracle.gptq_quantize_rows_lowmem(X, W, rows, bits=wl.bits, group=wl.group,
                                           block=wl.block, damp=wl.damp)
    print(f"oracle {time.time() - t0:.1f} s", flush=True)
    np.savez_compressed(
        OUT, rows=rows, codes=res["codes"].astype(np.uint8), scales=res["scales"],
        zeros=res["zeros"].astype(np.int16), row_loss=res["row_loss"],
        lam=np.array([res["lambda"]]), fingerprint=fingerprint(X, W, rows),
        config=np.array([wl.r, wl.d, wl.n, wl.bits, wl.group, wl.block, wl.seed]))
    print(f"wrote {OUT}", flush=True)


if __name__ == "__main__":
    main()
