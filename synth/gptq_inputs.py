"""Seeded calibration activations X and layer weights W for the GPTQ layer solve.

The GPTQ reading card (page "GPTQ: Accurate Post-Training Quantization for
Generative Pre-trained Transformers", section on the compute setup) calibrates
on 128 random 2048-token C4 segments.  Neither the dataset nor trained weights
are available here, so these generators stand in for them with the same shapes
and a value structure that matters to the solve:

* X [n x d] fp16: z ~ N(0,1) times a per-channel factor c_j ~ lognormal(0, s).
  A fraction of channels (0.1 %, at least one) is multiplied by a large factor,
  the activation-outlier structure that makes the Hessian ill-scaled.
* W [r x d] fp32: N(0, sigma^2), optionally with a few outlier columns (x10) or
  a fraction of heavy-tailed Student-t(3) rows.

Every array is a pure function of its seed: numpy PCG64 streams, one child
stream per 8192-token chunk (SeedSequence.spawn), so chunks can be filled by a
thread pool and still give identical bytes on any machine.
"""

from __future__ import annotations

import concurrent.futures as _fut
import dataclasses
import math
import os

import numpy as np

_CHUNK = 8192


def _threads() -> int:
    try:
        return max(1, len(os.sched_getaffinity(0)))
    except AttributeError:  # pragma: no cover
        return os.cpu_count() or 1


def channel_factors(d: int, sigma: float, outlier_frac: float, outlier_mult: float,
                    seed: int) -> np.ndarray:
    """Per-channel scale c_j (float64): lognormal(0, sigma), outliers multiplied."""
    rng = np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, 1])))
    c = rng.lognormal(mean=0.0, sigma=sigma, size=d)
    if outlier_frac > 0.0 and outlier_mult != 1.0:
        k = max(1, int(math.ceil(outlier_frac * d)))
        idx = rng.choice(d, size=k, replace=False)
        c[idx] *= outlier_mult
    return c


def make_activations(n: int, d: int, *, sigma: float = 1.0, outlier_frac: float = 0.0,
                     outlier_mult: float = 1.0, seed: int = 0) -> np.ndarray:
    """Calibration activations X [n x d] as C-contiguous float16."""
    c = channel_factors(d, sigma, outlier_frac, outlier_mult, seed).astype(np.float32)
    X = np.empty((n, d), dtype=np.float16)
    nchunks = (n + _CHUNK - 1) // _CHUNK
    children = np.random.SeedSequence([seed, 2]).spawn(max(nchunks, 1))

    def fill(i: int) -> None:
        t0, t1 = i * _CHUNK, min(n, (i + 1) * _CHUNK)
        rng = np.random.Generator(np.random.PCG64(children[i]))
        z = rng.standard_normal(size=(t1 - t0, d), dtype=np.float32)
        z *= c
        X[t0:t1] = z.astype(np.float16)

    if nchunks <= 1:
        for i in range(nchunks):
            fill(i)
    else:
        with _fut.ThreadPoolExecutor(max_workers=min(_threads(), nchunks)) as ex:
            list(ex.map(fill, range(nchunks)))
    if not np.isfinite(X).all():
        raise ValueError("synthetic activations overflowed float16")
    return X


def make_weights(r: int, d: int, *, std: float = 0.02, outlier_cols: int = 0,
                 outlier_col_mult: float = 10.0, t3_row_frac: float = 0.0,
                 seed: int = 0) -> np.ndarray:
    """Layer weights W [r x d] as C-contiguous float32."""
    W = np.empty((r, d), dtype=np.float32)
    rows_per = max(1, _CHUNK * 64 // max(d, 1))
    nchunks = (r + rows_per - 1) // rows_per
    children = np.random.SeedSequence([seed, 3]).spawn(max(nchunks, 1))

    def fill(i: int) -> None:
        r0, r1 = i * rows_per, min(r, (i + 1) * rows_per)
        rng = np.random.Generator(np.random.PCG64(children[i]))
        W[r0:r1] = (rng.standard_normal(size=(r1 - r0, d), dtype=np.float64) * std
                    ).astype(np.float32)

    if nchunks <= 1:
        for i in range(nchunks):
            fill(i)
    else:
        with _fut.ThreadPoolExecutor(max_workers=min(_threads(), nchunks)) as ex:
            list(ex.map(fill, range(nchunks)))
    rng = np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, 4])))
    if outlier_cols > 0:
        cols = rng.choice(d, size=outlier_cols, replace=False)
        W[:, cols] *= np.float32(outlier_col_mult)
    if t3_row_frac > 0.0:
        k = max(1, int(math.ceil(t3_row_frac * r)))
        rows = rng.choice(r, size=k, replace=False)
        W[rows] = (rng.standard_t(3.0, size=(k, d)) * std).astype(np.float32)
    return W


@dataclasses.dataclass(frozen=True)
class Workload:
    """One layer problem: shapes, input recipe and quantiser settings."""

    name: str
    r: int
    d: int
    n: int
    bits: int
    group: int
    act_order: bool
    x_sigma: float
    x_outlier_frac: float
    x_outlier_mult: float
    w_std: float
    w_outlier_cols: int = 0
    w_t3_row_frac: float = 0.0
    block: int = 128
    damp: float = 0.01
    seed: int = 1000

    @property
    def x_bytes(self) -> int:
        return self.n * self.d * 2


# The layer shapes named in the workload list: a tiny layer, a Llama-7B
# q_proj, the two MLP projections, an 8192-wide 3-bit layer and an
# OPT-175B fc2.  Seeds are 1000 + the position in that list.
WORKLOADS: dict[str, Workload] = {w.name: w for w in [
    Workload("tiny_128x256", 128, 256, 2048, 4, -1, False, 0.5, 0.0, 1.0, 0.02,
             w_outlier_cols=2, seed=1000),
    Workload("llama7b_q_proj_4096x4096", 4096, 4096, 262144, 4, 128, False, 1.0, 0.001, 50.0,
             0.02, seed=1001),
    Workload("llama7b_up_proj_11008x4096", 11008, 4096, 262144, 4, 128, False, 1.0, 0.001,
             50.0, 0.02, seed=1002),
    Workload("llama7b_up_proj_11008x4096_actorder", 11008, 4096, 262144, 4, 128, True, 1.0,
             0.001, 50.0, 0.02, seed=1002),
    Workload("llama7b_down_proj_4096x11008", 4096, 11008, 262144, 4, 128, False, 1.0, 0.001,
             50.0, 0.02, seed=1012),
    Workload("llama7b_down_proj_4096x11008_actorder", 4096, 11008, 262144, 4, 128, True, 1.0,
             0.001, 50.0, 0.02, seed=1012),
    Workload("w3_8192x8192_perrow", 8192, 8192, 262144, 3, -1, False, 1.0, 0.001, 50.0, 0.015,
             w_t3_row_frac=0.01, seed=1003),
    Workload("w3_8192x8192_g128", 8192, 8192, 262144, 3, 128, False, 1.0, 0.001, 50.0, 0.015,
             w_t3_row_frac=0.01, seed=1003),
    Workload("opt175b_fc2_12288x49152", 12288, 49152, 65536, 3, 128, False, 1.0, 0.001, 50.0,
             0.01, seed=1004),
]}


def workload(name: str) -> Workload:
    return WORKLOADS[name]


def workload_inputs(wl: Workload, *, n: int | None = None, r: int | None = None
                    ) -> tuple[np.ndarray, np.ndarray]:
    """(X fp16 [n x d], W fp32 [r x d]) for a workload.

    ``n``/``r`` take a leading sub-sample of the tokens/rows (same bytes as the
    full arrays' first rows, because chunks are seeded independently).
    """
    nn = wl.n if n is None else min(n, wl.n)
    rr = wl.r if r is None else min(r, wl.r)
    X = make_activations(nn, wl.d, sigma=wl.x_sigma, outlier_frac=wl.x_outlier_frac,
                         outlier_mult=wl.x_outlier_mult, seed=wl.seed)
    W = make_weights(wl.r, wl.d, std=wl.w_std, outlier_cols=wl.w_outlier_cols,
                     t3_row_frac=wl.w_t3_row_frac, seed=wl.seed)
    return X, np.ascontiguousarray(W[:rr])


def make_problem(r: int, d: int, n: int, *, seed: int, sigma: float = 1.0,
                 outlier_frac: float = 0.001, outlier_mult: float = 50.0,
                 w_std: float = 0.02) -> tuple[np.ndarray, np.ndarray]:
    """A small seeded layer problem with the workload value structure."""
    X = make_activations(n, d, sigma=sigma, outlier_frac=outlier_frac,
                         outlier_mult=outlier_mult, seed=seed)
    W = make_weights(r, d, std=w_std, seed=seed)
    return X, W
