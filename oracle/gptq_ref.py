"""Plain float64 CPU oracle for GPTQ's per-layer solve (test infrastructure).

TEST INFRASTRUCTURE ONLY.  Only the tests, ``__graft_entry__.smoke`` and the
benchmark's CPU-baseline leg may import this module.  It shares no code, table
or helper with the CUDA library; the two meet only at the seeded inputs of the
``synth`` package.

Every step follows the description on the source pages, cited by page title
and section:

* [Tutorial]  "GPTQ：一键量化大模型压缩" (aiqz.cc) -- sections 二阶信息 (Hessian
  H = 2 sum x x^T), 逐层量化 (layer objective ||W X - W^ X||_F^2), 误差补偿
  (OBS compensation delta_F = (q - w_q)/[H^-1]_qq [H^-1]_{F,q}), 分组方案
  (scale = (max - min)/(2^b - 1), zero = -min/scale, group-wise parameters).
* [Survey]    "LLM 量化技术" blog (astro-blog, llm-quantization-techniques) --
  §1.2 量化原理 (x_q = round(x/s + z), dequantised s(x_q - z)), §2.2 OBQ
  (the OBS update of the remaining weights), §2.3 items 1-3 (fixed column
  order, blocks of B = 128 columns, Cholesky for the needed rows of H^-1).
* [Card]      "GPTQ: Accurate Post-Training Quantization for Generative
  Pre-trained Transformers" reading card -- section 方法适配 (any fixed order,
  lazy batch of B = 128 columns with the global update deferred to the end of
  the block, Cholesky reformulation with mild damping).
* [Explainer] "一文读懂GPTQ" (mcipr.com) -- section 三 (int32 packing of 3/4-bit
  codes, group_size, desc_act).

Readings where the pages are silent or garbled (each one is listed in the
design notes):

* q in the compensation equation is the quantised value, so the remaining
  columns move by -(w_j - w^_j)/U_jj * U[j, j+1:] with U the upper Cholesky
  factor of H^-1 (the sign of the [Survey] §2.2 update).
* The error form "tr(dW^T H^-1 dW)" printed on two pages is garbled; the
  objective is ||(W - W^) X^T||_F^2 = 1/2 tr(dW H dW^T) with H = 2 X^T X.
* Damping adds lambda = damp * mean(diag H) to the diagonal.
* Quantiser: integer zero point.  xmin = min(0, min x), xmax = max(0, max x),
  s = (xmax - xmin)/(2^b - 1) (s = 1 when xmax == xmin), z = rint(-xmin/s),
  q = clip(rint(w/s) + z, 0, 2^b - 1), w^ = s (q - z).  rint rounds half to
  even.
* Group parameters are taken from the current (compensated) W when the sweep
  reaches a group's first column; with group = -1 they come from the original
  row.
* Act-order: stable argsort of -diag(H) (ties keep the lower index); groups
  are formed over permuted positions and g_idx maps original columns to them.
* Symmetric variant ([Survey] §1.2, whose formula is garbled): zero point 0,
  s = max|x| / (2^(b-1) - 1) (s = 1 for an all-zero row), signed codes
  clamped to [-2^(b-1), 2^(b-1) - 1] and stored as unsigned codes with
  z = 2^(b-1).
* Static groups (not on the pages; the plainest reading of parameters fixed
  before the sweep): every group's parameters come from the original W over
  the layer's own column groups, so under act-order g_idx[c] = c // group.
* Packing: per row, codes form an LSB-first bit stream along the input
  dimension, 32 bits per int32 word; 3-bit codes straddle words.

Parity status: every function here is pinned by tests under ``tests/``
(closed forms, invariants, special cases and brute force); none is unpinned.
"""

from __future__ import annotations

import itertools

import numpy as np

F64 = np.float64


# ---------------------------------------------------------------------------
# Hessian  ([Tutorial] §二阶信息: H = 2 * sum_i x_i x_i^T)
# ---------------------------------------------------------------------------

def hessian(X: np.ndarray, chunk: int = 8192) -> np.ndarray:
    """H = 2 * sum_t x_t x_t^T in float64 for X [n x d] (rows are tokens).

    fp16 inputs are exact in float64; the sum over tokens is taken in chunks of
    ``chunk`` rows with a float64 matrix product per chunk.
    """
    X = np.asarray(X)
    n, d = X.shape
    H = np.zeros((d, d), dtype=F64)
    for t0 in range(0, n, chunk):
        Xc = X[t0:t0 + chunk].astype(F64)
        H += Xc.T @ Xc
    return 2.0 * H


def hessian_rows(X: np.ndarray, rows: np.ndarray, chunk: int = 8192) -> np.ndarray:
    """Rows ``rows`` of H = 2 X^T X in float64, without forming all of H."""
    X = np.asarray(X)
    n, d = X.shape
    rows = np.asarray(rows, dtype=np.int64)
    out = np.zeros((rows.size, d), dtype=F64)
    for t0 in range(0, n, chunk):
        Xc = X[t0:t0 + chunk].astype(F64)
        out += Xc[:, rows].T @ Xc
    return 2.0 * out


# ---------------------------------------------------------------------------
# Damping, act-order, inverse-Hessian factor  ([Card] 方法适配; [Survey] §2.3)
# ---------------------------------------------------------------------------

def dampen(H: np.ndarray, damp: float) -> tuple[np.ndarray, float]:
    """H_d = H + lambda I with lambda = damp * mean(diag H)."""
    H = np.asarray(H, dtype=F64)
    lam = float(damp) * float(np.mean(np.diag(H)))
    Hd = H.copy()
    Hd[np.diag_indices_from(Hd)] += lam
    return Hd, lam


def act_order_perm(H: np.ndarray) -> np.ndarray:
    """Quantisation order: columns by descending diag(H), ties by lower index."""
    return np.argsort(-np.diag(np.asarray(H, dtype=F64)), kind="stable")


def inverse_upper_cholesky(Hd: np.ndarray) -> np.ndarray:
    """U upper triangular with positive diagonal and U^T U = Hd^-1.

    Plain definition: invert, then take the Cholesky factor of the inverse
    (numpy returns the lower factor L with Hd^-1 = L L^T; U = L^T).
    """
    Hinv = np.linalg.inv(np.asarray(Hd, dtype=F64))
    L = np.linalg.cholesky(Hinv)
    return np.ascontiguousarray(L.T)


def _lapack64():
    """dgemm of the OpenBLAS bundled with numpy, which takes
    64-bit integers (matrices of 2^31 elements and more), or None if absent.

    Reference BLAS/LAPACK calling convention: every argument by reference,
    column-major arrays, hidden lengths of the character arguments last.
    """
    import ctypes
    import glob
    import os

    site = os.path.dirname(os.path.dirname(np.__file__))
    found = glob.glob(os.path.join(site, "numpy.libs", "libscipy_openblas64_*.so"))
    if not found:
        return None
    lib = ctypes.CDLL(found[0])
    try:
        fns = {k: getattr(lib, f"scipy_{k}_64_") for k in ("dgemm",)}
    except AttributeError:
        return None
    for f in fns.values():
        f.restype = None
    return fns


_L64 = None


def _l64():
    global _L64
    if _L64 is None:
        _L64 = _lapack64() or {}
    return _L64


def _ref_args(*vals):
    import ctypes
    out = []
    for v in vals:
        if isinstance(v, bytes):
            out.append(ctypes.c_char_p(v))
        elif isinstance(v, float):
            out.append(ctypes.byref(ctypes.c_double(v)))
        else:
            out.append(ctypes.byref(ctypes.c_int64(v)))
    return out


def gemm_acc_inplace(H: np.ndarray, j0: int, j1: int, Xc: np.ndarray, alpha: float) -> None:
    """H[:j1, j0:j1] += alpha Xc[:, :j1]^T Xc[:, j0:j1] (library dgemm, in place).

    H: Fortran-ordered float64 d x d; Xc: C-ordered float64 t x d."""
    import ctypes

    if not (H.flags.f_contiguous and Xc.flags.c_contiguous and H.dtype == F64
            and Xc.dtype == F64):
        raise ValueError("gemm needs a Fortran-ordered H and a C-ordered Xc (float64)")
    t, d = Xc.shape
    L = _l64()
    if not L:
        H[:j1, j0:j1] += alpha * (Xc[:, :j1].T @ Xc[:, j0:j1])
        return
    # column-major view: Y = Xc^T is d x t with leading dimension d; the block is
    # Y[:j1, :] Y[j0:j1, :]^T
    m_, n_, k_, al, be, lda, ldb, ldc = _ref_args(j1, j1 - j0, t, float(alpha), 1.0, d, d, d)
    base = Xc.ctypes.data
    L["dgemm"](b"N", b"T", m_, n_, k_, al, ctypes.c_void_p(base), lda,
               ctypes.c_void_p(base + 8 * j0), ldb, be, ctypes.c_void_p(H.ctypes.data + 8 * d * j0),
               ldc, ctypes.c_size_t(1), ctypes.c_size_t(1))


def inverse_upper_cholesky_lowmem(box: list) -> np.ndarray:
    """``inverse_upper_cholesky`` of a d x d H_d held once, for very large d.

    ``box`` = [Hd]: Hd float64 in Fortran order with its upper triangle filled
    (the strictly lower triangle is ignored); the box is emptied so that Hd can
    be released as soon as it is no longer needed.  The same definition --
    invert, then take the Cholesky factor of the inverse -- with each step a
    LAPACK routine of PyTorch's CPU build: the Cholesky factor of Hd, the
    inverse from that factor (cholesky_inverse), and the upper Cholesky factor
    of the inverse.  At most two d x d arrays are alive at any time.
    """
    import torch

    Hd = box.pop()
    if Hd.dtype != F64 or not Hd.flags.f_contiguous:
        raise ValueError("Hd must be a Fortran-ordered float64 array")
    # Hd.T is C-ordered with the lower triangle filled
    L = torch.linalg.cholesky(torch.from_numpy(Hd.T), upper=False)
    del Hd
    Hinv = torch.cholesky_inverse(L, upper=False)
    del L
    U = torch.linalg.cholesky(Hinv, upper=True)
    del Hinv
    return U.numpy()


# ---------------------------------------------------------------------------
# Asymmetric min-max quantiser  ([Tutorial] §分组方案; [Survey] §1.2)
# ---------------------------------------------------------------------------

def quant_params(x: np.ndarray, bits: int, sym: bool = False) -> tuple[np.ndarray, np.ndarray]:
    """Per-row (scale, zero) of x [rows x cols] (float64 in, float64 out).

    ``sym``: the symmetric quantiser of [Survey] §1.2 (zero point 0, scale
    max|x| / (2^(b-1) - 1), signed codes clamped to [-2^(b-1), 2^(b-1) - 1]).
    The signed code is stored as the unsigned b-bit code code + 2^(b-1), so the
    same quantize/dequantize pair serves it with z = 2^(b-1).
    """
    x = np.asarray(x, dtype=F64)
    if sym:
        amax = np.abs(x).max(axis=1)
        half = 1 << (bits - 1)
        s = np.where(amax == 0.0, 1.0, amax / (half - 1))
        return s, np.full_like(s, float(half))
    maxq = (1 << bits) - 1
    xmin = np.minimum(x.min(axis=1), 0.0)
    xmax = np.maximum(x.max(axis=1), 0.0)
    flat = xmax == xmin
    s = np.where(flat, 1.0, (xmax - xmin) / maxq)
    z = np.rint(-xmin / s)
    return s, z


def quantize(w: np.ndarray, s: np.ndarray, z: np.ndarray, bits: int) -> np.ndarray:
    """Integer code clip(rint(w/s) + z, 0, 2^b - 1) (float64 holding integers)."""
    maxq = (1 << bits) - 1
    return np.clip(np.rint(np.asarray(w, dtype=F64) / s) + z, 0, maxq)


def dequantize(q: np.ndarray, s: np.ndarray, z: np.ndarray) -> np.ndarray:
    """w^ = s (q - z)."""
    return s * (q - z)


def rtn(W: np.ndarray, bits: int, group: int,
        sym: bool = False) -> tuple[np.ndarray, np.ndarray]:
    """Round-to-nearest baseline: same quantiser, parameters from W, no compensation.

    Returns (codes int64 [r x d], W^ float64 [r x d]).
    """
    W = np.asarray(W, dtype=F64)
    r, d = W.shape
    g = d if group == -1 else group
    codes = np.zeros((r, d), dtype=np.int64)
    What = np.zeros((r, d), dtype=F64)
    for c0 in range(0, d, g):
        blk = W[:, c0:c0 + g]
        s, z = quant_params(blk, bits, sym)
        q = quantize(blk, s[:, None], z[:, None], bits)
        codes[:, c0:c0 + g] = q.astype(np.int64)
        What[:, c0:c0 + g] = dequantize(q, s[:, None], z[:, None])
    return codes, What


# ---------------------------------------------------------------------------
# Column sweep with OBS compensation and lazy batches
# ([Tutorial] §误差补偿; [Survey] §2.2, §2.3; [Card] 方法适配)
# ---------------------------------------------------------------------------

def _check_groups(d: int, group: int, block: int) -> None:
    if group == -1:
        return
    if group <= 0 or d % group:
        raise ValueError("group must be -1 or a positive divisor of d")
    if block < d and not (block % group == 0 or group % block == 0):
        # A group that straddles a block end would read columns whose deferred
        # update has not been applied yet; the lazy form is then not exact.
        raise ValueError("lazy batches need block % group == 0 or group % block == 0")


def gptq_sweep(W: np.ndarray, U: np.ndarray, bits: int, group: int, block: int,
               sym: bool = False, fixed=None, forced=None):
    """Quantise W [r x d] column by column in fixed order.

    At column j: q = quantize(w_j), e_j = (w_j - w^_j)/U_jj, and the columns
    after j move by -e_j * U[j, j+1:].  Inside a block of ``block`` columns the
    move is applied at once; the move of the columns after the block is
    deferred to the block's end as one product E_blk @ U[blk, end:] (the lazy
    batch).  ``block >= d`` is the plain unblocked loop.

    ``fixed`` = (scales [r x G], zeros [r x G], col_group [d]) gives static
    group parameters chosen before the sweep: column j uses group col_group[j]
    and no parameters are taken from the compensated weights.

    ``forced`` = {j: codes [r]} replaces the rounding decision at column j by
    the given codes (then compensated as usual): for following another
    result's choice at a rounding tie, where both choices are correct.

    Returns (codes int64, scales, zeros (float64 holding integers), W^ float64,
    E float64 [r x d] with E[:, j] = e_j).
    """
    W = np.array(W, dtype=F64, copy=True)
    U = np.asarray(U, dtype=F64)
    r, d = W.shape
    G = 1 if group == -1 else d // group
    codes = np.zeros((r, d), dtype=np.int64)
    E = np.zeros((r, d), dtype=F64)
    if fixed is not None:
        scales = np.asarray(fixed[0], dtype=F64)
        zeros = np.asarray(fixed[1], dtype=F64)
        col_group = np.asarray(fixed[2], dtype=np.int64)
    else:
        _check_groups(d, group, block)
        scales = np.zeros((r, G), dtype=F64)
        zeros = np.zeros((r, G), dtype=F64)
        if group == -1:
            s, z = quant_params(W, bits, sym)
            scales[:, 0], zeros[:, 0] = s, z
    for b0 in range(0, d, block):
        b1 = min(d, b0 + block)
        for j in range(b0, b1):
            if fixed is not None:
                s, z = scales[:, col_group[j]], zeros[:, col_group[j]]
            elif group != -1 and j % group == 0:
                s, z = quant_params(W[:, j:j + group], bits, sym)
                scales[:, j // group], zeros[:, j // group] = s, z
            w = W[:, j]
            q = quantize(w, s, z, bits)
            if forced is not None and j in forced:
                q = np.asarray(forced[j], dtype=F64).copy()
            wq = dequantize(q, s, z)
            e = (w - wq) / U[j, j]
            codes[:, j] = q.astype(np.int64)
            E[:, j] = e
            W[:, j] = wq
            if j + 1 < b1:
                W[:, j + 1:b1] -= np.outer(e, U[j, j + 1:b1])
        if b1 < d:
            W[:, b1:] -= E[:, b0:b1] @ U[b0:b1, b1:]
    return codes, scales, zeros, W, E


# ---------------------------------------------------------------------------
# Layer objective  ([Tutorial] §逐层量化)
# ---------------------------------------------------------------------------

def layer_loss(W: np.ndarray, What: np.ndarray, H: np.ndarray) -> float:
    """||(W - W^) X^T||_F^2 written through H = 2 X^T X: 1/2 tr(D H D^T)."""
    D = np.asarray(W, dtype=F64) - np.asarray(What, dtype=F64)
    return 0.5 * float(np.sum((D @ np.asarray(H, dtype=F64)) * D))


def layer_loss_direct(W: np.ndarray, What: np.ndarray, X: np.ndarray) -> float:
    """||W X^T - W^ X^T||_F^2 straight from the activations (X [n x d])."""
    D = np.asarray(W, dtype=F64) - np.asarray(What, dtype=F64)
    Y = D @ np.asarray(X, dtype=F64).T
    return float(np.sum(Y * Y))


# ---------------------------------------------------------------------------
# The whole layer
# ---------------------------------------------------------------------------

def gptq_quantize_layer(W: np.ndarray, H: np.ndarray, *, bits: int, group: int,
                        block: int = 128, damp: float = 0.01,
                        act_order: bool = False, rows: np.ndarray | None = None,
                        sym: bool = False, static_groups: bool = False,
                        perm: np.ndarray | None = None) -> dict:
    """Damp, order, factor, sweep, score and unpermute one layer.

    ``rows`` restricts the sweep to a subset of output rows (rows are
    independent once U is fixed), for checks at full layer width.

    ``perm`` (act-order only) gives the column order instead of computing it
    from diag(H): for checking a result whose order differs from the oracle's
    only among columns whose diagonal entries are equal to within the
    precision of the H it was computed from (either order is then a stable
    descending order of the same values).

    ``sym`` selects the symmetric quantiser (see ``quant_params``).
    ``static_groups`` takes every group's parameters from the original W over
    the layer's own column groups (columns c with c // group = k) before the
    sweep, instead of from the compensated W when the sweep reaches a group;
    under act-order the groups then stay contiguous in the original column
    order, so g_idx[c] = c // group.  With group = -1 both rules coincide.
    """
    W = np.asarray(W, dtype=F64)
    H = np.asarray(H, dtype=F64)
    if rows is not None:
        W = W[np.asarray(rows)]
    r, d = W.shape
    Hd, lam = dampen(H, damp)
    if perm is not None:
        if not act_order:
            raise ValueError("a column order is given only with act-order")
        perm = np.asarray(perm, dtype=np.int64)
        if not np.array_equal(np.sort(perm), np.arange(d)):
            raise ValueError("perm is not a permutation")
    else:
        perm = act_order_perm(H) if act_order else np.arange(d)
    inv = np.argsort(perm)
    U = inverse_upper_cholesky(Hd[np.ix_(perm, perm)])
    fixed = None
    g_idx = (inv // group) if group != -1 else np.zeros(d, dtype=np.int64)
    if static_groups and group != -1:
        G = d // group
        fs = np.zeros((r, G), dtype=F64)
        fz = np.zeros((r, G), dtype=F64)
        for k in range(G):
            fs[:, k], fz[:, k] = quant_params(W[:, k * group:(k + 1) * group], bits, sym)
        # sweep position j holds original column perm[j]
        fixed = (fs, fz, perm // group)
        g_idx = np.arange(d) // group
    codes_p, scales, zeros, What_p, E = gptq_sweep(W[:, perm], U, bits, group, block,
                                                   sym=sym, fixed=fixed)
    codes = codes_p[:, inv]
    What = What_p[:, inv]
    return {
        "codes": codes,
        "scales": scales,
        "zeros": zeros.astype(np.int64),
        "g_idx": g_idx.astype(np.int64),
        "What": What,
        "loss": layer_loss(W, What, H),
        "obs_sum": 0.5 * float(np.sum(E * E)),
        "lambda": lam,
        "perm": perm,
        "U": U,
        "E": E,
    }


def gptq_quantize_rows_lowmem(X: np.ndarray, W: np.ndarray, rows: np.ndarray, *, bits: int,
                              group: int, block: int = 128, damp: float = 0.01,
                              chunk: int = 8192) -> dict:
    """``gptq_quantize_layer(W, hessian(X), rows=rows)`` holding one d x d array.

    For layers whose float64 H fits in host memory once but not the three or
    four times the plain path needs (the OPT-175B fc2 layer: d = 49152, one
    float64 H is 19.3 GB).  The steps are the same -- H = 2 sum x x^T
    ([Tutorial] §二阶信息), damping by damp * mean(diag H) and the upper
    Cholesky factor of H_d^-1 ([Card] 方法适配), the column sweep of the sampled
    rows -- with the upper triangle of H accumulated into a Fortran-ordered
    array by float64 matrix products (a band of columns at a time per token
    chunk; its diagonal checked against the column norms of X) and factored
    with at most two d x d arrays alive (``inverse_upper_cholesky_lowmem``);
    U^T U H_d e_j = e_j is checked on three columns.  H no longer exists after the
    factorisation, so each row's objective ||(w - w^) X^T||^2 is taken from X
    directly.  Natural column order only (no act-order).

    Returns codes/scales/zeros/What of the rows, ``row_loss`` [rows] and
    ``loss`` (their sum), ``lambda``.
    """
    X = np.asarray(X)
    n, d = X.shape
    rows = np.asarray(rows, dtype=np.int64)
    Wr = np.asarray(W, dtype=F64)[rows]
    H = np.zeros((d, d), dtype=F64, order="F")
    diag = np.zeros(d, dtype=F64)
    band = 4096
    for t0 in range(0, n, chunk):
        Xc = X[t0:t0 + chunk].astype(F64)
        diag += np.einsum("ij,ij->j", Xc, Xc)
        # the upper triangle, a band of columns at a time: H[:j1, j0:j1] +=
        # 2 Xc[:, :j1]^T Xc[:, j0:j1] (a float64 matrix product accumulated in place)
        for j0 in range(0, d, band):
            j1 = min(d, j0 + band)
            gemm_acc_inplace(H, j0, j1, Xc, 2.0)
    diag *= 2.0
    idx = np.arange(d)
    if not np.allclose(H[idx, idx], diag, rtol=1e-12, atol=0.0):
        raise RuntimeError("Hessian diagonal disagrees with the column norms")
    lam = float(damp) * float(np.mean(H[idx, idx]))
    H[idx, idx] += lam
    box = [H]
    del H
    U = inverse_upper_cholesky_lowmem(box)
    # U^T U H_d e_j = e_j on a few columns, with H_d e_j = 2 X^T (X e_j) + lambda e_j
    for j in (0, d // 3, d - 1):
        v = np.zeros(d)
        for t0 in range(0, n, chunk):
            Xc = X[t0:t0 + chunk]
            v += 2.0 * (Xc.T.astype(F64) @ Xc[:, j].astype(F64))
        v[j] += lam
        res = U.T @ (U @ v)
        res[j] -= 1.0
        if np.abs(res).max() > 1e-6:
            raise np.linalg.LinAlgError(f"U^T U H_d e_{j} is off the unit vector by {np.abs(res).max():.2e}")
    codes, scales, zeros, What, _ = gptq_sweep(Wr, U, bits, group, block)
    del U
    D = Wr - What
    row_loss = np.zeros(rows.size, dtype=F64)
    for t0 in range(0, n, chunk):
        Y = D @ X[t0:t0 + chunk].astype(F64).T
        row_loss += np.sum(Y * Y, axis=1)
    return {
        "codes": codes,
        "scales": scales,
        "zeros": zeros.astype(np.int64),
        "What": What,
        "row_loss": row_loss,
        "loss": float(np.sum(row_loss)),
        "lambda": lam,
    }


# ---------------------------------------------------------------------------
# Brute force for tiny rows (the grid is fixed by the row's own min/max)
# ---------------------------------------------------------------------------

def brute_force_min_loss(w: np.ndarray, H: np.ndarray, bits: int, sym: bool = False) -> float:
    """min over every code vector of 1/2 (w - w^) H (w - w^)^T for one row.

    The row's (s, z) come from its original values (group = -1), as in the
    sweep, so every candidate lies on the same grid.  Only for tiny d.
    """
    w = np.asarray(w, dtype=F64).reshape(1, -1)
    d = w.shape[1]
    s, z = quant_params(w, bits, sym)
    levels = np.arange(1 << bits, dtype=F64)
    cand = np.array(list(itertools.product(levels, repeat=d)), dtype=F64)
    D = w - dequantize(cand, s[0], z[0])
    return 0.5 * float(np.min(np.einsum("ij,jk,ik->i", D, np.asarray(H, dtype=F64), D)))


# ---------------------------------------------------------------------------
# int32 packing  ([Explainer] §三: 3/4-bit codes stored in 32-bit integers)
# ---------------------------------------------------------------------------

def pack_rows(codes: np.ndarray, bits: int) -> np.ndarray:
    """Pack codes [r x d] into int32 [r x d*bits/32]: LSB-first bit stream per row.

    Code c of a row occupies stream bits [c*bits, (c+1)*bits); stream bit k
    is bit (k mod 32) of word k // 32.
    """
    codes = np.asarray(codes)
    r, d = codes.shape
    if (d * bits) % 32:
        raise ValueError("d * bits must be a multiple of 32")
    words = np.zeros((r, d * bits // 32), dtype=np.uint64)
    for c in range(d):
        pos = c * bits
        wi, off = divmod(pos, 32)
        v = codes[:, c].astype(np.uint64) << np.uint64(off)
        words[:, wi] |= v & np.uint64(0xFFFFFFFF)
        if off + bits > 32:
            words[:, wi + 1] |= v >> np.uint64(32)
    return words.astype(np.uint32).view(np.int32)


def unpack_rows(words: np.ndarray, bits: int, d: int) -> np.ndarray:
    """Inverse of ``pack_rows``: int32 [r x d*bits/32] -> codes int64 [r x d]."""
    w = np.asarray(words).view(np.uint32).astype(np.uint64)
    r = w.shape[0]
    mask = np.uint64((1 << bits) - 1)
    out = np.zeros((r, d), dtype=np.int64)
    for c in range(d):
        pos = c * bits
        wi, off = divmod(pos, 32)
        v = w[:, wi] >> np.uint64(off)
        if off + bits > 32:
            v |= w[:, wi + 1] << np.uint64(32 - off)
        out[:, c] = (v & mask).astype(np.int64)
    return out


# ---------------------------------------------------------------------------
# Using the packed layer: y = W^ x  ([Card] §计算设置 -- the quantised layers
# are consumed by a dequantising matrix-vector kernel at inference; the
# packing of [Explainer] §三)
# ---------------------------------------------------------------------------

def dequant_gemv(qweight: np.ndarray, scales: np.ndarray, zeros: np.ndarray, bits: int,
                 group: int, x: np.ndarray, g_idx: np.ndarray | None = None) -> np.ndarray:
    """y [m x r] = x [m x d] @ W^^T with W^[row, c] = s[row, gi(c)] (q[row, c] - z[row, gi(c)]).

    q comes from unpacking ``qweight`` (LSB-first stream per row); gi(c) = g_idx[c]
    when given (act-order), else c // group (0 for group = -1).  float64 throughout.
    """
    x = np.atleast_2d(np.asarray(x, dtype=F64))
    d = x.shape[1]
    q = unpack_rows(qweight, bits, d).astype(F64)
    if g_idx is not None:
        gi = np.asarray(g_idx, dtype=np.int64)
    else:
        gi = np.zeros(d, dtype=np.int64) if group == -1 else np.arange(d) // group
    s = np.asarray(scales, dtype=F64)[:, gi]
    z = np.asarray(zeros, dtype=F64)[:, gi]
    return x @ (s * (q - z)).T



# ---------------------------------------------------------------------------
# Sequential layers  ([Card] §计算设置: quantise one block, then run the
# quantised block to produce the next block's calibration inputs; [Concept]
# §3 技術原理: at inference the codes are dequantised to FP16 and multiplied in
# floating point)
# ---------------------------------------------------------------------------

def quantize_chain(X0: np.ndarray, Ws: list, *, bits: int, group: int, block: int = 128,
                   damp: float = 0.01, act_order: bool = False, sym: bool = False,
                   static_groups: bool = False) -> list[dict]:
    """Quantise a chain of linear layers in order, each on its true inputs.

    Layer k (W_k [r_k x d_k], d_{k+1} = r_k) is solved with H_k = hessian(X_k);
    the next inputs are the quantised layer's outputs X_{k+1} = fp16(X_k
    fp16(W^_k)^T), accumulated in float64 over the fp16 values and rounded once
    to fp16 (an output beyond the fp16 range is an error).  Each entry is
    ``gptq_quantize_layer``'s result plus ``inputs`` = X_k (fp16).
    """
    X = np.asarray(X0, dtype=np.float16)
    outs = []
    for W in Ws:
        out = gptq_quantize_layer(W, hessian(X), bits=bits, group=group, block=block,
                                  damp=damp, act_order=act_order, sym=sym,
                                  static_groups=static_groups)
        out["inputs"] = X
        outs.append(out)
        Wh16 = out["What"].astype(np.float16).astype(F64)
        X = (X.astype(F64) @ Wh16.T).astype(np.float16)
        if not np.all(np.isfinite(X)):
            raise ValueError("layer outputs overflow fp16")
    return outs
