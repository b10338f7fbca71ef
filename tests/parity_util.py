"""Helpers shared by the GPU parity tests: run the CUDA path, compare with the oracle.

Tolerances (stated for the layer solve):
  H       relative Frobenius error <= 1e-5 against the float64 oracle;
  codes   >= 99.9 % identical and every mismatch exactly +-1 level;
  loss    within 0.5 % of the oracle's;
  packing bit-exact on identical codes.
"""

from __future__ import annotations

import numpy as np

H_REL_FRO = 1e-5
CODE_MATCH = 0.999
LOSS_REL = 5e-3


def rel_fro(a: np.ndarray, b: np.ndarray) -> float:
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    return float(np.linalg.norm(a - b) / np.linalg.norm(b))


def assert_codes_close(got: np.ndarray, ref: np.ndarray, frac: float = CODE_MATCH) -> float:
    diff = got.astype(np.int64) - ref.astype(np.int64)
    same = float(np.mean(diff == 0))
    worst = int(np.abs(diff).max()) if diff.size else 0
    assert worst <= 1, f"a code differs by {worst} levels"
    assert same >= frac, f"only {same:.6f} of codes identical"
    return same


def gpu_layer(X: np.ndarray | None, W: np.ndarray, *, bits: int, group: int, block: int = 128,
              damp: float = 0.01, act_order: bool = False, H32: np.ndarray | None = None,
              sym: bool = False, static_groups: bool = False) -> dict:
    """Run the CUDA path: H from X on the GPU (or a given fp32 H), then the solve."""
    import torch

    import post_weight_quantization_19_b200 as g

    dev = torch.device("cuda")
    r, d = W.shape
    Wd = torch.from_numpy(np.ascontiguousarray(W, dtype=np.float32)).to(dev)
    if H32 is None:
        Xd = torch.from_numpy(np.ascontiguousarray(X)).to(dev)
        H = torch.zeros((d, d), dtype=torch.float32, device=dev)
        g.gptq_hessian_accumulate(Xd, H)
    else:
        H = torch.from_numpy(np.ascontiguousarray(H32, dtype=np.float32)).to(dev)
    H_used = H.cpu().numpy().copy()
    W_hat = torch.empty_like(Wd)
    codes = torch.empty((r, d), dtype=torch.uint8, device=dev)
    g_idx = torch.empty((d,), dtype=torch.int32, device=dev)
    res = g.gptq_quantize_layer(Wd, H, bits=bits, group=group, block=block, damp=damp,
                                act_order=act_order, sym=sym, static_groups=static_groups,
                                W_hat=W_hat, codes=codes, g_idx=g_idx)
    torch.cuda.synchronize()
    return {
        "H": H_used,
        "codes": codes.cpu().numpy(),
        "W_hat": W_hat.cpu().numpy(),
        "g_idx": g_idx.cpu().numpy(),
        "qweight": res["qweight"].cpu().numpy(),
        "scales": res["scales"].cpu().numpy(),
        "zeros": res["zeros"].cpu().numpy(),
        "loss": res["loss"],
    }


def check_against_oracle(got: dict, ref: dict, W: np.ndarray, *, bits: int, group: int) -> dict:
    """Codes, loss, dequantisation consistency, packing and g_idx checks."""
    import oracle

    stats = {"code_match": assert_codes_close(got["codes"], ref["codes"])}
    rel = abs(got["loss"] - ref["loss"]) / max(abs(ref["loss"]), 1e-300)
    stats["loss_rel"] = rel
    assert rel <= LOSS_REL, f"loss {got['loss']} vs oracle {ref['loss']} ({rel:.2e})"
    # W^ = s (q - z) on the GPU's own parameters (same fp32 expression: exact)
    d = W.shape[1]
    g = d if group == -1 else group
    gi = got["g_idx"].astype(np.int64) if group != -1 else np.zeros(d, dtype=np.int64)
    s = got["scales"][:, gi].astype(np.float32)
    z = got["zeros"][:, gi].astype(np.float32)
    np.testing.assert_array_equal(got["W_hat"], s * (got["codes"].astype(np.float32) - z))
    np.testing.assert_array_equal(got["qweight"], oracle.pack_rows(got["codes"], bits))
    np.testing.assert_array_equal(got["g_idx"], ref["g_idx"] if group != -1 else 0)
    assert got["codes"].max() <= (1 << bits) - 1
    assert got["zeros"].min() >= 0 and got["zeros"].max() <= (1 << bits) - 1
    # scales: where every earlier code of the row agrees, the group started from
    # the same state up to rounding, so the scale agrees to fp32 accuracy.
    G = got["scales"].shape[1]
    order = np.argsort(ref["g_idx"], kind="stable") if group != -1 else np.arange(d)
    mism = got["codes"][:, order] != ref["codes"][:, order]
    first_bad = np.where(mism.any(axis=1), mism.argmax(axis=1), d)
    starts = np.arange(G) * g
    ok = starts[None, :] <= first_bad[:, None]
    sg, sr = got["scales"][ok], ref["scales"][ok]
    assert np.all(np.abs(sg - sr) <= 1e-4 * np.abs(sr)), "scale mismatch on agreeing groups"
    zmatch = float(np.mean(got["zeros"][ok] == ref["zeros"][ok]))
    assert zmatch >= CODE_MATCH
    stats["zero_match"] = zmatch
    return stats


def reconcile_at_ties(got_codes: np.ndarray, W: np.ndarray, ref: dict, *, bits: int, group: int,
                      block: int, max_ties: int = 16, delta: float = 1e-3) -> dict:
    """Rows whose codes differ from the oracle's: the first difference must sit at
    a rounding tie on the oracle's side (its value within ``delta`` code steps of a
    half-integer), where either choice is correct; the row is then re-swept by the
    oracle with the GPU's choice there, and so on until the row matches.

    After one tie is decided differently, the compensation of every later column
    of the row differs, so the rest of the row is another correct result, not a
    rounding error.  ``ref`` is ``oracle.gptq_quantize_layer``'s result for the
    rows of ``W`` (with "U", "perm", "scales", "zeros", "E", "What").  Returns
    the number of rows followed and of ties followed."""
    import oracle

    perm = np.asarray(ref["perm"])
    inv = np.argsort(perm)
    U = ref["U"]
    d = W.shape[1]
    gi = np.zeros(d, dtype=np.int64) if group == -1 else np.arange(d) // group
    rows_followed, ties = 0, 0
    for i in range(W.shape[0]):
        if np.array_equal(got_codes[i], ref["codes"][i]):
            continue
        rows_followed += 1
        want = np.asarray(got_codes[i], dtype=np.int64)[perm]    # sweep order
        forced = {}
        Wi = np.asarray(W[i:i + 1], dtype=np.float64)[:, perm]
        codes_p = ref["codes"][i][perm]
        E = ref["E"][i:i + 1]
        What_p = ref["What"][i:i + 1][:, perm]
        sc, zr = ref["scales"][i:i + 1], ref["zeros"][i:i + 1]
        for _ in range(max_ties + 1):
            diff = np.where(codes_p != want)[0]
            if diff.size == 0:
                break
            j = int(diff[0])
            t = (What_p[0, j] + E[0, j] * U[j, j]) / sc[0, gi[j]] + zr[0, gi[j]]
            off = abs(t - np.floor(t) - 0.5)
            assert off <= delta, f"row {i}: column {perm[j]} differs {off:.2e} code steps from a tie"
            assert abs(int(want[j]) - int(codes_p[j])) == 1, f"row {i}: not a neighbouring code"
            forced[j] = np.array([want[j]])
            ties += 1
            c, sc, zr, What_p, E = oracle.gptq_sweep(Wi, U, bits, group, block, forced=forced)
            codes_p = c[0]
        else:
            raise AssertionError(f"row {i}: more than {max_ties} ties to follow")
        assert np.array_equal(codes_p, want), f"row {i} does not reconcile"
    return {"rows": rows_followed, "ties": ties}
