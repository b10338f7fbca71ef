"""Full-size layers on the GPU, checked against the float64 oracle (needs a B200).

The GPU runs the whole layer in the launch configuration the benchmark times.
Where the float64 Hessian fits on the host, the oracle computes H and U in
full (rows are independent once U is fixed) and sweeps a seeded sample of rows.
The OPT-175B fc2 layer (d = 49152: a float64 H alone is 19 GB and the oracle
needs minutes of host time for it) is compared with the oracle's result for 16
seeded rows, stored by tests/golden/make_opt175b_fc2_rows.py from the same
seeded inputs (checked by a fingerprint), plus sampled rows of H and the
dequantisation and packing identities.
"""

import numpy as np
import pytest

import oracle
from parity_util import (CODE_MATCH, H_REL_FRO, LOSS_REL, assert_codes_close, gpu_layer,
                         reconcile_at_ties, rel_fro)
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
    del X
    err = rel_fro(got["H"], H)
    assert err <= H_REL_FRO, err
    rows = np.sort(np.random.default_rng(wl.seed).choice(wl.r, nrows, replace=False))
    perm = None
    if wl.act_order:
        # The order is a stable descending sort of diag(H).  The GPU sorts its
        # fp32 H, whose entries differ from the float64 ones by up to the H
        # tolerance, so columns whose diagonals agree to within it may come in
        # either order (both are valid).  Check that the GPU's order is
        # descending in the float64 diagonal up to that tolerance, then compare
        # with the oracle run in that order.
        perm = np.argsort(-np.diag(got["H"]).astype(np.float64), kind="stable")
        dg = np.diag(H)[perm]
        assert np.all(dg[1:] <= dg[:-1] * (1 + H_REL_FRO))
        swapped = int(np.sum(perm != oracle.act_order_perm(H)))
        print(f"{name}: {swapped} columns ordered differently from the float64 order "
              f"(near-equal diagonals)")
    ref = oracle.gptq_quantize_layer(W, H, bits=wl.bits, group=wl.group, block=wl.block,
                                     damp=wl.damp, act_order=wl.act_order, rows=rows, perm=perm)
    gc = got["codes"][rows].astype(np.int64)
    diff = gc - ref["codes"]
    match = float(np.mean(diff == 0))
    if np.abs(diff).max() > 1 or match < CODE_MATCH:
        # a rounding tie decided the other way sends the rest of its row down a
        # different correct path: follow the GPU's choice at each tie
        rec = reconcile_at_ties(gc, W[rows], ref, bits=wl.bits, group=wl.group, block=wl.block)
        print(f"{name}: {match:.5f} identical; {rec['rows']} rows reconcile through "
              f"{rec['ties']} rounding ties")
    gl = oracle.layer_loss(W[rows], got["W_hat"][rows], H)
    assert abs(gl - ref["loss"]) <= LOSS_REL * ref["loss"], (gl, ref["loss"])
    total = oracle.layer_loss(W, got["W_hat"], H)
    assert abs(got["loss"] - total) <= LOSS_REL * total, (got["loss"], total)
    np.testing.assert_array_equal(got["qweight"][rows],
                                  oracle.pack_rows(got["codes"][rows], wl.bits))
    if wl.act_order:
        np.testing.assert_array_equal(got["g_idx"], ref["g_idx"])
    print(f"{name}: H rel {err:.2e}, codes {match:.6f}, sampled loss rel "
          f"{abs(gl - ref['loss']) / ref['loss']:.2e}")


def test_llama7b_q_proj_4096x4096():
    _check_sampled("llama7b_q_proj_4096x4096")


@pytest.mark.parametrize("name", ["llama7b_up_proj_11008x4096",
                                  "llama7b_up_proj_11008x4096_actorder"])
def test_llama7b_up_proj(name):
    _check_sampled(name)


@pytest.mark.parametrize("name", ["llama7b_down_proj_4096x11008",
                                  "llama7b_down_proj_4096x11008_actorder"])
def test_llama7b_down_proj(name):
    _check_sampled(name, nrows=32)


@pytest.mark.parametrize("name", ["w3_8192x8192_perrow", "w3_8192x8192_g128"])
def test_w3_8192(name):
    _check_sampled(name, nrows=32)


def _row_losses(W, What, X, chunk=4096):
    # ||(w - w^) X^T||^2 per row, summed over token chunks in float64
    D = np.asarray(W, np.float64) - np.asarray(What, np.float64)
    out = np.zeros(D.shape[0])
    for t in range(0, X.shape[0], chunk):
        Y = D @ X[t:t + chunk].astype(np.float64).T
        out += np.sum(Y * Y, axis=1)
    return out


def test_opt175b_fc2_matches_stored_oracle_rows():
    # The OPT-175B fc2 layer (d = 49152) in the launch configuration the bench
    # times, against the float64 oracle's result for 16 seeded rows, written by
    # tests/golden/make_opt175b_fc2_rows.py from the same seeded inputs (the
    # oracle's float64 H alone is 19 GB and its factorisation takes minutes).
    import os

    import post_weight_quantization_19_b200 as g
    golden = os.path.join(os.path.dirname(__file__), "golden", "opt175b_fc2_rows.npz")
    if not os.path.exists(golden):
        pytest.skip("stored oracle rows not written yet")
    ref = np.load(golden)
    wl = workload("opt175b_fc2_12288x49152")
    assert list(ref["config"]) == [wl.r, wl.d, wl.n, wl.bits, wl.group, wl.block, wl.seed]
    X, W = workload_inputs(wl)
    rows = ref["rows"]
    import importlib.util
    spec = importlib.util.spec_from_file_location(
        "make_rows", os.path.join(os.path.dirname(golden), "make_opt175b_fc2_rows.py"))
    mk = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mk)
    np.testing.assert_array_equal(mk.fingerprint(X, W, rows), ref["fingerprint"])
    r, d = W.shape
    dev = torch.device("cuda")
    Xd = torch.from_numpy(X).to(dev)
    H = torch.zeros((d, d), dtype=torch.float32, device=dev)
    g.gptq_hessian_accumulate(Xd, H)
    del Xd
    hrows = np.array([0, 777, d // 2, d - 1])
    Hs = H[torch.from_numpy(hrows).to(dev)].cpu().numpy()
    assert rel_fro(Hs, oracle.hessian_rows(X, hrows)) <= H_REL_FRO
    Wd = torch.from_numpy(W).to(dev)
    W_hat = torch.empty_like(Wd)
    codes = torch.empty((r, d), dtype=torch.uint8, device=dev)
    g_idx = torch.empty((d,), dtype=torch.int32, device=dev)
    res = g.gptq_quantize_layer(Wd, H, bits=wl.bits, group=wl.group, block=wl.block,
                                damp=wl.damp, W_hat=W_hat, codes=codes, g_idx=g_idx)
    torch.cuda.synchronize()
    del H
    rt = torch.from_numpy(rows).to(dev)
    c = codes[rt].cpu().numpy()
    wh = W_hat[rt].cpu().numpy()
    sc = res["scales"][rt].cpu().numpy()
    zr = res["zeros"][rt].cpu().numpy()
    q = res["qweight"][rt].cpu().numpy()
    gi = np.arange(d) // wl.group
    np.testing.assert_array_equal(g_idx.cpu().numpy(), gi)
    match = assert_codes_close(c, ref["codes"])
    np.testing.assert_array_equal(wh, sc[:, gi] * (c.astype(np.float32) - zr[:, gi].astype(np.float32)))
    np.testing.assert_array_equal(q, oracle.pack_rows(c, wl.bits))
    # scales and zeros where every earlier code of the row agrees
    mism = c != ref["codes"]
    first_bad = np.where(mism.any(axis=1), mism.argmax(axis=1), d)
    ok = (np.arange(d // wl.group) * wl.group)[None, :] <= first_bad[:, None]
    assert np.all(np.abs(sc[ok] - ref["scales"][ok]) <= 1e-4 * np.abs(ref["scales"][ok]))
    assert float(np.mean(zr[ok] == ref["zeros"][ok])) >= 0.999
    # the objective of each sampled row, from X, against the oracle's
    lg = _row_losses(W[rows], wh, X)
    rel = np.abs(lg - ref["row_loss"]) / ref["row_loss"]
    assert rel.max() <= LOSS_REL, rel
    assert abs(lg.sum() - ref["row_loss"].sum()) <= LOSS_REL * ref["row_loss"].sum()
    assert np.isfinite(res["loss"]) and res["loss"] > 0
    print(f"opt175b fc2: codes {match:.6f} identical on {len(rows)} rows, row objective "
          f"within {rel.max():.2e} of the oracle")
