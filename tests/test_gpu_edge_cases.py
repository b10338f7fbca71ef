"""Edge cases of the quantiser and the factorisation on the GPU, against the
float64 oracle (needs a B200).

The quantiser of "GPTQ：一键量化大模型压缩" §分组方案 with the readings of the
oracle: the range widened to include 0, s = 1 for an empty range, rint half to
even.  Both sides get the same fp32 Hessian.
"""

import numpy as np
import pytest

import oracle
from parity_util import assert_codes_close, check_against_oracle, gpu_layer
from synth import make_problem

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import post_weight_quantization_19_b200 as g
    yield g
    assert g.gptq_check_device_status() == 0


def _H32(d, seed, n=None):
    X, _ = make_problem(1, d, n or 8 * d, seed=seed)
    return oracle.hessian(X).astype(np.float32)


@pytest.mark.parametrize("group", [-1, 128])
def test_zero_rows_and_a_zero_group_take_the_flat_range_branch(group):
    # Rows 0-3 are all zero; rows 4-7 have an all-zero first group (nothing has
    # been compensated into it when the sweep reaches column 0).  Their range is
    # empty, so s = 1 and z = 0 and every code there is 0; the rest of the layer
    # still matches the oracle.
    r, d = 24, 512
    H32 = _H32(d, 301)
    W = (0.02 * np.random.default_rng(302).standard_normal((r, d))).astype(np.float32)
    W[:4] = 0.0
    W[4:8, :128] = 0.0
    got = gpu_layer(None, W, bits=4, group=group, H32=H32)
    ref = oracle.gptq_quantize_layer(W, H32.astype(np.float64), bits=4, group=group)
    check_against_oracle(got, ref, W, bits=4, group=group)
    np.testing.assert_array_equal(got["codes"][:4], 0)
    assert np.all(got["scales"][:4] == 1.0) and np.all(got["zeros"][:4] == 0)
    np.testing.assert_array_equal(got["W_hat"][:4], 0.0)
    if group == 128:
        np.testing.assert_array_equal(got["codes"][4:8, :128], 0)
        assert np.all(got["scales"][4:8, 0] == 1.0) and np.all(got["zeros"][4:8, 0] == 0)
    np.testing.assert_array_equal(got["codes"], ref["codes"])


@pytest.mark.parametrize("bits,group", [(4, -1), (4, 128), (3, 64), (2, 32), (8, 128)])
def test_weights_on_a_power_of_two_grid_are_reproduced_with_zero_loss(bits, group):
    # W = s (q - z) with s a power of two and every group holding both code 0
    # and code 2^b - 1: the min-max parameters give back s and z exactly, every
    # column rounds without error, nothing is compensated, and the loss is 0
    # exactly on both sides.
    r, d = 40, 256
    rng = np.random.default_rng(bits * 1000 + max(group, 0))
    maxq = (1 << bits) - 1
    g = d if group == -1 else group
    q = rng.integers(0, maxq + 1, size=(r, d))
    q[:, 0::g] = 0
    q[:, 1::g] = maxq
    z = rng.integers(1, maxq, size=(r, d // g)) if maxq > 1 else np.ones((r, d // g), int)
    s = 2.0 ** rng.integers(-9, -5, size=(r, d // g))
    gi = np.arange(d) // g
    W = (s[:, gi] * (q - z[:, gi])).astype(np.float32)
    H32 = _H32(d, 303)
    got = gpu_layer(None, W, bits=bits, group=group, H32=H32)
    ref = oracle.gptq_quantize_layer(W, H32.astype(np.float64), bits=bits, group=group)
    np.testing.assert_array_equal(ref["codes"], q)
    np.testing.assert_array_equal(got["codes"], q)
    np.testing.assert_array_equal(got["W_hat"], W)
    np.testing.assert_array_equal(got["scales"], s.astype(np.float32))
    np.testing.assert_array_equal(got["zeros"], z)
    assert ref["loss"] == 0.0 and got["loss"] == 0.0


@pytest.mark.parametrize("group", [-1, 128])
def test_rows_above_zero_widen_the_range_to_zero(group):
    # Every weight positive: the range is widened to [0, max], so the zero point
    # of each row's first group is 0.
    r, d = 32, 384
    rng = np.random.default_rng(304)
    W = (0.005 + np.abs(0.02 * rng.standard_normal((r, d)))).astype(np.float32)
    H32 = _H32(d, 305)
    got = gpu_layer(None, W, bits=4, group=group, H32=H32)
    ref = oracle.gptq_quantize_layer(W, H32.astype(np.float64), bits=4, group=group)
    check_against_oracle(got, ref, W, bits=4, group=group)
    assert np.all(got["zeros"][:, 0] == 0) and np.all(ref["zeros"][:, 0] == 0)


def test_code_mismatches_sit_on_rounding_ties():
    # The GPU decides each code in fp32 (w * (1/s), rintf), the oracle in
    # float64.  Where they differ, the value being rounded must have been within
    # a hair of a half-integer step on the oracle's side (after the first
    # mismatch a row's later columns see different compensation, so only each
    # row's first mismatch is tested).  Column 0 of every row is put exactly on
    # a tie that both precisions see: columns 1 and 2 pin the first group's
    # range to [-z s, (7 - z) s] with s a power of two (the rest of the group
    # lies inside it), so s and z come out exactly, and w_0 = s (k + 1/2 - z)
    # is exact in fp32; both sides must round it to even.
    r, d, bits, group = 256, 1024, 3, 128
    X, W = make_problem(r, d, 8 * d, seed=306)
    H32 = oracle.hessian(X).astype(np.float32)
    rng = np.random.default_rng(309)
    s0 = np.float32(2.0 ** -5)
    z0 = rng.integers(2, 6, size=r).astype(np.float32)
    k = rng.integers(0, 7, size=r).astype(np.float32)
    lo, hi = -z0 * s0, (7 - z0) * s0
    W[:, 3:group] = np.clip(W[:, 3:group], 0.9 * lo[:, None], 0.9 * hi[:, None])
    W[:, 1], W[:, 2] = lo, hi
    W[:, 0] = s0 * (k + np.float32(0.5) - z0)
    got = gpu_layer(None, W, bits=bits, group=group, H32=H32)
    ref = oracle.gptq_quantize_layer(W, H32.astype(np.float64), bits=bits, group=group)
    np.testing.assert_array_equal(ref["scales"][:, 0], s0)
    np.testing.assert_array_equal(got["scales"][:, 0], s0)
    # rint(k - z + 1/2) is the even one of k - z and k - z + 1
    np.testing.assert_array_equal(ref["codes"][:, 0], np.where((k - z0) % 2 == 0, k, k + 1))
    np.testing.assert_array_equal(got["codes"][:, 0], ref["codes"][:, 0])
    assert_codes_close(got["codes"], ref["codes"])
    # the value rounded at column j, in code units: t = w_j / s + z, with
    # w_j = w^_j + e_j U_jj (e_j = (w_j - w^_j) / U_jj)
    U = ref["U"]
    gi = np.arange(d) // group
    w_pre = ref["What"] + ref["E"] * np.diag(U)[None, :]
    t = w_pre / ref["scales"][:, gi] + ref["zeros"][:, gi]
    off_tie = np.abs(t - np.floor(t) - 0.5)
    exact_ties = int(np.sum(off_tie == 0.0))
    mism = got["codes"] != ref["codes"]
    rows = np.where(mism.any(axis=1))[0]
    first = mism[rows].argmax(axis=1)
    worst = float(off_tie[rows, first].max()) if rows.size else 0.0
    print(f"exact ties {exact_ties}, rows with a mismatch {rows.size}/{r}, "
          f"largest distance of a first mismatch from a tie {worst:.2e} (code units)")
    assert exact_ties >= r   # the planted first-column ties (at least)
    assert worst <= 1e-3, worst


@pytest.mark.parametrize("d,act", [(1056, False), (6272, False), (6432, False), (6432, True)])
def test_factor_matches_oracle_U(d, act):
    # The factor alone: U from gptq_factor against the oracle's upper Cholesky
    # factor of H_d^-1.  1056: one block of 128-column steps with a ragged leaf;
    # 6272 and 6432: outer 1024-column blocks, the last one ragged (288 columns
    # in 6432).  fp32 with 3xTF32 products against float64: the bound is a
    # structural check (a missing or doubled update moves U by O(1)).
    import post_weight_quantization_19_b200 as g
    H32 = _H32(d, 307 + d, n=4 * d)
    fac = g.gptq_factor(torch.from_numpy(H32.copy()).cuda(), act_order=act)
    torch.cuda.synchronize()
    U = np.triu(fac["U"].cpu().numpy().astype(np.float64))
    H = H32.astype(np.float64)
    Hd, lam = oracle.dampen(H, 0.01)
    perm = oracle.act_order_perm(H) if act else np.arange(d)
    if act:
        np.testing.assert_array_equal(fac["perm"].cpu().numpy(), perm)
    Uref = oracle.inverse_upper_cholesky(Hd[np.ix_(perm, perm)])
    err = np.linalg.norm(U - Uref) / np.linalg.norm(Uref)
    print(f"d={d} act={act}: U rel Frobenius error {err:.2e}")
    assert err <= 1e-3, err
    assert abs(float(fac["lambda"][0]) - lam) <= 1e-6 * lam


def test_a_wait_that_runs_out_reports_timeout_and_the_device_stays_usable(lib):
    # A GEMM whose operand loads stop early: its bounded waits run out, the
    # status word says GPTQ_ERR_TIMEOUT (5), and the next solve on the same
    # device -- which allocates tensor memory again -- is still correct.
    import post_weight_quantization_19_b200 as g
    assert g.gptq_check_device_status() == 0
    buf = torch.zeros(81920, dtype=torch.float32, device="cuda")
    stream = torch.cuda.current_stream().cuda_stream
    assert lib.gptq_selftest_timeout(buf.data_ptr(), stream) == 0
    assert g.gptq_check_device_status() == 5
    assert g.gptq_check_device_status() == 0
    r, d = 48, 384
    X, W = make_problem(r, d, 3000, seed=308)
    H32 = oracle.hessian(X).astype(np.float32)
    got = gpu_layer(None, W, bits=4, group=128, H32=H32)
    ref = oracle.gptq_quantize_layer(W, H32.astype(np.float64), bits=4, group=128)
    check_against_oracle(got, ref, W, bits=4, group=128)
