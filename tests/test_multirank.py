"""One layer solved across ranks, on CPU: gloo ranks in separate processes.

The token-sharded Hessian with one all-reduce, the row-sharded solve and the
gathered outputs (``post_weight_quantization_19_b200.sharded``) run here with
the two GPU entry points played by the float64 oracle.
"""

import os
import socket
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


# ------------------------------------------------- one layer over two ranks ---

def test_shard_ranges_cover_every_item_once():
    from post_weight_quantization_19_b200.sharded import shard_range
    for count in (0, 1, 5, 11, 64, 4097):
        for world in (1, 2, 3, 8):
            spans = [shard_range(count, k, world) for k in range(world)]
            covered = [i for a, b in spans for i in range(a, b)]
            assert covered == list(range(count))
            sizes = [b - a for a, b in spans]
            assert max(sizes) - min(sizes) <= 1
            if count >= world:
                assert min(sizes) >= 1
    with pytest.raises(ValueError):
        shard_range(4, 2, 2)


def _integer_layer(rows=11):
    # Small integer activations: every partial Hessian and their all-reduced sum
    # are exact integers in fp32, so the sharded H equals the single-process H
    # bit for bit and so must every code.
    import numpy as np
    import torch
    rng = np.random.default_rng(5)
    X = rng.integers(-8, 9, size=(130, 64)).astype(np.float16)
    W = (0.02 * rng.standard_normal((rows, 64))).astype(np.float32)
    return torch.from_numpy(X), torch.from_numpy(W)


def _sharded_worker(rank, world, port, q, act_order, factor_once, rows=11):
    import numpy as np
    import torch
    import torch.distributed as dist

    import oracle
    from post_weight_quantization_19_b200 import sharded

    # The GPU entry points, played on the CPU by the oracle (same arguments and
    # outputs as the binding's; H exact in fp32, U and lambda rounded to fp32 as
    # the device keeps them).
    def hessian(X, H):
        H += torch.from_numpy(oracle.hessian(X.numpy())).to(H.dtype)

    def quantize_layer(W, H, *, bits, group, block, damp, act_order, g_idx=None):
        o = oracle.gptq_quantize_layer(W.numpy(), H.double().numpy(), bits=bits, group=group,
                                       block=block, damp=damp, act_order=act_order)
        if g_idx is not None:
            g_idx.copy_(torch.from_numpy(o["g_idx"]))
        return {"qweight": torch.from_numpy(oracle.pack_rows(o["codes"], bits)),
                "scales": torch.from_numpy(o["scales"]).float(),
                "zeros": torch.from_numpy(o["zeros"]).int(), "loss": o["loss"],
                "g_idx": g_idx}

    def factor(H, *, damp, act_order):
        U, perm, lam = _oracle_factor(H.double().numpy(), damp, act_order)
        H.copy_(torch.from_numpy(U))
        return {"U": H, "perm": torch.from_numpy(perm).int() if act_order else None,
                "lambda": torch.tensor([lam], dtype=torch.float32)}

    def quantize_with_factor(W, fac, *, bits, group, block, g_idx=None):
        d = W.shape[1]
        perm = fac["perm"].numpy().astype(np.int64) if fac["perm"] is not None else np.arange(d)
        o = _oracle_sweep(W.numpy(), fac["U"].double().numpy(), perm,
                          float(fac["lambda"][0]), bits, group, block)
        if g_idx is not None:
            g_idx.copy_(torch.from_numpy(o["g_idx"]))
        return {"qweight": torch.from_numpy(oracle.pack_rows(o["codes"], bits)),
                "scales": torch.from_numpy(o["scales"]).float(),
                "zeros": torch.from_numpy(o["zeros"]).int(), "loss": o["loss"], "g_idx": g_idx}

    sharded.gptq_hessian_accumulate = hessian
    sharded.gptq_quantize_layer = quantize_layer
    sharded.gptq_factor = factor
    sharded.gptq_quantize_with_factor = quantize_with_factor
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world)
    try:
        X, W = _integer_layer(rows)
        res = sharded.solve_layer_sharded(sharded.token_shard(X, rank, world), W, bits=4,
                                          group=16, act_order=act_order,
                                          factor_once=factor_once)
        q.put((rank, {k: v.numpy() if torch.is_tensor(v) else v for k, v in res.items()}))
    finally:
        dist.destroy_process_group()


def _oracle_factor(H, damp, act_order):
    # damping, order and U as the device keeps them (fp32)
    import numpy as np

    import oracle
    Hd, lam = oracle.dampen(H, damp)
    perm = oracle.act_order_perm(H) if act_order else np.arange(H.shape[0])
    U = oracle.inverse_upper_cholesky(Hd[np.ix_(perm, perm)]).astype(np.float32)
    return U, perm, np.float32(lam)


def _oracle_sweep(W, U, perm, lam, bits, group, block):
    # the sweep half from a given factor; the loss as the device forms it
    import numpy as np

    import oracle
    W = W.astype(np.float64)
    codes_p, scales, zeros, What_p, E = oracle.gptq_sweep(W[:, perm], U, bits, group, block)
    inv = np.argsort(perm)
    What = What_p[:, inv]
    D = W - What
    return {"codes": codes_p[:, inv], "scales": scales, "zeros": zeros.astype(np.int64),
            "g_idx": inv // group, "loss": 0.5 * float(np.sum(E * E)) - 0.5 * lam * float(np.sum(D * D))}


@pytest.mark.parametrize("world,rows", [(2, 11), (4, 9)])
@pytest.mark.parametrize("factor_once", [True, False])
@pytest.mark.parametrize("act_order", [False, True])
def test_ranks_solve_one_layer_like_one_process(act_order, factor_once, world, rows):
    # world 4 with 9 rows: shards of 3, 2, 2, 2 rows -- every rank solves rows,
    # and every rank returns the whole layer (g_idx included under act-order)
    import numpy as np

    import oracle
    mp = pytest.importorskip("torch.multiprocessing")
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_sharded_worker,
                         args=(r, world, port, q, act_order, factor_once, rows))
             for r in range(world)]
    for p in procs:
        p.start()
    results = dict(q.get(timeout=180) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    X, W = _integer_layer(rows)
    H = oracle.hessian(X.numpy())
    if factor_once:
        U, perm, lam = _oracle_factor(H, 0.01, act_order)
        ref = _oracle_sweep(W.numpy(), U.astype(np.float64), perm, float(lam), 4, 16, 128)
    else:
        ref = oracle.gptq_quantize_layer(W.numpy(), H, bits=4, group=16, act_order=act_order)
    for rank in range(world):
        got = results[rank]
        np.testing.assert_array_equal(got["qweight"], oracle.pack_rows(ref["codes"], 4))
        np.testing.assert_array_equal(got["scales"], ref["scales"].astype(np.float32))
        np.testing.assert_array_equal(got["zeros"], ref["zeros"])
        assert got["loss"] == pytest.approx(ref["loss"], rel=1e-12)
        if act_order:
            np.testing.assert_array_equal(got["g_idx"], ref["g_idx"])


def _failing_factor_worker(rank, world, port, q):
    import torch
    import torch.distributed as dist

    import oracle
    from post_weight_quantization_19_b200 import sharded
    from post_weight_quantization_19_b200.gptq import GPTQError

    def hessian(X, H):
        H += torch.from_numpy(oracle.hessian(X.numpy())).to(H.dtype)

    def factor(H, *, damp, act_order):
        raise GPTQError(2, "gptq_factor")   # GPTQ_ERR_NOT_PD, as the root would report it

    sharded.gptq_hessian_accumulate = hessian
    sharded.gptq_factor = factor
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world)
    try:
        X, W = _integer_layer()
        try:
            sharded.solve_layer_sharded(sharded.token_shard(X, rank, world), W, bits=4, group=16)
            q.put((rank, None))
        except GPTQError as e:
            q.put((rank, e.status))
    finally:
        dist.destroy_process_group()


def test_a_failed_factor_ends_every_rank_with_its_error():
    # The root's status is broadcast before U, so the other rank raises the same
    # error instead of waiting in the broadcast.
    mp = pytest.importorskip("torch.multiprocessing")
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_failing_factor_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    results = dict(q.get(timeout=180) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert results == {0: 2, 1: 2}
