"""One layer solved across the ranks of a process group (one process per GPU).

Token-sharded Hessian: H is a sum over calibration tokens ("GPTQ：一键量化大模型
压缩", §二阶信息), so rank i accumulates H_i = 2 X_i^T X_i over its own tokens with
``gptq_hessian_accumulate`` and one reduction (sum) gives H = 2 X^T X.
Row-sharded solve: every row of W is quantised in the same column order with the
same inverse-Hessian factor (GPTQ reading card, §方法适配), so once the factor is
known the rows are independent problems.  By default the root rank factors H
once (``gptq_factor``) and broadcasts U, the act-order permutation and the
damping; rank i then sweeps the rows ``row_shard(r, i, N)`` with
``gptq_quantize_with_factor``.  (``factor_once=False`` all-reduces H instead and
lets every rank factor its own copy with ``gptq_quantize_layer``.)  The packed
rows, scales and zeros are then all-gathered, so every rank returns the whole
layer, and the per-rank losses (sums over rows) are all-reduced.

The exchange is a reduce and a broadcast of d^2 fp32 words, the gather of the
packed layer and two scalars, issued through ``torch.distributed`` (NCCL on
GPUs); every rank takes the same collective steps, the error paths included.
"""

from __future__ import annotations

import torch

from .gptq import (GPTQError, gptq_factor, gptq_hessian_accumulate, gptq_quantize_layer,
                   gptq_quantize_with_factor)


def shard_range(count: int, rank: int, world: int) -> tuple[int, int]:
    """Contiguous slice [a, b) of ``count`` items for ``rank`` of ``world``.

    Balanced: the first ``count % world`` ranks get one item more than the
    others, so every rank has at least one item whenever count >= world.
    """
    if world < 1 or not 0 <= rank < world or count < 0:
        raise ValueError("need 0 <= rank < world and count >= 0")
    base, extra = divmod(count, world)
    a = rank * base + min(rank, extra)
    return a, a + base + (1 if rank < extra else 0)


def token_shard(X: torch.Tensor, rank: int, world: int) -> torch.Tensor:
    """This rank's calibration tokens (rows of X), as a contiguous view."""
    a, b = shard_range(X.shape[0], rank, world)
    return X[a:b]


def row_shard(r: int, rank: int, world: int) -> tuple[int, int]:
    """The output rows of W that ``rank`` solves."""
    return shard_range(r, rank, world)


def _gather_rows(local: torch.Tensor, r: int, world: int, dist, group) -> torch.Tensor:
    # all_gather needs equal shapes: every rank pads its rows to ceil(r / world),
    # and the padding is dropped rank by rank.
    per = -(-r // world)
    buf = local.new_zeros((per,) + tuple(local.shape[1:]))
    buf[:local.shape[0]] = local
    parts = [torch.empty_like(buf) for _ in range(world)]
    dist.all_gather(parts, buf, group=group)
    sizes = [b - a for a, b in (shard_range(r, k, world) for k in range(world))]
    return torch.cat([p[:n] for p, n in zip(parts, sizes)])


def _factor_on_root(H: torch.Tensor, rank: int, root: int, damp: float, act_order: bool,
                    dist, group) -> dict:
    # The root factors; its status goes out first, so that a failed factor ends
    # every rank with the same error instead of leaving them in the broadcast.
    d = H.shape[0]
    fac, err = None, None
    if rank == root:
        try:
            fac = gptq_factor(H, damp=damp, act_order=act_order)
        except GPTQError as e:
            err = e
    status = torch.tensor([0 if err is None else (err.status or 1)], dtype=torch.int32,
                          device=H.device)
    dist.broadcast(status, src=root, group=group)
    if int(status.item()) != 0:
        raise err if err is not None else GPTQError(int(status.item()), "gptq_factor on the root rank")
    if fac is None:
        fac = {"U": H,
               "perm": torch.empty(d, dtype=torch.int32, device=H.device) if act_order else None,
               "lambda": torch.empty(1, dtype=torch.float32, device=H.device)}
    dist.broadcast(fac["U"], src=root, group=group)
    if act_order:
        dist.broadcast(fac["perm"], src=root, group=group)
    dist.broadcast(fac["lambda"], src=root, group=group)
    return fac


def solve_layer_sharded(X_local: torch.Tensor, W: torch.Tensor, *, bits: int, group: int,
                        block: int = 128, damp: float = 0.01, act_order: bool = False,
                        factor_once: bool = True, root: int = 0, process_group=None) -> dict:
    """GPTQ solve of one layer W [r, d] spread over the ranks of ``process_group``.

    ``X_local`` holds this rank's calibration tokens (fp16 [n_i, d]); every rank
    passes the whole W (fp32).  Every rank must call this with the same W,
    shapes and options.  Returns the whole layer on every rank: ``qweight``,
    ``scales``, ``zeros``, ``g_idx`` (act-order only) and ``loss``.
    """
    import torch.distributed as dist

    world = dist.get_world_size(process_group)
    rank = dist.get_rank(process_group)
    r, d = W.shape
    if r < world:
        raise ValueError("need at least one row of W per rank")
    if X_local.shape[1] != d:
        raise ValueError("X_local must have d columns")
    H = torch.zeros((d, d), dtype=torch.float32, device=W.device)
    if X_local.shape[0] > 0:
        gptq_hessian_accumulate(X_local, H)
    a, b = row_shard(r, rank, world)
    g_idx = torch.empty(d, dtype=torch.int32, device=W.device) if act_order else None
    if factor_once:
        dist.reduce(H, dst=root, group=process_group)
        fac = _factor_on_root(H, rank, root, damp, act_order, dist, process_group)
        res = gptq_quantize_with_factor(W[a:b].contiguous(), fac, bits=bits, group=group,
                                        block=block, g_idx=g_idx)
    else:
        dist.all_reduce(H, group=process_group)
        res = gptq_quantize_layer(W[a:b].contiguous(), H, bits=bits, group=group, block=block,
                                  damp=damp, act_order=act_order, g_idx=g_idx)
    loss = torch.tensor([res["loss"]], dtype=torch.float64, device=W.device)
    dist.all_reduce(loss, group=process_group)
    out = {key: _gather_rows(res[key], r, world, dist, process_group)
           for key in ("qweight", "scales", "zeros")}
    out["loss"] = float(loss.item())
    if act_order:
        out["g_idx"] = res["g_idx"]
    return out
