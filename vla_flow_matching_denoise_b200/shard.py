"""Request sharding of a batch over the ranks of one node.

Requests of a batch are independent (each has its own prefix K/V and chunk;
all share the weights and the time grid), so a batch of B requests splits
over G GPUs with no collective on the data path: request b runs on rank
b mod G, every rank holds the full weights, and the finished chunks are
gathered back in request order ("LingBot-VLA v2 Examples", Configuration: one
full policy per GPU, no tensor or pipeline split).  The gather runs once per
call on the host side of the process group (gloo or NCCL), after the device
work.
"""
from __future__ import annotations

from typing import Callable, List, Optional, Sequence

import numpy as np


def rank_requests(n_requests: int, rank: int, world: int) -> List[int]:
    """Request indices rank `rank` of `world` runs: b with b mod world == rank."""
    if world < 1 or not 0 <= rank < world or n_requests < 0:
        raise ValueError(f"bad shard: {n_requests} requests, rank {rank} of {world}")
    return list(range(rank, n_requests, world))


def take_requests(arrays: Sequence[np.ndarray], idx: Sequence[int]) -> List[np.ndarray]:
    """Rows `idx` (axis 0, the request axis) of each array, contiguous."""
    return [np.ascontiguousarray(a[list(idx)]) for a in arrays]


def gather_in_order(local: np.ndarray, n_requests: int, rank: int, world: int, pg=None) -> np.ndarray:
    """Every rank's chunks [n_local, ...] -> all chunks [n_requests, ...] in
    request order, on every rank.  `pg` is torch.distributed (or None for a
    single process)."""
    if pg is None or world == 1:
        if local.shape[0] != n_requests:
            raise ValueError("a single rank must hold every request")
        return local
    parts: List[Optional[np.ndarray]] = [None] * world
    pg.all_gather_object(parts, local)
    out = np.empty((n_requests,) + tuple(local.shape[1:]), dtype=local.dtype)
    for r, part in enumerate(parts):
        idx = rank_requests(n_requests, r, world)
        if part is None or part.shape[0] != len(idx):
            raise RuntimeError(f"rank {r} returned {None if part is None else part.shape[0]} chunks, "
                               f"expected {len(idx)}")
        out[idx] = part
    return out


def denoise_sharded(run: Callable[[np.ndarray, Sequence[np.ndarray], Sequence[np.ndarray]], np.ndarray],
                    x0: np.ndarray, k_prefix: Sequence[np.ndarray], v_prefix: Sequence[np.ndarray],
                    rank: int, world: int, pg=None) -> np.ndarray:
    """Denoises this rank's share of a batch with `run(x0_local, k_local,
    v_local)` and gathers every rank's chunks in request order.

    x0: [B, T, A]; k_prefix / v_prefix: per layer [B, P, H_kv, hd] (the
    request axis first).  `run` is the caller's one-GPU call, e.g. an Expert's
    set_prefix + denoise; a rank with no request runs nothing."""
    B = x0.shape[0]
    idx = rank_requests(B, rank, world)
    if idx:
        (xl,) = take_requests([x0], idx)
        kl = take_requests(k_prefix, idx)
        vl = take_requests(v_prefix, idx)
        local = np.asarray(run(xl, kl, vl))
    else:
        local = np.empty((0,) + tuple(x0.shape[1:]), dtype=x0.dtype)
    return gather_in_order(local, B, rank, world, pg)
