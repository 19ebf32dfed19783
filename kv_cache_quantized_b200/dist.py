"""Multi-GPU plumbing (one process per GPU, torch.distributed).

Decode attention shards without any exchange: (batch row, KV head) units are independent, so each rank attends
over its own rows and caches.  The only exchange on the path is in sign-pattern selection: candidates are split
across ranks, each rank scores its share on its own GPU, and one all-gather of the per-candidate MSEs (n_cand
float64 values) gives every rank the full vector and the same pick.  Timings are reduced with a max over ranks.
"""

from __future__ import annotations

import torch
import torch.distributed as dist


def world() -> tuple[int, int]:
    """(rank, world size); (0, 1) without an initialised process group."""
    if dist.is_available() and dist.is_initialized():
        return dist.get_rank(), dist.get_world_size()
    return 0, 1


def shard_range(n: int, rank: int, size: int) -> tuple[int, int]:
    """Contiguous share [lo, hi) of n units for `rank` of `size` (the first n % size ranks get one extra)."""
    base, extra = divmod(n, size)
    lo = rank * base + min(rank, extra)
    return lo, lo + base + (1 if rank < extra else 0)


def max_over_ranks(values, device=None):
    """Element-wise max of a list of floats over all ranks (identity on one rank)."""
    t = torch.tensor(list(values), dtype=torch.float64, device=device)
    rank, size = world()
    if size > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def gather_candidate_mse(local_mse: torch.Tensor, n_cand: int) -> torch.Tensor:
    """All-gather each rank's MSEs for its shard_range() share of n_cand candidates into one [n_cand] vector."""
    rank, size = world()
    if size == 1:
        return local_mse.to(torch.float64)
    width = -(-n_cand // size)
    buf = torch.full((width,), float("nan"), dtype=torch.float64, device=local_mse.device)
    buf[: local_mse.numel()] = local_mse.to(torch.float64)
    parts = [torch.empty_like(buf) for _ in range(size)]
    dist.all_gather(parts, buf)
    out = []
    for r in range(size):
        lo, hi = shard_range(n_cand, r, size)
        out.append(parts[r][: hi - lo])
    return torch.cat(out)


def first_argmin(mse: torch.Tensor) -> int:
    """Index of the first minimum (the pick rule of the selector)."""
    m = torch.min(mse)
    return int(torch.nonzero(mse == m)[0, 0])


def select_signs_sharded(q, k, v, candidates, bits, causal=True, score_fn=None):
    """Sign-pattern selection with the candidates split across ranks.

    score_fn(q, k, v, candidates_share, bits, causal) -> mse tensor of the share; the default runs the library's
    axr_select_signs on this rank's GPU.  Returns (mse [n_cand] float64, best index), identical on every rank.
    """
    if score_fn is None:
        from . import ops

        def score_fn(q_, k_, v_, c_, b_, causal_):
            return ops.select_signs(q_, k_, v_, c_, b_, causal=causal_)[0]
    rank, size = world()
    n = candidates.shape[0]
    lo, hi = shard_range(n, rank, size)
    local = score_fn(q, k, v, candidates[lo:hi].contiguous(), bits, causal) if hi > lo else \
        torch.empty(0, dtype=torch.float64, device=candidates.device)
    mse = gather_candidate_mse(local, n)
    return mse, first_argmin(mse)


def select_signs_per_layer_sharded(q, k, v, candidates, bits, causal=True, score_fn=None):
    """One sign vector per layer with the candidates split across ranks: each rank scores its share of candidates
    on every layer, one all-gather of the [n_layers, share] MSEs per layer row assembles [n_layers, n_cand] on every
    rank, and each layer picks the first index of its minimum.

    score_fn(q, k, v, candidates_share, bits, causal) -> [n_layers, share] MSEs; the default runs the library's
    axr_select_signs_per_layer on this rank's GPU.  Returns (mse [n_layers, n_cand] float64, best [n_layers] list).
    """
    if score_fn is None:
        from . import ops

        def score_fn(q_, k_, v_, c_, b_, causal_):
            return ops.select_signs_per_layer(q_, k_, v_, c_, b_, causal=causal_)[0]
    rank, size = world()
    n = candidates.shape[0]
    lo, hi = shard_range(n, rank, size)
    n_layers = q.shape[0] if q is not None else None
    local = score_fn(q, k, v, candidates[lo:hi].contiguous(), bits, causal) if hi > lo else None
    if local is None:
        local = torch.empty((n_layers if n_layers is not None else 0, 0), dtype=torch.float64,
                            device=candidates.device)
    rows = [gather_candidate_mse(local[layer], n) for layer in range(local.shape[0])]
    mse = torch.stack(rows) if rows else torch.empty((0, n), dtype=torch.float64)
    return mse, [first_argmin(mse[layer]) for layer in range(mse.shape[0])]
