"""Sharding one long prefill over GPUs by query rows (one process per GPU, torch.distributed).

Each rank runs the row-block entry points (dsa_indexer_topk_rows, dsa_sparse_mla_prefill_rows)
on its own block of query rows.  Every rank needs the whole sequence's keys (k_I, k_scale) and
latent rows; the ranks hold them in equal row blocks and all-gather them once per sequence into
local memory (NCCL over NVLink on GPUs, gloo on CPU), so no kernel ever reads another GPU's
memory.  The query-row blocks are balanced on a cost model (dsa_row_partition in
include/dsa.h): the indexer's work grows with a row's causal prefix, sparse MLA's with its
selection.
"""

from __future__ import annotations

import torch

from . import dsa_row_partition


def row_blocks(L: int, k: int, world: int, indexer_cost: float, mla_cost: float) -> list[int]:
    """Query-row boundaries [0, ..., L] of balanced cost for `world` ranks, given the two
    kernels' measured times of one whole-sequence step."""
    return dsa_row_partition(L, k, world, indexer_cost, mla_cost)


def even_blocks(L: int, world: int) -> list[int]:
    """Equal row blocks: how the key and latent rows are spread over the ranks before the gather."""
    return [L * r // world for r in range(world + 1)]


def gather_sequence(local: torch.Tensor, full: torch.Tensor, world: int, rank: int) -> torch.Tensor:
    """All-gather of the ranks' row blocks (rank r holds rows even_blocks(L, world)[r:r+2] of a
    tensor of L rows) into `full` on every rank.  Blocks are padded to a common size for the
    collective, then the L real rows are copied out."""
    L = full.shape[0]
    if world == 1:
        full.copy_(local)
        return full
    import torch.distributed as dist

    bounds = even_blocks(L, world)
    assert local.shape[0] == bounds[rank + 1] - bounds[rank], "local block does not match the even split"
    per = max(bounds[r + 1] - bounds[r] for r in range(world))
    pad = torch.zeros((per,) + tuple(full.shape[1:]), dtype=full.dtype, device=full.device)
    pad[: local.shape[0]] = local
    if dist.get_backend() == "nccl":
        buf = torch.empty((world * per,) + tuple(full.shape[1:]), dtype=full.dtype, device=full.device)
        dist.all_gather_into_tensor(buf, pad)
        parts = [buf[r * per: r * per + bounds[r + 1] - bounds[r]] for r in range(world)]
    else:
        gathered = [torch.empty_like(pad) for _ in range(world)]
        dist.all_gather(gathered, pad)
        parts = [gathered[r][: bounds[r + 1] - bounds[r]] for r in range(world)]
    for r in range(world):
        full[bounds[r]: bounds[r + 1]] = parts[r]
    return full
