"""The lookup over a value table sharded by rows across ranks.

"Memory Layers at Scale" digest: memories of 64B and 128B parameters do not
fit one GPU's memory, so the value table is split by row id across the
ranks (contiguous ranges, ``shard_rows``) while the sub-keys, which are
small, stay replicated.  Per step, with every rank holding T tokens:

1. each rank selects the rows of its own tokens (``pkm_select``, the
   replicated sub-keys);
2. the selections (ids and weights, H*k per token) are all-gathered;
3. each rank sums, for the tokens of every rank, the selected rows it holds
   (``embbag_forward_range``, fp32 partial bags of world*T tokens);
4. a reduce-scatter over tokens sums the partials and hands each rank the
   bags of its own tokens (fp32, summed in rank order by the collective).

The exchange is one all-gather of T*H*k*8 bytes and one reduce-scatter of
world*T*d_v*4 bytes per rank, instead of moving value rows: a row is read
from HBM once, by its owner.  This module only orders the steps; every
step's arithmetic runs in the CUDA library (steps 1 and 3) or in the
collective (step 4).  ``comm`` is any object with ``all_gather(t) ->
[world, *t.shape]`` and ``reduce_scatter_sum(t [world*T, d]) -> [T, d]``;
``TorchComm`` wraps ``torch.distributed``.
"""

from __future__ import annotations

import torch


def shard_rows(n_rows: int, world: int, rank: int):
    """(first row, number of rows) of rank's contiguous share of a table of
    n_rows rows: ceil(n_rows / world) rows each, the last share shorter."""
    per = -(-n_rows // world)
    lo = min(n_rows, rank * per)
    return lo, max(0, min(n_rows, lo + per) - lo)


class TorchComm:
    """The two collectives over a torch.distributed process group:
    all_gather_into_tensor (concatenated along the first dimension) and
    reduce_scatter_tensor (sum).  The same calls run on NCCL and on gloo, so
    the host tests exercise the code path the GPUs take."""

    def __init__(self, group=None):
        import torch.distributed as dist

        self.dist = dist
        self.group = group
        self.world = dist.get_world_size(group)
        self.rank = dist.get_rank(group)

    def all_gather(self, t: torch.Tensor) -> torch.Tensor:
        t = t.contiguous()
        out = torch.empty((self.world * t.shape[0],) + tuple(t.shape[1:]), dtype=t.dtype,
                          device=t.device)
        self.dist.all_gather_into_tensor(out, t, group=self.group)
        return out.view((self.world,) + tuple(t.shape))

    def reduce_scatter_sum(self, t: torch.Tensor) -> torch.Tensor:
        T = t.shape[0] // self.world
        out = torch.empty((T,) + tuple(t.shape[1:]), dtype=t.dtype, device=t.device)
        self.dist.reduce_scatter_tensor(out, t.contiguous(), group=self.group)
        return out


class LocalComm:
    """The exchange of a single rank: the all-gather stacks its one input and
    the reduce-scatter returns it."""

    world, rank = 1, 0

    def all_gather(self, t: torch.Tensor) -> torch.Tensor:
        return t.unsqueeze(0)

    def reduce_scatter_sum(self, t: torch.Tensor) -> torch.Tensor:
        return t


def exchange_bytes(T: int, H: int, k: int, d_v: int, world: int) -> dict:
    """Bytes one rank receives per step: the other ranks' selections (ids
    and weights, 8 bytes per entry) in the all-gather, and their partial
    bags of this rank's tokens (fp32) in the reduce-scatter."""
    return {"all_gather": (world - 1) * T * H * k * 8,
            "reduce_scatter": (world - 1) * T * d_v * 4}


def sharded_lookup(query, subkeys, values_shard, k: int, row_lo: int, comm, select=None,
                   gather=None):
    """One rank's step of the row-sharded lookup (steps 1-4 above).

    query [T, H, 2, d_half] (this rank's tokens, T equal on every rank),
    subkeys [H, 2, n_sub, d_half] (replicated), values_shard [n_local, d_v]
    (rows row_lo .. of the full table).  Returns (y fp32 [T, d_v], idx,
    weights).  ``select`` / ``gather`` default to the CUDA library's
    pkm_select / embbag_forward_range."""
    if select is None or gather is None:
        import sparse_key_value_b200 as skv

        select = select or (lambda q, K, kk: skv.pkm_select(q, K, kk, d_v=values_shard.shape[1]))
        gather = gather or skv.embbag_forward_range
    T, H = query.shape[0], query.shape[1]
    idx, w = select(query, subkeys, k)
    all_idx = comm.all_gather(idx.reshape(T, H * k)).reshape(-1, H * k)
    all_w = comm.all_gather(w.reshape(T, H * k)).reshape(-1, H * k)
    if values_shard.shape[0] > 0:
        part = gather(values_shard, row_lo, all_idx, all_w)
    else:  # more ranks than rows: this rank holds none
        part = torch.zeros(all_idx.shape[0], values_shard.shape[1], dtype=torch.float32,
                           device=values_shard.device)
    return comm.reduce_scatter_sum(part), idx, w
