"""Row-sharded triangle attention over torch.distributed (one process per GPU).

One N x N problem is split over the ranks of a process group by problem rows:
rank r holds the slab of rows [r*S, min((r+1)*S, N)) of the pair tensor, with
S = ceil(N / world).  A starting-node block needs, for its rows, only their own
K and V and the logit bias of every pair, so the one exchange is an all-gather
of the bias (the 1D row sharding of the Design-CP technical summary,
§Metodología 1).  An ending-node block is the starting-node block of the
transposed pair tensor: its rows are the columns of Z, so the slabs are
transposed with one all-to-all before the block and one after it.

The per-rank compute is any object with the row-slab methods of
``binding.TriangleAttention``: ``bias_ld(N)``, ``rows_bias(Z_rows, N, row0,
mask)`` -> [H][nrows][ld] and ``rows_forward(Z_rows, N, row0, bias_all, mask)``
-> out_rows.  Collectives go through the group's backend (NCCL on GPUs); every
rank takes the same collective steps in the same order.  Slabs are padded to S
rows inside the collectives so that every rank sends and receives equal sizes.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

STARTING, ENDING = 0, 1


def row_shards(N: int, world: int) -> list[tuple[int, int]]:
    """(row0, nrows) of every rank; S = ceil(N / world) rows each, the last
    ranks fewer (N >= world is required so that every rank holds a row)."""
    if N < world:
        raise ValueError(f"N = {N} rows cannot be split over {world} ranks")
    S = -(-N // world)
    out = []
    for r in range(world):
        row0 = min(r * S, N)
        out.append((row0, max(0, min(S, N - row0))))
    if any(n == 0 for _, n in out):
        raise ValueError(f"N = {N} leaves a rank without rows at world size {world}")
    return out


class ShardedTriangleAttention:
    """The triangle attention block on a row-sharded pair tensor."""

    def __init__(self, block, group=None):
        self.block = block
        self.group = group
        self.rank = dist.get_rank(group)
        self.world = dist.get_world_size(group)

    # ---------------------------------------------------------------- public
    def shard(self, N: int) -> tuple[int, int]:
        """(row0, nrows) of this rank."""
        return row_shards(N, self.world)[self.rank]

    def forward(self, Z_rows: torch.Tensor, N: int, orientation: int = STARTING,
                mask: torch.Tensor | None = None) -> torch.Tensor:
        """This rank's rows of the block's output.  Z_rows: this rank's slab
        [nrows][N][c_z] of the pair tensor (rows of Z for both orientations)."""
        row0, nrows = self.shard(N)
        assert Z_rows.shape[0] == nrows and Z_rows.shape[1] == N, (Z_rows.shape, nrows, N)
        if orientation == STARTING:
            return self._starting(Z_rows, N, row0, mask)
        if orientation != ENDING:
            raise ValueError(f"orientation {orientation}")
        Zt_rows = self.transpose_rows(Z_rows, N)
        out_t = self._starting(Zt_rows, N, row0, mask)
        return self.transpose_rows(out_t, N)

    __call__ = forward

    # ------------------------------------------------------------ the steps
    def _starting(self, Z_rows, N, row0, mask):
        bias_rows = self.block.rows_bias(Z_rows, N, row0, mask)   # [H][nrows][ld]
        bias_all = self.gather_bias(bias_rows, N)                  # [H][N][ld]
        return self.block.rows_forward(Z_rows, N, row0, bias_all, mask)

    def gather_bias(self, bias_rows: torch.Tensor, N: int) -> torch.Tensor:
        """All-gather of every rank's bias rows into the whole [H][N][ld] bias
        (one all-gather per head, each slab padded to S rows)."""
        H, nrows, ld = bias_rows.shape
        S = -(-N // self.world)
        out = torch.empty(H, N, ld, dtype=bias_rows.dtype, device=bias_rows.device)
        for h in range(H):
            mine = torch.zeros(S, ld, dtype=bias_rows.dtype, device=bias_rows.device)
            mine[:nrows] = bias_rows[h]
            parts = [torch.empty_like(mine) for _ in range(self.world)]
            dist.all_gather(parts, mine, group=self.group)
            out[h] = torch.cat(parts, dim=0)[:N]
        return out

    def transpose_rows(self, X_rows: torch.Tensor, N: int) -> torch.Tensor:
        """This rank's rows of the transpose (pair (i, j) -> (j, i)) of a row-
        sharded N x N x C tensor, by one all-to-all of S x S blocks."""
        shards = row_shards(N, self.world)
        S = -(-N // self.world)
        row0, nrows = shards[self.rank]
        C = X_rows.shape[2]
        send = torch.zeros(self.world, S, S, C, dtype=X_rows.dtype, device=X_rows.device)
        for q, (c0, nc) in enumerate(shards):
            send[q, :nrows, :nc] = X_rows[:, c0:c0 + nc]           # X[R_me][R_q]
        recv = torch.empty_like(send)
        dist.all_to_all_single(recv, send, group=self.group)       # block p = X[R_p][R_me]
        out = torch.empty(nrows, N, C, dtype=X_rows.dtype, device=X_rows.device)
        for p, (c0, nc) in enumerate(shards):
            out[:, c0:c0 + nc] = recv[p, :nc, :nrows].transpose(0, 1)
        return out.contiguous()
