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
        """All-gather of every rank's bias rows into the whole [H][N][ld] bias:
        one all_gather_into_tensor over the slab-major layout [world][H][S][ld]
        (each rank's slab padded to S rows only if it has fewer), then one
        strided copy into the head-major layout the attention kernel reads."""
        H, nrows, ld = bias_rows.shape
        S = -(-N // self.world)
        mine = bias_rows
        if nrows < S or not bias_rows.is_contiguous():
            mine = torch.zeros(H, S, ld, dtype=bias_rows.dtype, device=bias_rows.device)
            mine[:, :nrows] = bias_rows
        flat = torch.empty(self.world * H, S, ld, dtype=bias_rows.dtype, device=bias_rows.device)
        dist.all_gather_into_tensor(flat, mine.contiguous(), group=self.group)
        gathered = flat.view(self.world, H, S, ld)
        out = torch.empty(H, N, ld, dtype=bias_rows.dtype, device=bias_rows.device)
        # rank p's rows are p*S .. p*S+S-1: out[h][p*S + r] = gathered[p][h][r]
        full = out.view(H, N, ld) if self.world * S == N else None
        if full is not None:
            full.view(H, self.world, S, ld).copy_(gathered.permute(1, 0, 2, 3))
        else:
            out.copy_(gathered.permute(1, 0, 2, 3).reshape(H, self.world * S, ld)[:, :N])
        return out

    def transpose_rows(self, X_rows: torch.Tensor, N: int) -> torch.Tensor:
        """This rank's rows of the transpose (pair (i, j) -> (j, i)) of a row-
        sharded N x N x C tensor, by one all-to-all of S x S blocks.  Block q of
        the send buffer is X[my rows][rows of q]; it is packed with one strided
        copy (X viewed as [S][world][S][C], columns padded to world*S when N is
        not a multiple of the world size) and unpacked with another."""
        shards = row_shards(N, self.world)
        S = -(-N // self.world)
        row0, nrows = shards[self.rank]
        C = X_rows.shape[2]
        W = self.world
        if nrows == S and W * S == N:
            src = X_rows.view(S, W, S, C)
        else:
            src = torch.zeros(S, W * S, C, dtype=X_rows.dtype, device=X_rows.device)
            src[:nrows, :N] = X_rows
            src = src.view(S, W, S, C)
        send = src.permute(1, 0, 2, 3).contiguous()                # [q][my row][col of q]
        recv = torch.empty_like(send)
        dist.all_to_all_single(recv, send, group=self.group)       # block p = X[R_p][R_me]
        # out[c][p*S + i] = recv[p][i][c]
        t = recv.permute(2, 0, 1, 3)                               # [my col][p][row of p]
        if nrows == S and W * S == N:
            return t.reshape(S, N, C).contiguous()
        return t.reshape(S, W * S, C)[:nrows, :N].contiguous()
