"""Triangle attention on a 2D grid of devices (one process per GPU).

The pair tensor Z[N][N][c_z] is split over a p x p grid of ranks: rank
r = a p + b holds the block of pairs (rows A_a, columns B_b), n = N / p rows
and columns each (the 2D grid sharding of the Design-CP technical summary,
§Metodología 1).  A starting-node block computes, for each pair (i, j) of the
block, o_ij = softmax_k(q_ij . k_ik + b(j, k)) v_ik over every key k, so rank
(a, b) needs:

- the K and V of its rows A_a over every column block B_c: held along its grid
  row, (a, c) for c = 0..p-1, and passed round that row as a ring, one block
  per step (K/V column blocks moving from device to device, as on the page);
- the logit bias b(j, k) of the pairs (B_b, B_c): the bias block of rank
  (b, c), gathered from every rank once (an all-gather of p^2 blocks of
  n x n, each with its masked padding).

Each ring step runs the flash attention kernel over one key block, giving the
block's output and log-sum-exp, and merges it into the running output by their
log-sum-exp (the online softmax across blocks); then the gate, output
projection and residual run on the block.  An ending-node block is the
starting-node block of the transposed pair tensor: block (a, b) of T(Z) is the
transpose of block (b, a) of Z, so ranks (a, b) and (b, a) swap their blocks
before the block and after it (the diagonal ranks transpose in place).

The per-rank compute is any object with the block-level methods of
``BlockOps`` (the library's kernels on a bf16 handle): ``block_project``,
``block_attend``, ``merge`` and ``block_gate``.  Collectives go through the
group's backend (NCCL on GPUs); every rank takes the same collective steps in
the same order.  ``grid2d_local`` runs the same steps for every block in one
process (a single-GPU emulation of the grid, with the ring order and the
merges of the distributed run).
"""
from __future__ import annotations

import torch
import torch.distributed as dist

STARTING, ENDING = 0, 1


def block_size(N: int, p: int) -> int:
    """n = N / p; the grid needs N divisible by p."""
    if p < 1 or N % p != 0:
        raise ValueError(f"N = {N} does not split into a {p} x {p} grid of equal blocks")
    return N // p


class BlockOps:
    """The library's block-level calls on a bf16 handle (binding.TriangleAttention)."""

    def __init__(self, handle_block):
        self.h = handle_block

    def block_project(self, Z_blk, mask_cols):
        return self.h.block_project(Z_blk, mask_cols)

    def block_attend(self, Q, K, V, bias, ld):
        return self.h.block_attend(Q, K, V, bias, ld)

    def block_gate(self, Z_blk, O):
        return self.h.block_gate(Z_blk, O)

    def merge(self, acc, O, lse, first: bool, last: bool):
        """Running (O fp32, lse, O bf16 or None) after merging one key block."""
        from . import binding
        if first:
            acc = (torch.empty(O.shape, dtype=torch.float32, device=O.device),
                   torch.empty(lse.shape, dtype=torch.float32, device=O.device), None)
        out = torch.empty_like(O) if last else None
        binding.merge_partial(acc[0], acc[1], O, lse, first, out)
        return acc[0], acc[1], out


def _attend_row_of_blocks(ops, Q, kv_at, bias_at, ld, b: int, p: int):
    """Steps of the ring for one block (a, b): key block c = (b + s) mod p at
    step s, its K, V from kv_at(s) and the bias of pairs (B_b, B_c) from
    bias_at(c); the partial outputs merged in that order."""
    acc = None
    for s in range(p):
        c = (b + s) % p
        K, V = kv_at(s)
        O, lse = ops.block_attend(Q, K, V, bias_at(c), ld)
        acc = ops.merge(acc, O, lse, s == 0, s == p - 1)
    return acc[2]


class Grid2DTriangleAttention:
    """The triangle attention block on a p x p grid of ranks."""

    def __init__(self, ops, p: int, group=None):
        self.ops = ops
        self.p = p
        self.group = group
        self.rank = dist.get_rank(group)
        world = dist.get_world_size(group)
        if world != p * p:
            raise ValueError(f"a {p} x {p} grid needs {p * p} ranks, the group has {world}")
        self.a, self.b = divmod(self.rank, p)

    def _global(self, group_rank: int) -> int:
        return group_rank if self.group is None else dist.get_global_rank(self.group, group_rank)

    def forward(self, Z_blk: torch.Tensor, N: int, orientation: int = STARTING,
                mask: torch.Tensor | None = None) -> torch.Tensor:
        """This rank's block of the block's output.  Z_blk: block (a, b) of Z,
        [n][n][c_z], for both orientations."""
        n = block_size(N, self.p)
        assert Z_blk.shape[0] == n and Z_blk.shape[1] == n, (Z_blk.shape, n)
        if orientation not in (STARTING, ENDING):
            raise ValueError(f"orientation {orientation}")
        if orientation == ENDING:
            Z_blk = self.swap_transpose(Z_blk)
        out = self._starting(Z_blk, n, mask)
        return self.swap_transpose(out) if orientation == ENDING else out

    __call__ = forward

    def _starting(self, Z_blk, n, mask):
        p, a, b = self.p, self.a, self.b
        m_b = None if mask is None else mask[b * n:(b + 1) * n]
        Q, K, V, bias, ld = self.ops.block_project(Z_blk, m_b)
        biases = self.gather_bias(bias)
        ring = [torch.stack([K, V])]

        def kv_at(s):
            if s > 0:
                ring[0] = self.ring_shift(ring[0])
            return ring[0][0], ring[0][1]

        O = _attend_row_of_blocks(self.ops, Q, kv_at, lambda c: biases[b * p + c], ld, b, p)
        return self.ops.block_gate(Z_blk, O)

    # ------------------------------------------------------------- exchanges
    def gather_bias(self, bias: torch.Tensor) -> torch.Tensor:
        """Every rank's bias block, [p^2][H][n][ld], rank order (block (x, y) at
        x p + y): one all_gather_into_tensor."""
        pp = self.p * self.p
        flat = torch.empty((pp * bias.shape[0],) + tuple(bias.shape[1:]), dtype=bias.dtype,
                           device=bias.device)
        dist.all_gather_into_tensor(flat, bias.contiguous(), group=self.group)
        return flat.view((pp,) + tuple(bias.shape))

    def ring_shift(self, kv: torch.Tensor) -> torch.Tensor:
        """Pass the K/V block one step round the grid row: send to (a, b-1),
        receive from (a, b+1)."""
        p, a, b = self.p, self.a, self.b
        left, right = a * p + (b - 1) % p, a * p + (b + 1) % p
        recv = torch.empty_like(kv)
        ops = [dist.P2POp(dist.isend, kv.contiguous(), self._global(left), self.group),
               dist.P2POp(dist.irecv, recv, self._global(right), self.group)]
        for req in dist.batch_isend_irecv(ops):
            req.wait()
        return recv

    def swap_transpose(self, X_blk: torch.Tensor) -> torch.Tensor:
        """Block (a, b) of the transposed pair tensor: block (b, a) of X,
        transposed (pair (i, j) -> (j, i))."""
        p, a, b = self.p, self.a, self.b
        peer = b * p + a
        if peer == self.rank:
            return X_blk.transpose(0, 1).contiguous()
        recv = torch.empty_like(X_blk)
        ops = [dist.P2POp(dist.isend, X_blk.contiguous(), self._global(peer), self.group),
               dist.P2POp(dist.irecv, recv, self._global(peer), self.group)]
        for req in dist.batch_isend_irecv(ops):
            req.wait()
        return recv.transpose(0, 1).contiguous()


def grid2d_local(ops, Z: torch.Tensor, N: int, p: int, orientation: int = STARTING,
                 mask: torch.Tensor | None = None) -> torch.Tensor:
    """The whole block computed block by block as the p x p grid computes it
    (same projections, ring order and merges), in one process."""
    n = block_size(N, p)
    Zp = Z if orientation == STARTING else Z.transpose(0, 1)
    blocks = {(x, y): Zp[x * n:(x + 1) * n, y * n:(y + 1) * n].contiguous()
              for x in range(p) for y in range(p)}
    proj = {(x, y): ops.block_project(blocks[(x, y)],
                                      None if mask is None else mask[y * n:(y + 1) * n])
            for x in range(p) for y in range(p)}
    out = torch.empty_like(Zp)
    for a in range(p):
        for b in range(p):
            Q, ld = proj[(a, b)][0], proj[(a, b)][4]
            O = _attend_row_of_blocks(
                ops, Q, lambda s, a=a, b=b: proj[(a, (b + s) % p)][1:3],
                lambda c, b=b: proj[(b, c)][3], ld, b, p)
            out[a * n:(a + 1) * n, b * n:(b + 1) * n] = ops.block_gate(blocks[(a, b)], O)
    return out if orientation == STARTING else out.transpose(0, 1)
