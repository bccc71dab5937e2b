"""The 2D-grid block (protein_pair_representation_layernorm_b200.grid2d) on CPU:
the in-process driver at p = 1, 2, 3 and 4 gloo ranks forming a 2 x 2 grid
must give exactly the whole block's output, for both orientations, with a key
mask.  The per-block compute is a stand-in built on the oracle (projections
from its pair features, each key block's output from its full softmax, the
block's log-sum-exp from the same scores), so what is checked here is the
grid: which K/V, bias and mask blocks each step uses, the ring order, the
merges and the transposes of the ending node.  The GPU block calls are checked
in tests/test_gpu_grid2d.py."""
import dataclasses
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

H, D = 4, 32


class OracleBlockOps:
    """Block-level calls with the oracle's arithmetic (fp64).  Conventions as
    the library's, in natural units: bias -inf at masked keys, lse natural,
    +inf for a key block with no unmasked key."""

    def __init__(self, prob):
        self.prob = prob

    def _features(self, Z_blk):
        import oracle
        p = dataclasses.replace(self.prob, Z=np.ascontiguousarray(Z_blk.numpy()), mask=None)
        return oracle.pair_features(p)

    def block_project(self, Z_blk, mask_cols):
        q, k, v, _, b = self._features(Z_blk)
        n = Z_blk.shape[0]
        to_heads = lambda a: torch.from_numpy(a.reshape(n, n, H, D).transpose(0, 2, 1, 3).copy())  # noqa: E731
        if mask_cols is not None:
            b = b.copy()
            b[:, :, np.asarray(mask_cols) == 0] = -np.inf
        return to_heads(q), to_heads(k), to_heads(v), torch.from_numpy(b), n

    def block_attend(self, Q, K, V, bias, ld):
        import oracle
        b = bias.numpy()
        valid = ~np.isneginf(b[0, 0])
        bn = np.where(np.isneginf(b), 0.0, b)
        O, L = [], []
        for r in range(Q.shape[0]):
            q, k, v = (t[r].numpy().transpose(1, 0, 2) for t in (Q, K, V))  # (n, H, d)
            O.append(oracle.attend(q, k, v, bn, valid.astype(np.uint8)).transpose(1, 0, 2))
            s = np.einsum("jhd,khd->hjk", q, k) / np.sqrt(D) + bn
            s[:, :, ~valid] = -np.inf
            m = s.max(axis=2, keepdims=True)
            with np.errstate(invalid="ignore"):
                lse = (m + np.log(np.exp(s - m).sum(axis=2, keepdims=True)))[:, :, 0]
            L.append(np.where(valid.any(), lse, np.inf))
        return torch.from_numpy(np.stack(O)), torch.from_numpy(np.stack(L))

    def merge(self, acc, O, lse, first, last):
        o2, l2 = O.numpy(), lse.numpy()
        o1, l1 = (np.zeros_like(o2), np.full_like(l2, np.inf)) if first else acc[:2]
        e1, e2 = np.isposinf(l1), np.isposinf(l2)
        m = np.where(e1, l2, np.where(e2, l1, np.maximum(l1, l2)))
        with np.errstate(invalid="ignore"):
            w1 = np.where(e1, 0.0, np.exp(l1 - m))
            w2 = np.where(e2, 0.0, np.exp(l2 - m))
        tot = w1 + w2
        lse_new = np.where(e1 & e2, np.inf, m + np.log(np.where(tot > 0, tot, 1.0)))
        tot = np.where(tot > 0, tot, 1.0)
        o = (w1 / tot)[..., None] * o1 + (w2 / tot)[..., None] * o2
        return o, lse_new, (torch.from_numpy(o) if last else None)

    def block_gate(self, Z_blk, O):
        _, _, _, g, _ = self._features(Z_blk)
        n = Z_blk.shape[0]
        o = O.numpy().transpose(0, 2, 1, 3).reshape(n, n, H * D)
        upd = (g * o) @ np.asarray(self.prob.Wo, dtype=np.float64).T
        if self.prob.bo is not None:
            upd = upd + np.asarray(self.prob.bo, dtype=np.float64)
        return torch.from_numpy(Z_blk.numpy().astype(np.float64) + upd)


def _problem(N, seed):
    from conftest import to_problem
    from protein_pair_representation_layernorm_b200 import workloads
    inp = workloads.make_inputs(N, "f32", seed, "random:0.25")
    return inp, to_problem(inp)


@pytest.mark.parametrize("p,N", [(1, 12), (2, 12), (3, 12)])
def test_grid2d_local_equals_the_whole_block(p, N):
    import oracle
    from protein_pair_representation_layernorm_b200.grid2d import grid2d_local
    inp, prob = _problem(N, 90 + p)
    ops = OracleBlockOps(prob)
    for orientation in (0, 1):
        want = oracle.tri_attn_full(prob, orientation)
        got = grid2d_local(ops, inp.Z.double(), N, p, orientation, inp.mask).numpy()
        assert np.abs(got - want).max() < 1e-9, (p, orientation, np.abs(got - want).max())


def test_block_size_rejects_uneven_grids():
    from protein_pair_representation_layernorm_b200.grid2d import block_size
    assert block_size(12, 3) == 4
    with pytest.raises(ValueError):
        block_size(13, 2)


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, N, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), OMP_NUM_THREADS="1")
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    import datetime
    import torch.distributed as dist
    import oracle
    from protein_pair_representation_layernorm_b200.grid2d import Grid2DTriangleAttention
    try:
        dist.init_process_group("gloo", rank=rank, world_size=world,
                                timeout=datetime.timedelta(seconds=120))
        inp, prob = _problem(N, 95)
        p = int(round(world ** 0.5))
        grid = Grid2DTriangleAttention(OracleBlockOps(prob), p)
        n = N // p
        a, b = grid.a, grid.b
        errs = []
        for orientation in (0, 1):
            want = oracle.tri_attn_full(prob, orientation)[a * n:(a + 1) * n, b * n:(b + 1) * n]
            Z_blk = inp.Z.double()[a * n:(a + 1) * n, b * n:(b + 1) * n].contiguous()
            got = grid(Z_blk, N, orientation, inp.mask).numpy()
            errs.append(float(np.abs(got - want).max()))
        dist.barrier()
        dist.destroy_process_group()
        q.put((rank, errs))
    except Exception as e:  # report, never hang the parent
        q.put((rank, [repr(e)]))


def test_grid2d_on_four_gloo_ranks():
    world, N = 4, 12
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, N, q)) for r in range(world)]
    for pr in procs:
        pr.start()
    res = sorted(q.get(timeout=300) for _ in procs)
    for pr in procs:
        pr.join(timeout=60)
        assert pr.exitcode == 0
    for rank, errs in res:
        assert all(isinstance(e, float) for e in errs), errs
        assert max(errs) < 1e-9, (rank, errs)
