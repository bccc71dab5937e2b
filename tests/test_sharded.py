"""The row-sharded block (protein_pair_representation_layernorm_b200.sharded) on
CPU gloo ranks: the bias all-gather and the all-to-all transposes must give
every rank exactly its rows of the whole block, for both orientations, with
slabs of unequal size.  The per-rank compute is a stand-in built on the
oracle (a starting-node block on a row slab given the whole bias), so what is
checked here is the sharding and the exchange; the GPU row-slab kernels are
checked against the unsharded path in tests/test_gpu_parity.py."""
import dataclasses
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


class OracleSlabBlock:
    """rows_bias / rows_forward of the oracle for a problem of which only the
    slab's rows are known (the other rows of Z are zeros and never read)."""

    def __init__(self, prob):
        self.prob = prob

    def bias_ld(self, N):
        return N

    def _problem(self, Z_rows, N, row0):
        Z = np.zeros((N, N, Z_rows.shape[2]), dtype=np.float32)
        Z[row0:row0 + Z_rows.shape[0]] = Z_rows.numpy()
        return dataclasses.replace(self.prob, Z=Z)

    def rows_bias(self, Z_rows, N, row0, mask):
        import oracle
        b = oracle.bias_all(self._problem(Z_rows, N, row0))
        return torch.from_numpy(np.ascontiguousarray(b[:, row0:row0 + Z_rows.shape[0]]))

    def rows_forward(self, Z_rows, N, row0, bias_all, mask):
        import oracle
        lines = list(range(row0, row0 + Z_rows.shape[0]))
        out = oracle.tri_attn(self._problem(Z_rows, N, row0), 0, lines, bias=bias_all.numpy())
        return torch.from_numpy(out)


def _rank_main(rank, world, port, N, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), OMP_NUM_THREADS="2")
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    import datetime
    import torch.distributed as dist
    import oracle
    from conftest import to_problem
    from protein_pair_representation_layernorm_b200 import workloads
    from protein_pair_representation_layernorm_b200.sharded import ShardedTriangleAttention
    try:
        dist.init_process_group("gloo", rank=rank, world_size=world,
                                timeout=datetime.timedelta(seconds=120))
        inp = workloads.make_inputs(N, "f32", 70 + N, "random:0.25")
        prob = to_problem(inp)
        sharded = ShardedTriangleAttention(OracleSlabBlock(prob))
        row0, nrows = sharded.shard(N)
        errs = []
        for orientation in (0, 1):
            want = oracle.tri_attn_full(prob, orientation)[row0:row0 + nrows]
            got = sharded(inp.Z[row0:row0 + nrows].contiguous(), N, orientation,
                          inp.mask).numpy()
            errs.append(float(np.abs(got - want).max()))
        dist.barrier()
        dist.destroy_process_group()
        q.put((rank, row0, nrows, errs))
    except Exception as e:  # report, never hang the parent
        q.put((rank, -1, -1, [repr(e)]))


@pytest.mark.parametrize("world,N", [(2, 13), (3, 13)])
def test_row_sharded_block_gloo(world, N):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, N, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=300) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    covered = []
    for rank, row0, nrows, errs in res:
        assert row0 >= 0, errs
        assert max(errs) < 1e-9, (rank, errs)
        covered += list(range(row0, row0 + nrows))
    assert covered == list(range(N))


def test_row_shards_split():
    sys.path.insert(0, ROOT)
    from protein_pair_representation_layernorm_b200.sharded import row_shards
    assert row_shards(13, 2) == [(0, 7), (7, 6)]
    assert row_shards(13, 3) == [(0, 5), (5, 5), (10, 3)]
    assert row_shards(8, 8) == [(r, 1) for r in range(8)]
    with pytest.raises(ValueError):
        row_shards(3, 4)
    with pytest.raises(ValueError):
        row_shards(5, 4)  # ceil(5/4) = 2 rows each leaves the fourth rank empty
