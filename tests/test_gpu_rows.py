"""Row-slab entry points (tri_attn_rows_bias / tri_attn_rows_forward) on one
GPU: the slabs of two or three emulated ranks, with the bias gathered on the
device, give bitwise the output of tri_attn_forward on the whole tensor, for
both orientations (the ending node through the transposed tensor); bad row
ranges are rejected before anything runs."""
import pytest
import torch

from protein_pair_representation_layernorm_b200 import binding, workloads
from protein_pair_representation_layernorm_b200.sharded import row_shards

pytestmark = pytest.mark.gpu


def _sharded_emulation(blk, Zp, mask, world):
    """Starting-node block of Zp computed slab by slab (the exchange done
    locally: concatenation of the bias rows)."""
    N = Zp.shape[0]
    shards = row_shards(N, world)
    bias_rows = [blk.rows_bias(Zp[r0:r0 + n].contiguous(), N, r0, mask) for r0, n in shards]
    bias_all = torch.cat(bias_rows, dim=1).contiguous()   # [H][N][ld]
    outs = [blk.rows_forward(Zp[r0:r0 + n].contiguous(), N, r0, bias_all, mask)
            for r0, n in shards]
    torch.cuda.synchronize()
    return torch.cat(outs, dim=0), bias_all


@pytest.mark.parametrize("N,world", [(200, 2), (300, 3), (97, 2)])
def test_rows_equal_whole_tensor_bitwise(N, world):
    inp = workloads.make_inputs(N, "bf16", 300 + N, "random:0.1")
    blk = binding.TriangleAttention(inp.weights())
    Z = inp.Z.cuda()
    mask = inp.mask.cuda()
    ld = blk.bias_ld(N)
    assert ld % 64 == 0 and ld >= N
    # starting node
    ref = blk.forward(Z, 0, mask, flags=binding.TRI_ATTN_FLAG_SYNC)
    got, bias_all = _sharded_emulation(blk, Z, mask, world)
    assert bias_all.shape == (4, N, ld)
    assert torch.equal(got, ref)
    # ending node = starting node of the transposed pair tensor
    ref_e = blk.forward(Z, 1, mask, flags=binding.TRI_ATTN_FLAG_SYNC)
    got_t, _ = _sharded_emulation(blk, Z.transpose(0, 1).contiguous(), mask, world)
    assert torch.equal(got_t.transpose(0, 1), ref_e)
    assert blk.status() == binding.TRI_ATTN_OK
    blk.close()


def test_rows_in_place_and_chunked():
    N = 160
    inp = workloads.make_inputs(N, "bf16", 77, "random:0.2")
    blk = binding.TriangleAttention(inp.weights())
    Z = inp.Z.cuda()
    mask = inp.mask.cuda()
    ref = blk.forward(Z, 0, mask, flags=binding.TRI_ATTN_FLAG_SYNC)
    bias_all = torch.cat([blk.rows_bias(Z[r0:r0 + n].contiguous(), N, r0, mask)
                          for r0, n in row_shards(N, 2)], dim=1).contiguous()
    # a workspace limit small enough to split each slab into several row chunks
    blk.set_workspace_limit(binding.tri_attn_workspace_bytes(binding.TRI_ATTN_BF16, N) // 8)
    outs = []
    for r0, n in row_shards(N, 2):
        slab = Z[r0:r0 + n].clone()
        blk.rows_forward(slab, N, r0, bias_all, mask, out=slab)  # in place
        outs.append(slab)
    torch.cuda.synchronize()
    assert torch.equal(torch.cat(outs), ref)
    blk.close()


def test_rows_reject_bad_ranges():
    N = 64
    inp = workloads.make_inputs(N, "bf16", 5)
    blk = binding.TriangleAttention(inp.weights())
    Z = inp.Z.cuda()
    bias = torch.empty(4, N, blk.bias_ld(N), dtype=torch.bfloat16, device="cuda")
    for row0, rows in ((-1, 8), (60, 8), (0, 0)):
        slab = torch.empty(max(rows, 1), N, 128, dtype=torch.bfloat16, device="cuda")
        rc = binding.lib().tri_attn_rows_bias(blk.handle, slab.data_ptr(), N, row0, rows, None,
                                              bias.data_ptr(), None, 0)
        assert rc == binding.TRI_ATTN_ERR_INVALID_ARG, (row0, rows, rc)
    # overlapping but unequal out and Z
    rc = binding.lib().tri_attn_rows_forward(blk.handle, Z.data_ptr(), N, 0, 8, None,
                                             bias.data_ptr(), Z[1:].data_ptr(), None, 0)
    assert rc == binding.TRI_ATTN_ERR_ALIAS
    blk.close()
    f32 = binding.TriangleAttention(workloads.make_inputs(8, "f32", 6).weights(),
                                    dtype=torch.float32)
    z32 = torch.zeros(8, 8, 128, device="cuda")
    rc = binding.lib().tri_attn_rows_bias(f32.handle, z32.data_ptr(), 8, 0, 8, None,
                                          bias.data_ptr(), None, 0)
    assert rc == binding.TRI_ATTN_ERR_UNSUPPORTED
    f32.close()
