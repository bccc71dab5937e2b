"""The 2D grid on one GPU: grid2d_local runs every block of a p x p grid with
the library's block-level calls (tri_attn_block_project, tri_attn_block_attend,
tri_attn_merge_partial, tri_attn_block_gate) in the ring order of the
distributed run.  At p = 1 it must equal tri_attn_forward bit for bit (the same
three kernels on the same pairs, and a merge of one block that only rounds
its fp32 copy back to bf16); at p = 2, 3, 4 the outputs of the split softmax
must match the fp64 oracle within the bf16 tolerances, both orientations, with
a key mask."""
import numpy as np
import pytest
import torch

import oracle
from conftest import to_problem
from gpu_util import assert_within, compare, log_parity, run_gpu
from protein_pair_representation_layernorm_b200 import binding, workloads
from protein_pair_representation_layernorm_b200.grid2d import BlockOps, grid2d_local

pytestmark = pytest.mark.gpu


def _grid(inp, blk, p, orientation):
    Z = inp.Z.cuda()
    mask = None if inp.mask is None else inp.mask.cuda()
    out = grid2d_local(BlockOps(blk), Z, inp.N, p, orientation, mask)
    torch.cuda.synchronize()
    assert blk.status() == binding.TRI_ATTN_OK
    return out


@pytest.mark.parametrize("N", [200, 130])
def test_one_block_grid_equals_the_forward(N):
    inp = workloads.make_inputs(N, "bf16", 120 + N, "random:0.1")
    want0, blk = run_gpu(inp, 0)
    want1, _ = run_gpu(inp, 1, blk=blk)
    got0 = _grid(inp, blk, 1, 0)
    got1 = _grid(inp, blk, 1, 1)
    assert torch.equal(got0.view(torch.int16), want0.view(torch.int16))
    assert torch.equal(got1.contiguous().view(torch.int16), want1.view(torch.int16))
    blk.close()


@pytest.mark.parametrize("p,N", [(2, 256), (3, 192), (4, 256)])
def test_grid_matches_oracle(p, N):
    inp = workloads.make_inputs(N, "bf16", 130 + p, "random:0.1")
    blk = binding.TriangleAttention(inp.weights(), dtype=torch.bfloat16)
    prob = to_problem(inp)
    z = inp.Z.double().numpy()
    for orientation in (0, 1):
        got = _grid(inp, blk, p, orientation).double().cpu().numpy()
        ref = oracle.tri_attn_full(prob, orientation)
        st = compare(got, ref, z, "bf16")
        log_parity(f"2D grid p={p} N={N} orientation {orientation}", st)
        assert st["finite"]
        assert_within(st, "bf16", f"2D grid p={p} orientation {orientation}")
    blk.close()


def test_merge_of_split_keys_equals_one_block():
    """tri_attn_merge_partial on the two halves of a key range gives the
    output and log-sum-exp of the whole range (to bf16 rounding of the parts)."""
    N, rows = 128, 3
    inp = workloads.make_inputs(N, "bf16", 140, "random:0.1")
    blk = binding.TriangleAttention(inp.weights(), dtype=torch.bfloat16)
    Q, K, V, bias, ld = blk.block_project(inp.Z.cuda(), inp.mask.cuda())
    Q, K, V = (t[:rows].contiguous() for t in (Q, K, V))  # the bias is of all N queries
    O_all, l_all = blk.block_attend(Q, K, V, bias, ld)
    # the same keys as two blocks of 64: each block masks the other's keys
    parts = []
    for h in range(2):
        b2 = bias.clone()
        cols = slice(64, 128) if h == 0 else slice(0, 64)
        b2[:, :, cols] = torch.tensor(-3e38, dtype=torch.bfloat16)
        parts.append(blk.block_attend(Q, K, V, b2, ld))
    acc_o = torch.empty(O_all.shape, dtype=torch.float32, device="cuda")
    acc_l = torch.empty(l_all.shape, dtype=torch.float32, device="cuda")
    out = torch.empty_like(O_all)
    binding.merge_partial(acc_o, acc_l, parts[0][0], parts[0][1], True)
    binding.merge_partial(acc_o, acc_l, parts[1][0], parts[1][1], False, out)
    torch.cuda.synchronize()
    fin = torch.isfinite(l_all)
    assert torch.equal(fin, torch.isfinite(acc_l))
    assert (acc_l[fin] - l_all[fin]).abs().max().item() < 1e-4
    rel = ((out.float() - O_all.float()).norm() / O_all.float().norm()).item()
    assert rel < 5e-3, rel
    blk.close()


@pytest.mark.parametrize("masked", ["first_block", "all"])
def test_grid_with_fully_masked_key_blocks(masked):
    """A key block whose every key is masked has lse = +inf and weight 0 in the
    merge; with every key masked o = 0 and out = z + bo (bo = 0 here)."""
    N, p = 256, 2
    inp = workloads.make_inputs(N, "bf16", 150, "random:0.1")
    mask = torch.ones(N, dtype=torch.uint8)
    if masked == "first_block":
        mask[: N // p] = 0
    else:
        mask[:] = 0
    inp = workloads.Inputs(**{**{f: getattr(inp, f) for f in (
        "Z", "gamma", "beta", "Wq", "Wk", "Wv", "Wg", "bg", "Wb", "Wo", "bo")}, "mask": mask})
    blk = binding.TriangleAttention(inp.weights(), dtype=torch.bfloat16)
    for orientation in (0, 1):
        got = _grid(inp, blk, p, orientation)
        if masked == "all":
            assert torch.equal(got.contiguous().view(torch.int16), inp.Z.cuda().view(torch.int16))
        else:
            ref = oracle.tri_attn_full(to_problem(inp), orientation)
            st = compare(got.double().cpu().numpy(), ref, inp.Z.double().numpy(), "bf16")
            assert_within(st, "bf16", f"2D grid, first key block masked, orientation {orientation}")
    blk.close()


def test_block_gate_in_place():
    N = 128
    inp = workloads.make_inputs(N, "bf16", 160, "random:0.1")
    blk = binding.TriangleAttention(inp.weights(), dtype=torch.bfloat16)
    Z = inp.Z.cuda()
    Q, K, V, bias, ld = blk.block_project(Z, inp.mask.cuda())
    O, _ = blk.block_attend(Q, K, V, bias, ld)
    want = blk.block_gate(Z, O)
    Z2 = Z.clone()
    got = blk.block_gate(Z2, O, out=Z2)
    torch.cuda.synchronize()
    assert got.data_ptr() == Z2.data_ptr()
    assert torch.equal(got.view(torch.int16), want.view(torch.int16))
    # an output that overlaps Z without being Z (one row of pairs apart) is rejected
    big = torch.empty(N + 1, N, 128, dtype=torch.bfloat16, device="cuda")
    big[:N].copy_(Z)
    with pytest.raises(binding.TriAttnError) as err:
        blk.block_gate(big[:N], O, out=big[1:])
    assert err.value.code == binding.TRI_ATTN_ERR_ALIAS
    blk.close()
