"""GPU parity: the CUDA path against the fp64 CPU oracle on the same seeded
inputs, through the C ABI.

Tolerances (on out): fp32 inputs max-abs 1e-4; bf16 inputs with fp32
accumulation rel-L2 5e-3 and max-abs 2e-2.  Full tensors where the oracle
finishes in seconds; at the large workloads the oracle evaluates sampled
lines (rows for the starting node, columns for the ending node) one by one,
in the same launch configuration the benchmark times.
"""
import numpy as np
import pytest
import torch

import oracle
from conftest import to_problem
from gpu_util import (assert_within, block_for, compare, lines_of, run_gpu, z_lines)
from protein_pair_representation_layernorm_b200 import binding, workloads

pytestmark = pytest.mark.gpu


def _check_full(inp, orientation, dtype, what):
    out, _ = run_gpu(inp, orientation)
    p = to_problem(inp)
    ref = oracle.tri_attn_full(p, orientation)
    st = compare(out.double().cpu().numpy(), ref, inp.Z.double().numpy(), dtype)
    assert_within(st, dtype, what)
    return st


def _check_lines(inp, orientation, lines, dtype, what, out=None):
    if out is None:
        out, _ = run_gpu(inp, orientation)
    p = to_problem(inp)
    bias = oracle.bias_all(p)
    ref = oracle.tri_attn(p, orientation, lines, bias=bias)
    got = lines_of(out, orientation, lines)
    st = compare(got, ref, z_lines(inp.Z, orientation, lines), dtype)
    assert_within(st, dtype, what)
    return st


def _sample_lines(N, n, seed):
    rng = np.random.default_rng(seed)
    fixed = [0, N - 1, N // 2]
    rest = rng.choice(N, size=min(N, n) - len(fixed), replace=False).tolist()
    return sorted(set(fixed + rest))


def test_workload0_fp32_full():
    inp = workloads.workload_inputs(0)
    _check_full(inp, 0, "f32", "workload 0")


@pytest.mark.parametrize("orientation", [0, 1])
def test_workload1_full(orientation):
    inp = workloads.workload_inputs(1)
    _check_full(inp, orientation, "bf16", f"workload 1 orient {orientation}")


@pytest.mark.parametrize("orientation", [0, 1])
def test_workload2_sampled(orientation):
    inp = workloads.workload_inputs(2)
    # rows spanning all three chains, chain boundaries included
    lines = sorted(set(_sample_lines(768, 16, 2) + [255, 256, 511, 512]))
    _check_lines(inp, orientation, lines, "bf16", f"workload 2 orient {orientation}")


@pytest.mark.parametrize("orientation", [0, 1])
def test_workload3_sampled(orientation):
    inp = workloads.workload_inputs(3)
    _check_lines(inp, orientation, _sample_lines(1536, 8, 3), "bf16",
                 f"workload 3 orient {orientation}")


@pytest.mark.parametrize("orientation", [0, 1])
def test_workload4_sampled(orientation):
    inp = workloads.workload_inputs(4)
    masked = np.flatnonzero(inp.mask.numpy() == 0)
    lines = sorted(set(_sample_lines(4096, 5, 4) + [int(masked[0])]))
    _check_lines(inp, orientation, lines, "bf16", f"workload 4 orient {orientation}")


# key-tile counts T = ceil(N / 64): 1, 1, 2, 3, 4, 5, 7 (the attention kernel's
# issue loops are unrolled over its 4 stages: 300 and 420 end one and three
# tiles into a second round); query tiles of 128 are ragged for all but N = 1
@pytest.mark.parametrize("N", [1, 7, 97, 130, 200, 300, 420])
@pytest.mark.parametrize("orientation", [0, 1])
def test_ragged_sizes(N, orientation):
    inp = workloads.make_inputs(N, "bf16", 100 + N, "random:0.15" if N > 1 else "none")
    _check_full(inp, orientation, "bf16", f"N={N} orient {orientation}")


@pytest.mark.parametrize("mask", ["first:70", "first:130", "tail:1", "random:0.9"])
def test_mask_patterns(mask):
    inp = workloads.make_inputs(160, "bf16", 31, mask)
    for orientation in (0, 1):
        _check_full(inp, orientation, "bf16", f"mask {mask} orient {orientation}")


@pytest.mark.parametrize("N", [5, 70])
def test_fp32_small(N):
    inp = workloads.make_inputs(N, "f32", 50 + N, "random:0.2")
    for orientation in (0, 1):
        _check_full(inp, orientation, "f32", f"fp32 N={N} orient {orientation}")


def test_in_place_equals_out_of_place():
    inp = workloads.make_inputs(150, "bf16", 41, "random:0.1")
    for orientation in (0, 1):
        ref, blk = run_gpu(inp, orientation)
        got, _ = run_gpu(inp, orientation, blk=blk, inplace=True)
        assert torch.equal(ref.view(torch.int16), got.view(torch.int16))


def test_deterministic():
    inp = workloads.make_inputs(300, "bf16", 42, "random:0.05")
    a, blk = run_gpu(inp, 1)
    b, _ = run_gpu(inp, 1, blk=blk)
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))


def test_row_chunking_matches_single_pass():
    inp = workloads.make_inputs(260, "bf16", 43, "random:0.1")
    blk = block_for(inp)
    ref, _ = run_gpu(inp, 0, blk=blk)
    ref_e, _ = run_gpu(inp, 1, blk=blk)
    full = binding.tri_attn_workspace_bytes(binding.TRI_ATTN_BF16, 260)
    blk.set_workspace_limit(full // 3)
    got, _ = run_gpu(inp, 0, blk=blk)
    got_e, _ = run_gpu(inp, 1, blk=blk)
    ws = blk.debug_workspace()
    assert ws["rows"] < 260
    assert torch.equal(ref.view(torch.int16), got.view(torch.int16))
    assert torch.equal(ref_e.view(torch.int16), got_e.view(torch.int16))


def test_sequence_starting_then_ending():
    """The benchmark step: starting node, then ending node on its output."""
    inp = workloads.make_inputs(96, "bf16", 44, "random:0.1")
    out1, blk = run_gpu(inp, 0)
    out2 = blk.forward(out1, 1, inp.mask.cuda(), flags=binding.TRI_ATTN_FLAG_SYNC)
    p = to_problem(inp)
    r1 = oracle.tri_attn_full(p, 0)
    # the second block reads the GPU's own bf16 output of the first
    inp2 = workloads.Inputs(Z=out1.cpu(), **{k: getattr(inp, k) for k in (
        "mask", "gamma", "beta", "Wq", "Wk", "Wv", "Wg", "bg", "Wb", "Wo", "bo")})
    r2 = oracle.tri_attn_full(to_problem(inp2), 1)
    st = compare(out2.double().cpu().numpy(), r2, out1.double().cpu().numpy(), "bf16")
    assert_within(st, "bf16", "start then end")


# The last block of a host-buffer call runs in ~8 row chunks whose outputs are
# read back while later chunks compute (rows of Z when the starting node comes
# last, strided columns when the ending node does): the result must equal the
# device path bit for bit.
@pytest.mark.parametrize("N,dtype,orients", [(120, "bf16", [0, 1]), (97, "bf16", [1, 0]),
                                             (130, "bf16", [1]), (64, "bf16", [0]),
                                             (70, "f32", [0, 1]), (33, "bf16", [])])
def test_host_buffer_entry_point(N, dtype, orients):
    inp = workloads.make_inputs(N, dtype, 45 + N, "random:0.1")
    blk = block_for(inp)
    z_host = inp.Z.clone().pin_memory()
    got = blk.forward_host(z_host, orients, inp.mask)
    want = inp.Z.cuda()
    for o in orients:
        want = blk.forward(want, o, inp.mask.cuda(), flags=binding.TRI_ATTN_FLAG_SYNC)
    bits = torch.int16 if dtype == "bf16" else torch.int32
    assert torch.equal(got.view(bits), want.cpu().view(bits))
    assert torch.equal(z_host, inp.Z)  # the input buffer is left alone


def test_kernel_times_reported():
    inp = workloads.make_inputs(256, "bf16", 46)
    blk = block_for(inp)
    run_gpu(inp, 0, blk=blk, flags=binding.TRI_ATTN_FLAG_TIME_KERNELS)
    ms, n = blk.kernel_times()
    assert len(ms) == 3 and all(m > 0 for m in ms) and n == [1, 1, 1]
    ms, n = blk.kernel_times()
    assert n == [0, 0, 0]


def test_invalid_arguments_do_not_launch():
    inp = workloads.make_inputs(16, "bf16", 47)
    blk = block_for(inp)
    Z = inp.Z.cuda()
    h = blk.handle
    L = binding
    assert L.tri_attn_forward(h, None, 16, None, 0, Z.data_ptr(), None, 0) == L.TRI_ATTN_ERR_INVALID_ARG
    assert L.tri_attn_forward(h, Z.data_ptr(), 0, None, 0, Z.data_ptr(), None, 0) == L.TRI_ATTN_ERR_INVALID_ARG
    assert L.tri_attn_forward(h, Z.data_ptr(), 16, None, 2, Z.data_ptr(), None, 0) == L.TRI_ATTN_ERR_INVALID_ARG
    assert L.tri_attn_forward(h, Z.data_ptr() + 2, 16, None, 0, Z.data_ptr(), None, 0) == L.TRI_ATTN_ERR_INVALID_ARG
    big = torch.empty(16 * 16 * 128 + 64, dtype=torch.bfloat16, device="cuda")
    assert L.tri_attn_forward(h, big.data_ptr(), 16, None, 0, big.data_ptr() + 256, None, 0) == L.TRI_ATTN_ERR_ALIAS


def test_bounded_wait_reports_timeout_and_recovers():
    """Fault injection on the host side of a bounded wait: the producer of one
    CTA withholds a stage, its consumers give up after the wait limit, the call
    reports TRI_ATTN_ERR_TIMEOUT, and the next call on the same context works."""
    inp = workloads.make_inputs(64, "bf16", 48)
    blk = block_for(inp)
    Z = inp.Z.cuda()
    out = torch.empty_like(Z)
    rc = binding.tri_attn_forward(blk.handle, Z.data_ptr(), 64, None, 0, out.data_ptr(), None,
                                  binding.TRI_ATTN_FLAG_DEBUG_STALL | binding.TRI_ATTN_FLAG_SYNC)
    assert rc == binding.TRI_ATTN_ERR_TIMEOUT
    assert blk.status() == binding.TRI_ATTN_OK  # status cleared
    _check_full(inp, 0, "bf16", "after timeout")
