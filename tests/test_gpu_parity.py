"""GPU parity: the CUDA path against the fp64 CPU oracle on the same seeded
inputs, through the C ABI.

Tolerances (on out): fp32 inputs max-abs 1e-4; bf16 inputs with fp32
accumulation rel-L2 5e-3 and max-abs 2e-2.  The attention update is held to
rel-L2 2e-2 as well: the GPU's attention output o (before the gate, read from
the workspace) against the oracle's, at every bf16 workload and both
orientations; and out - z against oracle - z on inputs scaled by 2^-4 (exact
in bf16; LayerNorm leaves the update almost unchanged while the residual
shrinks sixteenfold, so the bf16 rounding of out no longer hides the update).
Full tensors where the oracle finishes in seconds; at the large workloads the
oracle evaluates sampled lines (rows for the starting node, columns for the
ending node) one by one, in the same launch configuration the benchmark
times.
"""
import functools

import numpy as np
import pytest
import torch

import oracle
from conftest import to_problem
from gpu_util import (assert_within, attn_output_lines, block_for, compare, lines_of,
                      log_parity, run_gpu, z_lines)
from protein_pair_representation_layernorm_b200 import binding, workloads

pytestmark = pytest.mark.gpu

NAMES = {0: "starting", 1: "ending"}


def _check_full(inp, orientation, dtype, what, with_o=True):
    out, blk = run_gpu(inp, orientation)
    p = to_problem(inp)
    if dtype == "bf16" and with_o:
        ref, ref_o = oracle.tri_attn(p, orientation, want_o=True)
        got_o = attn_output_lines(blk, inp.N, range(inp.N))
    else:
        ref, ref_o, got_o = oracle.tri_attn(p, orientation), None, None
    if orientation == 1:
        ref = np.ascontiguousarray(ref.transpose(1, 0, 2))
    st = compare(out.double().cpu().numpy(), ref, inp.Z.double().numpy(), dtype, got_o, ref_o)
    assert_within(st, dtype, what)
    log_parity(what, st, inp.N)
    return st


def _check_lines(inp, orientation, lines, dtype, what, update_at_out=False):
    out, blk = run_gpu(inp, orientation)
    p = to_problem(inp)
    bias = oracle.bias_all(p)
    ref, ref_o = oracle.tri_attn(p, orientation, lines, bias=bias, want_o=True)
    got = lines_of(out, orientation, lines)
    got_o = attn_output_lines(blk, inp.N, lines)
    st = compare(got, ref, z_lines(inp.Z, orientation, lines), dtype, got_o, ref_o)
    assert_within(st, dtype, what, update_at_out=update_at_out)
    log_parity(what, st, len(lines))
    blk.close()
    return st


def _sample_lines(N, n, seed, extra=()):
    """n distinct lines: 0, N-1, N/2, the extra ones, the rest seeded random."""
    rng = np.random.default_rng(seed)
    fixed = sorted(set([0, N - 1, N // 2] + [int(x) for x in extra]))
    pool = np.setdiff1d(np.arange(N), fixed)
    rest = rng.choice(pool, size=max(0, min(N, n) - len(fixed)), replace=False).tolist()
    return sorted(fixed + rest)


@functools.lru_cache(maxsize=1)
def _workload(w: int, scale_pow2: int = 0):
    inp = workloads.workload_inputs(w)
    if scale_pow2:
        # exact in bf16 (a power of two; no value of these workloads comes near underflow)
        inp = workloads.Inputs(Z=inp.Z * (2.0 ** scale_pow2), **{k: getattr(inp, k) for k in (
            "mask", "gamma", "beta", "Wq", "Wk", "Wv", "Wg", "bg", "Wb", "Wo", "bo")})
    return inp


def _lines_for(w: int, inp):
    N = inp.N
    if w == 2:  # rows spanning all three chains, chain boundaries included
        return _sample_lines(N, 24, 2, extra=[255, 256, 511, 512])
    if w == 3:
        return _sample_lines(N, 32, 3, extra=[127, 128, 1535 - 63])
    if w == 4:  # masked residues among the lines
        masked = np.flatnonzero(inp.mask.numpy() == 0)
        return _sample_lines(N, 32, 4, extra=masked[:3].tolist() + [4095 - 64])
    raise ValueError(w)
def test_workload0_fp32_full():
    inp = workloads.workload_inputs(0)
    _check_full(inp, 0, "f32", "workload 0")


@pytest.mark.parametrize("orientation", [0, 1])
def test_workload1_full(orientation):
    inp = workloads.workload_inputs(1)
    _check_full(inp, orientation, "bf16", f"workload 1 (N=384) {NAMES[orientation]}")


@pytest.mark.parametrize("orientation", [0, 1])
@pytest.mark.parametrize("w", [2, 3])
def test_workload_full_tensor(w, orientation):
    """Every line of the block's output (and of the attention output o) at
    N = 768 (three chains) and N = 1536 (the benchmark's size) against the
    oracle: a few minutes of fp64 on the host's cores."""
    inp = _workload(w)
    _check_full(inp, orientation, "bf16", f"workload {w} (N={inp.N}) full {NAMES[orientation]}")


@pytest.mark.parametrize("orientation", [0, 1])
@pytest.mark.parametrize("w", [2, 3, 4])
def test_workload_sampled(w, orientation):
    inp = _workload(w)
    lines = _lines_for(w, inp)
    _check_lines(inp, orientation, lines, "bf16", f"workload {w} (N={inp.N}) {NAMES[orientation]}")


@pytest.mark.parametrize("orientation", [0, 1])
@pytest.mark.parametrize("w", [1, 2, 3, 4])
def test_update_small_residual(w, orientation):
    """The attention update asserted at out level: the workload's Z times 2^-4,
    so out - z is no longer dwarfed by z and the update error is measured
    through every kernel, gate and output projection included."""
    inp = _workload(w, scale_pow2=-4)
    lines = list(range(inp.N)) if w == 1 else _lines_for(w, inp)
    _check_lines(inp, orientation, lines, "bf16",
                 f"workload {w} (N={inp.N}) x 2^-4 {NAMES[orientation]}", update_at_out=True)


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
