"""The allocation-free entry point, tri_attn_forward_noalloc, against the
regular handle-based entry point.

It exists for callers that must not allocate device memory (a host application
that owns all device memory, or latency-critical paths that cannot afford a
cudaMalloc): all its scratch sits in one static device array inside the
library.  Both paths run the same kernels, and row chunking leaves results
unchanged bit for bit, so the no-alloc output must equal the handle path's
exactly.  Kept in a file of its own that pytest collects last; it passes alone
in a fresh process and after the other tests.
"""
import ctypes

import pytest
import torch

from protein_pair_representation_layernorm_b200 import binding, workloads

pytestmark = pytest.mark.gpu

MAX_N = 1856  # the largest N whose whole bias plus one three-row chunk fits the 32 MiB array


def _params(w: dict) -> binding.tri_attn_params:
    p = binding.tri_attn_params()
    p.c_z, p.n_heads, p.head_dim = 128, 4, 32
    p.dtype = binding.TRI_ATTN_BF16
    p.ln_eps = 1e-5
    p.ln_gamma, p.ln_beta = w["gamma"].data_ptr(), w["beta"].data_ptr()
    p.w_q, p.w_k, p.w_v, p.w_g = (w[k].data_ptr() for k in ("Wq", "Wk", "Wv", "Wg"))
    p.b_g, p.w_b = w["bg"].data_ptr(), w["Wb"].data_ptr()
    p.w_o, p.b_o = w["Wo"].data_ptr(), w["bo"].data_ptr()
    return p


def _device_weights(inp):
    return {k: v.cuda().to(torch.bfloat16).contiguous() for k, v in inp.weights().items()}


def _noalloc(p, Z, N, mask, orientation, out):
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return binding.tri_attn_forward_noalloc(
        p, ctypes.c_void_p(Z.data_ptr()), N,
        None if mask is None else ctypes.c_void_p(mask.data_ptr()), orientation,
        ctypes.c_void_p(out.data_ptr()), stream, binding.TRI_ATTN_FLAG_SYNC)


def _bits(t):
    return t.view(torch.int16)


def test_noalloc_matches_handle_entry_point_twice():
    """Two calls in a row (both orientations) equal the handle path bit for
    bit, and the second call leaves the device's free memory unchanged."""
    N = 200
    inp = workloads.make_inputs(N, "bf16", 61, "random:0.1")
    w = _device_weights(inp)
    Z = inp.Z.cuda()
    mask = inp.mask.cuda()
    blk = binding.TriangleAttention(inp.weights(), dtype=torch.bfloat16)
    p = _params(w)
    refs = [blk.forward(Z, o, mask, flags=binding.TRI_ATTN_FLAG_SYNC)
            for o in (binding.TRI_ATTN_STARTING, binding.TRI_ATTN_ENDING)]
    outs = [torch.empty_like(Z) for _ in refs]
    torch.cuda.synchronize()
    free_before = None
    for k, orientation in enumerate((binding.TRI_ATTN_STARTING, binding.TRI_ATTN_ENDING)):
        if k == 1:
            free_before = torch.cuda.mem_get_info()[0]
        rc = _noalloc(p, Z, N, mask, orientation, outs[k])
        assert rc == binding.TRI_ATTN_OK, binding.tri_attn_status_string(rc)
    torch.cuda.synchronize()
    free_after = torch.cuda.mem_get_info()[0]
    assert free_after == free_before, (free_before, free_after)
    for got, ref in zip(outs, refs):
        assert torch.equal(_bits(got), _bits(ref))
    blk.close()


def test_noalloc_largest_supported_size():
    """N = 1856 runs (in three-row chunks) and equals the handle path on
    sampled rows and columns, bit for bit; N = 1857 is rejected before any
    launch."""
    N = MAX_N
    inp = workloads.make_inputs(N, "bf16", 63, "random:0.05")
    w = _device_weights(inp)
    Z = inp.Z.cuda()
    mask = inp.mask.cuda()
    p = _params(w)
    out = torch.empty_like(Z)
    rc = _noalloc(p, Z, N, mask, binding.TRI_ATTN_ENDING, out)
    assert rc == binding.TRI_ATTN_OK, binding.tri_attn_status_string(rc)
    blk = binding.TriangleAttention(inp.weights(), dtype=torch.bfloat16)
    ref = blk.forward(Z, binding.TRI_ATTN_ENDING, mask, flags=binding.TRI_ATTN_FLAG_SYNC)
    idx = torch.tensor([0, 1, 2, 3, 895, 896, N - 4, N - 1], device="cuda")
    assert torch.equal(_bits(out.index_select(1, idx)), _bits(ref.index_select(1, idx)))
    assert torch.equal(_bits(out.index_select(0, idx)), _bits(ref.index_select(0, idx)))
    blk.close()
    rc = _noalloc(p, Z, N + 1, mask, binding.TRI_ATTN_STARTING, out)
    assert rc == binding.TRI_ATTN_ERR_UNSUPPORTED


def test_noalloc_rejects_sizes_beyond_its_scratch():
    inp = workloads.make_inputs(8, "bf16", 62)
    p = _params(_device_weights(inp))
    N = 4096  # needs far more than the 32 MiB static scratch; nothing is launched
    dummy = torch.empty(16, dtype=torch.bfloat16, device="cuda")
    rc = binding.tri_attn_forward_noalloc(p, ctypes.c_void_p(dummy.data_ptr()), N, None, 0,
                                          ctypes.c_void_p(dummy.data_ptr()), None, 0)
    assert rc == binding.TRI_ATTN_ERR_UNSUPPORTED
