"""The allocation-free entry point, tri_attn_forward_noalloc, against the
regular handle-based entry point.

It exists for callers that must not allocate device memory (a host application
that owns all device memory, or latency-critical paths that cannot afford a
cudaMalloc): all its scratch sits in one static device array inside the
library.  Kept in a file of its own that pytest collects last; it passes alone
in a fresh process and after the other tests.
"""
import ctypes

import pytest
import torch

from gpu_util import TOL_BF16_MAXABS, TOL_BF16_RELL2
from protein_pair_representation_layernorm_b200 import binding, workloads

pytestmark = pytest.mark.gpu


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


def _close(got: torch.Tensor, ref: torch.Tensor):
    d = (got.double() - ref.double())
    rel = (d.norm() / ref.double().norm()).item()
    mx = d.abs().max().item()
    assert torch.isfinite(got.float()).all()
    assert rel <= TOL_BF16_RELL2 and mx <= TOL_BF16_MAXABS, (rel, mx)


def test_noalloc_matches_handle_entry_point_twice():
    inp = workloads.make_inputs(200, "bf16", 61, "random:0.1")
    w = {k: v.cuda().to(torch.bfloat16).contiguous() for k, v in inp.weights().items()}
    Z = inp.Z.cuda()
    mask = inp.mask.cuda()
    blk = binding.TriangleAttention(inp.weights(), dtype=torch.bfloat16)
    p = _params(w)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for orientation in (binding.TRI_ATTN_STARTING, binding.TRI_ATTN_ENDING):  # two calls in a row
        out = torch.empty_like(Z)
        rc = binding.tri_attn_forward_noalloc(p, ctypes.c_void_p(Z.data_ptr()), 200,
                                              ctypes.c_void_p(mask.data_ptr()), orientation,
                                              ctypes.c_void_p(out.data_ptr()), stream,
                                              binding.TRI_ATTN_FLAG_SYNC)
        assert rc == binding.TRI_ATTN_OK, binding.tri_attn_status_string(rc)
        ref = blk.forward(Z, orientation, mask, flags=binding.TRI_ATTN_FLAG_SYNC)
        _close(out, ref)
    blk.close()


def test_noalloc_rejects_sizes_beyond_its_scratch():
    inp = workloads.make_inputs(8, "bf16", 62)
    w = {k: v.cuda().to(torch.bfloat16).contiguous() for k, v in inp.weights().items()}
    p = _params(w)
    N = 4096  # needs far more than the 32 MiB static scratch; nothing is launched
    dummy = torch.empty(16, dtype=torch.bfloat16, device="cuda")
    rc = binding.tri_attn_forward_noalloc(p, ctypes.c_void_p(dummy.data_ptr()), N, None, 0,
                                          ctypes.c_void_p(dummy.data_ptr()), None, 0)
    assert rc == binding.TRI_ATTN_ERR_UNSUPPORTED
