"""Error paths, driven from the host: a withheld copy in each kernel (its
consumers' bounded waits expire, they release TMEM and leave, the call
reports TRI_ATTN_ERR_TIMEOUT) and a failed workspace allocation (the call
returns TRI_ATTN_ERR_OOM before any launch and leaks nothing).  Nothing here
faults, traps or hangs the GPU; after each failure the next call on the same
handle and context must be correct."""
import numpy as np
import pytest
import torch

import oracle
from conftest import to_problem
from gpu_util import assert_within, compare, run_gpu
from protein_pair_representation_layernorm_b200 import binding, workloads

pytestmark = pytest.mark.gpu


def _parity(inp, blk, orientation):
    out, _ = run_gpu(inp, orientation, blk=blk)
    ref = oracle.tri_attn_full(to_problem(inp), orientation)
    st = compare(out.double().cpu().numpy(), ref, inp.Z.double().numpy(), "bf16")
    assert_within(st, "bf16", "after the injected failure")


@pytest.mark.parametrize("flag", [binding.TRI_ATTN_FLAG_DEBUG_STALL_PROJ,
                                  binding.TRI_ATTN_FLAG_DEBUG_STALL,
                                  binding.TRI_ATTN_FLAG_DEBUG_STALL_GATE],
                         ids=["pair_ln_proj", "tri_attn_fwd", "gate_out"])
def test_withheld_copy_reports_timeout_and_recovers(flag):
    # N = 200: the persistent kernels' CTA 0 owns several tiles, so the
    # producer also meets a stage that will never be released
    inp = workloads.make_inputs(200, "bf16", 48, "random:0.1")
    blk = binding.TriangleAttention(inp.weights(), dtype=torch.bfloat16)
    Z = inp.Z.cuda()
    mask = inp.mask.cuda()
    out = torch.empty_like(Z)
    rc = binding.tri_attn_forward(blk.handle, Z.data_ptr(), 200, mask.data_ptr(), 1,
                                  out.data_ptr(), None, flag | binding.TRI_ATTN_FLAG_SYNC)
    assert rc == binding.TRI_ATTN_ERR_TIMEOUT, binding.tri_attn_status_string(rc)
    assert blk.status() == binding.TRI_ATTN_OK  # the sticky status was cleared
    _parity(inp, blk, 1)
    blk.close()


def test_failed_workspace_allocation_returns_oom_and_recovers():
    N = 160
    inp = workloads.make_inputs(N, "bf16", 49, "random:0.1")
    blk = binding.TriangleAttention(inp.weights(), dtype=torch.bfloat16)
    # a first, smaller call leaves a workspace that the size-160 call must grow
    small = workloads.make_inputs(48, "bf16", 49)
    run_gpu(small, 0, blk=blk)
    Z = inp.Z.cuda()
    out = torch.empty_like(Z)
    torch.cuda.synchronize()
    free_before = torch.cuda.mem_get_info()[0]
    rc = binding.tri_attn_forward(blk.handle, Z.data_ptr(), N, None, 0, out.data_ptr(), None,
                                  binding.TRI_ATTN_FLAG_DEBUG_FAIL_ALLOC)
    assert rc == binding.TRI_ATTN_ERR_OOM
    torch.cuda.synchronize()
    # the old workspace was released and nothing new is held
    assert torch.cuda.mem_get_info()[0] >= free_before
    ws = blk.debug_workspace()
    assert ws["q"] is None and ws["o"] is None and ws["rows"] == 0
    assert blk.status() == binding.TRI_ATTN_OK
    _parity(inp, blk, 0)
    # with a workspace already large enough the flag has nothing to fail
    rc = binding.tri_attn_forward(blk.handle, Z.data_ptr(), N, None, 0, out.data_ptr(), None,
                                  binding.TRI_ATTN_FLAG_DEBUG_FAIL_ALLOC | binding.TRI_ATTN_FLAG_SYNC)
    assert rc == binding.TRI_ATTN_OK
    blk.close()
