"""Out-of-bounds writes and non-finite values, without a sanitizer: every
buffer the library writes for the caller (out on the device, out on the host,
the row-slab bias and output) sits between guard bands filled with a canary
pattern, which must be intact after the call; the inputs must be unchanged
and the outputs finite.  Sizes are ragged in both tile dimensions (queries in
tiles of 128, keys in tiles of 64)."""
import pytest
import torch

from protein_pair_representation_layernorm_b200 import binding, workloads
from protein_pair_representation_layernorm_b200.sharded import row_shards

pytestmark = pytest.mark.gpu

GUARD = 4096          # elements on each side
CANARY = -12345.0     # exactly representable in bf16 and fp32


def _guarded(shape, dtype, device):
    n = 1
    for s in shape:
        n *= s
    big = torch.full((n + 2 * GUARD,), CANARY, dtype=dtype, device=device)
    return big, big[GUARD:GUARD + n].view(shape)


def _guards_intact(big):
    return bool((big[:GUARD] == CANARY).all()) and bool((big[-GUARD:] == CANARY).all())


@pytest.mark.parametrize("N", [97, 130, 300])
@pytest.mark.parametrize("orientation", [0, 1])
def test_forward_writes_only_out(N, orientation):
    inp = workloads.make_inputs(N, "bf16", 900 + N, "random:0.2")
    blk = binding.TriangleAttention(inp.weights())
    Z = inp.Z.cuda()
    Z0 = Z.clone()
    big, out = _guarded(tuple(Z.shape), torch.bfloat16, "cuda")
    blk.forward(Z, orientation, inp.mask.cuda(), out=out, flags=binding.TRI_ATTN_FLAG_SYNC)
    assert _guards_intact(big)
    assert torch.equal(Z, Z0)
    assert torch.isfinite(out.float()).all()
    blk.close()


def test_rows_calls_write_only_their_buffers():
    N = 200
    inp = workloads.make_inputs(N, "bf16", 901, "random:0.2")
    blk = binding.TriangleAttention(inp.weights())
    Z = inp.Z.cuda()
    mask = inp.mask.cuda()
    ld = blk.bias_ld(N)
    parts, bigs = [], []
    for r0, n in row_shards(N, 3):
        bigb, b = _guarded((4, n, ld), torch.bfloat16, "cuda")
        blk.rows_bias(Z[r0:r0 + n].contiguous(), N, r0, mask, bias_rows=b)
        parts.append(b)
        bigs.append(bigb)
    torch.cuda.synchronize()
    assert all(_guards_intact(b) for b in bigs)
    bias_all = torch.cat(parts, dim=1).contiguous()
    for r0, n in row_shards(N, 3):
        bigo, o = _guarded((n, N, 128), torch.bfloat16, "cuda")
        blk.rows_forward(Z[r0:r0 + n].contiguous(), N, r0, bias_all, mask, out=o)
        torch.cuda.synchronize()
        assert _guards_intact(bigo)
        assert torch.isfinite(o.float()).all()
    blk.close()


def test_forward_host_writes_only_out():
    N = 150
    inp = workloads.make_inputs(N, "bf16", 902, "random:0.2")
    blk = binding.TriangleAttention(inp.weights())
    z_host = inp.Z.clone().pin_memory()
    big, out = _guarded(tuple(z_host.shape), torch.bfloat16, "cpu")
    big = big.pin_memory()
    out = big[GUARD:GUARD + out.numel()].view(out.shape)
    blk.forward_host(z_host, [0, 1], inp.mask, out=out)
    assert _guards_intact(big)
    assert torch.equal(z_host, inp.Z)
    assert torch.isfinite(out.float()).all()
    blk.close()
