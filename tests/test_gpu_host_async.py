"""The asynchronous host-buffer entry point: a stream of independent problems
enqueued back to back (uploads, blocks and downloads overlapping across
calls) must give, for every call, exactly the result of the synchronous call
on the same inputs, bit for bit."""
import pytest
import torch

from protein_pair_representation_layernorm_b200 import binding, workloads
from gpu_util import block_for

pytestmark = pytest.mark.gpu


def _sync_ref(blk, inp, orients):
    return blk.forward_host(inp.Z.clone().pin_memory(), orients, inp.mask)


def test_pipelined_calls_equal_synchronous_calls():
    N = 160
    base = workloads.make_inputs(N, "bf16", 300, "random:0.1")
    blk = block_for(base)
    # six problems on the same weights (three go round the staging ring twice),
    # each its own input and output buffer, orientation sequences mixed
    probs = []
    for k in range(6):
        inp = workloads.make_inputs(N, "bf16", 301 + k, "random:0.1")
        inp = workloads.Inputs(Z=inp.Z, **{a: getattr(base, a) for a in (
            "mask", "gamma", "beta", "Wq", "Wk", "Wv", "Wg", "bg", "Wb", "Wo", "bo")})
        probs.append(inp)
    orients = [[0, 1], [1, 0], [0, 1], [1], [0, 1], []]
    st = torch.cuda.Stream()
    outs = []
    zs = [p.Z.clone().pin_memory() for p in probs]
    for z, o in zip(zs, orients):
        outs.append(blk.forward_host_async(z, o, base.mask, stream=st))
    assert blk.host_wait() == binding.TRI_ATTN_OK
    for p, o, got, z in zip(probs, orients, outs, zs):
        want = _sync_ref(blk, p, o)
        assert torch.equal(got.view(torch.int16), want.view(torch.int16))
        assert torch.equal(z, p.Z)  # inputs untouched
    blk.close()


def test_pipelined_in_place_and_shared_output():
    """A call may write its result over its own input; several in-flight calls
    may share one output buffer (their downloads run in call order)."""
    N = 128
    inp = workloads.make_inputs(N, "bf16", 310, "random:0.2")
    blk = block_for(inp)
    want = _sync_ref(blk, inp, [0, 1])
    st = torch.cuda.Stream()
    inplace = inp.Z.clone().pin_memory()
    blk.forward_host_async(inplace, [0, 1], inp.mask, out=inplace, stream=st)
    shared = torch.empty_like(inplace).pin_memory()
    srcs = [inp.Z.clone().pin_memory() for _ in range(4)]
    for z in srcs:
        blk.forward_host_async(z, [0, 1], inp.mask, out=shared, stream=st)
    assert blk.host_wait() == binding.TRI_ATTN_OK
    assert torch.equal(inplace.view(torch.int16), want.view(torch.int16))
    assert torch.equal(shared.view(torch.int16), want.view(torch.int16))
    blk.close()


def test_pipelined_growing_problem_size():
    """A larger N waits for the calls in flight, then reallocates the ring."""
    small = workloads.make_inputs(96, "bf16", 320, "random:0.1")
    blk = block_for(small)
    big = workloads.make_inputs(200, "bf16", 321, "random:0.1")
    big = workloads.Inputs(Z=big.Z, mask=None, **{a: getattr(small, a) for a in (
        "gamma", "beta", "Wq", "Wk", "Wv", "Wg", "bg", "Wb", "Wo", "bo")})
    st = torch.cuda.Stream()
    z1, z2 = small.Z.clone().pin_memory(), big.Z.clone().pin_memory()
    o1 = blk.forward_host_async(z1, [0, 1], small.mask, stream=st)
    o2 = blk.forward_host_async(z2, [1, 0], None, stream=st)
    assert blk.host_wait() == binding.TRI_ATTN_OK
    assert torch.equal(o1.view(torch.int16), _sync_ref(blk, small, [0, 1]).view(torch.int16))
    assert torch.equal(o2.view(torch.int16), _sync_ref(blk, big, [1, 0]).view(torch.int16))
    blk.close()


def test_pipelined_calls_at_the_benchmark_size():
    """N = 1536 (the benchmark's problem), four pipelined calls on two
    alternating inputs: each result equals the synchronous call bit for bit."""
    N = 1536
    a = workloads.workload_inputs(3)
    b = workloads.make_inputs(N, "bf16", 333)
    b = workloads.Inputs(Z=b.Z, **{k: getattr(a, k) for k in (
        "mask", "gamma", "beta", "Wq", "Wk", "Wv", "Wg", "bg", "Wb", "Wo", "bo")})
    blk = block_for(a)
    want = [_sync_ref(blk, p, [0, 1]) for p in (a, b)]
    st = torch.cuda.Stream()
    zs = [a.Z.clone().pin_memory(), b.Z.clone().pin_memory()]
    outs = [blk.forward_host_async(zs[k % 2], [0, 1], a.mask, stream=st) for k in range(4)]
    assert blk.host_wait() == binding.TRI_ATTN_OK
    for k, got in enumerate(outs):
        assert torch.equal(got.view(torch.int16), want[k % 2].view(torch.int16)), k
    blk.close()


def test_pipelined_calls_on_an_fp32_handle():
    """fp32 handles upload Z whole (no piecewise projection) and run the SIMT
    kernels; pipelined calls must still equal synchronous ones bit for bit."""
    N = 70
    inp = workloads.make_inputs(N, "f32", 340, "random:0.1")
    blk = block_for(inp)
    st = torch.cuda.Stream()
    zs = [inp.Z.clone().pin_memory() for _ in range(4)]
    orients = [[0, 1], [1], [1, 0], [0]]
    outs = [blk.forward_host_async(z, o, inp.mask, stream=st) for z, o in zip(zs, orients)]
    assert blk.host_wait() == binding.TRI_ATTN_OK
    for got, o in zip(outs, orients):
        want = _sync_ref(blk, inp, o)
        assert torch.equal(got.view(torch.int32), want.view(torch.int32))
    blk.close()
