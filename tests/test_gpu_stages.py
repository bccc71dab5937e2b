"""Step-by-step checks of the three bf16 kernels on the GPU.

Each kernel's output (read from the handle's workspace after a forward call)
is compared with a plain PyTorch fp32 evaluation of that step computed from
the previous step's GPU output, so a failure names the kernel at fault.
"""
import math

import pytest
import torch
import torch.nn.functional as F

from protein_pair_representation_layernorm_b200 import binding, workloads
from gpu_util import device_view, run_gpu

pytestmark = pytest.mark.gpu

LOG2E = 1.0 / math.log(2.0)


def _setup(N, orientation, mask="random:0.2", seed=21):
    inp = workloads.make_inputs(N, "bf16", seed, mask)
    out, blk = run_gpu(inp, orientation)
    ws = blk.debug_workspace()
    assert ws["g"] is None  # the bf16 path recomputes the gate in gate_out
    rows = ws["rows"]
    assert rows == N
    ld = ws["ld_bias"]
    bf = torch.bfloat16
    t = {
        "q": device_view(ws["q"], (N, 4, N, 32), bf).float(),
        "k": device_view(ws["k"], (N, 4, N, 32), bf).float(),
        "v": device_view(ws["v"], (N, 4, N, 32), bf).float(),
        "o": device_view(ws["o"], (N, 4, N, 32), bf).float(),
        "bias": device_view(ws["bias"], (4, N, ld), bf).float(),
    }
    return inp, out, blk, t, ld


def _problem_view(z, orientation):
    return z if orientation == 0 else z.transpose(0, 1)


@pytest.mark.parametrize("orientation", [0, 1])
def test_pair_ln_proj_matches_torch(orientation):
    N = 200
    inp, out, blk, t, ld = _setup(N, orientation)
    w = {k: v.cuda().float() for k, v in inp.weights().items()}
    zf = _problem_view(inp.Z.cuda().float(), orientation)
    x = F.layer_norm(zf, (128,), w["gamma"], w["beta"], eps=1e-5)
    xb = x.bfloat16().float()  # the MMA consumes x rounded to bf16
    qs = LOG2E / math.sqrt(32.0)
    q = (xb @ w["Wq"].T * qs).reshape(N, N, 4, 32).permute(0, 2, 1, 3)
    k = (xb @ w["Wk"].T).reshape(N, N, 4, 32).permute(0, 2, 1, 3)
    v = (xb @ w["Wv"].T).reshape(N, N, 4, 32).permute(0, 2, 1, 3)
    bias = (x @ w["Wb"].T * LOG2E).permute(2, 0, 1)
    valid = inp.mask.cuda().bool()
    for name, ref in (("q", q), ("k", k), ("v", v)):
        got = t[name]
        err = (got - ref).abs().max().item()
        assert err < 2e-2 + 1e-2 * ref.abs().max().item(), f"{name}: max err {err}"
    gb = t["bias"]
    # masked keys and padding columns carry a huge finite negative logit (-3e38)
    assert (gb[:, :, :N][:, :, ~valid] <= -1e38).all() and torch.isfinite(gb).all()
    assert (gb[:, :, N:] <= -1e38).all()
    err = (gb[:, :, :N][:, :, valid] - bias[:, :, valid]).abs().max().item()
    assert err < 3e-2, f"bias max err {err}"


@pytest.mark.parametrize("orientation", [0, 1])
def test_tri_attn_fwd_matches_torch(orientation):
    N = 200
    inp, out, blk, t, ld = _setup(N, orientation)
    q, k, v, o = t["q"], t["k"], t["v"], t["o"]
    b = t["bias"][:, :, :N]                      # (H, j, k), base-2 logits
    s = torch.einsum("rhjc,rhkc->rhjk", q, k) + b.unsqueeze(0)
    p = torch.softmax(s * math.log(2.0), dim=-1)
    ref = torch.einsum("rhjk,rhkc->rhjc", p, v)
    err = (o - ref).abs().max().item()
    rel = ((o - ref).norm() / ref.norm()).item()
    assert err < 2e-2 and rel < 1e-2, f"attention max err {err} rel {rel}"


@pytest.mark.parametrize("orientation", [0, 1])
def test_gate_out_matches_torch(orientation):
    N = 200
    inp, out, blk, t, ld = _setup(N, orientation)
    w = {k: v.cuda().float() for k, v in inp.weights().items()}
    o = t["o"].permute(0, 2, 1, 3).reshape(N, N, 128)
    z = _problem_view(inp.Z.cuda().float(), orientation)
    # the gate, recomputed from LayerNorm(z) rounded to bf16 (the MMA operand)
    xb = F.layer_norm(z, (128,), w["gamma"], w["beta"], eps=1e-5).bfloat16().float()
    g = torch.sigmoid(xb @ w["Wg"].T + w["bg"])
    go = (g * o).bfloat16().float()
    ref = z + go @ w["Wo"].T + w["bo"]
    got = _problem_view(out.float(), orientation)
    err = (got - ref).abs().max().item()
    assert err < 2e-2, f"gate_out max err {err}"


def test_all_masked_leaves_z():
    inp = workloads.make_inputs(70, "bf16", 3, "all")
    for orientation in (0, 1):
        out, _ = run_gpu(inp, orientation)
        assert torch.equal(out.cpu().view(torch.int16), inp.Z.view(torch.int16))
