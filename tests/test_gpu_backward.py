"""Parity of the attention-core backward (tri_attn_attention_backward, fp32)
with the fp64 oracle's gradients, element by element, on seeded inputs that
span several tiles and a ragged tail, with masks, an all-masked problem and
N = 1; at N = 768 (every row on the GPU) sampled rows against the oracle and
the softmax-Jacobian property sum_k dbias[h][j][k] = 0 for every query."""
import numpy as np
import pytest
import torch

import oracle
from protein_pair_representation_layernorm_b200 import binding
from gpu_util import PARITY_LOG

pytestmark = pytest.mark.gpu

H, D = 4, 32
REL_TOL = 1e-4  # fp32 products and sums against fp64, relative to the largest |gradient|


def _inputs(seed, rows, N, mask_kind):
    rng = np.random.default_rng(seed)
    q = rng.normal(size=(rows, H, N, D)).astype(np.float32)
    k = rng.normal(size=(rows, H, N, D)).astype(np.float32)
    v = rng.normal(size=(rows, H, N, D)).astype(np.float32)
    g = rng.normal(size=(rows, H, N, D)).astype(np.float32)
    bias = rng.normal(size=(H, N, N)).astype(np.float32)
    if mask_kind is None:
        mask = None
    elif mask_kind == "random":
        mask = (rng.random(N) > 0.2).astype(np.uint8)
    elif mask_kind == "head":
        mask = np.ones(N, np.uint8)
        mask[:10] = 0
    elif mask_kind == "all":
        mask = np.zeros(N, np.uint8)
    return q, k, v, g, bias, mask


def _gpu(q, k, v, g, bias, mask):
    T = lambda a: torch.from_numpy(a).cuda()  # noqa: E731
    m = None if mask is None else torch.from_numpy(mask).cuda()
    out = binding.attention_backward(T(q), T(k), T(v), T(bias), T(g), m)
    torch.cuda.synchronize()
    return [t.cpu().numpy().astype(np.float64) for t in out]


def _to_oracle(a):  # [rows][H][N][d] -> (rows, N, H, d)
    return np.ascontiguousarray(a.transpose(0, 2, 1, 3)).astype(np.float64)


def _check(name, got, ref):
    scale = max(float(np.abs(ref).max()), 1e-30)
    err = float(np.abs(got - ref).max())
    PARITY_LOG.append(f"backward {name}: max_abs {err:.2e}, relative to max {err / scale:.2e}")
    assert err <= REL_TOL * scale + 1e-6, (name, err, scale)


@pytest.mark.parametrize("rows,N,mask_kind,seed", [
    (3, 70, None, 1), (2, 133, "random", 2), (2, 64, "head", 3), (4, 200, "random", 4),
    (2, 1, None, 5)])
def test_backward_matches_oracle(rows, N, mask_kind, seed):
    q, k, v, g, bias, mask = _inputs(seed, rows, N, mask_kind)
    dq, dk, dv, db = _gpu(q, k, v, g, bias, mask)
    rq, rk, rv, rb = oracle.tri_attn_core_bwd(_to_oracle(q), _to_oracle(k), _to_oracle(v),
                                              bias.astype(np.float64), _to_oracle(g), mask)
    tag = f"N={N} rows={rows} mask={mask_kind}"
    _check(f"dQ {tag}", _to_oracle(dq), rq)
    _check(f"dK {tag}", _to_oracle(dk), rk)
    _check(f"dV {tag}", _to_oracle(dv), rv)
    _check(f"dbias {tag}", db, rb)


def test_all_masked_gives_zero_gradients():
    q, k, v, g, bias, mask = _inputs(6, 2, 40, "all")
    for t in _gpu(q, k, v, g, bias, mask):
        assert not np.any(t)


def test_backward_is_deterministic():
    q, k, v, g, bias, mask = _inputs(7, 3, 150, "random")
    a = _gpu(q, k, v, g, bias, mask)
    b = _gpu(q, k, v, g, bias, mask)
    for x, y in zip(a, b):
        assert np.array_equal(x, y)


def test_backward_at_n768_sampled_rows_and_jacobian_property():
    rows, N = 768, 768
    q, k, v, g, bias, mask = _inputs(8, rows, N, "random")
    dq, dk, dv, db = _gpu(q, k, v, g, bias, mask)
    # dQ, dK, dV of a row depend on that row (and the shared bias) only
    for r in (0, 1, 383, 767):
        rq, rk, rv, _ = oracle.attend_bwd(_to_oracle(q[r:r + 1])[0], _to_oracle(k[r:r + 1])[0],
                                          _to_oracle(v[r:r + 1])[0], bias.astype(np.float64),
                                          _to_oracle(g[r:r + 1])[0], mask)
        _check(f"dQ N=768 row {r}", _to_oracle(dq[r:r + 1])[0], rq)
        _check(f"dK N=768 row {r}", _to_oracle(dk[r:r + 1])[0], rk)
        _check(f"dV N=768 row {r}", _to_oracle(dv[r:r + 1])[0], rv)
    # every softmax row's Jacobian annihilates constants: sum_k ds_jk = 0 for
    # each (row, h, j), hence for the bias gradient summed over rows
    sums = db.sum(axis=2)
    assert float(np.abs(sums).max()) <= 1e-4 * float(np.abs(db).max()) * np.sqrt(N)
    # masked keys receive no bias gradient
    assert not np.any(db[:, :, mask == 0])


@pytest.mark.parametrize("rows,N,mask_kind,seed", [(3, 70, None, 11), (2, 133, "random", 12),
                                                   (1, 40, "all", 13)])
def test_core_forward_matches_oracle(rows, N, mask_kind, seed):
    q, k, v, g, bias, mask = _inputs(seed, rows, N, mask_kind)
    T = lambda a: torch.from_numpy(a).cuda()  # noqa: E731
    o, lse = binding.attention_forward(T(q), T(k), T(v), T(bias),
                                       None if mask is None else T(mask))
    torch.cuda.synchronize()
    o = o.cpu().numpy().astype(np.float64)
    for r in range(rows):
        ref = oracle.attend(_to_oracle(q[r:r + 1])[0], _to_oracle(k[r:r + 1])[0],
                            _to_oracle(v[r:r + 1])[0], bias.astype(np.float64), mask)
        _check(f"core forward N={N} row {r} mask={mask_kind}", _to_oracle(o[r:r + 1])[0], ref)
    if mask_kind == "all":
        assert torch.isinf(lse).all() and (lse > 0).all()


def test_autograd_function_gives_the_oracle_gradients():
    """AttentionCore.apply inside a torch graph: a scalar loss that weights o
    by a fixed tensor G has d loss / d o = G, so every input's gradient must be
    the oracle's gradient for dout = G."""
    q, k, v, g, bias, mask = _inputs(14, 2, 90, "random")
    T = lambda a: torch.from_numpy(a).cuda().requires_grad_()  # noqa: E731
    tq, tk, tv, tb = T(q), T(k), T(v), T(bias)
    o = binding.AttentionCore.apply(tq, tk, tv, tb, torch.from_numpy(mask).cuda())
    (o * torch.from_numpy(g).cuda()).sum().backward()
    rq, rk, rv, rb = oracle.tri_attn_core_bwd(_to_oracle(q), _to_oracle(k), _to_oracle(v),
                                              bias.astype(np.float64), _to_oracle(g), mask)
    _check("autograd dQ", _to_oracle(tq.grad.cpu().numpy().astype(np.float64)), rq)
    _check("autograd dK", _to_oracle(tk.grad.cpu().numpy().astype(np.float64)), rk)
    _check("autograd dV", _to_oracle(tv.grad.cpu().numpy().astype(np.float64)), rv)
    _check("autograd dbias", tb.grad.cpu().numpy().astype(np.float64), rb)
