"""Parity of the tensor-core attention core with the fp64 oracle.

tri_attn_attention_forward_bf16 and tri_attn_attention_backward_bf16 take
bf16 operands and accumulate in fp32.  The oracle runs on the same
bf16-rounded inputs.  Checks:
- element by element, at sizes that span several tiles and a ragged tail, with
  masks, with row counts that leave the kernels' row groups partly empty, on an
  all-masked problem and at N = 1;
- at N = 768 (every row on the GPU): sampled rows of dQ, dK and dV, and
  sampled query lines of the bias gradient, against the oracle;
- the softmax-Jacobian property sum_k dbias[h][j][k] = 0;
- bitwise determinism."""
import numpy as np
import pytest
import torch

import oracle
from protein_pair_representation_layernorm_b200 import binding
from gpu_util import PARITY_LOG

pytestmark = pytest.mark.gpu

H, D = 4, 32
# Tolerances, from the arithmetic: q * log2(e)/sqrt(d) and the base-2 bias are
# rounded to bf16 before the score MMA, and P and ds to bf16 before the
# gradient MMAs (relative 2^-9 each); on these O(1) logits that moves a
# probability by a few tenths of a percent, and every sum runs in fp32.
GRAD_REL_L2 = 1e-2
GRAD_MAX_REL = 4e-2  # max |error| relative to the largest |gradient|
O_REL_L2, O_MAX_ABS = 5e-3, 2e-2  # the bf16 tolerance of the attention output
P_MAX_ABS = 1e-2  # probabilities implied by the returned lse, against the oracle's


def _inputs(seed, rows, N, mask_kind):
    rng = np.random.default_rng(seed)
    bf = lambda a: torch.from_numpy(a.astype(np.float32)).to(torch.bfloat16)  # noqa: E731
    q, k, v, g = (bf(rng.normal(size=(rows, H, N, D))) for _ in range(4))
    bias = bf(rng.normal(size=(H, N, N)))
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
    m = None if mask is None else torch.from_numpy(mask).cuda()
    Q, K, V, G, B = (t.cuda() for t in (q, k, v, g, bias))
    O, lse = binding.attention_forward_bf16(Q, K, V, B, m)
    grads = binding.attention_backward_bf16(Q, K, V, B, O, lse, G, m, sync=True)
    torch.cuda.synchronize()
    # fp32 as computed (the comparisons promote to fp64)
    return O.float().cpu().numpy(), lse.cpu().numpy(), [t.cpu().numpy() for t in grads]


def _f64(t):
    return t.float().numpy().astype(np.float64)


def _to_oracle(a):  # [rows][H][N][d] -> (rows, N, H, d)
    return np.ascontiguousarray(a.transpose(0, 2, 1, 3))


def _check(name, got, ref):
    scale = max(float(np.abs(ref).max()), 1e-30)
    err = float(np.abs(got - ref).max())
    rel_l2 = float(np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-30))
    PARITY_LOG.append(f"tensor-core backward {name}: rel_l2 {rel_l2:.2e}, "
                      f"max_abs/max {err / scale:.2e}")
    assert rel_l2 <= GRAD_REL_L2 and err <= GRAD_MAX_REL * scale + 1e-6, (name, rel_l2, err, scale)


def _check_forward(tag, q, k, v, bias, mask, O, lse):
    """o against the oracle's attention; lse through the probabilities it implies."""
    qo, ko, vo = (_to_oracle(_f64(t)) for t in (q, k, v))
    b = _f64(bias)
    rows, N = qo.shape[0], qo.shape[1]
    for r in range(rows):
        o_ref, p_ref = oracle.attend(qo[r], ko[r], vo[r], b, mask, want_probs=True)
        o_got = _to_oracle(O)[r]
        rel = float(np.linalg.norm(o_got - o_ref) / max(np.linalg.norm(o_ref), 1e-30))
        mx = float(np.abs(o_got - o_ref).max())
        assert rel <= O_REL_L2 and mx <= O_MAX_ABS, (tag, r, rel, mx)
        # s_jk in natural units from the same bf16 inputs; p = exp(s - lse)
        s = np.einsum("jhd,khd->hjk", qo[r], ko[r]) / np.sqrt(D) + b
        with np.errstate(invalid="ignore", over="ignore"):
            p_got = np.exp(s - lse[r][:, :, None])
        if mask is not None:
            p_got[:, :, mask == 0] = 0.0
        p_got[~np.isfinite(p_got)] = 0.0
        assert float(np.abs(p_got - p_ref).max()) <= P_MAX_ABS, (tag, r)


@pytest.mark.parametrize("rows,N,mask_kind,seed", [
    (4, 70, None, 11), (5, 133, "random", 12), (2, 64, "head", 13), (3, 200, "random", 14),
    (1, 1, None, 15), (2, 257, None, 16)])
def test_tensor_core_core_matches_oracle(rows, N, mask_kind, seed):
    q, k, v, g, bias, mask = _inputs(seed, rows, N, mask_kind)
    O, lse, (dq, dk, dv, db) = _gpu(q, k, v, g, bias, mask)
    tag = f"N={N} rows={rows} mask={mask_kind}"
    _check_forward(tag, q, k, v, bias, mask, O, lse)
    rq, rk, rv, rb = oracle.tri_attn_core_bwd(*(_to_oracle(_f64(t)) for t in (q, k, v)),
                                              _f64(bias), _to_oracle(_f64(g)), mask)
    _check(f"dQ {tag}", _to_oracle(dq), rq)
    _check(f"dK {tag}", _to_oracle(dk), rk)
    _check(f"dV {tag}", _to_oracle(dv), rv)
    _check(f"dbias {tag}", db, rb)


def test_tensor_core_all_masked():
    """Every key masked: o = 0, lse = +inf, every gradient exactly 0."""
    q, k, v, g, bias, mask = _inputs(17, 2, 40, "all")
    O, lse, grads = _gpu(q, k, v, g, bias, mask)
    assert not np.any(O)
    assert np.all(np.isposinf(lse))
    for t in grads:
        assert not np.any(t)


def test_tensor_core_backward_is_deterministic():
    q, k, v, g, bias, mask = _inputs(18, 3, 150, "random")
    a = _gpu(q, k, v, g, bias, mask)
    b = _gpu(q, k, v, g, bias, mask)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])
    for x, y in zip(a[2], b[2]):
        assert np.array_equal(x, y)


@pytest.mark.parametrize("N", [768, 1536])
def test_tensor_core_full_size_sampled(N):
    """Every row at N = 768 and at N = 1536 (the size bench.py --backward
    times): rows 0, N/2 - 1 and N - 1 of dQ, dK, dV and query lines 0, N/2 + 16
    and N - 1 of the bias gradient (summed over all N rows) against the
    oracle; sum_k dbias[h][j][k] = 0 for every (h, j)."""
    rows = N
    q, k, v, g, bias, mask = _inputs(19, rows, N, "random")
    _, _, (dq, dk, dv, db) = _gpu(q, k, v, g, bias, mask)
    row = lambda t, r: t[r].float().numpy().transpose(1, 0, 2).astype(np.float64)  # noqa: E731
    b = _f64(bias)
    for r in (0, N // 2 - 1, N - 1):
        rq, rk, rv, _ = oracle.attend_bwd(row(q, r), row(k, r), row(v, r), b, row(g, r), mask)
        _check(f"dQ N={N} row {r}", dq[r].transpose(1, 0, 2), rq)
        _check(f"dK N={N} row {r}", dk[r].transpose(1, 0, 2), rk)
        _check(f"dV N={N} row {r}", dv[r].transpose(1, 0, 2), rv)
    lines = (0, N // 2 + 16, N - 1)
    refs = {j: np.zeros((H, N)) for j in lines}
    for r in range(rows):
        kr, vr = row(k, r), row(v, r)
        qr, gr = row(q, r), row(g, r)
        for j in lines:
            refs[j] += oracle.attend_bwd(qr[j:j + 1], kr, vr, b[:, j:j + 1, :], gr[j:j + 1],
                                         mask)[3][:, 0, :]
    for j in lines:
        _check(f"dbias N={N} line {j}", db[:, j, :], refs[j])
    row_sums = np.abs(db.sum(axis=2)).max()
    assert row_sums <= 1e-3 * np.abs(db).sum(axis=2).max(), row_sums


def test_autograd_op_on_bf16_inputs():
    """binding.AttentionCore on bf16 tensors runs the tensor-core forward and
    backward: its output equals attention_forward_bf16's, its gradients
    (returned in bf16) the fp32 gradients of attention_backward_bf16 rounded,
    and both agree with the oracle."""
    q, k, v, g, bias, mask = _inputs(20, 3, 90, "random")
    m = torch.from_numpy(mask).cuda()
    leaves = [t.cuda().requires_grad_() for t in (q, k, v, bias)]
    out = binding.AttentionCore.apply(*leaves, m)
    out.backward(g.cuda())
    Q, K, V, B = (t.detach() for t in leaves)
    O, lse = binding.attention_forward_bf16(Q, K, V, B, m)
    assert torch.equal(out.detach(), O)
    want = binding.attention_backward_bf16(Q, K, V, B, O, lse, g.cuda(), m, sync=True)
    for leaf, w in zip(leaves, want):
        assert leaf.grad.dtype == torch.bfloat16
        assert torch.equal(leaf.grad, w.to(torch.bfloat16))
    rq, rk, rv, rb = oracle.tri_attn_core_bwd(*(_to_oracle(_f64(t)) for t in (q, k, v)),
                                              _f64(bias), _to_oracle(_f64(g)), mask)
    for name, leaf, ref, tr in (("dQ", leaves[0], rq, True), ("dK", leaves[1], rk, True),
                                ("dV", leaves[2], rv, True), ("dbias", leaves[3], rb, False)):
        got = leaf.grad.float().cpu().numpy().astype(np.float64)
        _check(f"autograd {name}", _to_oracle(got) if tr else got, ref)


def test_withheld_copy_reports_timeout_and_recovers():
    """A withheld stage in CTA 0 of each tensor-core kernel (forward: one; backward:
    dQ, dK dV and dbias) makes its bounded waits expire: the call returns
    TRI_ATTN_ERR_TIMEOUT with SYNC, the other CTAs finish, and the next call on the
    same workspace and context is correct."""
    import ctypes
    q, k, v, g, bias, mask = _inputs(21, 2, 70, "random")
    m = torch.from_numpy(mask).cuda()
    Q, K, V, G, B = (t.cuda() for t in (q, k, v, g, bias))
    rows, N = 2, 70
    nbytes = binding.tri_attn_attention_bf16_workspace_bytes(rows, N)
    ws = torch.empty((nbytes + 15) // 16 * 4, dtype=torch.float32, device="cuda")
    O = torch.empty_like(Q)
    lse = torch.empty(rows, H, N, dtype=torch.float32, device="cuda")
    f32 = dict(dtype=torch.float32, device="cuda")
    dq, dk, dv = (torch.empty(rows, H, N, D, **f32) for _ in range(3))
    db = torch.empty(H, N, N, **f32)
    P = lambda t: ctypes.c_void_p(t.data_ptr())  # noqa: E731
    stall = binding.TRI_ATTN_FLAG_DEBUG_STALL | binding.TRI_ATTN_FLAG_SYNC
    rc = binding.tri_attn_attention_forward_bf16(P(Q), P(K), P(V), P(B), P(m), rows, N, P(O),
                                                 P(lse), P(ws), nbytes, None, stall)
    assert rc == binding.TRI_ATTN_ERR_TIMEOUT, binding.tri_attn_status_string(rc)
    rc = binding.tri_attn_attention_forward_bf16(P(Q), P(K), P(V), P(B), P(m), rows, N, P(O),
                                                 P(lse), P(ws), nbytes, None,
                                                 binding.TRI_ATTN_FLAG_SYNC)
    assert rc == binding.TRI_ATTN_OK
    args = (P(Q), P(K), P(V), P(B), P(m), P(O), P(lse), P(G), rows, N, P(dq), P(dk), P(dv), P(db),
            P(ws), nbytes, None)
    rc = binding.tri_attn_attention_backward_bf16(*args, stall)
    assert rc == binding.TRI_ATTN_ERR_TIMEOUT, binding.tri_attn_status_string(rc)
    rc = binding.tri_attn_attention_backward_bf16(*args, binding.TRI_ATTN_FLAG_SYNC)
    assert rc == binding.TRI_ATTN_OK
    got = [t.cpu().numpy().astype(np.float64) for t in (dq, dk, dv, db)]
    rq, rk, rv, rb = oracle.tri_attn_core_bwd(*(_to_oracle(_f64(t)) for t in (q, k, v)),
                                              _f64(bias), _to_oracle(_f64(g)), mask)
    _check("dQ after timeout", _to_oracle(got[0]), rq)
    _check("dK after timeout", _to_oracle(got[1]), rk)
    _check("dV after timeout", _to_oracle(got[2]), rv)
    _check("dbias after timeout", got[3], rb)
