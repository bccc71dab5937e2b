"""Host-side checks of the C ABI that need no GPU: the library loads, exports
every function include/tri_attn.h declares, and rejects bad arguments before
touching a device."""
import ctypes
import os
import re
import subprocess

import pytest
import torch

from protein_pair_representation_layernorm_b200 import binding

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_library_exports_every_declared_function():
    L = binding.lib()
    declared = binding.declared_functions()
    assert len(declared) >= 9
    for name in declared:
        assert hasattr(L, name), name
    out = subprocess.run(["nm", "-D", "--defined-only", binding.library_path()],
                         capture_output=True, text=True, check=True).stdout
    exported = set(re.findall(r"\bT (tri_attn_\w+)", out))
    assert set(declared) <= exported


def test_status_strings():
    for code in range(0, -8, -1):
        s = binding.tri_attn_status_string(code)
        assert s and s != "unknown status"
    assert binding.tri_attn_status_string(-99) == "unknown status"


def test_workspace_bytes():
    ws = binding.tri_attn_workspace_bytes
    assert ws(binding.TRI_ATTN_BF16, 0) == 0
    assert ws(7, 10) == 0
    # bf16: q, k, v, o (N*N*128 each; the gate is recomputed, never stored) +
    # bias H*N*roundup(N,64), 2 bytes per element; fp32: q, k, v, g, o + bias, 4 bytes
    for N in (1536, 200):
        ld = -(-N // 64) * 64
        bias = -(-4 * N * ld * 2 // 256) * 256
        assert ws(binding.TRI_ATTN_BF16, N) == 4 * N * N * 128 * 2 + bias
        bias = -(-4 * N * ld * 4 // 256) * 256
        assert ws(binding.TRI_ATTN_F32, N) == 5 * N * N * 128 * 4 + bias
    assert ws(binding.TRI_ATTN_BF16, 4096) > ws(binding.TRI_ATTN_BF16, 1536)


def test_create_rejects_bad_params_without_device():
    L = binding.lib()
    h = ctypes.c_void_p()
    assert L.tri_attn_create(None, ctypes.byref(h)) == binding.TRI_ATTN_ERR_INVALID_ARG
    p = binding.tri_attn_params()
    p.c_z, p.n_heads, p.head_dim, p.dtype, p.ln_eps = 64, 4, 32, binding.TRI_ATTN_BF16, 1e-5
    assert L.tri_attn_create(ctypes.byref(p), ctypes.byref(h)) == binding.TRI_ATTN_ERR_UNSUPPORTED
    p.c_z = 128
    # weight pointers missing
    assert L.tri_attn_create(ctypes.byref(p), ctypes.byref(h)) == binding.TRI_ATTN_ERR_INVALID_ARG
    p.dtype = 5
    assert L.tri_attn_create(ctypes.byref(p), ctypes.byref(h)) == binding.TRI_ATTN_ERR_INVALID_ARG


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-device error path")
def test_no_device_fails_loudly():
    L = binding.lib()
    p = binding.tri_attn_params()
    p.c_z, p.n_heads, p.head_dim, p.dtype, p.ln_eps = 128, 4, 32, binding.TRI_ATTN_BF16, 1e-5
    fake = ctypes.c_void_p(0x1000)
    for f in ("ln_gamma", "ln_beta", "w_q", "w_k", "w_v", "w_g", "w_b", "w_o"):
        setattr(p, f, fake.value)
    h = ctypes.c_void_p()
    assert L.tri_attn_create(ctypes.byref(p), ctypes.byref(h)) == binding.TRI_ATTN_ERR_NO_DEVICE
    with pytest.raises(binding.TriAttnError):
        binding.tri_attn_create(p)


def test_null_handle_calls():
    L = binding.lib()
    assert L.tri_attn_forward(None, None, 1, None, 0, None, None, 0) == binding.TRI_ATTN_ERR_INVALID_ARG
    assert L.tri_attn_get_status(None, None) == binding.TRI_ATTN_ERR_INVALID_ARG
    assert L.tri_attn_destroy(None) == binding.TRI_ATTN_OK
    assert L.tri_attn_set_workspace_limit(None, 0) == binding.TRI_ATTN_ERR_INVALID_ARG


def test_product_path_never_touches_the_oracle():
    """The package (kernels, binding, workloads) must not import, load or call oracle/."""
    pkg = os.path.join(ROOT, "protein_pair_representation_layernorm_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h", ".cpp")):
                text = open(os.path.join(dirpath, f), encoding="utf-8").read()
                assert not re.search(r"^\s*(import|from)\s+oracle\b", text, re.M), f
                assert "liboracle" not in text, f
                assert "oracle.c" not in text, f


def test_row_slab_calls_reject_bad_arguments_without_device():
    L = binding.lib()
    assert L.tri_attn_bias_ld(0) == 0
    assert L.tri_attn_bias_ld(1) == 64 and L.tri_attn_bias_ld(64) == 64
    assert L.tri_attn_bias_ld(65) == 128 and L.tri_attn_bias_ld(1536) == 1536
    buf = ctypes.c_void_p(0x10000)
    # no handle: rejected before anything else
    assert L.tri_attn_rows_bias(None, buf, 16, 0, 16, None, buf, None, 0) == \
        binding.TRI_ATTN_ERR_INVALID_ARG
    assert L.tri_attn_rows_forward(None, buf, 16, 0, 16, None, buf, buf, None, 0) == \
        binding.TRI_ATTN_ERR_INVALID_ARG


def test_binding_constants_match_the_header():
    """Every status code and flag the header defines has the same value in the binding."""
    with open(os.path.join(ROOT, "include", "tri_attn.h")) as f:
        text = f.read()
    defs = re.findall(r"#define\s+(TRI_ATTN_(?:OK|ERR_\w+|FLAG_\w+))\s+(-?\d+)u?", text)
    assert len(defs) >= 14
    for name, value in defs:
        assert getattr(binding, name) == int(value), name


def test_attention_backward_rejects_bad_arguments_without_device():
    L = binding.lib()
    ws_bytes = binding.tri_attn_attention_backward_workspace_bytes
    assert ws_bytes(0, 10) == 0 and ws_bytes(3, 0) == 0
    assert ws_bytes(3, 70) == 2 * 3 * 4 * 70 * 4  # log-sum-exp and D per (row, head, query)
    buf = 0x10000
    ok = dict(Q=buf, K=buf, V=buf, bias=buf, mask=None, dO=buf, rows=3, N=70, dQ=buf, dK=buf,
              dV=buf, dbias=buf, workspace=buf, workspace_bytes=ws_bytes(3, 70), stream=None,
              flags=0)

    def call(**kw):
        a = dict(ok, **kw)
        return L.tri_attn_attention_backward(*a.values())

    assert call(Q=None) == binding.TRI_ATTN_ERR_INVALID_ARG
    assert call(dbias=None) == binding.TRI_ATTN_ERR_INVALID_ARG
    assert call(dK=buf + 4) == binding.TRI_ATTN_ERR_INVALID_ARG  # misaligned
    assert call(rows=0) == binding.TRI_ATTN_ERR_INVALID_ARG
    assert call(N=0) == binding.TRI_ATTN_ERR_INVALID_ARG
    assert call(workspace_bytes=ws_bytes(3, 70) - 4) == binding.TRI_ATTN_ERR_INVALID_ARG
    assert call(N=46341, workspace_bytes=ws_bytes(3, 46341)) == binding.TRI_ATTN_ERR_UNSUPPORTED
    if not torch.cuda.is_available():
        assert call() == binding.TRI_ATTN_ERR_NO_DEVICE


def test_async_host_calls_reject_bad_arguments_without_device():
    L = binding.lib()
    buf = ctypes.c_void_p(0x10000)
    orients = (ctypes.c_int * 2)(0, 1)
    assert L.tri_attn_forward_host_async(None, buf, 16, None, orients, 2, buf, None, 0) == \
        binding.TRI_ATTN_ERR_INVALID_ARG
    assert L.tri_attn_host_wait(None) == binding.TRI_ATTN_ERR_INVALID_ARG


def test_core_forward_rejects_bad_arguments_without_device():
    L = binding.lib()
    buf = 0x10000
    ok = dict(Q=buf, K=buf, V=buf, bias=buf, mask=None, rows=2, N=40, O=buf, lse=buf,
              stream=None, flags=0)

    def call(**kw):
        return L.tri_attn_attention_forward(*dict(ok, **kw).values())

    assert call(Q=None) == binding.TRI_ATTN_ERR_INVALID_ARG
    assert call(O=buf + 8) == binding.TRI_ATTN_ERR_INVALID_ARG
    assert call(lse=None) == binding.TRI_ATTN_ERR_INVALID_ARG
    assert call(N=0) == binding.TRI_ATTN_ERR_INVALID_ARG
    assert call(rows=70000) == binding.TRI_ATTN_ERR_UNSUPPORTED
    if not torch.cuda.is_available():
        assert call() == binding.TRI_ATTN_ERR_NO_DEVICE


def test_tensor_core_core_calls_reject_bad_arguments_without_device():
    L = binding.lib()
    ws_bytes = binding.tri_attn_attention_bf16_workspace_bytes
    assert ws_bytes(0, 10) == 0 and ws_bytes(3, 0) == 0
    # status word, Qs, b2 and b2T, -lse2 and -D, each 256-byte aligned (ld = 128 here)
    al = lambda x: (x + 255) // 256 * 256  # noqa: E731
    want = al(4) + al(3 * 4 * 70 * 32 * 2) + 2 * al(4 * 70 * 128 * 2) + 2 * al(3 * 4 * 128 * 4)
    assert ws_bytes(3, 70) == want
    buf = 0x10000
    fwd = dict(Q=buf, K=buf, V=buf, bias=buf, mask=None, rows=3, N=70, O=buf, lse=buf,
               workspace=buf, workspace_bytes=want, stream=None, flags=0)
    bwd = dict(Q=buf, K=buf, V=buf, bias=buf, mask=None, O=buf, lse=buf, dO=buf, rows=3, N=70,
               dQ=buf, dK=buf, dV=buf, dbias=buf, workspace=buf, workspace_bytes=want,
               stream=None, flags=0)

    def f(**kw):
        return L.tri_attn_attention_forward_bf16(*dict(fwd, **kw).values())

    def b(**kw):
        return L.tri_attn_attention_backward_bf16(*dict(bwd, **kw).values())

    bad = binding.TRI_ATTN_ERR_INVALID_ARG
    for call in (f, b):
        assert call(Q=None) == bad
        assert call(V=buf + 8) == bad  # misaligned
        assert call(bias=None) == bad
        assert call(rows=0) == bad and call(N=0) == bad
        assert call(workspace=None) == bad
        assert call(workspace_bytes=want - 1) == bad
        assert call(rows=70000, workspace_bytes=ws_bytes(70000, 70)) == \
            binding.TRI_ATTN_ERR_UNSUPPORTED
        assert call(lse=buf + 2) == bad
    assert b(lse=None) == bad and b(dO=None) == bad and b(dbias=buf + 4) == bad
    if not torch.cuda.is_available():
        assert f() == binding.TRI_ATTN_ERR_NO_DEVICE
        assert f(lse=None) == binding.TRI_ATTN_ERR_NO_DEVICE  # lse is optional in the forward
        assert b() == binding.TRI_ATTN_ERR_NO_DEVICE


def test_block_calls_reject_bad_arguments_without_device():
    L = binding.lib()
    buf, bad = 0x10000, binding.TRI_ATTN_ERR_INVALID_ARG
    # no handle
    assert L.tri_attn_block_project(None, buf, 8, 8, None, buf, buf, buf, buf, None, 0) == bad
    assert L.tri_attn_block_attend(None, buf, buf, buf, buf, 64, 8, 8, buf, buf, None, 0) == bad
    assert L.tri_attn_block_gate(None, buf, 8, 8, buf, buf, None, 0) == bad
    # the merge needs no handle: pointers, alignment and count are checked first
    assert L.tri_attn_merge_partial(None, buf, buf, buf, 10, 1, None, None, 0) == bad
    assert L.tri_attn_merge_partial(buf + 4, buf, buf, buf, 10, 1, None, None, 0) == bad
    assert L.tri_attn_merge_partial(buf, buf, buf, buf, 0, 1, None, None, 0) == bad
    assert L.tri_attn_merge_partial(buf, buf + 2, buf, buf, 10, 1, None, None, 0) == bad
    assert L.tri_attn_merge_partial(buf, buf, buf, buf, 10, 1, buf + 8, None, 0) == bad
    if not torch.cuda.is_available():
        assert L.tri_attn_merge_partial(buf, buf, buf, buf, 10, 1, None, None, 0) == \
            binding.TRI_ATTN_ERR_NO_DEVICE
