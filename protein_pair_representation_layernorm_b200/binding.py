"""Thin ctypes binding of the C ABI in include/tri_attn.h.

Each ``tri_attn_*`` function here marshals its arguments and calls the C
function of the same name; every step of the computation runs in the CUDA
kernels of ``_lib/libtriattn.so``.  PyTorch is used only to hold device
memory and to name streams.  There is no CPU fallback: if the library is
missing or no sm_100 device is present the calls raise.
"""
from __future__ import annotations

import ctypes
import os
import re

import torch

from . import build as _build

TRI_ATTN_OK = 0
TRI_ATTN_ERR_INVALID_ARG = -1
TRI_ATTN_ERR_UNSUPPORTED = -2
TRI_ATTN_ERR_ALIAS = -3
TRI_ATTN_ERR_OOM = -4
TRI_ATTN_ERR_CUDA = -5
TRI_ATTN_ERR_TIMEOUT = -6
TRI_ATTN_ERR_NO_DEVICE = -7

TRI_ATTN_FLAG_SYNC = 1
TRI_ATTN_FLAG_TIME_KERNELS = 2
TRI_ATTN_FLAG_DEBUG_STALL = 4
TRI_ATTN_FLAG_DEBUG_STALL_PROJ = 8
TRI_ATTN_FLAG_DEBUG_STALL_GATE = 16
TRI_ATTN_FLAG_DEBUG_FAIL_ALLOC = 32

TRI_ATTN_F32 = 0
TRI_ATTN_BF16 = 1
TRI_ATTN_STARTING = 0
TRI_ATTN_ENDING = 1

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include",
                      "tri_attn.h")


class TriAttnError(RuntimeError):
    def __init__(self, code: int, what: str):
        super().__init__(f"{what}: {tri_attn_status_string(code)} ({code})")
        self.code = code


class tri_attn_params(ctypes.Structure):
    _fields_ = [
        ("c_z", ctypes.c_int), ("n_heads", ctypes.c_int), ("head_dim", ctypes.c_int),
        ("dtype", ctypes.c_int),
        ("ln_eps", ctypes.c_float),
        ("ln_gamma", ctypes.c_void_p), ("ln_beta", ctypes.c_void_p),
        ("w_q", ctypes.c_void_p), ("w_k", ctypes.c_void_p), ("w_v", ctypes.c_void_p),
        ("w_g", ctypes.c_void_p),
        ("b_g", ctypes.c_void_p),
        ("w_b", ctypes.c_void_p),
        ("w_o", ctypes.c_void_p),
        ("b_o", ctypes.c_void_p),
    ]


_lib = None


def library_path() -> str:
    return _build.LIB


def lib() -> ctypes.CDLL:
    """Load (building first if the sources are newer) the CUDA library."""
    global _lib
    if _lib is None:
        path = _build.build() if _build.needs_build() else _build.LIB
        if not os.path.exists(path):
            raise RuntimeError(f"CUDA extension missing: {path}")
        L = ctypes.CDLL(path)
        vp, ci, cu, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_uint, ctypes.c_size_t
        L.tri_attn_create.argtypes = [ctypes.POINTER(tri_attn_params), ctypes.POINTER(vp)]
        L.tri_attn_forward.argtypes = [vp, vp, ci, vp, ci, vp, vp, cu]
        L.tri_attn_forward_host.argtypes = [vp, vp, ci, vp, vp, ci, vp, vp, cu]
        L.tri_attn_forward_host_async.argtypes = [vp, vp, ci, vp, vp, ci, vp, vp, cu]
        L.tri_attn_host_wait.argtypes = [vp]
        L.tri_attn_get_status.argtypes = [vp, vp]
        L.tri_attn_kernel_times.argtypes = [vp, ctypes.POINTER(ctypes.c_float),
                                            ctypes.POINTER(ctypes.c_int)]
        L.tri_attn_set_workspace_limit.argtypes = [vp, sz]
        L.tri_attn_workspace_bytes.argtypes = [ci, ci]
        L.tri_attn_workspace_bytes.restype = sz
        L.tri_attn_debug_workspace.argtypes = [vp] + [ctypes.POINTER(vp)] * 6 + [
            ctypes.POINTER(ci), ctypes.POINTER(ci)]
        L.tri_attn_forward_noalloc.argtypes = [ctypes.POINTER(tri_attn_params), vp, ci, vp, ci,
                                               vp, vp, cu]
        L.tri_attn_bias_ld.argtypes = [ci]
        L.tri_attn_rows_bias.argtypes = [vp, vp, ci, ci, ci, vp, vp, vp, cu]
        L.tri_attn_rows_forward.argtypes = [vp, vp, ci, ci, ci, vp, vp, vp, vp, cu]
        L.tri_attn_block_project.argtypes = [vp, vp, ci, ci, vp, vp, vp, vp, vp, vp, cu]
        L.tri_attn_block_attend.argtypes = [vp, vp, vp, vp, vp, ci, ci, ci, vp, vp, vp, cu]
        L.tri_attn_block_gate.argtypes = [vp, vp, ci, ci, vp, vp, vp, cu]
        L.tri_attn_merge_partial.argtypes = [vp, vp, vp, vp, ctypes.c_longlong, ci, vp, vp, cu]
        L.tri_attn_attention_backward_workspace_bytes.argtypes = [ci, ci]
        L.tri_attn_attention_backward_workspace_bytes.restype = sz
        L.tri_attn_attention_backward.argtypes = [vp, vp, vp, vp, vp, vp, ci, ci, vp, vp, vp, vp,
                                                  vp, sz, vp, cu]
        L.tri_attn_attention_forward.argtypes = [vp, vp, vp, vp, vp, ci, ci, vp, vp, vp, cu]
        L.tri_attn_attention_bf16_workspace_bytes.argtypes = [ci, ci]
        L.tri_attn_attention_bf16_workspace_bytes.restype = sz
        L.tri_attn_attention_forward_bf16.argtypes = [vp, vp, vp, vp, vp, ci, ci, vp, vp, vp, sz,
                                                      vp, cu]
        L.tri_attn_attention_backward_bf16.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, ci, ci, vp,
                                                       vp, vp, vp, vp, sz, vp, cu]
        L.tri_attn_destroy.argtypes = [vp]
        L.tri_attn_status_string.argtypes = [ci]
        L.tri_attn_status_string.restype = ctypes.c_char_p
        _lib = L
    return _lib


def declared_functions() -> list[str]:
    """Names of the functions include/tri_attn.h declares."""
    text = open(HEADER).read()
    return sorted(set(re.findall(r"\b(tri_attn_[a-z_]+)\s*\(", text)))


# ---------------------------------------------------------------- C ABI calls

def tri_attn_status_string(code: int) -> str:
    return lib().tri_attn_status_string(int(code)).decode()


def tri_attn_workspace_bytes(dtype: int, N: int) -> int:
    return int(lib().tri_attn_workspace_bytes(int(dtype), int(N)))


def tri_attn_create(params: tri_attn_params) -> ctypes.c_void_p:
    h = ctypes.c_void_p()
    rc = lib().tri_attn_create(ctypes.byref(params), ctypes.byref(h))
    if rc != TRI_ATTN_OK:
        raise TriAttnError(rc, "tri_attn_create")
    return h


def tri_attn_forward(h, Z_ptr: int, N: int, mask_ptr, orientation: int, out_ptr: int,
                     stream: int = 0, flags: int = 0) -> int:
    return lib().tri_attn_forward(h, Z_ptr, int(N), mask_ptr, int(orientation), out_ptr, stream,
                                  int(flags))


def tri_attn_forward_host(h, Z_host_ptr: int, N: int, mask_host_ptr, orientations,
                          out_host_ptr: int, stream: int = 0, flags: int = 0) -> int:
    arr = (ctypes.c_int * len(orientations))(*[int(o) for o in orientations])
    return lib().tri_attn_forward_host(h, Z_host_ptr, int(N), mask_host_ptr, arr,
                                       len(orientations), out_host_ptr, stream, int(flags))


def tri_attn_forward_host_async(h, Z_host_ptr: int, N: int, mask_host_ptr, orientations,
                                out_host_ptr: int, stream: int = 0, flags: int = 0) -> int:
    arr = (ctypes.c_int * len(orientations))(*[int(o) for o in orientations])
    return lib().tri_attn_forward_host_async(h, Z_host_ptr, int(N), mask_host_ptr, arr,
                                             len(orientations), out_host_ptr, stream, int(flags))


def tri_attn_host_wait(h) -> int:
    return lib().tri_attn_host_wait(h)


def tri_attn_get_status(h, stream: int = 0) -> int:
    return lib().tri_attn_get_status(h, stream)


def tri_attn_kernel_times(h) -> tuple[list[float], list[int]]:
    ms = (ctypes.c_float * 3)()
    n = (ctypes.c_int * 3)()
    rc = lib().tri_attn_kernel_times(h, ms, n)
    if rc != TRI_ATTN_OK:
        raise TriAttnError(rc, "tri_attn_kernel_times")
    return [float(x) for x in ms], [int(x) for x in n]


def tri_attn_set_workspace_limit(h, nbytes: int) -> int:
    return lib().tri_attn_set_workspace_limit(h, int(nbytes))


def tri_attn_debug_workspace(h) -> dict:
    ptrs = [ctypes.c_void_p() for _ in range(6)]
    ld, rows = ctypes.c_int(), ctypes.c_int()
    rc = lib().tri_attn_debug_workspace(h, *[ctypes.byref(p) for p in ptrs], ctypes.byref(ld),
                                        ctypes.byref(rows))
    if rc != TRI_ATTN_OK:
        raise TriAttnError(rc, "tri_attn_debug_workspace")
    names = ["q", "k", "v", "g", "bias", "o"]
    d = {n: p.value for n, p in zip(names, ptrs)}
    d["ld_bias"] = ld.value
    d["rows"] = rows.value
    return d


def tri_attn_forward_noalloc(params: tri_attn_params, Z_ptr, N: int, mask_ptr, orientation: int,
                             out_ptr, stream=None, flags: int = 0) -> int:
    """Forward that allocates no device memory (bf16 only); see tri_attn.h."""
    return lib().tri_attn_forward_noalloc(ctypes.byref(params), Z_ptr, int(N), mask_ptr,
                                          int(orientation), out_ptr, stream, int(flags))


def tri_attn_destroy(h) -> int:
    return lib().tri_attn_destroy(h)


def tri_attn_attention_forward(Q, K, V, bias, mask, rows: int, N: int, O, lse, stream=None,
                               flags: int = 0) -> int:
    """Forward of the attention core (device pointers); see tri_attn.h."""
    return lib().tri_attn_attention_forward(Q, K, V, bias, mask, int(rows), int(N), O, lse,
                                            stream, int(flags))


def tri_attn_attention_bf16_workspace_bytes(rows: int, N: int) -> int:
    return int(lib().tri_attn_attention_bf16_workspace_bytes(int(rows), int(N)))


def tri_attn_attention_forward_bf16(Q, K, V, bias, mask, rows: int, N: int, O, lse, workspace,
                                    workspace_bytes: int, stream=None, flags: int = 0) -> int:
    """Tensor-core forward of the attention core (device pointers); see tri_attn.h."""
    return lib().tri_attn_attention_forward_bf16(Q, K, V, bias, mask, int(rows), int(N), O, lse,
                                                 workspace, int(workspace_bytes), stream,
                                                 int(flags))


def tri_attn_attention_backward_bf16(Q, K, V, bias, mask, O, lse, dO, rows: int, N: int, dQ, dK,
                                     dV, dbias, workspace, workspace_bytes: int, stream=None,
                                     flags: int = 0) -> int:
    """Tensor-core backward of the attention core (device pointers); see tri_attn.h."""
    return lib().tri_attn_attention_backward_bf16(Q, K, V, bias, mask, O, lse, dO, int(rows),
                                                  int(N), dQ, dK, dV, dbias, workspace,
                                                  int(workspace_bytes), stream, int(flags))


def tri_attn_attention_backward_workspace_bytes(rows: int, N: int) -> int:
    return int(lib().tri_attn_attention_backward_workspace_bytes(int(rows), int(N)))


def tri_attn_attention_backward(Q, K, V, bias, mask, dO, rows: int, N: int, dQ, dK, dV, dbias,
                                workspace, workspace_bytes: int, stream=None, flags: int = 0) -> int:
    """Backward pass of the attention core (device pointers); see tri_attn.h."""
    return lib().tri_attn_attention_backward(Q, K, V, bias, mask, dO, int(rows), int(N), dQ, dK,
                                             dV, dbias, workspace, int(workspace_bytes), stream,
                                             int(flags))


# ---------------------------------------------------------------- convenience

def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream_handle(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


class TriangleAttention:
    """One block's weights on the device plus its handle.

    ``weights`` maps gamma, beta, Wq, Wk, Wv, Wg, bg, Wb, Wo, bo to tensors
    (any device; they are copied to the current CUDA device in ``dtype``)."""

    def __init__(self, weights: dict, dtype: torch.dtype = torch.bfloat16, eps: float = 1e-5):
        if dtype not in (torch.float32, torch.bfloat16):
            raise ValueError("dtype must be float32 or bfloat16")
        self.dtype = dtype
        dev = torch.device("cuda", torch.cuda.current_device())
        self._w = {k: v.detach().to(dev, dtype).contiguous() for k, v in weights.items()
                   if v is not None}
        w = self._w
        p = tri_attn_params()
        p.c_z, p.n_heads = w["Wo"].shape[0], w["Wb"].shape[0]
        p.head_dim = w["Wq"].shape[0] // p.n_heads
        p.dtype = TRI_ATTN_F32 if dtype == torch.float32 else TRI_ATTN_BF16
        p.ln_eps = eps
        p.ln_gamma, p.ln_beta = w["gamma"].data_ptr(), w["beta"].data_ptr()
        p.w_q, p.w_k, p.w_v, p.w_g = (w[k].data_ptr() for k in ("Wq", "Wk", "Wv", "Wg"))
        p.b_g = w["bg"].data_ptr() if "bg" in w else None
        p.w_b, p.w_o = w["Wb"].data_ptr(), w["Wo"].data_ptr()
        p.b_o = w["bo"].data_ptr() if "bo" in w else None
        self.handle = tri_attn_create(p)

    def forward(self, Z: torch.Tensor, orientation: int = TRI_ATTN_STARTING, mask=None,
                out: torch.Tensor | None = None, stream=None, flags: int = 0) -> torch.Tensor:
        assert Z.is_cuda and Z.dtype == self.dtype and Z.is_contiguous()
        N = Z.shape[0]
        if out is None:
            out = torch.empty_like(Z)
        if mask is not None:
            mask = mask.to(device=Z.device, dtype=torch.uint8).contiguous()
        rc = tri_attn_forward(self.handle, _ptr(Z), N, _ptr(mask), orientation, _ptr(out),
                              _stream_handle(stream), flags)
        if rc != TRI_ATTN_OK:
            raise TriAttnError(rc, "tri_attn_forward")
        return out

    __call__ = forward

    def forward_host(self, Z_host: torch.Tensor, orientations, mask=None,
                     out: torch.Tensor | None = None, stream=None, flags: int = 0):
        assert not Z_host.is_cuda and Z_host.is_contiguous()
        if out is None:
            out = torch.empty_like(Z_host)
        if mask is not None:
            mask = mask.to(torch.uint8).contiguous()
        rc = tri_attn_forward_host(self.handle, _ptr(Z_host), Z_host.shape[0], _ptr(mask),
                                   list(orientations), _ptr(out), _stream_handle(stream), flags)
        if rc != TRI_ATTN_OK:
            raise TriAttnError(rc, "tri_attn_forward_host")
        return out

    def forward_host_async(self, Z_host: torch.Tensor, orientations, mask=None,
                           out: torch.Tensor | None = None, stream=None, flags: int = 0):
        """Enqueue tri_attn_forward_host_async; the result is in `out` after
        host_wait().  The tensors must stay alive and unmodified until then."""
        assert not Z_host.is_cuda and Z_host.is_contiguous()
        if out is None:
            out = torch.empty_like(Z_host)
        if mask is not None:
            mask = mask.to(torch.uint8).contiguous()
        keep = getattr(self, "_async_keep", [])
        keep.append((Z_host, out, mask))  # alive until host_wait
        self._async_keep = keep
        rc = tri_attn_forward_host_async(self.handle, _ptr(Z_host), Z_host.shape[0], _ptr(mask),
                                         list(orientations), _ptr(out), _stream_handle(stream),
                                         flags)
        if rc != TRI_ATTN_OK:
            raise TriAttnError(rc, "tri_attn_forward_host_async")
        return out

    def host_wait(self) -> int:
        rc = tri_attn_host_wait(self.handle)
        self._async_keep = []
        return rc

    # ---- row-sharded execution (bf16): see tri_attn_rows_bias / _forward in
    # include/tri_attn.h.  Z_rows is the slab of problem rows row0.. of an
    # N x N problem ([nrows][N][c_z]); the starting-node formula applies (an
    # ending-node block is the starting-node block of the transposed tensor).
    def bias_ld(self, N: int) -> int:
        return int(lib().tri_attn_bias_ld(int(N)))

    def rows_bias(self, Z_rows: torch.Tensor, N: int, row0: int, mask=None,
                  bias_rows: torch.Tensor | None = None, stream=None, flags: int = 0):
        """The slab's logit-bias rows, [H][nrows][ld] bf16."""
        assert Z_rows.is_cuda and Z_rows.dtype == self.dtype and Z_rows.is_contiguous()
        nrows = Z_rows.shape[0]
        if bias_rows is None:
            bias_rows = torch.empty(4, nrows, self.bias_ld(N), dtype=torch.bfloat16,
                                    device=Z_rows.device)
        if mask is not None:
            mask = mask.to(device=Z_rows.device, dtype=torch.uint8).contiguous()
        rc = lib().tri_attn_rows_bias(self.handle, _ptr(Z_rows), int(N), int(row0), nrows,
                                      _ptr(mask), _ptr(bias_rows), _stream_handle(stream), flags)
        if rc != TRI_ATTN_OK:
            raise TriAttnError(rc, "tri_attn_rows_bias")
        return bias_rows

    def rows_forward(self, Z_rows: torch.Tensor, N: int, row0: int, bias_all: torch.Tensor,
                     mask=None, out: torch.Tensor | None = None, stream=None, flags: int = 0):
        """The starting-node block on the slab, given the whole [H][N][ld] bias."""
        assert Z_rows.is_cuda and Z_rows.dtype == self.dtype and Z_rows.is_contiguous()
        assert bias_all.is_cuda and bias_all.is_contiguous()
        if out is None:
            out = torch.empty_like(Z_rows)
        if mask is not None:
            mask = mask.to(device=Z_rows.device, dtype=torch.uint8).contiguous()
        rc = lib().tri_attn_rows_forward(self.handle, _ptr(Z_rows), int(N), int(row0),
                                         Z_rows.shape[0], _ptr(mask), _ptr(bias_all), _ptr(out),
                                         _stream_handle(stream), flags)
        if rc != TRI_ATTN_OK:
            raise TriAttnError(rc, "tri_attn_rows_forward")
        return out

    # ------------------------------------------------ block-level calls (bf16)
    def block_project(self, Z_blk: torch.Tensor, mask=None, stream=None, flags: int = 0):
        """(Q, K, V, bias, ld) of a block of pairs Z_blk [rows][cols][c_z]:
        Q, K, V [rows][H][cols][d] (q scaled by log2(e)/sqrt(d)), bias
        [H][rows][ld] (times log2(e), -3e38 at masked keys and padding)."""
        assert Z_blk.is_cuda and Z_blk.dtype == torch.bfloat16 and Z_blk.is_contiguous()
        rows, cols = Z_blk.shape[0], Z_blk.shape[1]
        ld = self.bias_ld(cols)
        Q, K, V = (torch.empty(rows, 4, cols, 32, dtype=torch.bfloat16, device=Z_blk.device)
                   for _ in range(3))
        bias = torch.empty(4, rows, ld, dtype=torch.bfloat16, device=Z_blk.device)
        if mask is not None:
            mask = mask.to(device=Z_blk.device, dtype=torch.uint8).contiguous()
        rc = lib().tri_attn_block_project(self.handle, _ptr(Z_blk), rows, cols, _ptr(mask),
                                          _ptr(Q), _ptr(K), _ptr(V), _ptr(bias),
                                          _stream_handle(stream), flags)
        if rc != TRI_ATTN_OK:
            raise TriAttnError(rc, "tri_attn_block_project")
        return Q, K, V, bias, ld

    def block_attend(self, Q, K, V, bias, ld: int, stream=None, flags: int = 0):
        """(O, lse) of the rows' queries over one key block (O bf16
        [rows][H][n][d] normalised within the block, lse fp32 [rows][H][n])."""
        rows, _, n, _ = Q.shape
        O = torch.empty_like(Q)
        lse = torch.empty(rows, 4, n, dtype=torch.float32, device=Q.device)
        rc = lib().tri_attn_block_attend(self.handle, _ptr(Q), _ptr(K), _ptr(V), _ptr(bias),
                                         int(ld), rows, n, _ptr(O), _ptr(lse),
                                         _stream_handle(stream), flags)
        if rc != TRI_ATTN_OK:
            raise TriAttnError(rc, "tri_attn_block_attend")
        return O, lse

    def block_gate(self, Z_blk: torch.Tensor, O: torch.Tensor, out=None, stream=None,
                   flags: int = 0):
        """out = z + Wo (g * o) + bo for the block's pairs."""
        rows, cols = Z_blk.shape[0], Z_blk.shape[1]
        if out is None:
            out = torch.empty_like(Z_blk)
        rc = lib().tri_attn_block_gate(self.handle, _ptr(Z_blk), rows, cols, _ptr(O), _ptr(out),
                                       _stream_handle(stream), flags)
        if rc != TRI_ATTN_OK:
            raise TriAttnError(rc, "tri_attn_block_gate")
        return out

    def status(self, stream=None) -> int:
        return tri_attn_get_status(self.handle, _stream_handle(stream))

    def kernel_times(self) -> tuple[list[float], list[int]]:
        """(ms per kernel, launches per kernel) since the previous call."""
        return tri_attn_kernel_times(self.handle)

    def set_workspace_limit(self, nbytes: int):
        rc = tri_attn_set_workspace_limit(self.handle, nbytes)
        if rc != TRI_ATTN_OK:
            raise TriAttnError(rc, "tri_attn_set_workspace_limit")

    def debug_workspace(self) -> dict:
        return tri_attn_debug_workspace(self.handle)

    def close(self):
        if getattr(self, "handle", None) is not None:
            tri_attn_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def attention_backward(Q: torch.Tensor, K: torch.Tensor, V: torch.Tensor, bias: torch.Tensor,
                       dO: torch.Tensor, mask: torch.Tensor | None = None, stream=None):
    """Gradients (dQ, dK, dV, dbias) of the attention core on the GPU.

    Q, K, V, dO: fp32 CUDA tensors [rows][H][N][d] (H = 4, d = 32); bias: fp32
    [H][N][N] (natural-unit logits); mask: uint8 [N] or None.  Allocates the
    outputs and the row-statistics workspace with torch and calls
    tri_attn_attention_backward on `stream` (default: the current stream)."""
    rows, H, N, d = Q.shape
    for t in (Q, K, V, dO):
        if t.dtype != torch.float32 or not t.is_cuda or tuple(t.shape) != (rows, H, N, d):
            raise ValueError("Q, K, V, dO must be fp32 CUDA tensors of one shape [rows][H][N][d]")
    if bias.dtype != torch.float32 or tuple(bias.shape) != (H, N, N):
        raise ValueError("bias must be an fp32 CUDA tensor [H][N][N]")
    Q, K, V, dO, bias = (t.contiguous() for t in (Q, K, V, dO, bias))
    m = None if mask is None else mask.to(device=Q.device, dtype=torch.uint8).contiguous()
    dQ, dK, dV = torch.empty_like(Q), torch.empty_like(K), torch.empty_like(V)
    dB = torch.empty_like(bias)
    nbytes = tri_attn_attention_backward_workspace_bytes(rows, N)
    ws = torch.empty(max(nbytes // 4, 4), dtype=torch.float32, device=Q.device)
    rc = tri_attn_attention_backward(_ptr(Q), _ptr(K), _ptr(V), _ptr(bias), _ptr(m), _ptr(dO),
                                     rows, N, _ptr(dQ), _ptr(dK), _ptr(dV), _ptr(dB), _ptr(ws),
                                     ws.numel() * 4, _stream_handle(stream), 0)
    if rc != TRI_ATTN_OK:
        raise TriAttnError(rc, "tri_attn_attention_backward")
    return dQ, dK, dV, dB


def _core_checked(Q, K, V, bias):
    rows, H, N, d = Q.shape
    for t in (Q, K, V):
        if t.dtype != torch.float32 or not t.is_cuda or tuple(t.shape) != (rows, H, N, d):
            raise ValueError("Q, K, V must be fp32 CUDA tensors of one shape [rows][H][N][d]")
    if bias.dtype != torch.float32 or tuple(bias.shape) != (H, N, N):
        raise ValueError("bias must be an fp32 CUDA tensor [H][N][N]")
    return rows, N


def attention_forward(Q: torch.Tensor, K: torch.Tensor, V: torch.Tensor, bias: torch.Tensor,
                      mask: torch.Tensor | None = None, stream=None):
    """(o, lse) of the attention core on the GPU (fp32; layouts as attention_backward)."""
    rows, N = _core_checked(Q, K, V, bias)
    Q, K, V, bias = (t.contiguous() for t in (Q, K, V, bias))
    m = None if mask is None else mask.to(device=Q.device, dtype=torch.uint8).contiguous()
    O = torch.empty_like(Q)
    lse = torch.empty(Q.shape[:3], dtype=torch.float32, device=Q.device)
    rc = tri_attn_attention_forward(_ptr(Q), _ptr(K), _ptr(V), _ptr(bias), _ptr(m), rows, N,
                                    _ptr(O), _ptr(lse), _stream_handle(stream), 0)
    if rc != TRI_ATTN_OK:
        raise TriAttnError(rc, "tri_attn_attention_forward")
    return O, lse


def merge_partial(O_acc: torch.Tensor, lse_acc: torch.Tensor, O_part: torch.Tensor,
                  lse_part: torch.Tensor, first: bool, O_out: torch.Tensor | None = None,
                  stream=None):
    """Merge one key block's (O_part bf16, lse_part) into the running (O_acc
    fp32, lse_acc), in place; O_out (bf16) receives the merged output."""
    count = lse_part.numel()
    rc = lib().tri_attn_merge_partial(_ptr(O_acc), _ptr(lse_acc), _ptr(O_part), _ptr(lse_part),
                                      count, 1 if first else 0, _ptr(O_out),
                                      _stream_handle(stream), 0)
    if rc != TRI_ATTN_OK:
        raise TriAttnError(rc, "tri_attn_merge_partial")


def _core_checked_bf16(Q, K, V, bias, *more):
    rows, H, N, d = Q.shape
    for t in (Q, K, V) + more:
        if t.dtype != torch.bfloat16 or not t.is_cuda or tuple(t.shape) != (rows, H, N, d):
            raise ValueError("Q, K, V (O, dO) must be bf16 CUDA tensors of one shape "
                             "[rows][H][N][d]")
    if bias.dtype != torch.bfloat16 or tuple(bias.shape) != (H, N, N):
        raise ValueError("bias must be a bf16 CUDA tensor [H][N][N]")
    return rows, N


def _core_workspace(rows, N, device):
    nbytes = tri_attn_attention_bf16_workspace_bytes(rows, N)
    return torch.empty((nbytes + 15) // 16 * 4, dtype=torch.float32, device=device), nbytes


def attention_forward_bf16(Q: torch.Tensor, K: torch.Tensor, V: torch.Tensor, bias: torch.Tensor,
                           mask: torch.Tensor | None = None, stream=None):
    """(o, lse) of the attention core on the tensor cores: bf16 Q, K, V
    [rows][H][N][d] and bias [H][N][N] (natural-unit logits), o bf16, lse fp32
    [rows][H][N] (natural log; +inf for a query whose every key is masked)."""
    rows, N = _core_checked_bf16(Q, K, V, bias)
    Q, K, V, bias = (t.contiguous() for t in (Q, K, V, bias))
    m = None if mask is None else mask.to(device=Q.device, dtype=torch.uint8).contiguous()
    O = torch.empty_like(Q)
    lse = torch.empty(Q.shape[:3], dtype=torch.float32, device=Q.device)
    ws, nbytes = _core_workspace(rows, N, Q.device)
    rc = tri_attn_attention_forward_bf16(_ptr(Q), _ptr(K), _ptr(V), _ptr(bias), _ptr(m), rows, N,
                                         _ptr(O), _ptr(lse), _ptr(ws), nbytes,
                                         _stream_handle(stream), 0)
    if rc != TRI_ATTN_OK:
        raise TriAttnError(rc, "tri_attn_attention_forward_bf16")
    return O, lse


def attention_backward_bf16(Q: torch.Tensor, K: torch.Tensor, V: torch.Tensor, bias: torch.Tensor,
                            O: torch.Tensor, lse: torch.Tensor, dO: torch.Tensor,
                            mask: torch.Tensor | None = None, stream=None, sync: bool = False):
    """Gradients (dQ, dK, dV, dbias), fp32, of the attention core on the tensor
    cores, from the bf16 operands, the forward's o (bf16) and lse (fp32) and
    the bf16 dO.  With sync, waits and raises on a device-side timeout."""
    rows, N = _core_checked_bf16(Q, K, V, bias, O, dO)
    if lse.dtype != torch.float32 or tuple(lse.shape) != tuple(Q.shape[:3]):
        raise ValueError("lse must be an fp32 CUDA tensor [rows][H][N]")
    Q, K, V, bias, O, lse, dO = (t.contiguous() for t in (Q, K, V, bias, O, lse, dO))
    m = None if mask is None else mask.to(device=Q.device, dtype=torch.uint8).contiguous()
    dQ = torch.empty(Q.shape, dtype=torch.float32, device=Q.device)
    dK, dV = torch.empty_like(dQ), torch.empty_like(dQ)
    dB = torch.empty(bias.shape, dtype=torch.float32, device=Q.device)
    ws, nbytes = _core_workspace(rows, N, Q.device)
    rc = tri_attn_attention_backward_bf16(_ptr(Q), _ptr(K), _ptr(V), _ptr(bias), _ptr(m),
                                          _ptr(O), _ptr(lse), _ptr(dO), rows, N, _ptr(dQ),
                                          _ptr(dK), _ptr(dV), _ptr(dB), _ptr(ws), nbytes,
                                          _stream_handle(stream), TRI_ATTN_FLAG_SYNC if sync else 0)
    if rc != TRI_ATTN_OK:
        raise TriAttnError(rc, "tri_attn_attention_backward_bf16")
    return dQ, dK, dV, dB


class AttentionCore(torch.autograd.Function):
    """The attention core as a differentiable torch op: o = softmax_k(q . k /
    sqrt(d) + bias, masked) v per problem row, with gradients for q, k, v and
    the (row-shared) bias.  fp32 inputs run the library's fp32 SIMT kernels;
    bf16 inputs run the tensor-core forward and backward (gradients returned in
    bf16, computed in fp32).  Call as AttentionCore.apply(Q, K, V, bias, mask)."""

    @staticmethod
    def forward(ctx, Q, K, V, bias, mask=None):
        if Q.dtype == torch.bfloat16:
            O, lse = attention_forward_bf16(Q, K, V, bias, mask)
            ctx.save_for_backward(Q, K, V, bias, O, lse)
        else:
            O, _ = attention_forward(Q, K, V, bias, mask)
            ctx.save_for_backward(Q, K, V, bias)
        ctx.mask = mask
        return O

    @staticmethod
    def backward(ctx, dO):
        if len(ctx.saved_tensors) == 6:
            Q, K, V, bias, O, lse = ctx.saved_tensors
            grads = attention_backward_bf16(Q, K, V, bias, O, lse,
                                            dO.to(torch.bfloat16).contiguous(), ctx.mask)
            return tuple(g.to(torch.bfloat16) for g in grads) + (None,)
        Q, K, V, bias = ctx.saved_tensors
        dQ, dK, dV, dB = attention_backward(Q, K, V, bias, dO.contiguous(), ctx.mask)
        return dQ, dK, dV, dB, None
