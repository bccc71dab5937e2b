"""CPU fp64 oracle for the pair-biased triangle attention block.

TEST INFRASTRUCTURE ONLY: the tests, the smoke check and the benchmark's
CPU-baseline leg are the only callers.  The GPU product path never imports
this package.

The arithmetic lives in ``oracle.c`` (plain C, fp64, one softmax row
materialised at a time); this module only compiles it with gcc and marshals
numpy arrays through ctypes.  See ``oracle.c`` for the definition that is
followed and the passages it cites.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

Z_F64, Z_F32, Z_BF16 = 0, 1, 2


def build(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so (gcc, -O2, OpenMP, no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call([
            "gcc", "-O2", "-std=c11", "-fopenmp", "-shared", "-fPIC",
            _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


class _Params(ctypes.Structure):
    _fields_ = [
        ("N", ctypes.c_int), ("c_z", ctypes.c_int), ("H", ctypes.c_int), ("d", ctypes.c_int),
        ("eps", ctypes.c_double),
        ("z_dtype", ctypes.c_int),
        ("Z", ctypes.c_void_p),
        ("mask", ctypes.c_void_p),
        ("gamma", ctypes.c_void_p), ("beta", ctypes.c_void_p),
        ("Wq", ctypes.c_void_p), ("Wk", ctypes.c_void_p), ("Wv", ctypes.c_void_p), ("Wg", ctypes.c_void_p),
        ("bg", ctypes.c_void_p),
        ("Wb", ctypes.c_void_p),
        ("Wo", ctypes.c_void_p),
        ("bo", ctypes.c_void_p),
    ]


_lib = None


def lib():
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
        vp, ci, cl = ctypes.c_void_p, ctypes.c_int, ctypes.c_long
        _lib.oracle_layer_norm.argtypes = [vp, cl, ci, ctypes.c_double, vp, vp, vp]
        _lib.oracle_pair_features.argtypes = [ctypes.POINTER(_Params), vp, vp, vp, vp, vp]
        _lib.oracle_attend.argtypes = [vp, vp, vp, vp, vp, ci, ci, ci, ci, vp, vp]
        _lib.oracle_attend_blockwise.argtypes = [vp, vp, vp, vp, vp, ci, ci, ci, ci, ci, vp]
        _lib.oracle_attend_bwd.argtypes = [vp, vp, vp, vp, vp, vp, ci, ci, ci, ci, vp, vp, vp, vp]
        _lib.oracle_tri_attn.argtypes = [ctypes.POINTER(_Params), ci, vp, ci, vp, vp, vp]
        _lib.oracle_num_threads.restype = ci
    return _lib


def num_threads() -> int:
    return int(lib().oracle_num_threads())


def _ptr(a):
    return None if a is None else a.ctypes.data


def _f64(a):
    return None if a is None else np.ascontiguousarray(a, dtype=np.float64)


@dataclass
class Problem:
    """One block instance.  Z is (N, N, c_z) as float64, float32 or bf16 bits
    (uint16); weights are float64 (exact upcasts of whatever precision the
    GPU side stores)."""
    Z: np.ndarray
    gamma: np.ndarray
    beta: np.ndarray
    Wq: np.ndarray
    Wk: np.ndarray
    Wv: np.ndarray
    Wg: np.ndarray
    Wb: np.ndarray
    Wo: np.ndarray
    bg: np.ndarray | None = None
    bo: np.ndarray | None = None
    mask: np.ndarray | None = None
    H: int = 4
    d: int = 32
    eps: float = 1e-5

    def _keep(self):
        # keep contiguous copies alive for as long as the ctypes struct is used
        self._arrs = {
            "Z": np.ascontiguousarray(self.Z),
            "mask": None if self.mask is None else np.ascontiguousarray(self.mask, dtype=np.uint8),
            "gamma": _f64(self.gamma), "beta": _f64(self.beta),
            "Wq": _f64(self.Wq), "Wk": _f64(self.Wk), "Wv": _f64(self.Wv), "Wg": _f64(self.Wg),
            "bg": _f64(self.bg), "Wb": _f64(self.Wb), "Wo": _f64(self.Wo), "bo": _f64(self.bo),
        }
        return self._arrs

    def params(self) -> _Params:
        a = self._keep()
        z = a["Z"]
        if z.dtype == np.float64:
            zt = Z_F64
        elif z.dtype == np.float32:
            zt = Z_F32
        elif z.dtype == np.uint16:
            zt = Z_BF16
        else:
            raise TypeError(f"unsupported Z dtype {z.dtype}")
        N, N2, cz = z.shape
        assert N == N2
        return _Params(N, cz, self.H, self.d, self.eps, zt, _ptr(z), _ptr(a["mask"]),
                       _ptr(a["gamma"]), _ptr(a["beta"]), _ptr(a["Wq"]), _ptr(a["Wk"]),
                       _ptr(a["Wv"]), _ptr(a["Wg"]), _ptr(a["bg"]), _ptr(a["Wb"]),
                       _ptr(a["Wo"]), _ptr(a["bo"]))

    @property
    def N(self) -> int:
        return int(self.Z.shape[0])

    @property
    def c_z(self) -> int:
        return int(self.Z.shape[2])


def layer_norm(z: np.ndarray, gamma, beta, eps: float) -> np.ndarray:
    z = _f64(z)
    cz = z.shape[-1]
    x = np.empty_like(z)
    g, b = _f64(gamma), _f64(beta)
    rc = lib().oracle_layer_norm(_ptr(z), z.size // cz, cz, eps, _ptr(g), _ptr(b), _ptr(x))
    assert rc == 0
    return x


def pair_features(p: Problem):
    """q, k, v, g as (N, N, H*d) and the unmasked bias as (H, N, N)."""
    N, HD = p.N, p.H * p.d
    q = np.empty((N, N, HD)); k = np.empty_like(q); v = np.empty_like(q); g = np.empty_like(q)
    b = np.empty((p.H, N, N))
    prm = p.params()
    rc = lib().oracle_pair_features(ctypes.byref(prm), _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(b))
    assert rc == 0
    return q, k, v, g, b


def bias_all(p: Problem) -> np.ndarray:
    N = p.N
    b = np.empty((p.H, N, N))
    prm = p.params()
    rc = lib().oracle_pair_features(ctypes.byref(prm), None, None, None, None, _ptr(b))
    assert rc == 0
    return b


def attend(q, k, v, bias, mask=None, want_probs=False):
    """q: (Nq, H, d); k, v: (Nk, H, d); bias: (H, Nq, Nk).  Full softmax."""
    q, k, v, bias = _f64(q), _f64(k), _f64(v), _f64(bias)
    Nq, H, d = q.shape
    Nk = k.shape[0]
    o = np.empty((Nq, H, d))
    probs = np.empty((H, Nq, Nk)) if want_probs else None
    m = None if mask is None else np.ascontiguousarray(mask, dtype=np.uint8)
    rc = lib().oracle_attend(_ptr(q), _ptr(k), _ptr(v), _ptr(bias), _ptr(m), Nq, Nk, H, d,
                             _ptr(o), _ptr(probs))
    assert rc == 0
    return (o, probs) if want_probs else o


def attend_blockwise(q, k, v, bias, mask=None, block=7):
    q, k, v, bias = _f64(q), _f64(k), _f64(v), _f64(bias)
    Nq, H, d = q.shape
    Nk = k.shape[0]
    o = np.empty((Nq, H, d))
    m = None if mask is None else np.ascontiguousarray(mask, dtype=np.uint8)
    rc = lib().oracle_attend_blockwise(_ptr(q), _ptr(k), _ptr(v), _ptr(bias), _ptr(m), Nq, Nk,
                                       H, d, block, _ptr(o))
    assert rc == 0
    return o


def attend_bwd(q, k, v, bias, dout, mask=None):
    """Gradients (dq, dk, dv, dbias) of attend(q, k, v, bias, mask) given the
    gradient dout of a loss with respect to its output (shapes as attend)."""
    q, k, v, bias, dout = _f64(q), _f64(k), _f64(v), _f64(bias), _f64(dout)
    Nq, H, d = q.shape
    Nk = k.shape[0]
    dq, dk, dv = np.empty_like(q), np.empty_like(k), np.empty_like(v)
    dbias = np.empty((H, Nq, Nk))
    m = None if mask is None else np.ascontiguousarray(mask, dtype=np.uint8)
    rc = lib().oracle_attend_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(bias), _ptr(m), _ptr(dout), Nq,
                                 Nk, H, d, _ptr(dq), _ptr(dk), _ptr(dv), _ptr(dbias))
    assert rc == 0
    return dq, dk, dv, dbias


def tri_attn_core_bwd(q, k, v, bias, dout, mask=None):
    """Backward of the starting-node attention core over R problem rows, each
    row an attend() call with its own q, k, v and the shared bias:
    q, k, v, dout: (R, N, H, d); bias: (H, N, N).  Returns dq, dk, dv
    (R, N, H, d) and dbias (H, N, N), the bias gradient summed over the rows.
    (The ending-node core is the same computation on the transposed problem.)"""
    R = q.shape[0]
    outs = [attend_bwd(q[r], k[r], v[r], bias, dout[r], mask) for r in range(R)]
    dq = np.stack([o[0] for o in outs])
    dk = np.stack([o[1] for o in outs])
    dv = np.stack([o[2] for o in outs])
    dbias = np.zeros_like(_f64(bias))
    for o in outs:
        dbias += o[3]
    return dq, dk, dv, dbias


def tri_attn(p: Problem, orientation: int, lines=None, bias=None, want_o: bool = False):
    """The whole block.  orientation 0 (starting node): returns out[lines, :, :];
    orientation 1 (ending node): returns out[:, lines, :] laid out as
    (len(lines), N, c_z), i.e. result[r, i] = out[i, lines[r]].
    With want_o, returns (out, o): o is the attention output before the gate,
    (len(lines), N, H, d), in the same line layout."""
    N, cz = p.N, p.c_z
    if lines is None:
        ln_arr, n = None, N
    else:
        ln_arr = np.ascontiguousarray(np.asarray(lines, dtype=np.int32))
        n = len(ln_arr)
    out = np.empty((n, N, cz))
    o = np.empty((n, N, p.H, p.d)) if want_o else None
    b = None if bias is None else _f64(bias)
    prm = p.params()
    rc = lib().oracle_tri_attn(ctypes.byref(prm), int(orientation), _ptr(ln_arr), n, _ptr(b),
                               _ptr(out), _ptr(o))
    assert rc == 0, rc
    return (out, o) if want_o else out


def tri_attn_full(p: Problem, orientation: int, bias=None) -> np.ndarray:
    """out as (N, N, c_z) in Z's own indexing for either orientation."""
    r = tri_attn(p, orientation, None, bias)
    return r if orientation == 0 else np.ascontiguousarray(r.transpose(1, 0, 2))
