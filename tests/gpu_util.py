"""Helpers shared by the GPU tests: run the CUDA path, view workspace pointers,
compare against the oracle at the stated tolerances."""
from __future__ import annotations

import numpy as np
import torch

from protein_pair_representation_layernorm_b200 import binding, workloads

ORIENT = {"starting": binding.TRI_ATTN_STARTING, "ending": binding.TRI_ATTN_ENDING}

# fp32 inputs: max-abs 1e-4.  bf16 inputs with fp32 accumulation: rel-L2 5e-3
# and max-abs 2e-2 on out.
TOL_F32_MAXABS = 1e-4
TOL_BF16_RELL2 = 5e-3
TOL_BF16_MAXABS = 2e-2


def block_for(inp: workloads.Inputs) -> binding.TriangleAttention:
    return binding.TriangleAttention(inp.weights(), dtype=inp.Z.dtype)


def run_gpu(inp: workloads.Inputs, orientation: int, blk=None, flags=0, inplace=False):
    """Returns (out on device, block)."""
    blk = blk or block_for(inp)
    Z = inp.Z.cuda()
    mask = None if inp.mask is None else inp.mask.cuda()
    if inplace:
        out = blk.forward(Z, orientation, mask, out=Z, flags=flags | binding.TRI_ATTN_FLAG_SYNC)
    else:
        out = blk.forward(Z, orientation, mask, flags=flags | binding.TRI_ATTN_FLAG_SYNC)
    torch.cuda.synchronize()
    return out, blk


class _CAI:
    def __init__(self, ptr, shape, typestr):
        self.__cuda_array_interface__ = {"shape": tuple(shape), "typestr": typestr,
                                         "data": (int(ptr), False), "version": 3}


def device_view(ptr: int, shape, dtype: torch.dtype) -> torch.Tensor:
    """Zero-copy tensor over library-owned device memory (valid while the handle lives)."""
    if dtype == torch.bfloat16:
        t = torch.as_tensor(_CAI(ptr, shape, "<i2"), device="cuda")
        return t.view(torch.bfloat16)
    if dtype == torch.float32:
        return torch.as_tensor(_CAI(ptr, shape, "<f4"), device="cuda")
    raise TypeError(dtype)


def compare(got: np.ndarray, ref: np.ndarray, z: np.ndarray, dtype: str) -> dict:
    """Errors of out and of the attention update (out - z)."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    diff = got - ref
    st = {
        "max_abs": float(np.abs(diff).max()) if diff.size else 0.0,
        "rel_l2": float(np.linalg.norm(diff) / max(np.linalg.norm(ref), 1e-300)),
        "upd_rel_l2": float(np.linalg.norm(diff) / max(np.linalg.norm(ref - z), 1e-300)),
        "max_ref": float(np.abs(ref).max()) if ref.size else 0.0,
        "finite": bool(np.isfinite(got).all()),
    }
    return st


def assert_within(st: dict, dtype: str, what: str = ""):
    assert st["finite"], f"{what}: non-finite output"
    if dtype == "f32":
        assert st["max_abs"] <= TOL_F32_MAXABS, f"{what}: {st}"
    else:
        # bf16 rounding of out adds <= half an ulp of |out|; below 8 that is <= 0.0156
        assert st["max_ref"] < 8.0, f"{what}: |out| too large for the bf16 bound: {st}"
        assert st["rel_l2"] <= TOL_BF16_RELL2, f"{what}: {st}"
        assert st["max_abs"] <= TOL_BF16_MAXABS, f"{what}: {st}"


def lines_of(out_dev: torch.Tensor, orientation: int, lines) -> np.ndarray:
    """GPU output at the oracle's line layout: rows (starting) or columns (ending)."""
    idx = torch.as_tensor(list(lines), device=out_dev.device, dtype=torch.long)
    sel = out_dev.index_select(0, idx) if orientation == 0 else out_dev.index_select(1, idx).transpose(0, 1)
    return sel.to(torch.float64).cpu().numpy()


def z_lines(z: torch.Tensor, orientation: int, lines) -> np.ndarray:
    idx = torch.as_tensor(list(lines), dtype=torch.long)
    sel = z.index_select(0, idx) if orientation == 0 else z.index_select(1, idx).transpose(0, 1)
    return sel.to(torch.float64).numpy()
