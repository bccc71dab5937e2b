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
# The attention update itself: rel-L2 of the GPU's attention output o against
# the oracle's (and, where the residual does not dominate out, of out - z
# against oracle - z).  The residual z is ~94% of |out| at N = 1536, so the
# out-level bounds above alone would admit an update several percent off.
TOL_UPD_RELL2 = 2e-2

# one line per comparison, printed in the terminal summary (conftest.py)
PARITY_LOG: list[str] = []


def log_parity(what: str, st: dict, n_lines=None):
    keys = ["max_abs", "rel_l2", "upd_rel_l2", "upd_floor", "o_rel_l2", "o_max_abs"]
    parts = [f"{k} {st[k]:.2e}" for k in keys if k in st]
    if n_lines is not None:
        parts.append(f"lines {n_lines}")
    PARITY_LOG.append(f"{what}: " + ", ".join(parts))


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


def _bf16_round(x: np.ndarray) -> np.ndarray:
    return torch.from_numpy(np.asarray(x, dtype=np.float32)).to(torch.bfloat16).double().numpy()


def compare(got: np.ndarray, ref: np.ndarray, z: np.ndarray, dtype: str,
            got_o: np.ndarray | None = None, ref_o: np.ndarray | None = None) -> dict:
    """Errors of out and of the attention update.

    upd_rel_l2 = |out - oracle| / |oracle - z|: the out-level error relative to
    the update.  upd_floor is what the bf16 rounding of out alone contributes to
    it (|bf16(oracle) - oracle| / |oracle - z|): out is stored in Z's dtype, and
    where z dominates out that rounding is a sizeable fraction of the update.
    With got_o/ref_o (the attention output o before the gate, GPU and oracle),
    o_rel_l2 = |o_gpu - o_oracle| / |o_oracle| measures the update directly."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    diff = got - ref
    upd = max(np.linalg.norm(ref - z), 1e-300)
    st = {
        "max_abs": float(np.abs(diff).max()) if diff.size else 0.0,
        "rel_l2": float(np.linalg.norm(diff) / max(np.linalg.norm(ref), 1e-300)),
        "upd_rel_l2": float(np.linalg.norm(diff) / upd),
        "upd_norm_frac": float(upd / max(np.linalg.norm(ref), 1e-300)),
        "max_ref": float(np.abs(ref).max()) if ref.size else 0.0,
        "finite": bool(np.isfinite(got).all()),
    }
    if dtype == "bf16":
        st["upd_floor"] = float(np.linalg.norm(_bf16_round(ref) - ref) / upd)
    if got_o is not None:
        got_o = np.asarray(got_o, dtype=np.float64)
        ref_o = np.asarray(ref_o, dtype=np.float64)
        do = got_o - ref_o
        st["o_rel_l2"] = float(np.linalg.norm(do) / max(np.linalg.norm(ref_o), 1e-300))
        st["o_max_abs"] = float(np.abs(do).max()) if do.size else 0.0
        st["o_finite"] = bool(np.isfinite(got_o).all())
    return st


def assert_within(st: dict, dtype: str, what: str = "", update_at_out: bool = False):
    """The parity tolerances on out (fp32: max-abs 1e-4; bf16: rel-L2 5e-3 and
    max-abs 2e-2); for bf16 also the update target on the
    attention output (when given) and, with update_at_out, on out - z (for
    inputs whose residual does not dominate out)."""
    assert st["finite"], f"{what}: non-finite output"
    if dtype == "f32":
        assert st["max_abs"] <= TOL_F32_MAXABS, f"{what}: {st}"
    else:
        # bf16 rounding of out adds <= half an ulp of |out|; below 8 that is <= 0.0156
        assert st["max_ref"] < 8.0, f"{what}: |out| too large for the bf16 bound: {st}"
        assert st["rel_l2"] <= TOL_BF16_RELL2, f"{what}: {st}"
        assert st["max_abs"] <= TOL_BF16_MAXABS, f"{what}: {st}"
        if "o_rel_l2" in st:
            assert st["o_finite"], f"{what}: non-finite attention output"
            assert st["o_rel_l2"] <= TOL_UPD_RELL2, f"{what}: attention output {st}"
        if update_at_out:
            assert st["upd_rel_l2"] <= TOL_UPD_RELL2, f"{what}: update {st}"


def attn_output_lines(blk, N: int, lines, dtype: torch.dtype = torch.bfloat16) -> np.ndarray:
    """The GPU's attention output o (before the gate) of the block's last,
    unchunked forward, for the given lines, as (len(lines), N, H, d): the
    workspace holds o head-major per problem row ([row][H][N][d]), and problem
    rows are the oracle's lines (rows of Z for the starting node, columns for
    the ending node)."""
    ws = blk.debug_workspace()
    assert ws["rows"] == N, "the last forward ran in row chunks; o of every row is not resident"
    O = device_view(ws["o"], (N, 4, N, 32), dtype)
    idx = torch.as_tensor(list(lines), device="cuda", dtype=torch.long)
    return O.index_select(0, idx).permute(0, 2, 1, 3).to(torch.float64).cpu().numpy()


def lines_of(out_dev: torch.Tensor, orientation: int, lines) -> np.ndarray:
    """GPU output at the oracle's line layout: rows (starting) or columns (ending)."""
    idx = torch.as_tensor(list(lines), device=out_dev.device, dtype=torch.long)
    sel = out_dev.index_select(0, idx) if orientation == 0 else out_dev.index_select(1, idx).transpose(0, 1)
    return sel.to(torch.float64).cpu().numpy()


def z_lines(z: torch.Tensor, orientation: int, lines) -> np.ndarray:
    idx = torch.as_tensor(list(lines), dtype=torch.long)
    sel = z.index_select(0, idx) if orientation == 0 else z.index_select(1, idx).transpose(0, 1)
    return sel.to(torch.float64).numpy()
