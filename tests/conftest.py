import os
import sys

import numpy as np
import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_terminal_summary(terminalreporter, exitstatus, config):
    """One line per GPU parity comparison (errors and lines compared)."""
    try:
        from gpu_util import PARITY_LOG
    except Exception:
        return
    if PARITY_LOG:
        terminalreporter.section("parity against the oracle")
        for line in PARITY_LOG:
            terminalreporter.write_line(line)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running CPU oracle case")


def to_numpy_f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to(torch.float64).cpu().numpy()


def z_for_oracle(z: torch.Tensor) -> np.ndarray:
    """Z in a form the oracle reads exactly: fp32 as float32, bf16 as raw bits."""
    z = z.detach().cpu().contiguous()
    if z.dtype == torch.bfloat16:
        return z.view(torch.int16).numpy().view(np.uint16)
    if z.dtype == torch.float32:
        return z.numpy()
    return z.to(torch.float64).numpy()


def to_problem(inp, eps: float = 1e-5):
    """Oracle problem from workload inputs (weights upcast exactly to fp64)."""
    import oracle
    f = to_numpy_f64
    return oracle.Problem(
        Z=z_for_oracle(inp.Z), gamma=f(inp.gamma), beta=f(inp.beta),
        Wq=f(inp.Wq), Wk=f(inp.Wk), Wv=f(inp.Wv), Wg=f(inp.Wg), Wb=f(inp.Wb), Wo=f(inp.Wo),
        bg=f(inp.bg), bo=f(inp.bo),
        mask=None if inp.mask is None else inp.mask.numpy().astype(np.uint8),
        H=inp.Wb.shape[0], d=inp.Wq.shape[0] // inp.Wb.shape[0], eps=eps)
