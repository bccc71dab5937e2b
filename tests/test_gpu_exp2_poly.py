"""exp2_poly2 (the FMA-pipe 2^x of the attention softmax) against CUDA's exp2.

The device function is compiled on its own into a small test library with
nvcc and evaluated over the range the softmax feeds it (x - m <= 8, down to
the masked-key logit); it must stay within the error bound of its fitted
polynomial (csrc/fit_exp2_poly.py: 7.5e-5 relative) where 2^x is a normal
float, give at most 2^-126 below that, and exactly 0 for -3e38 and -inf.
"""
import ctypes
import os
import shutil
import subprocess

import pytest
import torch

pytestmark = pytest.mark.gpu

CSRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                    "protein_pair_representation_layernorm_b200", "csrc")

SRC = r"""
#include "sm100.cuh"
__global__ void eval_poly(const float* x, float* y, int pairs) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < pairs) {
    const float2 r = tri::exp2_poly2(make_float2(x[2 * i], x[2 * i + 1]));
    y[2 * i] = r.x;
    y[2 * i + 1] = r.y;
  }
}
extern "C" int run_exp2_poly(const float* x, float* y, int pairs) {
  eval_poly<<<(pairs + 255) / 256, 256>>>(x, y, pairs);
  return static_cast<int>(cudaDeviceSynchronize());
}
"""


@pytest.fixture(scope="module")
def poly_lib(tmp_path_factory):
    nvcc = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    d = tmp_path_factory.mktemp("exp2poly")
    src = d / "poly.cu"
    src.write_text(SRC)
    lib = d / "libpoly.so"
    subprocess.check_call([nvcc, "-gencode", "arch=compute_100a,code=sm_100a", "-O3",
                           "-std=c++17", "-Xcompiler", "-fPIC", "-shared", "-I" + CSRC,
                           str(src), "-o", str(lib)])
    L = ctypes.CDLL(str(lib))
    L.run_exp2_poly.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int]
    return L


def _eval(L, x):
    x = x.to(torch.float32).cuda().contiguous()
    assert x.numel() % 2 == 0
    y = torch.empty_like(x)
    assert L.run_exp2_poly(x.data_ptr(), y.data_ptr(), x.numel() // 2) == 0
    return y


def test_exp2_poly_relative_error(poly_lib):
    # results stay normal floats down to x = -125 (2^n with n >= -125)
    x = torch.linspace(-125.0, 8.0, 2_000_000, dtype=torch.float32)
    y = _eval(poly_lib, x)
    ref = torch.exp2(x.cuda())  # CUDA's exp2 in fp32
    rel = ((y - ref).abs() / ref).max().item()
    assert rel < 8e-5, rel


def test_exp2_poly_underflow_and_masked_logits(poly_lib):
    x = torch.tensor([-125.9, -126.5, -126.9, -127.0, -150.0, -1000.0, -1.0e30, -3.0e38,
                      float("-inf"), 0.0, 1.0, 8.0], dtype=torch.float32)
    y = _eval(poly_lib, x).cpu()
    assert torch.all(y[:3] <= 2.0 ** -125) and torch.all(y[:3] >= 0)
    assert torch.all(y[3:9] == 0)
    assert abs(y[9].item() - 1.0) < 8e-5 and abs(y[10].item() - 2.0) < 1.6e-4
    assert abs(y[11].item() - 256.0) < 256.0 * 8e-5
