"""The FMA-pipe 2^x of the attention forward against CUDA's exp2f.

exp2_poly2 (csrc/tc.cuh) reduces x = n + f with n = round(x) and evaluates a
degree-3 minimax polynomial for 2^f on [-1/2, 1/2]; its stated bound is a
relative error of 7.5e-5 (from the Remez exchange in gen_exp2_poly.py) plus
fp32 rounding.  A small kernel built here evaluates it next to exp2f.
"""
import ctypes
import os
import subprocess
import tempfile

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = r"""
#include "tc.cuh"
extern "C" __global__ void k(const float* x, float* yp, float* yr, int n) {
  int i = 2 * (blockIdx.x * blockDim.x + threadIdx.x);
  if (i + 1 >= n) return;
  float2 y = lh::tc::exp2_poly2(make_float2(x[i], x[i + 1]));
  yp[i] = y.x; yp[i + 1] = y.y;
  yr[i] = exp2f(x[i]); yr[i + 1] = exp2f(x[i + 1]);
}
extern "C" int run(const float* x, float* yp, float* yr, int n) {
  k<<<(n / 2 + 255) / 256, 256>>>(x, yp, yr, n);
  return (int)cudaDeviceSynchronize();
}
"""


def test_exp2_poly_within_bound():
    d = tempfile.mkdtemp()
    cu, so = os.path.join(d, "e.cu"), os.path.join(d, "e.so")
    open(cu, "w").write(SRC)
    inc = os.path.join(ROOT, "long_context_hierarchical_b200", "csrc")
    subprocess.run(["nvcc", "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-shared",
                    "-Xcompiler", "-fPIC", f"-I{inc}", "-o", so, cu], check=True)
    lib = ctypes.CDLL(so)
    x = torch.cat([torch.linspace(-124.0, 8.0, 1 << 20), torch.rand(1 << 20) * -30.0,
                   torch.tensor([0.0, -0.5, 0.5, -1.0, 1.0, -124.5, 7.999])]).float()
    n = x.numel() - (x.numel() % 2)
    x = x[:n].cuda()
    yp, yr = torch.empty_like(x), torch.empty_like(x)
    assert lib.run(ctypes.c_void_p(x.data_ptr()), ctypes.c_void_p(yp.data_ptr()),
                   ctypes.c_void_p(yr.data_ptr()), n) == 0
    rel = ((yp.double() - yr.double()).abs() / yr.double()).cpu().numpy()
    assert np.all(np.isfinite(rel))
    assert rel.max() <= 7.5e-5 + 3e-7, rel.max()
