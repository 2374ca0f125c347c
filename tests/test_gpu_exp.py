"""Accuracy of the sampler's own fp64 exp (Tang's table-driven method: a
64-entry table of 2^(j/64) built with CUDA's exp2, a degree-5 Taylor series
on |r| <= ln2/128) against CUDA's exp: at most 3 ulp apart on [-745, 0]
(table entries within exp2's 1-ulp bound, the series and the final multiply
within about 1 ulp, CUDA's exp within its own 1-ulp bound), exact at 0, and
0 below the subnormal range."""
import ctypes
import os
import subprocess
import tempfile

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu
HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)


@pytest.fixture(scope="module")
def exp_pair():
    out = os.path.join(tempfile.mkdtemp(), "exp_check.so")
    subprocess.check_call(["/usr/local/cuda/bin/nvcc", "-gencode", "arch=compute_100a,code=sm_100a",
                           "-O3", "-std=c++17", "-Xcompiler", "-fPIC", "-shared", "-I",
                           os.path.join(ROOT, "include"), "-o", out,
                           os.path.join(HERE, "gpu_helpers", "exp_check.cu")])
    lib = ctypes.CDLL(out)
    lib.exp_pair.argtypes = [ctypes.c_void_p] * 3 + [ctypes.c_int]
    lib.exp_pair.restype = ctypes.c_int

    def run(x: np.ndarray):
        xt = torch.as_tensor(x, dtype=torch.float64).cuda()
        a = torch.empty_like(xt)
        b = torch.empty_like(xt)
        assert lib.exp_pair(xt.data_ptr(), a.data_ptr(), b.data_ptr(), xt.numel()) == 0
        return a.cpu().numpy(), b.cpu().numpy()
    return run


def ulps(a, b):
    ia = a.view(np.int64)
    ib = b.view(np.int64)
    return np.abs(ia - ib)


def test_exp_within_three_ulp_of_cuda(exp_pair):
    rng = np.random.default_rng(0)
    x = np.concatenate([-rng.random(1_000_000) * 745.0, -rng.random(1_000_000) * 40.0,
                        -rng.random(100_000) * 1e-6, -np.arange(0, 746, 0.5)])
    mine, ref = exp_pair(x)
    normal = ref > 2.3e-308
    d = ulps(mine[normal], ref[normal])
    print(f"max ulp difference {d.max()}, mean {d.mean():.3f}")
    assert d.max() <= 3
    # subnormal results: agree to the subnormal spacing
    assert np.abs(mine[~normal] - ref[~normal]).max() <= 4 * 5e-324


def test_exp_special_points(exp_pair):
    x = np.array([0.0, -0.0, -1e-300, -745.3, -800.0, -np.inf, np.log(0.5)])
    mine, ref = exp_pair(x)
    assert mine[0] == 1.0 and mine[1] == 1.0 and mine[2] == 1.0
    assert mine[3] == 0.0 and mine[4] == 0.0 and mine[5] == 0.0
    assert abs(mine[6] - 0.5) <= 2.3e-16
