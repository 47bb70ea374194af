"""The GPU's approximate base-2 exponential against the error bound the
oracle's ambiguity band assumes.

The attention kernel evaluates P~ = 2^x with ex2.approx.ftz.f32.  The oracle
(sage_oracle.c, orc_p_band) counts its error as at most 2^-22 relative -- two
units in the last place of a float32 result, the documented bound.  This test
builds a small probe (tests/probes/ex2_error.cu, not part of the library) and
measures the largest relative error over every float32 argument in
[-40, 11], the range the kernel's arguments fall in (log2 448 + tau at the
top; below -40 every P~ rounds to 0 in E4M3 and in binary16)."""
import ctypes
import os
import subprocess
import tempfile

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

HERE = os.path.dirname(os.path.abspath(__file__))
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")


@pytest.fixture(scope="module")
def probe():
    d = tempfile.mkdtemp(prefix="ex2probe")
    so = os.path.join(d, "ex2_error.so")
    subprocess.check_call([NVCC, "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-shared", "-Xcompiler",
                           "-fPIC", "-o", so, os.path.join(HERE, "probes", "ex2_error.cu")])
    L = ctypes.CDLL(so)
    L.ex2_max_rel_error.restype = ctypes.c_int
    L.ex2_max_rel_error.argtypes = [ctypes.c_float, ctypes.c_float, ctypes.c_void_p, ctypes.c_void_p]
    return L


def test_ex2_approx_within_the_band_assumption(probe):
    worst = torch.zeros(1, dtype=torch.int32, device="cuda")
    rc = probe.ex2_max_rel_error(-40.0, 11.0, worst.data_ptr(), torch.cuda.current_stream().cuda_stream)
    assert rc == 0
    torch.cuda.synchronize()
    w = float(np.array([worst.item()], np.int32).view(np.float32)[0])
    print(f"ex2.approx.ftz.f32: largest relative error over [-40, 11] = {w:.3e} = 2^{np.log2(w):.2f}")
    assert 0 < w <= 2.0 ** -22, w
