"""The FMA-pipe exp2 used by the forward sweep (Cody-Waite reduction + degree-5 Chebyshev
interpolation polynomial) against float64 and against CUDA's exp2f, on 4M inputs in
[-124, 0.5] (the range the stabilised sweep feeds it)."""
import os
import subprocess
import tempfile

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
pytestmark = pytest.mark.gpu


def test_fma_exp2_error_bound():
    with tempfile.TemporaryDirectory() as td:
        exe = os.path.join(td, "exp2_check")
        subprocess.check_call(["/usr/local/cuda/bin/nvcc", "-O3", "-gencode", "arch=compute_100a,code=sm_100a",
                               os.path.join(ROOT, "tests", "cuda", "exp2_check.cu"), "-o", exe])
        out = os.path.join(td, "y.bin")
        subprocess.check_call([exe, out])
        raw = np.fromfile(out, dtype=np.float32)
    n = raw.size // 3
    x, y_fma, y_cuda = raw[:n], raw[n:2 * n], raw[2 * n:]
    ref = np.exp2(x.astype(np.float64))
    rel_fma = np.abs(y_fma.astype(np.float64) - ref) / ref
    rel_cuda = np.abs(y_cuda.astype(np.float64) - ref) / ref
    assert rel_fma.max() <= 5e-7, rel_fma.max()
    # no worse than a few ulp of CUDA's own exp2f
    assert rel_fma.max() <= 4.0 * max(rel_cuda.max(), 2.0 ** -23)
