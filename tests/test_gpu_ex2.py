"""The prefill softmax's exponential on the FMA pipe against the hardware's
ex2.approx, on the GPU (test build libflint_hooks.so).  ex2_fma2 computes 2^x
as 2^rint(x) times a degree-4 Chebyshev interpolant of 2^f on [-1/2, 1/2];
its bound (relative error below 3.6e-6 wherever 2^x is a normal float) is
derived in tests/test_kernel_math.py.  ex2.approx has a relative error of
about 2^-22 and flushes denormal results to zero."""
import ctypes

import numpy as np
import pytest
import torch

from long_context_decode_flash_b200 import build as cuda_build
from long_context_decode_flash_b200 import flint

pytestmark = pytest.mark.gpu


def test_ex2_on_the_fma_pipe_matches_ex2_approx():
    lib = flint.open_library(cuda_build.build_hooks())
    x = np.concatenate([np.linspace(-140.0, 8.0, 1_000_001), [-np.inf, 0.0, 8.0, -0.5, 0.5, -126.0, -125.5]])
    xd = torch.tensor(x, dtype=torch.float32, device="cuda")
    y_fma, y_mufu = torch.empty_like(xd), torch.empty_like(xd)
    assert lib.flint_test_ex2(ctypes.c_void_p(xd.data_ptr()), ctypes.c_void_p(y_fma.data_ptr()),
                              ctypes.c_void_p(y_mufu.data_ptr()), xd.numel(), None) == 0
    torch.cuda.synchronize()
    a, b = y_fma.cpu().numpy().astype(np.float64), y_mufu.cpu().numpy().astype(np.float64)
    normal = b >= 2.0 ** -126
    assert normal.sum() > 800_000
    rel = np.abs(a[normal] / b[normal] - 1.0)
    assert rel.max() <= 3.6e-6 + 2.0 ** -21, rel.max()
    # below the normal range both are negligible next to anything fp16 P keeps
    assert np.all(np.abs(a[~normal]) <= 2.0 ** -126) and np.all(b[~normal] == 0.0)
    assert list(a[-7:-4]) == [0.0, 1.0, 256.0]
