"""The polynomial base-2 exponential the kernels use for part of their
probabilities: its coefficients, re-fitted by the committed Remez script,
and the device evaluation against CUDA's exp2f."""
import ctypes
import os
import re

import numpy as np
import pytest
import torch

from kv_cache_sparse_b200.fit_exp2 import remez_exp2

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
BOUND = 3e-6   # fitted 2.6e-6, plus fp32 evaluation


def kernel_coefficients():
    src = open(os.path.join(ROOT, "kv_cache_sparse_b200", "csrc", "sm100.cuh")).read()
    body = src[src.index("float ex2_poly(float x)"):]
    body = body[:body.index("}")]
    vals = [float(v) for v in re.findall(r"(?<![\d.])(\d+\.\d+)f", body)]
    return [v for v in vals if v not in (125.0, 12582912.0)]


def f32_fma(a, b, c):
    return np.float32(np.float64(a) * np.float64(b) + np.float64(c))


def emulate(x):
    """The kernel's sequence of fp32 operations."""
    c4, c3, c2, c1, c0 = [np.float32(v) for v in kernel_coefficients()[:5]]
    x = np.maximum(np.float32(x), np.float32(-125.0))
    t = np.float32(x + np.float32(12582912.0))
    r = np.float32(t - np.float32(12582912.0))
    f = np.float32(x - r)
    p = f32_fma(c4, f, c3)
    p = f32_fma(p, f, c2)
    p = f32_fma(p, f, c1)
    p = f32_fma(p, f, c0)
    bits = (np.array(p, np.float32).view(np.int32) + (np.array(t, np.float32).view(np.int32) << 23))
    return bits.astype(np.int32).view(np.float32)


def test_coefficients_are_the_remez_fit():
    coef, err = remez_exp2(4)
    k = kernel_coefficients()
    # the kernel lists c4, c3, c2, c1, c0
    assert np.allclose(k[:5], coef[::-1], rtol=1e-6, atol=0)
    assert err < 2.7e-6


def test_emulated_polynomial_error_bound():
    xs = np.float32(-np.linspace(0, 125, 250001))
    got = np.array([emulate(x) for x in xs[::97]])
    ref = np.exp2(xs[::97].astype(np.float64))
    assert np.max(np.abs(got - ref) / ref) < BOUND
    # clamped region returns ~2^-125, a normal float (p(0) = c0 ~ 1)
    v = float(emulate(np.float32(-np.inf)))
    assert abs(v - 2.0 ** -125) / 2.0 ** -125 < BOUND


@pytest.mark.gpu
def test_device_polynomial_against_exp2f(cuda_ok):
    from kv_cache_sparse_b200 import binding
    from kv_cache_sparse_b200.build import build
    build()
    L = binding.load_library()
    L.h2o_selftest_exp2.argtypes = [ctypes.c_void_p] * 3 + [ctypes.c_int32, ctypes.c_void_p]
    x = -torch.linspace(0, 125, 1 << 20, device="cuda")
    yp, yl = torch.empty_like(x), torch.empty_like(x)
    st = L.h2o_selftest_exp2(ctypes.c_void_p(x.data_ptr()), ctypes.c_void_p(yp.data_ptr()),
                             ctypes.c_void_p(yl.data_ptr()), x.numel(), None)
    assert st == 0
    torch.cuda.synchronize()
    rel = ((yp.double() - yl.double()).abs() / yl.double()).max().item()
    assert rel < BOUND + 2e-7
    # bit-identical to the fp32 emulation of the same operations
    sample = x[:: 4099].cpu().numpy()
    assert np.array_equal(np.array([emulate(v) for v in sample]).view(np.int32),
                          yp[:: 4099].cpu().numpy().view(np.int32))
