"""The FMA-pipe exponential of the attention kernels: its polynomial is the
relative-error minimax fit of 2^f on [0, 1] (Remez exchange), the constants
in the device header are that fit, the error bound holds, and (on a GPU) the
device routine agrees with the library exp2f within the bound."""
import ctypes
import os
import re

import numpy as np
import pytest

from kv_cache_sparse_b200.exp2_poly import max_rel_error, remez_exp2

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
BOUND = 7.5e-5


def header_coefficients():
    text = open(os.path.join(ROOT, "kv_cache_sparse_b200", "csrc", "sm100.cuh")).read()
    return [float(re.search(rf"kExp2C{i} = ([0-9.eE+-]+)f;", text).group(1)) for i in range(4)]


def test_remez_fit_equioscillates_and_meets_the_bound():
    c, E = remez_exp2(3)
    assert E < BOUND
    # minimax: the largest error on a fine grid equals the levelled error
    assert abs(max_rel_error(c) - E) < 1e-3 * E
    # a plain least-squares fit of the same degree is worse in the max norm
    f = np.linspace(0, 1, 4001)
    ls = np.polyfit(f, 2.0 ** f, 3)[::-1]
    assert max_rel_error(ls) > E


def test_header_constants_are_the_fit():
    c, _ = remez_exp2(3)
    assert np.allclose(header_coefficients(), c, rtol=0, atol=1e-9)


def _emulate_fp32(x):
    """The device routine's steps in float32 (numpy; fma rounding aside)."""
    c = np.array(header_coefficients(), np.float32)
    x = np.maximum(np.asarray(x, np.float32), np.float32(-125))
    j = np.floor(x).astype(np.float32)
    f = (x - j).astype(np.float32)
    p = ((c[3] * f + c[2]) * f + c[1]) * f + c[0]
    return np.ldexp(p.astype(np.float64), j.astype(np.int64))


def test_range_reduction_steps_meet_the_bound_in_fp32():
    x = np.concatenate([np.linspace(-125, 0, 200001, dtype=np.float32),
                        np.float32([-0.0, -1e-7, -0.5, -1.0, -124.99, -125.0])])
    y = _emulate_fp32(x)
    rel = np.abs(y / np.exp2(x.astype(np.float64)) - 1)
    assert rel.max() < BOUND + 1e-6


@pytest.mark.gpu
def test_device_exp2_agrees_with_exp2f(cuda_ok):
    import torch
    from kv_cache_sparse_b200 import binding
    from kv_cache_sparse_b200.build import build
    build()
    lib = binding.load_library()
    x = torch.cat([torch.linspace(-125, 0, 1 << 20), torch.tensor([-0.0, -1e-7, 1e-7, -0.5,
                                                                   -1.0, -124.99, -125.0])])
    x = x.cuda()
    y = torch.empty_like(x)
    assert lib.h2o_selftest_exp2(ctypes.c_void_p(x.data_ptr()), ctypes.c_void_p(y.data_ptr()),
                                 x.numel(), None) == 0
    torch.cuda.synchronize()
    ref = torch.exp2(x)                      # the CUDA library's exp2f
    rel = ((y.double() - ref.double()).abs() / ref.double()).max().item()
    assert rel < BOUND + 1e-6
    # below the range: about 2^-125 (the callers treat it as zero)
    z = torch.tensor([-float("inf"), -1000.0, -127.5, -125.5], device="cuda")
    w = torch.empty_like(z)
    assert lib.h2o_selftest_exp2(ctypes.c_void_p(z.data_ptr()), ctypes.c_void_p(w.data_ptr()),
                                 4, None) == 0
    torch.cuda.synchronize()
    assert torch.all(w <= 2.0 ** -125 * (1 + BOUND))
