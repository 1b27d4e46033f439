"""Failure detection without faulting the GPU: a bounded wait that can never
be satisfied gives up, latches the timeout bit and returns; the context stays
usable and the cache reports device errors through h2o_cache_check.  Host
validation rejects bad arguments before anything is launched."""
import ctypes
import time

import numpy as np
import pytest
import torch

import gpu_helpers as gh
from kv_cache_sparse_b200 import binding

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lib(cuda_ok):
    gh.ensure_built()
    L = binding.load_library()
    L.h2o_selftest_wait_timeout.argtypes = [ctypes.c_void_p, ctypes.c_uint32, ctypes.c_void_p]
    return L


def test_bounded_wait_times_out_and_context_survives(lib):
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    t = time.time()
    assert lib.h2o_selftest_wait_timeout(ctypes.c_void_p(err.data_ptr()), 20000, None) == 0
    torch.cuda.synchronize()
    elapsed = time.time() - t
    assert err.item() == 1            # the timeout bit
    assert elapsed < 5.0
    # the context still works: a normal step afterwards is correct
    shape = gh.shape_of(1, 4, 2, 128, 256, 128, 0)
    gpu = binding.H2OCache(shape)
    ref = gh.oracle_for(shape)
    q = torch.randn(1, 128, 4, 128).to(torch.bfloat16)
    kn = torch.randn(1, 128, 2, 128).to(torch.bfloat16)
    vn = torch.randn(1, 128, 2, 128).to(torch.bfloat16)
    O, cs = gpu.attention(q.cuda(), kn.cuda(), vn.cuda())
    O_ref, cs_ref, _ = ref.attention(gh.np64(q), gh.np64(kn), gh.np64(vn))
    gh.assert_attention_close(O, cs, O_ref, cs_ref, 128, 2, "after timeout")
    assert gpu.check() == 0


def test_state_word_reports_device_errors(lib):
    """h2o_cache_check maps the latched device bits to statuses."""
    shape = gh.shape_of(1, 4, 2, 128, 256, 128, 0)
    gpu = binding.H2OCache(shape)
    assert gpu.check() == 0
    gpu.state[2] = 1          # as a timed-out wait would leave it
    assert gpu.check() == 6   # H2O_ERR_TIMEOUT
    gpu.state[2] = 2          # inconsistent eviction plan
    assert gpu.check() == 7   # H2O_ERR_STATE
    st = gpu.read()
    gpu.write(st["k"], st["v"], st["scores"], st["pos"], st["n"], st["t0"])  # clears the bits
    assert gpu.check() == 0


def test_host_validation_rejects_before_launch(lib):
    shape = gh.shape_of(1, 4, 2, 128, 256, 64, 0)
    gpu = binding.H2OCache(shape)
    q = torch.zeros(1, 65, 4, 128, dtype=torch.bfloat16, device="cuda")
    kv = torch.zeros(1, 65, 2, 128, dtype=torch.bfloat16, device="cuda")
    L = binding.lib()
    out = torch.empty_like(q)
    P = ctypes.c_void_p
    # n_q above max_chunk
    assert L.h2o_chunk_step(gpu._h, P(q.data_ptr()), P(kv.data_ptr()), P(kv.data_ptr()), 65,
                            P(out.data_ptr()), None, None) == 1
    # misaligned pointer
    assert L.h2o_chunk_step(gpu._h, P(q.data_ptr() + 2), P(kv.data_ptr()), P(kv.data_ptr()), 8,
                            P(out.data_ptr()), None, None) == 4
    # n_q = 0 is a no-op
    assert L.h2o_chunk_step(gpu._h, None, None, None, 0, None, None, None) == 0
    assert gpu.info()["kernel_launches"] == 0
    assert gpu.info()["n"] == 0
