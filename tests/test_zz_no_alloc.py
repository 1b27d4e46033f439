"""h2o_attention_static_scratch, the entry point for callers that cannot
allocate device memory (plugin hosts that hand over only inputs and outputs,
serving loops that must not allocate once running), gives the same attention
output and summed weights as h2o_attention.

The test itself allocates its tensors with torch as any test does; the entry
point under test is handed only inputs and outputs and keeps its row
statistics in the library's static device array.  Two calls in a row with
different shapes check that the shared array's leftover contents from the
previous call do not leak into the next.
"""
import ctypes

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
    P, I = ctypes.c_void_p, ctypes.c_int32
    L.h2o_attention_static_scratch.argtypes = [ctypes.POINTER(binding.Config), P, P, I, P, P, P,
                                              I, P, P, P]
    L.h2o_attention_static_scratch.restype = ctypes.c_int
    return L


def call_static(L, shape, gpu, n, q, kn, vn):
    s = shape
    out = torch.empty(s.batch, q.shape[1], s.n_q_heads, s.head_dim, dtype=s.dtype, device="cuda")
    cs = torch.full((s.batch, s.n_kv_heads, s.capacity + q.shape[1]), float("nan"),
                    dtype=torch.float32, device="cuda")
    cfg = s.config()
    st = L.h2o_attention_static_scratch(
        ctypes.byref(cfg), ctypes.c_void_p(gpu.k.data_ptr()), ctypes.c_void_p(gpu.v.data_ptr()),
        n, ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(kn.data_ptr()),
        ctypes.c_void_p(vn.data_ptr()), q.shape[1], ctypes.c_void_p(out.data_ptr()),
        ctypes.c_void_p(cs.data_ptr()), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == 0, binding.STATUS_NAMES.get(st, st)
    torch.cuda.synchronize()
    return out, cs


CALLS = [
    # B, Hq, Hkv, d, C, n, nq, dtype
    (1, 8, 2, 128, 1024, 1000, 384, torch.bfloat16),
    (2, 4, 2, 128, 300, 77, 129, torch.bfloat16),
    (1, 4, 2, 64, 256, 256, 64, torch.float32),
]


def test_static_scratch_matches_h2o_attention(lib):
    rng = np.random.default_rng(5)
    for B, Hq, Hkv, d, C, n, nq, dt in CALLS:   # calls in a row share the static array
        shape = gh.shape_of(B, Hq, Hkv, d, C, nq, 0, dt)
        gpu = binding.H2OCache(shape)
        K, V, sc, pos = gh.random_state(shape, n, n + 1, rng)
        gpu.write(K, V, torch.from_numpy(sc), torch.from_numpy(pos), n, n + 1)
        q = torch.randn(B, nq, Hq, d).to(dt).cuda()
        kn = torch.randn(B, nq, Hkv, d).to(dt).cuda()
        vn = torch.randn(B, nq, Hkv, d).to(dt).cuda()
        O_ref, cs_ref = gpu.attention(q, kn, vn)
        O, cs = call_static(lib, shape, gpu, n, q, kn, vn)
        gh.assert_attention_close(O, cs, gh.np64(O_ref), gh.np64(cs_ref), nq, Hq // Hkv,
                                  f"static scratch {B, Hq, Hkv, d, C, n, nq}")
        assert not torch.isnan(cs).any()


def test_static_scratch_rejects_oversize(lib):
    # 144 caches x 32 heads x 1024 rows exceed the 4 Mi-row static array
    shape = gh.shape_of(144, 32, 8, 128, 1024, 1024, 0)
    cfg = shape.config()
    dummy = torch.empty(16, dtype=torch.uint8, device="cuda")
    p = ctypes.c_void_p(dummy.data_ptr())
    st = lib.h2o_attention_static_scratch(ctypes.byref(cfg), p, p, 0, p, p, p, 1024, p, p, None)
    assert st == 2  # H2O_ERR_SHAPE, before anything is launched
