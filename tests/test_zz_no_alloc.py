"""h2o_attention_static_scratch, the entry point for callers that cannot
allocate device memory (plugin hosts that hand over only inputs and outputs,
serving loops that must not allocate once running), gives exactly the
attention output and summed weights of h2o_attention.

Both calls run the same two kernels on the same inputs and both kernels are
deterministic, so the outputs must be identical bit for bit; one case is also
checked against the CPU oracle.  The test itself allocates its tensors with
torch as any test does; the entry point under test is handed only inputs and
outputs and keeps its row statistics in the library's static device array.
The calls run back to back with different shapes, so leftovers of one call in
the shared array would show up in the next.  The last test drives the
failure path: a bounded wait that expires latches the static error word,
h2o_static_scratch_check reports it, and the next call clears it.
"""
import ctypes

import numpy as np
import pytest
import torch

import gpu_helpers as gh
from kv_cache_sparse_b200 import binding

pytestmark = pytest.mark.gpu

H2O_ERR_SHAPE, H2O_ERR_TIMEOUT = 2, 6


@pytest.fixture(scope="module")
def lib(cuda_ok):
    gh.ensure_built()
    return binding.load_library()


def call_static(L, shape, gpu, n, q, kn, vn):
    s = shape
    out = torch.full((s.batch, q.shape[1], s.n_q_heads, s.head_dim), float("nan"),
                     dtype=s.dtype, device="cuda")
    cs = torch.full((s.batch, s.n_kv_heads, s.capacity + q.shape[1]), float("nan"),
                    dtype=torch.float32, device="cuda")
    cfg = s.config()
    st = L.h2o_attention_static_scratch(
        ctypes.byref(cfg), ctypes.c_void_p(gpu.k.data_ptr()), ctypes.c_void_p(gpu.v.data_ptr()),
        n, ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(kn.data_ptr()),
        ctypes.c_void_p(vn.data_ptr()), q.shape[1], ctypes.c_void_p(out.data_ptr()),
        ctypes.c_void_p(cs.data_ptr()), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == 0, binding.STATUS_NAMES.get(st, st)
    assert L.h2o_static_scratch_check(None) == 0
    return out, cs


CALLS = [
    # B, Hq, Hkv, d, C, n, nq, dtype
    (1, 8, 2, 128, 1024, 1000, 384, torch.bfloat16),
    (2, 4, 2, 128, 300, 77, 129, torch.bfloat16),
    (1, 4, 2, 128, 256, 0, 100, torch.bfloat16),     # empty cache
    (1, 4, 2, 64, 256, 256, 64, torch.float32),
    (1, 4, 2, 64, 256, 130, 64, torch.float32),      # n < C: the empty slots read 0
    (1, 4, 2, 64, 256, 0, 33, torch.float32),        # empty cache
]


def test_static_scratch_matches_h2o_attention_bit_for_bit(lib):
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
        torch.cuda.synchronize()
        what = f"static scratch {B, Hq, Hkv, d, C, n, nq, dt}"
        assert not torch.isnan(cs).any(), what
        assert torch.equal(O, O_ref), what
        assert torch.equal(cs, cs_ref), what
        assert torch.equal(cs[:, :, n:C], torch.zeros_like(cs[:, :, n:C])), what


def test_static_scratch_against_oracle(lib):
    rng = np.random.default_rng(7)
    B, Hq, Hkv, d, C, n, nq = 1, 8, 2, 128, 512, 400, 200
    shape = gh.shape_of(B, Hq, Hkv, d, C, nq, 0)
    gpu = binding.H2OCache(shape)
    K, V, sc, pos = gh.random_state(shape, n, n + 1, rng)
    gpu.write(K, V, torch.from_numpy(sc), torch.from_numpy(pos), n, n + 1)
    ref = gh.oracle_for(shape)
    ref.load(gh.np64(K), gh.np64(V), sc, pos, n, n + 1)
    q = torch.randn(B, nq, Hq, d).to(torch.bfloat16)
    kn = torch.randn(B, nq, Hkv, d).to(torch.bfloat16)
    vn = torch.randn(B, nq, Hkv, d).to(torch.bfloat16)
    O, cs = call_static(lib, shape, gpu, n, q.cuda(), kn.cuda(), vn.cuda())
    O_ref, cs_ref, _ = ref.attention(gh.np64(q), gh.np64(kn), gh.np64(vn))
    gh.assert_attention_close(O, cs, O_ref, cs_ref, nq, Hq // Hkv, "static scratch vs oracle")


def test_static_scratch_rejects_oversize(lib):
    # 144 caches x 32 heads x 1024 rows exceed the 4 Mi-row static array
    shape = gh.shape_of(144, 32, 8, 128, 1024, 1024, 0)
    cfg = shape.config()
    dummy = torch.empty(16, dtype=torch.uint8, device="cuda")
    p = ctypes.c_void_p(dummy.data_ptr())
    st = lib.h2o_attention_static_scratch(ctypes.byref(cfg), p, p, 0, p, p, p, 1024, p, p, None)
    assert st == H2O_ERR_SHAPE  # before anything is launched


def test_static_scratch_reports_and_clears_an_expired_wait(lib):
    # a bounded wait that nothing completes, latching into the static word
    assert lib.h2o_selftest_wait_timeout(None, 5000, None) == 0
    assert lib.h2o_static_scratch_check(None) == H2O_ERR_TIMEOUT
    # the next call starts from a clean word and completes normally
    B, Hq, Hkv, d, C, n, nq, dt = CALLS[1]
    shape = gh.shape_of(B, Hq, Hkv, d, C, nq, 0, dt)
    gpu = binding.H2OCache(shape)
    q = torch.randn(B, nq, Hq, d).to(dt).cuda()
    kn = torch.randn(B, nq, Hkv, d).to(dt).cuda()
    vn = torch.randn(B, nq, Hkv, d).to(dt).cuda()
    call_static(lib, shape, gpu, 0, q, kn, vn)   # asserts the check returns 0
