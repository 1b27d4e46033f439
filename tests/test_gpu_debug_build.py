"""The bounds-checked build (libh2o_debug.so, compiled with -DH2O_DEBUG):
small parity cases of every kernel family run through it and match the
oracle, and no bounds check fires (the state word stays clear).  The checks
latch an error bit and skip the access; they never trap."""
import numpy as np
import pytest
import torch

import gpu_helpers as gh
from kv_cache_sparse_b200 import binding
from kv_cache_sparse_b200.build import build
from kv_cache_sparse_b200.workloads import QWEN_C8K, ChunkSource

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def debug_lib(cuda_ok):
    gh.ensure_built()
    path = build(debug=True)
    saved = binding._lib
    binding._lib = binding.load_library(path)
    yield binding._lib
    binding._lib = saved


def test_debug_build_chunk_steps_and_decode(debug_lib):
    wl = QWEN_C8K.scaled(name="debug", n_q_heads=8, n_kv_heads=2, chunk=128, capacity=384,
                         window=32, seq_len=128 * 5)
    shape = gh.shape_of(1, 8, 2, 128, 384, 128, 32)
    gpu = binding.H2OCache(shape)
    ref = gh.oracle_for(shape)
    src = ChunkSource(wl, seed=8)
    for c in range(5):                      # fill, then eviction
        q, kn, vn = src.chunk(c)
        O, cs = gpu.step(q.cuda(), kn.cuda(), vn.cuda(), return_colsum=True)
        O_ref, cs_ref, _ = ref.attention(gh.np64(q), gh.np64(kn), gh.np64(vn))
        gh.assert_attention_close(O, cs, O_ref, cs_ref, 128, 4, f"debug step {c}")
        ref.evict(gh.np64(cs).astype(np.float32), gh.np64(kn), gh.np64(vn))
        gh.assert_state_equal(gpu.read(), ref, torch.bfloat16, f"debug step {c}")
        assert gpu.check() == 0
    g = torch.Generator().manual_seed(1)
    q1 = torch.randn(1, 1, 8, 128, generator=g).to(torch.bfloat16)
    k1 = torch.randn(1, 1, 2, 128, generator=g).to(torch.bfloat16)
    v1 = torch.randn(1, 1, 2, 128, generator=g).to(torch.bfloat16)
    O1, cs1 = gpu.step(q1.cuda(), k1.cuda(), v1.cuda(), return_colsum=True)
    O1_ref, cs1_ref, _ = ref.attention(gh.np64(q1), gh.np64(k1), gh.np64(v1))
    gh.assert_attention_close(O1, cs1, O1_ref, cs1_ref, 1, 4, "debug decode")
    ref.evict(gh.np64(cs1).astype(np.float32), gh.np64(k1), gh.np64(v1))
    gh.assert_state_equal(gpu.read(), ref, torch.bfloat16, "debug decode")
    assert gpu.check() == 0


@pytest.mark.parametrize("B,Hkv,C,n,nq,W", [(1, 2, 256, 256, 64, 8), (40, 8, 96, 96, 32, 4),
                                             (4, 8, 256, 200, 64, 0)])
def test_debug_build_eviction(debug_lib, B, Hkv, C, n, nq, W):
    rng = np.random.default_rng(B + C)
    shape = gh.shape_of(B, Hkv, Hkv, 128, C, nq, W)
    gpu = binding.H2OCache(shape)
    ref = gh.oracle_for(shape)
    t0 = n + 3
    K, V, sc, pos = gh.random_state(shape, n, t0, rng)
    gh.install_state(gpu, ref, K, V, sc, pos, n, t0)
    cs = (rng.random((B, Hkv, C + nq)) * 2).astype(np.float32)
    cs[:, :, n:C] = 0
    kn = torch.randn(B, nq, Hkv, 128).to(torch.bfloat16)
    vn = torch.randn(B, nq, Hkv, 128).to(torch.bfloat16)
    gpu.evict(torch.from_numpy(cs).cuda(), kn.cuda(), vn.cuda())
    assert gpu.check() == 0
    ref.evict(cs, gh.np64(kn), gh.np64(vn))
    gh.assert_state_equal(gpu.read(), ref, torch.bfloat16, "debug evict")


def test_debug_build_int8_cache(debug_lib):
    rng = np.random.default_rng(12)
    shape = gh.shape_of(1, 8, 2, 128, 384, 128, 16, torch.int8)
    gpu = binding.H2OCache(shape)
    ref = gh.oracle_for(shape)
    gh.install_state_q8(gpu, ref, *gh.random_state_q8(shape, 384, 390, rng), 384, 390)
    g = torch.Generator().manual_seed(2)
    q = torch.randn(1, 128, 8, 128, generator=g).to(torch.bfloat16)
    kn = torch.randn(1, 128, 2, 128, generator=g).to(torch.bfloat16)
    vn = torch.randn(1, 128, 2, 128, generator=g).to(torch.bfloat16)
    O, cs = gpu.step(q.cuda(), kn.cuda(), vn.cuda(), return_colsum=True)
    O_ref, cs_ref, _ = ref.attention(gh.np64(q), gh.np64(kn), gh.np64(vn))
    gh.assert_attention_close(O, cs, O_ref, cs_ref, 128, 4, "debug int8")
    ref.evict(gh.np64(cs).astype(np.float32), gh.np64(kn), gh.np64(vn))
    gh.assert_state_equal(gpu.read(), ref, torch.int8, "debug int8")
    assert gpu.check() == 0
