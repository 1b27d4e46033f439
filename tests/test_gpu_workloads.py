"""Every workload at full size, in the launch configuration the benchmark
uses: the cache is filled on the GPU with device-drawn chunks, then one
steady-state step is checked against the oracle on sampled (cache, KV group)
units read back from the GPU, and the eviction is checked bit-exactly on
sampled caches when fed the GPU's own summed weights."""
import numpy as np
import pytest
import torch

import gpu_helpers as gh
from kv_cache_sparse_b200 import binding
from kv_cache_sparse_b200.workloads import QWEN_C16K, STACK36, STREAM1M, DeviceChunkSource
from oracle import h2o_oracle as orc

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built(cuda_ok):
    gh.ensure_built()


def steady_state_check(wl, fill_steps, samples, evict_caches):
    dev = torch.device("cuda")
    shape = gh.shape_of(wl.batch, wl.n_q_heads, wl.n_kv_heads, wl.head_dim, wl.capacity,
                        wl.chunk, wl.window, wl.torch_dtype())
    gpu = binding.H2OCache(shape)
    src = DeviceChunkSource(wl, 0, dev)
    for c in range(fill_steps):
        gpu.step(*src.chunk(c))
    assert gpu.check() == 0
    st = gpu.read()
    assert st["n"] == wl.capacity
    q, kn, vn = src.chunk(fill_steps)
    O, cs = gpu.attention(q, kn, vn)
    G = wl.group
    assert np.allclose(gh.np64(cs).sum(-1), wl.chunk * G, rtol=1e-4)
    scale = 1.0 / np.sqrt(wl.head_dim)
    for b, g in samples:
        heads = list(range(g * G, (g + 1) * G))
        o_ref, cs_ref, _ = orc.attention_one_cache(
            gh.np64(q[b, :, heads]), gh.np64(st["k"][b, g:g + 1]), gh.np64(st["v"][b, g:g + 1]),
            st["n"], gh.np64(kn[b, :, g:g + 1]), gh.np64(vn[b, :, g:g + 1]), scale)
        gh.assert_attention_close(O[b, :, heads], cs[b, g:g + 1], o_ref, cs_ref, wl.chunk, G,
                                  f"{wl.name} cache {b} group {g}")
    ref = orc.OracleCache(len(evict_caches), wl.n_q_heads, wl.n_kv_heads, wl.head_dim,
                          wl.capacity, wl.window)
    idx = torch.tensor(evict_caches)
    ref.load(gh.np64(st["k"][idx]), gh.np64(st["v"][idx]), st["scores"][idx].cpu().numpy(),
             st["pos"][idx].cpu().numpy(), st["n"], st["t0"])
    gpu.evict(cs, kn, vn)
    ref.evict(gh.np64(cs[idx]).astype(np.float32), gh.np64(kn[idx]), gh.np64(vn[idx]))
    after = gpu.read()
    sub = {k: (v[idx] if isinstance(v, torch.Tensor) else v) for k, v in after.items()}
    gh.assert_state_equal(sub, ref, shape.dtype, f"{wl.name} eviction")
    assert gpu.check() == 0


def test_qwen_c16k_q2048_w512():
    wl = QWEN_C16K
    steady_state_check(wl, wl.capacity // wl.chunk + 1, [(0, 1), (0, 6)], [0])


def test_stack_of_144_caches():
    wl = STACK36
    steady_state_check(wl, wl.capacity // wl.chunk + 1, [(0, 3), (77, 0), (143, 7)],
                       [0, 77, 143])


def test_stream_c32k_window_equals_chunk():
    wl = STREAM1M
    steady_state_check(wl, wl.capacity // wl.chunk + 1, [(0, 2)], [0])
