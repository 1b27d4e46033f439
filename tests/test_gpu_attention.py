"""Attention output and summed weights of the CUDA path (h2o_attention: the
forward and column-sum kernels) against the fp64 oracle on the same inputs."""
import numpy as np
import pytest
import torch

import gpu_helpers as gh
from kv_cache_sparse_b200 import binding
from kv_cache_sparse_b200.workloads import TINY, ChunkSource

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built(cuda_ok):
    gh.ensure_built()


CASES = [
    # B, Hq, Hkv, d, C, n, nq, dtype                       what it covers
    (1, 8, 2, 128, 384, 300, 200, torch.bfloat16),   # ragged cache tile + ragged chunk tail
    (2, 4, 4, 64, 256, 256, 130, torch.bfloat16),    # d = 64, G = 1, two caches
    (1, 2, 1, 128, 128, 0, 1, torch.bfloat16),       # empty cache, a single query
    (1, 8, 1, 128, 640, 640, 256, torch.bfloat16),   # G = 8, full cache
    (1, 4, 2, 128, 1024, 1000, 384, torch.bfloat16), # several tiles each way
    (3, 4, 2, 128, 200, 77, 129, torch.bfloat16),    # odd sizes everywhere
    (1, 4, 2, 64, 256, 256, 64, torch.float32),      # fp32 path (tiny workload's shape)
    (2, 6, 3, 128, 96, 50, 33, torch.float32),       # fp32, d = 128, ragged
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "B{}_Hq{}_Hkv{}_d{}_C{}_n{}_nq{}_{}".format(
    *c[:7], str(c[7]).split(".")[-1]))
def test_attention_matches_oracle(case):
    B, Hq, Hkv, d, C, n, nq, dt = case
    rng = np.random.default_rng(sum(case[:7]))
    shape = gh.shape_of(B, Hq, Hkv, d, C, max(nq, 1), 0, dt)
    gpu = binding.H2OCache(shape)
    ref = gh.oracle_for(shape)
    K, V, sc, pos = gh.random_state(shape, n, n + 5, rng)
    gh.install_state(gpu, ref, K, V, sc, pos, n, n + 5)
    g = torch.Generator().manual_seed(7)
    q = torch.randn(B, nq, Hq, d, generator=g).to(dt)
    kn = torch.randn(B, nq, Hkv, d, generator=g).to(dt)
    vn = torch.randn(B, nq, Hkv, d, generator=g).to(dt)
    O, cs = gpu.attention(q.cuda(), kn.cuda(), vn.cuda())
    assert gpu.check() == 0
    O_ref, cs_ref, _ = ref.attention(gh.np64(q), gh.np64(kn), gh.np64(vn))
    gh.assert_attention_close(O, cs, O_ref, cs_ref, nq, Hq // Hkv, str(case))
    # the summed weights of each KV head add up to n_q * G
    tot = gh.np64(cs).sum(-1)
    assert np.allclose(tot, nq * (Hq // Hkv), rtol=1e-4)
    # state unchanged by h2o_attention
    st = gpu.read()
    assert st["n"] == n and st["t0"] == n + 5


def test_uniform_queries_closed_form():
    """Q = 0: every visible key gets the same logit, so the weights are sums
    of 1/(n+i+1) -- compared with the closed form, not only the oracle."""
    B, Hq, Hkv, d, C, n, nq = 1, 4, 2, 128, 256, 200, 160
    shape = gh.shape_of(B, Hq, Hkv, d, C, nq, 0)
    gpu = binding.H2OCache(shape)
    ref = gh.oracle_for(shape)
    rng = np.random.default_rng(1)
    K, V, sc, pos = gh.random_state(shape, n, n, rng)
    gh.install_state(gpu, ref, K, V, sc, pos, n, n)
    q = torch.zeros(B, nq, Hq, d, dtype=torch.bfloat16)
    kn = torch.randn(B, nq, Hkv, d).to(torch.bfloat16)
    vn = torch.randn(B, nq, Hkv, d).to(torch.bfloat16)
    O, cs = gpu.attention(q.cuda(), kn.cuda(), vn.cuda())
    cs = gh.np64(cs)
    G = Hq // Hkv
    harm = np.array([1.0 / (n + i + 1) for i in range(nq)])
    slot_w = G * harm.sum()
    chunk_w = G * np.cumsum(harm[::-1])[::-1]
    for g in range(Hkv):
        assert np.max(np.abs(cs[0, g, :n] - slot_w) / slot_w) < 1e-3
        assert np.all(cs[0, g, n:C] == 0)
        assert np.max(np.abs(cs[0, g, C:] - chunk_w) / chunk_w) < 1e-3
    O_ref, cs_ref, _ = ref.attention(gh.np64(q), gh.np64(kn), gh.np64(vn))
    gh.assert_attention_close(O, cs, O_ref, cs_ref, nq, G, "uniform")


def test_tiny_workload_first_chunks_fp32():
    """The tiny fp32 workload's generator output through h2o_attention."""
    src = ChunkSource(TINY, seed=0)
    shape = gh.shape_of(1, 4, 2, 64, 256, 64, 0, torch.float32)
    gpu = binding.H2OCache(shape)
    ref = gh.oracle_for(shape)
    for c in range(5):   # fill phase: n = 0, 64, 128, 192, 256
        q, kn, vn = src.chunk(c)
        O, cs = gpu.attention(q.cuda(), kn.cuda(), vn.cuda())
        O_ref, cs_ref, _ = ref.attention(gh.np64(q), gh.np64(kn), gh.np64(vn))
        gh.assert_attention_close(O, cs, O_ref, cs_ref, 64, 2, f"chunk {c}")
        ref.evict(cs_ref.astype(np.float32), gh.np64(kn), gh.np64(vn))
        gh.push_oracle_state(gpu, ref)


def test_deterministic():
    shape = gh.shape_of(1, 8, 2, 128, 512, 256, 0)
    rng = np.random.default_rng(3)
    K, V, sc, pos = gh.random_state(shape, 500, 600, rng)
    q = torch.randn(1, 256, 8, 128).to(torch.bfloat16).cuda()
    kn = torch.randn(1, 256, 2, 128).to(torch.bfloat16).cuda()
    vn = torch.randn(1, 256, 2, 128).to(torch.bfloat16).cuda()
    outs = []
    for _ in range(2):
        gpu = binding.H2OCache(shape)
        gpu.write(K, V, torch.from_numpy(sc), torch.from_numpy(pos), 500, 600)
        outs.append(gpu.attention(q, kn, vn))
    assert torch.equal(gh.bits(outs[0][0]), gh.bits(outs[1][0]))
    assert torch.equal(gh.bits(outs[0][1]), gh.bits(outs[1][1]))
