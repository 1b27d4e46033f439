"""The decode step (n_q = 1: split-KV attention that returns the summed
weights, then the single-token eviction) against the oracle: single steps
from installed states, a prefill-then-decode trajectory, and the full-size
Qwen3-4B-shaped cache."""
import numpy as np
import pytest
import torch

import gpu_helpers as gh
from kv_cache_sparse_b200 import binding
from kv_cache_sparse_b200.workloads import QWEN_C8K, ChunkSource

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built(cuda_ok):
    gh.ensure_built()


CASES = [
    # B, Hq, Hkv, d, C, n, W, dtype, score levels       what it covers
    (1, 32, 8, 128, 1024, 1024, 64, torch.bfloat16, 0),   # Qwen heads, full cache, window
    (2, 8, 2, 128, 600, 600, 0, torch.bfloat16, 0),       # W = 0: the new token competes
    (2, 8, 2, 128, 600, 600, 0, torch.bfloat16, 3),       # many equal scores: tie-break
    (1, 4, 4, 64, 300, 299, 10, torch.bfloat16, 0),       # room left (n < C), G = 1, d = 64
    (3, 16, 2, 64, 513, 513, 1, torch.bfloat16, 0),       # G = 8, 514 keys: ragged last chunk
    (1, 4, 2, 128, 256, 0, 0, torch.bfloat16, 0),         # empty cache: the first token
    (1, 4, 2, 128, 255, 255, 255, torch.bfloat16, 0),     # W = C, 256 keys: one full chunk
    (2, 6, 3, 128, 200, 200, 5, torch.float32, 0),        # float inputs
    (1, 4, 2, 64, 300, 120, 0, torch.float32, 0),         # float, room left
]


def _ids(c):
    return "B{}_Hq{}_Hkv{}_d{}_C{}_n{}_W{}_{}_lv{}".format(*c[:7], str(c[7]).split(".")[-1], c[8])


@pytest.mark.parametrize("case", CASES, ids=_ids)
def test_decode_step_matches_oracle(case):
    B, Hq, Hkv, d, C, n, W, dt, levels = case
    G = Hq // Hkv
    rng = np.random.default_rng(sum(case[:7]) + levels)
    shape = gh.shape_of(B, Hq, Hkv, d, C, 4, W, dt)
    gpu = binding.H2OCache(shape)
    ref = gh.oracle_for(shape)
    t0 = n + 17
    K, V, sc, pos = gh.random_state(shape, n, t0, rng, score_levels=levels or None)
    gh.install_state(gpu, ref, K, V, sc, pos, n, t0)
    g = torch.Generator().manual_seed(int(rng.integers(1 << 30)))
    q = torch.randn(B, 1, Hq, d, generator=g).to(dt)
    kn = torch.randn(B, 1, Hkv, d, generator=g).to(dt)
    vn = torch.randn(B, 1, Hkv, d, generator=g).to(dt)
    launches0 = gpu.info()["kernel_launches"]
    O, cs = gpu.step(q.cuda(), kn.cuda(), vn.cuda(), return_colsum=True)
    assert gpu.check() == 0
    assert gpu.info()["kernel_launches"] - launches0 == 2  # split-KV pass, then the merge
    O_ref, cs_ref, _ = ref.attention(gh.np64(q), gh.np64(kn), gh.np64(vn))
    gh.assert_attention_close(O, cs, O_ref, cs_ref, 1, G, str(case))
    # every KV head's summed weights add up to G (one query per head)
    assert np.allclose(gh.np64(cs).sum(-1), G, rtol=1e-4)
    # the eviction, fed the same summed weights, matches bit for bit
    ref.evict(gh.np64(cs).astype(np.float32), gh.np64(kn), gh.np64(vn))
    gh.assert_state_equal(gpu.read(), ref, dt, str(case))


def test_decode_attention_only_leaves_state():
    """h2o_attention with n_q = 1 returns O and the summed weights and
    changes nothing in the cache."""
    shape = gh.shape_of(1, 8, 2, 128, 512, 4, 16)
    gpu = binding.H2OCache(shape)
    ref = gh.oracle_for(shape)
    rng = np.random.default_rng(5)
    K, V, sc, pos = gh.random_state(shape, 512, 700, rng)
    gh.install_state(gpu, ref, K, V, sc, pos, 512, 700)
    before = gpu.read()
    q = torch.randn(1, 1, 8, 128).to(torch.bfloat16)
    kn = torch.randn(1, 1, 2, 128).to(torch.bfloat16)
    vn = torch.randn(1, 1, 2, 128).to(torch.bfloat16)
    O, cs = gpu.attention(q.cuda(), kn.cuda(), vn.cuda())
    O_ref, cs_ref, _ = ref.attention(gh.np64(q), gh.np64(kn), gh.np64(vn))
    gh.assert_attention_close(O, cs, O_ref, cs_ref, 1, 4)
    after = gpu.read()
    for key in ("k", "v", "scores", "pos"):
        assert torch.equal(gh.bits(before[key]), gh.bits(after[key])), key
    assert after["n"] == 512 and after["t0"] == 700


def test_prefill_then_decode_trajectory():
    """Chunked prefill (n_q = 128) up to a full cache, then 40 decode steps,
    free running against the oracle on the same inputs."""
    wl = QWEN_C8K.scaled(name="decode_small", n_q_heads=8, n_kv_heads=2, chunk=128,
                         capacity=512, window=32, seq_len=128 * 5)
    src = ChunkSource(wl, seed=11)
    shape = gh.shape_of(1, 8, 2, 128, 512, 128, 32)
    gpu = binding.H2OCache(shape)
    ref = gh.oracle_for(shape)
    near_ties = 0

    def one(q, kn, vn, nq, what):
        nonlocal near_ties
        O, cs = gpu.step(q.cuda(), kn.cuda(), vn.cuda(), return_colsum=True)
        O_ref, cs_ref, _ = ref.attention(gh.np64(q), gh.np64(kn), gh.np64(vn))
        gh.assert_attention_close(O, cs, O_ref, cs_ref, nq, 4, what)
        cs32 = cs_ref.astype(np.float32)
        gap = gh.min_gap(ref, cs32, nq)
        ref.evict(cs32, gh.np64(kn), gh.np64(vn))
        st = gpu.read()
        if gap > gh.GAP_RTOL:
            assert np.array_equal(st["pos"].cpu().numpy(), ref.pos), f"{what}: kept set"
            assert np.allclose(st["scores"].cpu().numpy(), ref.scores, rtol=2e-3, atol=1e-6)
        else:
            near_ties += 1
            gh.push_oracle_state(gpu, ref)
        assert st["n"] == ref.n and st["t0"] == ref.t0

    for c in range(5):  # 640 tokens: fill, then one evicting chunk
        one(*src.chunk(c), 128, f"prefill {c}")
    g = torch.Generator().manual_seed(3)
    for s in range(40):
        q = torch.randn(1, 1, 8, 128, generator=g).to(torch.bfloat16)
        kn = torch.randn(1, 1, 2, 128, generator=g).to(torch.bfloat16)
        vn = torch.randn(1, 1, 2, 128, generator=g).to(torch.bfloat16)
        one(q, kn, vn, 1, f"decode {s}")
    assert gpu.check() == 0
    assert near_ties <= 4


def test_decode_full_size_qwen_cache():
    """The Qwen3-4B-shaped cache (C 8192, 32/8 heads, d 128, W 256), full,
    one decode step from a random state, checked in full against the oracle."""
    shape = gh.shape_of(1, 32, 8, 128, 8192, 1024, 256)
    gpu = binding.H2OCache(shape)
    ref = gh.oracle_for(shape)
    rng = np.random.default_rng(8192)
    K, V, sc, pos = gh.random_state(shape, 8192, 65536, rng)
    gh.install_state(gpu, ref, K, V, sc, pos, 8192, 65536)
    q = torch.randn(1, 1, 32, 128).to(torch.bfloat16)
    kn = torch.randn(1, 1, 8, 128).to(torch.bfloat16)
    vn = torch.randn(1, 1, 8, 128).to(torch.bfloat16)
    O, cs = gpu.step(q.cuda(), kn.cuda(), vn.cuda(), return_colsum=True)
    O_ref, cs_ref, _ = ref.attention(gh.np64(q), gh.np64(kn), gh.np64(vn))
    gh.assert_attention_close(O, cs, O_ref, cs_ref, 1, 4, "C 8192 decode")
    ref.evict(gh.np64(cs).astype(np.float32), gh.np64(kn), gh.np64(vn))
    gh.assert_state_equal(gpu.read(), ref, torch.bfloat16, "C 8192 decode")


def test_one_token_step_with_unsupported_group_runs_the_chunk_kernels():
    """G = 3 is not a decode-kernel group size: a one-token step takes the
    chunk kernels (three launches) and still matches the oracle."""
    B, Hq, Hkv, d, C, n = 1, 6, 2, 128, 300, 300
    shape = gh.shape_of(B, Hq, Hkv, d, C, 4, 8)
    gpu = binding.H2OCache(shape)
    ref = gh.oracle_for(shape)
    rng = np.random.default_rng(33)
    K, V, sc, pos = gh.random_state(shape, n, n + 20, rng)
    gh.install_state(gpu, ref, K, V, sc, pos, n, n + 20)
    g = torch.Generator().manual_seed(5)
    q = torch.randn(B, 1, Hq, d, generator=g).to(torch.bfloat16)
    kn = torch.randn(B, 1, Hkv, d, generator=g).to(torch.bfloat16)
    vn = torch.randn(B, 1, Hkv, d, generator=g).to(torch.bfloat16)
    launches0 = gpu.info()["kernel_launches"]
    O, cs = gpu.step(q.cuda(), kn.cuda(), vn.cuda(), return_colsum=True)
    assert gpu.info()["kernel_launches"] - launches0 == 3
    O_ref, cs_ref, _ = ref.attention(gh.np64(q), gh.np64(kn), gh.np64(vn))
    gh.assert_attention_close(O, cs, O_ref, cs_ref, 1, 3, "G = 3 one-token step")
    ref.evict(gh.np64(cs).astype(np.float32), gh.np64(kn), gh.np64(vn))
    gh.assert_state_equal(gpu.read(), ref, torch.bfloat16, "G = 3 one-token step")
