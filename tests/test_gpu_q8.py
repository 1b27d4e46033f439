"""The int8 cache of the Q-Hitter variant (dtype Q8) against the oracle's
reading of it: placement quantises the kept tokens bit for bit, the attention
and summed weights over a quantised state match at the bf16 tolerances, a
trajectory of chunk steps and the decode step follow the oracle, and the
cache's codes and scales survive a checkpoint round trip."""
import numpy as np
import pytest
import torch

import gpu_helpers as gh
from kv_cache_sparse_b200 import binding
from kv_cache_sparse_b200.workloads import QH2O_C8K, ChunkSource
from oracle import h2o_oracle as orc

pytestmark = pytest.mark.gpu
Q8 = torch.int8


@pytest.fixture(scope="module", autouse=True)
def _built(cuda_ok):
    gh.ensure_built()


EVICT_CASES = [
    # B, Hkv, d, C, n, nq, W        launch shape / what
    (1, 2, 128, 256, 256, 64, 8),    # cluster kernel, eviction
    (1, 2, 128, 256, 100, 64, 0),    # fill phase: every token placed
    (4, 8, 64, 256, 256, 64, 16),    # 1024-thread kernel, d = 64
    (40, 8, 128, 96, 96, 32, 4),     # many units
]


@pytest.mark.parametrize("case", EVICT_CASES, ids=lambda c: "B{}_Hkv{}_d{}_C{}_n{}".format(*c[:5]))
def test_q8_placement_quantises_bit_exact(case):
    B, Hkv, d, C, n, nq, W = case
    rng = np.random.default_rng(C + n + d)
    shape = gh.shape_of(B, Hkv, Hkv, d, C, nq, W, Q8)
    gpu = binding.H2OCache(shape)
    ref = gh.oracle_for(shape)
    t0 = n + 3
    gh.install_state_q8(gpu, ref, *gh.random_state_q8(shape, n, t0, rng), n, t0)
    cs = (rng.random((B, Hkv, C + nq)) * 2).astype(np.float32)
    cs[:, :, n:C] = 0
    g = torch.Generator().manual_seed(int(rng.integers(1 << 30)))
    kn = (torch.randn(B, nq, Hkv, d, generator=g) * 3).to(torch.bfloat16)
    vn = torch.randn(B, nq, Hkv, d, generator=g).to(torch.bfloat16)
    kn[:, 0] = 0   # an all-zero row: scale 0, codes 0
    gpu.evict(torch.from_numpy(cs).cuda(), kn.cuda(), vn.cuda())
    assert gpu.check() == 0
    ref.evict(cs, gh.np64(kn), gh.np64(vn))
    gh.assert_state_equal(gpu.read(), ref, Q8, str(case))


ATTN_CASES = [
    # B, Hq, Hkv, d, C, n, nq
    (1, 8, 2, 128, 512, 512, 256),    # full cache, two query tiles per CTA
    (2, 4, 2, 128, 300, 277, 129),    # ragged cache and chunk
    (1, 32, 8, 128, 1024, 1000, 128),  # Qwen heads
    (1, 4, 1, 64, 256, 200, 64),      # d = 64, G = 4
]


@pytest.mark.parametrize("case", ATTN_CASES, ids=lambda c: "B{}_Hq{}_Hkv{}_d{}_C{}_n{}_nq{}".format(*c))
def test_q8_attention_matches_oracle(case):
    B, Hq, Hkv, d, C, n, nq = case
    rng = np.random.default_rng(sum(case))
    shape = gh.shape_of(B, Hq, Hkv, d, C, nq, 0, Q8)
    gpu = binding.H2OCache(shape)
    ref = gh.oracle_for(shape)
    gh.install_state_q8(gpu, ref, *gh.random_state_q8(shape, n, n + 1, rng), n, n + 1)
    g = torch.Generator().manual_seed(int(rng.integers(1 << 30)))
    q = torch.randn(B, nq, Hq, d, generator=g).to(torch.bfloat16)
    kn = torch.randn(B, nq, Hkv, d, generator=g).to(torch.bfloat16)
    vn = torch.randn(B, nq, Hkv, d, generator=g).to(torch.bfloat16)
    O, cs = gpu.attention(q.cuda(), kn.cuda(), vn.cuda())
    assert gpu.check() == 0
    O_ref, cs_ref, _ = ref.attention(gh.np64(q), gh.np64(kn), gh.np64(vn))
    gh.assert_attention_close(O, cs, O_ref, cs_ref, nq, Hq // Hkv, str(case))


def test_q8_trajectory_teacher_forced():
    """Chunk steps on a small Qwen-shaped int8 cache: each step's attention is
    checked against the oracle, then both sides evict with the GPU's summed
    weights, and the states (codes, scales, scores, positions) stay equal."""
    wl = QH2O_C8K.scaled(name="q8_small", n_q_heads=8, n_kv_heads=2, chunk=128, capacity=384,
                         window=32, seq_len=128 * 6)
    shape = gh.shape_of(1, 8, 2, 128, 384, 128, 32, Q8)
    gpu = binding.H2OCache(shape)
    ref = gh.oracle_for(shape)
    src = ChunkSource(wl, seed=4)
    for c in range(6):
        q, kn, vn = src.chunk(c)
        O, cs = gpu.step(q.cuda(), kn.cuda(), vn.cuda(), return_colsum=True)
        O_ref, cs_ref, _ = ref.attention(gh.np64(q), gh.np64(kn), gh.np64(vn))
        gh.assert_attention_close(O, cs, O_ref, cs_ref, 128, 4, f"step {c}")
        ref.evict(gh.np64(cs).astype(np.float32), gh.np64(kn), gh.np64(vn))
        gh.assert_state_equal(gpu.read(), ref, Q8, f"step {c}")
    assert gpu.check() == 0


@pytest.mark.parametrize("G,W", [(4, 16), (8, 0)])
def test_q8_decode_step(G, W):
    B, Hkv, d, C, n = 2, 2, 128, 600, 600
    Hq = G * Hkv
    rng = np.random.default_rng(G + W)
    shape = gh.shape_of(B, Hq, Hkv, d, C, 4, W, Q8)
    gpu = binding.H2OCache(shape)
    ref = gh.oracle_for(shape)
    gh.install_state_q8(gpu, ref, *gh.random_state_q8(shape, n, n + 11, rng), n, n + 11)
    g = torch.Generator().manual_seed(5)
    q = torch.randn(B, 1, Hq, d, generator=g).to(torch.bfloat16)
    kn = torch.randn(B, 1, Hkv, d, generator=g).to(torch.bfloat16)
    vn = torch.randn(B, 1, Hkv, d, generator=g).to(torch.bfloat16)
    launches0 = gpu.info()["kernel_launches"]
    O, cs = gpu.step(q.cuda(), kn.cuda(), vn.cuda(), return_colsum=True)
    assert gpu.check() == 0
    assert gpu.info()["kernel_launches"] - launches0 == 2  # split-KV pass, then the merge
    O_ref, cs_ref, _ = ref.attention(gh.np64(q), gh.np64(kn), gh.np64(vn))
    gh.assert_attention_close(O, cs, O_ref, cs_ref, 1, G, f"decode G={G}")
    ref.evict(gh.np64(cs).astype(np.float32), gh.np64(kn), gh.np64(vn))
    gh.assert_state_equal(gpu.read(), ref, Q8, f"decode G={G}")


def test_q8_checkpoint_round_trip_and_backward_rejected():
    shape = gh.shape_of(1, 4, 2, 128, 256, 64, 0, Q8)
    a = binding.H2OCache(shape)
    src = ChunkSource(QH2O_C8K.scaled(name="q8_ckpt", n_q_heads=4, n_kv_heads=2, chunk=64,
                                      capacity=256, window=0, seq_len=64 * 6), seed=6)
    chunks = [src.chunk(c) for c in range(6)]
    for c in chunks[:5]:
        a.step(*(t.cuda() for t in c))
    snap = a.read()
    b = binding.H2OCache(shape)
    b.write(snap["k"], snap["v"], snap["scores"], snap["pos"], snap["n"], snap["t0"],
            k_scale=snap["k_scale"], v_scale=snap["v_scale"])
    Oa = a.step(*(t.cuda() for t in chunks[5]))
    Ob = b.step(*(t.cuda() for t in chunks[5]))
    assert torch.equal(gh.bits(Oa), gh.bits(Ob))
    sa, sb = a.read(), b.read()
    for key in ("k", "v", "k_scale", "v_scale", "scores", "pos"):
        assert torch.equal(gh.bits(sa[key]), gh.bits(sb[key])), key
    q, kn, vn = (t.cuda() for t in chunks[5])
    O, _ = a.attention(q, kn, vn)
    with pytest.raises(binding.H2OError):
        a.attention_backward(q, kn, vn, O, torch.randn_like(O))
