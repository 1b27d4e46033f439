"""Score update, selection, placement and scatter of the CUDA path
(h2o_evict) fed the oracle's fp32 summed weights: always bit-exact."""
import numpy as np
import pytest
import torch

import gpu_helpers as gh
from kv_cache_sparse_b200 import binding

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built(cuda_ok):
    gh.ensure_built()


CASES = [
    # B, Hkv, d, C, n, nq, W, levels, dtype       what it covers
    (1, 2, 128, 64, 64, 16, 0, None, torch.bfloat16),    # full cache, no window
    (1, 2, 128, 64, 64, 16, 16, None, torch.bfloat16),   # window = chunk
    (1, 2, 128, 64, 64, 16, 40, None, torch.bfloat16),   # window wider than the chunk
    (2, 3, 64, 100, 80, 64, 8, None, torch.bfloat16),    # partially full: n < C < n + nq
    (1, 2, 128, 256, 100, 64, 8, None, torch.bfloat16),  # fill phase: no eviction
    (1, 4, 128, 512, 512, 128, 0, 4, torch.bfloat16),    # heavy ties (4 score levels)
    (1, 4, 128, 512, 512, 128, 32, 1, torch.bfloat16),   # all scores equal
    (1, 1, 128, 2048, 2048, 1, 0, None, torch.bfloat16),  # single new token
    (1, 8, 128, 8192, 8192, 1024, 256, None, torch.bfloat16),  # full-size shape
    (1, 2, 64, 256, 256, 64, 0, None, torch.float32),    # fp32 cache
    (4, 2, 64, 33, 20, 20, 5, 3, torch.float32),         # tiny, odd sizes
    (1, 1, 64, 5, 5, 1, 0, None, torch.bfloat16),        # 6 candidates: some cluster CTAs hold none
    (4, 8, 128, 512, 512, 128, 16, None, torch.bfloat16),  # 32 units: one 1024-thread CTA each
    (3, 8, 64, 300, 250, 100, 120, 3, torch.bfloat16),   # 24 units, partial fill, W > nq, ties
    (1, 1, 64, 49152, 49152, 1024, 64, None, torch.bfloat16),  # the most candidates a cache takes (C + nq = 50176)
    (40, 8, 64, 96, 96, 32, 8, 3, torch.bfloat16),       # 320 units: the many-cache variant
    (40, 8, 64, 300, 250, 100, 120, None, torch.bfloat16),  # many units, partial fill, W > nq
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "B{}_Hkv{}_d{}_C{}_n{}_nq{}_W{}_lv{}".format(*c[:8]))
def test_evict_fed_oracle_weights_is_bit_exact(case):
    B, Hkv, d, C, n, nq, W, levels, dt = case
    rng = np.random.default_rng(C + n + nq + W)
    shape = gh.shape_of(B, Hkv, Hkv, d, C, nq, W, dt)
    gpu = binding.H2OCache(shape)
    ref = gh.oracle_for(shape)
    t0 = n + 3
    K, V, sc, pos = gh.random_state(shape, n, t0, rng, score_levels=levels)
    gh.install_state(gpu, ref, K, V, sc, pos, n, t0)
    if levels:
        cs = (rng.integers(0, levels, (B, Hkv, C + nq)) / levels).astype(np.float32)
    else:
        cs = (rng.random((B, Hkv, C + nq)) * 2).astype(np.float32)
    cs[:, :, n:C] = 0
    kn = torch.randn(B, nq, Hkv, d).to(dt)
    vn = torch.randn(B, nq, Hkv, d).to(dt)
    gpu.evict(torch.from_numpy(cs).cuda(), kn.cuda(), vn.cuda())
    assert gpu.check() == 0
    ref.evict(cs, gh.np64(kn), gh.np64(vn))
    gh.assert_state_equal(gpu.read(), ref, dt, str(case))


def test_evict_many_steps_bit_exact():
    """A run of evictions on one cache (each fed the same weights on both
    sides) stays bit-identical, through the fill phase into eviction."""
    B, Hkv, d, C, nq, W = 2, 2, 128, 96, 40, 10
    shape = gh.shape_of(B, Hkv, Hkv, d, C, nq, W)
    gpu = binding.H2OCache(shape)
    ref = gh.oracle_for(shape)
    rng = np.random.default_rng(9)
    for step in range(8):
        m = int(rng.integers(1, nq + 1))
        cs = (rng.random((B, Hkv, C + m)) * 3).astype(np.float32)
        cs[:, :, ref.n:C] = 0
        kn = torch.randn(B, m, Hkv, d).to(torch.bfloat16)
        vn = torch.randn(B, m, Hkv, d).to(torch.bfloat16)
        gpu.evict(torch.from_numpy(cs).cuda(), kn.cuda(), vn.cuda())
        ref.evict(cs, gh.np64(kn), gh.np64(vn))
        gh.assert_state_equal(gpu.read(), ref, torch.bfloat16, f"step {step}")
    assert gpu.check() == 0


SIGNED_CASES = [
    # B, Hkv, d, C, n, nq, W      launch shape
    (1, 2, 128, 256, 256, 64, 8),     # cluster of CTAs per unit
    (4, 8, 64, 256, 256, 64, 0),      # one 1024-thread CTA per unit
    (40, 8, 64, 96, 96, 32, 4),       # many units: 256-thread CTAs
]


@pytest.mark.parametrize("case", SIGNED_CASES, ids=lambda c: "B{}_Hkv{}_C{}_nq{}".format(
    c[0], c[1], c[3], c[5]))
def test_evict_negative_scores_bit_exact(case):
    """Scores restored by h2o_cache_write and summed weights given to
    h2o_evict may be negative (and -0): the selection orders them by value
    like the oracle, which sorts the fp32 values themselves."""
    B, Hkv, d, C, n, nq, W = case
    rng = np.random.default_rng(C * 7 + B)
    shape = gh.shape_of(B, Hkv, Hkv, d, C, nq, W)
    gpu = binding.H2OCache(shape)
    ref = gh.oracle_for(shape)
    t0 = n + 5
    K, V, sc, pos = gh.random_state(shape, n, t0, rng)
    sc = (sc - 2.0).astype(np.float32)           # about half of the scores below zero
    sc[:, :, : n // 8] = np.float32(-0.0)
    sc[:, :, n:] = 0
    gh.install_state(gpu, ref, K, V, sc, pos, n, t0)
    cs = (rng.random((B, Hkv, C + nq)) * 2 - 1).astype(np.float32)
    cs[:, :, n:C] = 0
    cs[:, :, C:C + nq // 4] = np.float32(-0.0)
    kn = torch.randn(B, nq, Hkv, d).to(torch.bfloat16)
    vn = torch.randn(B, nq, Hkv, d).to(torch.bfloat16)
    gpu.evict(torch.from_numpy(cs).cuda(), kn.cuda(), vn.cuda())
    assert gpu.check() == 0
    ref.evict(cs, gh.np64(kn), gh.np64(vn))
    gh.assert_state_equal(gpu.read(), ref, torch.bfloat16, str(case))


def test_decode_eviction_with_negative_scores():
    """The decode step's single-token eviction ranks negative scores by
    value too (the lowest score leaves, the highest index on ties)."""
    B, Hq, Hkv, d, C, n, W = 2, 8, 2, 128, 600, 600, 0
    rng = np.random.default_rng(77)
    shape = gh.shape_of(B, Hq, Hkv, d, C, 4, W)
    gpu = binding.H2OCache(shape)
    ref = gh.oracle_for(shape)
    t0 = n + 9
    K, V, sc, pos = gh.random_state(shape, n, t0, rng)
    sc = (sc - 5.0).astype(np.float32)
    gh.install_state(gpu, ref, K, V, sc, pos, n, t0)
    g = torch.Generator().manual_seed(3)
    q = torch.randn(B, 1, Hq, d, generator=g).to(torch.bfloat16)
    kn = torch.randn(B, 1, Hkv, d, generator=g).to(torch.bfloat16)
    vn = torch.randn(B, 1, Hkv, d, generator=g).to(torch.bfloat16)
    O, cs = gpu.step(q.cuda(), kn.cuda(), vn.cuda(), return_colsum=True)
    assert gpu.check() == 0
    ref.evict(gh.np64(cs).astype(np.float32), gh.np64(kn), gh.np64(vn))
    gh.assert_state_equal(gpu.read(), ref, torch.bfloat16, "decode, negative scores")


@pytest.mark.parametrize("B,Hkv,C,nq,W,tie", [(40, 8, 96, 32, 0, False), (40, 8, 96, 32, 0, True),
                                              (4, 8, 256, 64, 0, False), (40, 8, 96, 32, 4, False)])
def test_evict_no_new_key_above_the_cache(B, Hkv, C, nq, W, tie):
    """Every new token's weight at or below every old slot's score: with no
    recent window nothing enters the cache (an old slot also wins a tie); with
    a window the protected tokens still enter.  Bit-exact against the oracle."""
    rng = np.random.default_rng(C + nq + W + int(tie))
    shape = gh.shape_of(B, Hkv, Hkv, 64, C, nq, W)
    gpu = binding.H2OCache(shape)
    ref = gh.oracle_for(shape)
    t0 = C + 7
    K, V, _, pos = gh.random_state(shape, C, t0, rng)
    sc = (1.0 + rng.random((B, Hkv, C)) * 3).astype(np.float32)   # old scores in [1, 4)
    gh.install_state(gpu, ref, K, V, sc, pos, C, t0)
    cs = np.zeros((B, Hkv, C + nq), np.float32)
    cs[:, :, :C] = (rng.random((B, Hkv, C)) * 0.5).astype(np.float32)
    cs[:, :, C:] = (rng.random((B, Hkv, nq)) * 0.5).astype(np.float32)   # new: below 1
    if tie:   # a new token exactly at the lowest updated old score
        low = (sc + cs[:, :, :C]).astype(np.float32).min(axis=-1)
        cs[:, :, C + 3] = low
    kn = torch.randn(B, nq, Hkv, 64).to(torch.bfloat16)
    vn = torch.randn(B, nq, Hkv, 64).to(torch.bfloat16)
    gpu.evict(torch.from_numpy(cs).cuda(), kn.cuda(), vn.cuda())
    assert gpu.check() == 0
    ref.evict(cs, gh.np64(kn), gh.np64(vn))
    gh.assert_state_equal(gpu.read(), ref, torch.bfloat16, f"W={W} tie={tie}")
