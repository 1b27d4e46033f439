"""The score-free eviction policies (LR: the most recent tokens stay; SLR: the
first sink positions and the most recent ones) through the CUDA path against
the oracle.  Positions are distinct, so the kept sets and the whole cache
state must match bit for bit at every step."""
import numpy as np
import pytest
import torch

import gpu_helpers as gh
from kv_cache_sparse_b200 import binding
from oracle import h2o_oracle as orc

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built(cuda_ok):
    gh.ensure_built()


def _pair(B, Hq, Hkv, d, C, max_chunk, W, policy, sinks, dt=torch.bfloat16):
    shape = binding.CacheShape(B, Hq, Hkv, d, C, max_chunk, W, dt, 0.0, policy, sinks)
    gpu = binding.H2OCache(shape)
    ref = orc.OracleCache(B, Hq, Hkv, d, C, W, policy=policy, sinks=sinks)
    return shape, gpu, ref


def _inputs(B, nq, Hq, Hkv, d, g, dt=torch.bfloat16):
    q = torch.randn(B, nq, Hq, d, generator=g).to(dt)
    kn = torch.randn(B, nq, Hkv, d, generator=g).to(dt)
    vn = torch.randn(B, nq, Hkv, d, generator=g).to(dt)
    return q, kn, vn


CASES = [
    # B, Hq, Hkv, d, C, n_q, W, policy, sinks
    (1, 8, 2, 128, 512, 128, 0, "lr", 0),
    (2, 8, 2, 128, 512, 100, 64, "lr", 0),
    (1, 8, 2, 64, 384, 130, 32, "slr", 4),
    (1, 8, 2, 128, 512, 1, 16, "slr", 4),      # decode step
    (2, 4, 4, 128, 300, 1, 0, "lr", 0),        # decode, W = 0
    (40, 8, 8, 64, 256, 64, 16, "slr", 2),     # 320 (cache, KV head) units
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "B{}_Hq{}_Hkv{}_d{}_C{}_nq{}_W{}_{}_s{}".format(*c))
def test_policy_step_matches_oracle(case):
    B, Hq, Hkv, d, C, nq, W, policy, sinks = case
    shape, gpu, ref = _pair(B, Hq, Hkv, d, C, nq, W, policy, sinks)
    rng = np.random.default_rng(sum(case[:7]))
    t0 = 4 * C
    K, V, sc, pos = gh.random_state(shape, C, t0, rng)
    # SLR: the sink positions are in the cache, as they would be after a run
    if policy == "slr":
        for b in range(B):
            for h in range(Hkv):
                pos[b, h, :sinks] = np.arange(sinks)
                rest = rng.permutation(np.arange(sinks, t0))[:C - sinks]
                pos[b, h, sinks:] = rest
    gh.install_state(gpu, ref, K, V, sc, pos, C, t0)
    g = torch.Generator().manual_seed(9)
    for step in range(3):
        q, kn, vn = _inputs(B, nq, Hq, Hkv, d, g)
        launches0 = gpu.info()["kernel_launches"]
        O = gpu.step(q.cuda(), kn.cuda(), vn.cuda())
        # no summed weights asked for: the column-sum kernel is skipped (a
        # decode step is two launches either way)
        assert gpu.info()["kernel_launches"] - launches0 == 2
        O_ref, _ = ref.step(gh.np64(q), gh.np64(kn), gh.np64(vn))
        assert float(np.max(np.abs(gh.np64(O) - O_ref))) <= gh.O_TOL
        gh.assert_state_equal(gpu.read(), ref, shape.dtype, f"{case} step {step}")
    assert gpu.check() == 0


@pytest.mark.parametrize("policy,sinks", [("lr", 0), ("slr", 3)])
def test_policy_prefill_then_decode_trajectory(policy, sinks):
    """Prefill in chunks of 96 from an empty cache past its capacity, then
    decode steps; the state equals the oracle's after every step."""
    B, Hq, Hkv, d, C, W = 1, 8, 2, 128, 320, 8
    shape, gpu, ref = _pair(B, Hq, Hkv, d, C, 96, W, policy, sinks)
    g = torch.Generator().manual_seed(4)
    for step, nq in enumerate([96] * 5 + [1] * 20):
        q, kn, vn = _inputs(B, nq, Hq, Hkv, d, g)
        O = gpu.step(q.cuda(), kn.cuda(), vn.cuda())
        O_ref, _ = ref.step(gh.np64(q), gh.np64(kn), gh.np64(vn))
        assert float(np.max(np.abs(gh.np64(O) - O_ref))) <= gh.O_TOL
        gh.assert_state_equal(gpu.read(), ref, shape.dtype, f"step {step}")
    held = np.sort(ref.pos[0, 0])
    t = ref.t0
    expect = list(range(sinks)) + list(range(t - (C - sinks), t))
    assert list(held) == expect


def test_policy_with_summed_weights_requested():
    """Asking for the summed weights under LR runs the column-sum kernel and
    returns the same values as under H2O; the eviction still ignores them."""
    B, Hq, Hkv, d, C, nq = 1, 8, 2, 128, 256, 64
    out = {}
    for policy in ("h2o", "lr"):
        shape, gpu, ref = _pair(B, Hq, Hkv, d, C, nq, 0, policy, 0)
        rng = np.random.default_rng(1)
        K, V, sc, pos = gh.random_state(shape, C, 1000, rng)
        gh.install_state(gpu, ref, K, V, sc, pos, C, 1000)
        q, kn, vn = _inputs(B, nq, Hq, Hkv, d, torch.Generator().manual_seed(2))
        launches0 = gpu.info()["kernel_launches"]
        O, cs = gpu.step(q.cuda(), kn.cuda(), vn.cuda(), return_colsum=True)
        assert gpu.info()["kernel_launches"] - launches0 == 3
        out[policy] = (gh.np64(O), gh.np64(cs))
        if policy == "lr":
            ref.step(gh.np64(q), gh.np64(kn), gh.np64(vn))
            gh.assert_state_equal(gpu.read(), ref, shape.dtype, "lr with colsum")
    assert np.array_equal(out["h2o"][0], out["lr"][0])
    assert np.array_equal(out["h2o"][1], out["lr"][1])


def test_policy_with_float_inputs():
    """The fp32 path (FMA attention kernels) under SLR: chunk steps past the
    capacity, then decode steps; the state equals the oracle's each step."""
    B, Hq, Hkv, d, C, W, sinks = 1, 4, 2, 64, 192, 4, 2
    shape, gpu, ref = _pair(B, Hq, Hkv, d, C, 64, W, "slr", sinks, dt=torch.float32)
    g = torch.Generator().manual_seed(8)
    for step, nq in enumerate([64] * 4 + [1] * 6):
        q, kn, vn = _inputs(B, nq, Hq, Hkv, d, g, dt=torch.float32)
        O = gpu.step(q.cuda(), kn.cuda(), vn.cuda())
        O_ref, _ = ref.step(gh.np64(q), gh.np64(kn), gh.np64(vn))
        assert float(np.max(np.abs(gh.np64(O) - O_ref))) <= gh.O_TOL
        gh.assert_state_equal(gpu.read(), ref, torch.float32, f"fp32 slr step {step}")
