"""Backward of the attention (h2o_attention_backward: dQ, dK and dV of the
cache slots and of the chunk's keys, eviction held fixed) against the oracle's
fp64 gradients on the same inputs.

Tolerance, from the arithmetic: the tensor cores take P, scale*dS, Q, K, V
and dO as bf16 (relative rounding 2^-9) and accumulate in fp32 over the
queries or keys; each gradient is compared to the oracle with a max-abs error
bound of 3 % of the tensor's largest magnitude and a relative Frobenius error
of 2 %."""
import numpy as np
import pytest
import torch

import gpu_helpers as gh
from kv_cache_sparse_b200 import binding

pytestmark = pytest.mark.gpu

MAX_REL = 3e-2
FRO_REL = 2e-2


@pytest.fixture(scope="module", autouse=True)
def _built(cuda_ok):
    gh.ensure_built()


def _close(got, ref, name):
    got = gh.np64(got)
    scale = max(float(np.max(np.abs(ref))), 1e-12)
    err = float(np.max(np.abs(got - ref)))
    fro = float(np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-30))
    assert err <= MAX_REL * scale, f"{name}: max-abs error {err:.3e} vs scale {scale:.3e}"
    assert fro <= FRO_REL, f"{name}: relative Frobenius error {fro:.3e}"


CASES = [
    # B, Hq, Hkv, d, C, n, nq                        what it covers
    (1, 8, 2, 128, 384, 300, 200),   # ragged cache tile, ragged chunk tail
    (2, 4, 4, 64, 256, 256, 130),    # d = 64, G = 1, two caches
    (1, 4, 2, 128, 256, 0, 96),      # empty cache: chunk keys only
    (1, 8, 1, 128, 640, 640, 256),   # G = 8
    (1, 32, 8, 128, 1024, 1024, 256),  # Qwen3-4B heads
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "B{}_Hq{}_Hkv{}_d{}_C{}_n{}_nq{}".format(*c))
def test_backward_matches_oracle(case):
    B, Hq, Hkv, d, C, n, nq = case
    rng = np.random.default_rng(sum(case))
    shape = gh.shape_of(B, Hq, Hkv, d, C, nq, 0)
    gpu = binding.H2OCache(shape)
    ref = gh.oracle_for(shape)
    K, V, sc, pos = gh.random_state(shape, n, n + 3, rng)
    gh.install_state(gpu, ref, K, V, sc, pos, n, n + 3)
    g = torch.Generator().manual_seed(int(rng.integers(1 << 30)))
    q = torch.randn(B, nq, Hq, d, generator=g).to(torch.bfloat16)
    kn = torch.randn(B, nq, Hkv, d, generator=g).to(torch.bfloat16)
    vn = torch.randn(B, nq, Hkv, d, generator=g).to(torch.bfloat16)
    dO = torch.randn(B, nq, Hq, d, generator=g).to(torch.bfloat16)
    O, _ = gpu.attention(q.cuda(), kn.cuda(), vn.cuda())
    grads = gpu.attention_backward(q.cuda(), kn.cuda(), vn.cuda(), O, dO.cuda())
    assert gpu.check() == 0
    want = ref.attention_backward(gh.np64(q), gh.np64(kn), gh.np64(vn), gh.np64(dO))
    for name, a, b in zip(("dq", "dk_cache", "dv_cache", "dk_new", "dv_new"), grads, want):
        _close(a, b, f"{case} {name}")
    # slots past the valid ones get exactly zero
    assert not grads[1][:, :, n:].any() and not grads[2][:, :, n:].any()


def test_backward_is_deterministic_and_needs_its_forward():
    shape = gh.shape_of(1, 8, 2, 128, 256, 128, 0)
    gpu = binding.H2OCache(shape)
    ref = gh.oracle_for(shape)
    rng = np.random.default_rng(1)
    K, V, sc, pos = gh.random_state(shape, 200, 210, rng)
    gh.install_state(gpu, ref, K, V, sc, pos, 200, 210)
    q = torch.randn(1, 128, 8, 128).to(torch.bfloat16).cuda()
    kn = torch.randn(1, 128, 2, 128).to(torch.bfloat16).cuda()
    vn = torch.randn(1, 128, 2, 128).to(torch.bfloat16).cuda()
    dO = torch.randn(1, 128, 8, 128).to(torch.bfloat16).cuda()
    O, _ = gpu.attention(q, kn, vn)
    a = gpu.attention_backward(q, kn, vn, O, dO)
    b = gpu.attention_backward(q, kn, vn, O, dO)
    for x, y in zip(a, b):
        assert torch.equal(x, y)
    # after the eviction the forward's statistics no longer describe the cache
    gpu.evict(torch.zeros(1, 2, 256 + 128).cuda(), kn, vn)
    with pytest.raises(binding.H2OError):
        gpu.attention_backward(q, kn, vn, O, dO)
