"""Backward of the attention (h2o_attention_backward: dQ, dK and dV of the
cache slots and of the chunk's keys, eviction held fixed) against the oracle's
fp64 gradients on the same inputs, within an elementwise error bound derived
from the kernels' arithmetic (`gradient_bounds`).

The arithmetic: the tensor cores take bf16 operands and accumulate in fp32.
Q, K, V, dO are bf16 inputs (exact); O is the forward's bf16 output; P is
recomputed in fp32 from the stored row statistic and rounded to bf16 for the
dV product; scale*dS is formed in fp32 and rounded to bf16 for the dQ and dK
products.  With u = 2^-8 (bf16 unit roundoff: 8 significant bits, round to
nearest), e = 2^-24 (fp32), N the length of
a sum and Nk = n + n_q the keys of a row, first-order worst-case bounds
(every error of one sign) are
  P's error before rounding: p = 2^-12 + Nk e  (fp32 logits and ex2 far below
      2^-12; the forward's fp32 row sum of Nk terms)
  a = u + p                                   (P or dS rounded to bf16)
  |dO_i err|_c <= a sum_j P_ij |V_jc| + u |O_ic|  (the forward's bf16 O)
  |dD_i|    <= sum_c |dO_ic| |O_i err|_c + d e sum_c |dO_ic O_ic|
  |dP_ij|   <= d e sum_c |dO_ic V_jc|
  |ddS_ij|  <= a |dS_ij| + P_ij (|dP_ij err| + |dD_i|)
  |ddV_j|   <= (a + N e) sum_i P_ij |dO_i|
  |ddK_j|   <= scale (sum_i |ddS_ij| |Q_i| + N e sum_i |dS_ij| |Q_i|)
  |ddQ_i|   <= scale (sum_j |ddS_ij| |K_j| + Nk e sum_j |dS_ij| |K_j|)
Every element of every gradient must lie within its bound (plus 1e-6 of the
tensor's largest magnitude for elements whose bound is zero)."""
import numpy as np
import pytest
import torch

import gpu_helpers as gh
from kv_cache_sparse_b200 import binding

pytestmark = pytest.mark.gpu

U = 2.0 ** -8
E = 2.0 ** -24


@pytest.fixture(scope="module", autouse=True)
def _built(cuda_ok):
    gh.ensure_built()


def gradient_bounds(q, kc, vc, n, kn, vn, do, o_bf16, scale):
    """Elementwise error bounds of (dq, dk_cache, dv_cache, dk_new, dv_new)
    for one cache (layouts of the oracle's attention_backward_one_cache)."""
    n_q, H_q, d = q.shape
    H_kv, C, _ = kc.shape
    G = H_q // H_kv
    vis = np.zeros((n_q, n + n_q), dtype=bool)
    vis[:, :n] = True
    vis[:, n:] = np.tril(np.ones((n_q, n_q), dtype=bool))
    bq = np.zeros_like(q)
    bkc, bvc = np.zeros_like(kc), np.zeros_like(vc)
    bkn, bvn = np.zeros_like(kn), np.zeros_like(vn)
    for h in range(H_q):
        g = h // G
        keys = np.concatenate([kc[g, :n], kn[:, g]], axis=0)
        vals = np.concatenate([vc[g, :n], vn[:, g]], axis=0)
        s = np.where(vis, scale * (q[:, h] @ keys.T), -np.inf)
        P = np.exp(s - s.max(axis=1, keepdims=True))
        P /= P.sum(axis=1, keepdims=True)
        dP = do[:, h] @ vals.T
        D = (do[:, h] * o_bf16[:, h]).sum(axis=1, keepdims=True)
        dS = P * (dP - D)
        A = U + 2.0 ** -12 + (n + n_q) * E
        err_O = A * (P @ np.abs(vals)) + U * np.abs(o_bf16[:, h])
        err_D = ((np.abs(do[:, h]) * err_O).sum(axis=1, keepdims=True)
                 + d * E * np.abs(do[:, h] * o_bf16[:, h]).sum(axis=1, keepdims=True))
        err_dP = d * E * (np.abs(do[:, h]) @ np.abs(vals).T)
        err_dS = A * np.abs(dS) + P * (err_dP + err_D)
        N = G * n_q
        dv = (A + N * E) * (P.T @ np.abs(do[:, h]))
        dk = scale * (err_dS.T @ np.abs(q[:, h]) + N * E * (np.abs(dS).T @ np.abs(q[:, h])))
        dq = scale * (err_dS @ np.abs(keys) + (n + n_q) * E * (np.abs(dS) @ np.abs(keys)))
        bq[:, h] += dq
        bkc[g, :n] += dk[:n]
        bvc[g, :n] += dv[:n]
        bkn[:, g] += dk[n:]
        bvn[:, g] += dv[n:]
    return bq, bkc, bvc, bkn, bvn


def _within(got, ref, bound, name):
    got = gh.np64(got)
    floor = 1e-6 * max(float(np.max(np.abs(ref))), 1e-30)
    excess = np.abs(got - ref) - bound - floor
    worst = float(np.max(excess)) if excess.size else -1.0
    assert worst <= 0, (f"{name}: an element exceeds its bound by {worst:.3e} "
                        f"(largest error {float(np.max(np.abs(got - ref))):.3e})")


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
    bounds = [np.zeros_like(w) for w in want]
    for bb in range(B):
        parts = gradient_bounds(gh.np64(q)[bb], ref.K[bb], ref.V[bb], n, gh.np64(kn)[bb],
                                gh.np64(vn)[bb], gh.np64(dO)[bb], gh.np64(O)[bb], ref.scale)
        for dst, part in zip(bounds, parts):
            dst[bb] = part
    for name, a, b, bd in zip(("dq", "dk_cache", "dv_cache", "dk_new", "dv_new"), grads, want,
                              bounds):
        _within(a, b, bd, f"{case} {name}")
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
