"""The device-side generator the benchmark uses (DeviceChunkSource, run here
on the CPU) draws the distributions the workloads state, like the CPU
generator (ChunkSource) that feeds the parity tests: one fixed heavy-hitter
direction per cache, the stated heavy density (per chunk from a range where
the workload gives one), and a per-token random walk of the K mean with
steps of the stated norm that carries over chunk boundaries."""
import numpy as np
import torch

from kv_cache_sparse_b200.workloads import (HEAVY_SHIFT, QWEN_C8K, QWEN_C16K, STREAM1M,
                                            ChunkSource, DeviceChunkSource, heavy_direction)


def test_heavy_direction_is_fixed_per_cache_and_shared_with_the_cpu_source():
    wl = QWEN_C8K.scaled(batch=3, n_q_heads=4, n_kv_heads=2, head_dim=64, chunk=128)
    dev = DeviceChunkSource(wl, seed=4, device="cpu")
    for b in range(3):
        assert torch.equal(dev.u[b], heavy_direction(wl, 4, b))
    # heavy keys carry +3.0 u_b in every KV head, in every chunk: the
    # projection of (heavy mean - light mean) on u_b is about 3
    for c in range(3):
        q, k, v = dev.chunk(c)
        k = k.float()
        for b in range(3):
            h = dev.last_heavy[b]
            if h.sum() < 2:
                continue
            proj = (k[b] @ dev.u[b])              # [n_q, H_kv]
            diff = proj[h].mean() - proj[~h].mean()
            assert abs(float(diff) - HEAVY_SHIFT) < 1.0


def test_heavy_density_matches_the_cpu_source():
    wl = QWEN_C8K.scaled(batch=8, n_q_heads=4, n_kv_heads=2, head_dim=64, chunk=1024)
    dev = DeviceChunkSource(wl, seed=1, device="cpu")
    fr = [float(dev.chunk(c)[1].shape[1] and dev.last_heavy.float().mean()) for c in range(6)]
    assert abs(np.mean(fr) - wl.heavy_p) < 0.004
    assert torch.allclose(dev.last_p, torch.full((8,), wl.heavy_p))
    # the CPU source's heavy keys sit at +3 along u: same rate of outliers
    cpu = ChunkSource(wl, seed=1)
    hits = []
    for c in range(6):
        _, k, _ = cpu.chunk(c)
        for b in range(8):
            proj = k[b].float() @ heavy_direction(wl, 1, b)
            hits.append(float((proj.mean(-1) > 1.5).float().mean()))
    # a light key's projection exceeds 1.5 with probability ~0.017 (mean of
    # two N(0,1)): the heavy rate shows on top of that
    assert abs(np.mean(hits) - (wl.heavy_p + 0.017)) < 0.006


def test_density_is_drawn_per_chunk_from_the_range():
    wl = QWEN_C16K.scaled(batch=16, n_q_heads=4, n_kv_heads=2, head_dim=64, chunk=2048)
    lo, hi = wl.heavy_p_range
    dev = DeviceChunkSource(wl, seed=2, device="cpu")
    ps, fracs = [], []
    for c in range(8):
        dev.chunk(c)
        assert ((dev.last_p >= lo) & (dev.last_p <= hi)).all()
        ps.append(dev.last_p.clone())
        fracs.append(dev.last_heavy.float().mean(dim=1))
    ps, fracs = torch.stack(ps), torch.stack(fracs)
    assert float(ps.std()) > 0.005                         # varies between chunks and caches
    assert abs(float(ps.mean()) - (lo + hi) / 2) < 0.006   # U[lo, hi] mean
    # each (chunk, cache) draws heavy positions at its own density
    assert float((fracs - ps).abs().max()) < 0.025


def test_drift_is_a_per_token_walk_carried_across_chunks():
    wl = STREAM1M.scaled(n_q_heads=4, n_kv_heads=2, head_dim=64, chunk=256)
    dev = DeviceChunkSource(wl, seed=0, device="cpu")
    dev.chunk(0)
    w0 = dev.last_walk.clone()                 # [1, n_q, H_kv, d]
    dev.chunk(1)
    w1 = dev.last_walk.clone()
    walk = torch.cat([w0, w1], dim=1)[0].double()          # [2 n_q, H_kv, d]
    steps = walk[1:] - walk[:-1]
    norms = steps.norm(dim=-1)
    assert torch.allclose(norms, torch.full_like(norms, wl.drift_step), rtol=1e-4)
    # the first step from the origin has the same norm; heads walk independently
    assert torch.allclose(walk[0].norm(dim=-1), torch.full((2,), wl.drift_step,
                                                          dtype=torch.float64), rtol=1e-4)
    assert float((steps[:, 0] - steps[:, 1]).abs().max()) > 1e-3
    # the CPU source's walk has the same step norm (it only exposes K): the
    # mean over a chunk of consecutive K differences is the mean step
    cpu = ChunkSource(wl, seed=0)
    mu = cpu._mu_at(2, 256)
    assert mu.shape == (1, 2, 64)
    # the walk's spread after m steps of norm s in d dims: |mu|^2 ~ m s^2
    m = 2 * 256
    for w_end in (dev.mu, mu):
        sq = float((w_end.double() ** 2).sum(-1).mean())
        assert 0.3 * m * wl.drift_step ** 2 < sq < 3.0 * m * wl.drift_step ** 2
