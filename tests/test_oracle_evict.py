"""Oracle score update / selection / placement against the rank-count
definition, hand-worked examples, fp32 rounding, and a token-centric
re-implementation of the whole multi-step run."""
import numpy as np
import pytest

import pins
from oracle import h2o_oracle as orc


@pytest.mark.parametrize("pin", pins.ALL_EVICT_PINS, ids=lambda f: f.__name__)
def test_evict_pin(pin):
    pin()


@pytest.mark.parametrize("args", [
    dict(seed=10, C=12, W=2, chunk_sizes=(5, 5, 3, 6, 4, 5)),
    dict(seed=11, C=7, W=0, chunk_sizes=(4, 4, 4, 1, 3)),            # partial fill, N_q = 1
    dict(seed=12, C=9, W=6, chunk_sizes=(3, 3, 3, 3, 3)),            # window wider than chunk
    dict(seed=13, C=6, W=2, chunk_sizes=(6, 1, 1, 1, 1, 1, 1, 1)),   # decode steps on a full cache
    dict(seed=14, C=5, W=0, chunk_sizes=(5, 1, 1, 1, 1, 1)),         # decode, the new token competes
])
def test_trajectory_token_centric(args):
    pins.check_trajectory(**args)


def test_checkpoint_resume_bit_exact():
    rng = np.random.default_rng(20)
    B, H_q, H_kv, d, C, W = 2, 4, 2, 4, 10, 2
    chunks = [(rng.standard_normal((B, 4, H_q, d)), rng.standard_normal((B, 4, H_kv, d)),
               rng.standard_normal((B, 4, H_kv, d))) for _ in range(6)]
    a = orc.OracleCache(B, H_q, H_kv, d, C, W)
    for c in chunks[:3]:
        a.step(*c)
    snap = a.state()
    b = orc.OracleCache(B, H_q, H_kv, d, C, W)
    b.load(*snap)
    for c in chunks[3:]:
        Oa, Wa = a.step(*c)
        Ob, Wb = b.step(*c)
        assert np.array_equal(Oa, Ob) and np.array_equal(Wa, Wb)
    for x, y in zip(a.state(), b.state()):
        assert np.array_equal(np.asarray(x), np.asarray(y))


def test_invariants_after_many_steps():
    rng = np.random.default_rng(21)
    B, H_q, H_kv, d, C, W = 1, 6, 3, 8, 16, 3
    cache = orc.OracleCache(B, H_q, H_kv, d, C, W)
    for step in range(8):
        n_q = int(rng.integers(1, 9))
        q = rng.standard_normal((B, n_q, H_q, d))
        kn = rng.standard_normal((B, n_q, H_kv, d))
        vn = rng.standard_normal((B, n_q, H_kv, d))
        n_before, t0 = cache.n, cache.t0
        O, colsum = cache.step(q, kn, vn)
        assert np.allclose(colsum.sum(-1), n_q * (H_q // H_kv))
        assert cache.n == min(C, n_before + n_q) and cache.t0 == t0 + n_q
        for g in range(H_kv):
            p = cache.pos[0, g]
            valid = p[p >= 0]
            assert len(valid) == cache.n and len(set(valid.tolist())) == cache.n
            assert np.all(p[:cache.n] >= 0) and np.all(p[cache.n:] == -1)
            # the recent window is always kept
            lim = cache.t0 - W
            assert set(range(max(lim, 0), cache.t0)) <= set(valid.tolist())


def test_gap_at_boundary():
    sc = np.array([1.0, 0.5, 0.25], np.float32)
    pos = np.array([0, 1, 2], np.int32)
    colsum = np.array([0, 0, 0, 0.75, 0.125], np.float32)
    # candidates 1.0, 0.5, 0.25, 0.75, 0.125; keep 3 -> boundary between 0.5 and 0.25
    g = orc.gap_at_boundary(sc, pos, 3, 3, colsum, 2, 0)
    assert abs(g - 0.5) < 1e-12
