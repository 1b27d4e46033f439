"""Pins of the oracle's score-free policies ("lr": the most recent tokens;
"slr": the first `sinks` positions plus the most recent ones) against their
closed forms: which positions a cache holds after any sequence of steps,
where each token's K/V row sits, and that the scores are left alone."""
import numpy as np
import pytest

from oracle import h2o_oracle as orc


def _run(policy, C, W, sinks, chunk_sizes, seed=0):
    """Steps an oracle cache (1 cache, 1 KV head, 2 query heads, d = 4) over
    chunks of the given sizes.  Each token's key row starts with its own
    position, so a slot's row tells which token it holds.  Yields the cache
    after every step."""
    rng = np.random.default_rng(seed)
    ref = orc.OracleCache(1, 2, 1, 4, C, W, policy=policy, sinks=sinks)
    ref.scores[:] = rng.random(ref.scores.shape).astype(np.float32)
    t = 0
    for nq in chunk_sizes:
        q = rng.standard_normal((1, nq, 2, 4))
        kn = rng.standard_normal((1, nq, 1, 4))
        kn[0, :, 0, 0] = np.arange(t, t + nq)  # the token's position, recoverable
        vn = rng.standard_normal((1, nq, 1, 4))
        before = (ref.scores.copy(), ref.pos.copy())
        ref.step(q, kn, vn)
        t += nq
        yield ref, before, t


SIZES = [5, 1, 7, 3, 1, 1, 6, 2, 9, 1, 4, 8, 1, 1, 3]


@pytest.mark.parametrize("W", [0, 3])
def test_lr_holds_the_most_recent_positions(W):
    C = 16
    for ref, _, t in _run("lr", C, W, 0, SIZES):
        held = sorted(int(p) for p in ref.pos[0, 0] if p >= 0)
        assert held == list(range(max(0, t - C), t))
        assert ref.n == min(C, t) and ref.t0 == t


@pytest.mark.parametrize("sinks,W", [(2, 0), (4, 5), (1, 1)])
def test_slr_holds_the_sinks_and_the_most_recent_positions(sinks, W):
    C = 16
    for ref, _, t in _run("slr", C, W, sinks, SIZES):
        held = sorted(int(p) for p in ref.pos[0, 0] if p >= 0)
        if t <= C:
            assert held == list(range(t))
        else:
            assert held == list(range(sinks)) + list(range(t - (C - sinks), t))


def test_slr_without_sinks_is_lr():
    a = [(r.pos.copy(), r.K.copy()) for r, _, _ in _run("slr", 12, 2, 0, SIZES, seed=3)]
    b = [(r.pos.copy(), r.K.copy()) for r, _, _ in _run("lr", 12, 2, 0, SIZES, seed=3)]
    for (pa, ka), (pb, kb) in zip(a, b):
        assert np.array_equal(pa, pb) and np.array_equal(ka, kb)


@pytest.mark.parametrize("policy,sinks", [("lr", 0), ("slr", 3)])
def test_rows_follow_their_tokens_and_survivors_keep_their_slot(policy, sinks):
    C = 16
    prev = None
    for ref, (sc_before, pos_before), t in _run(policy, C, 2, sinks, SIZES):
        pos = ref.pos[0, 0]
        for s in range(C):
            if pos[s] >= 0:  # the row in slot s is the token at position pos[s]
                assert ref.K[0, 0, s, 0] == pos[s]
        if prev is not None:  # an entry that stays keeps its slot
            for s in range(C):
                p = pos_before[0, 0, s]
                if p >= 0 and p in pos:
                    assert pos[s] == p
        prev = pos.copy()


@pytest.mark.parametrize("policy,sinks", [("lr", 0), ("slr", 2)])
def test_scores_are_not_accumulated(policy, sinks):
    """Old slots keep their score; placed tokens get 0."""
    C = 16
    for ref, (sc_before, pos_before), t in _run(policy, C, 0, sinks, SIZES, seed=7):
        for s in range(C):
            if ref.pos[0, 0, s] == pos_before[0, 0, s]:
                assert ref.scores[0, 0, s] == sc_before[0, 0, s]
            else:
                assert ref.scores[0, 0, s] == 0.0


def test_new_tokens_take_free_slots_in_ascending_order():
    """lr, full cache, chunk of 4: the 4 oldest leave; the new tokens, in
    order, take the freed slots in ascending slot order."""
    C = 8
    ref = orc.OracleCache(1, 1, 1, 2, C, 0, policy="lr")
    pos = np.array([3, 0, 6, 1, 7, 2, 5, 4], dtype=np.int32)  # oldest in slots 1, 3, 5, 0
    ref.load(np.zeros((1, 1, C, 2)), np.zeros((1, 1, C, 2)), np.zeros((1, 1, C), np.float32),
             pos[None, None], C, 8)
    kn = np.zeros((1, 4, 1, 2))
    kn[0, :, 0, 0] = [8, 9, 10, 11]
    ref.step(np.zeros((1, 4, 1, 2)), kn, np.zeros((1, 4, 1, 2)))
    assert list(ref.pos[0, 0]) == [8, 9, 6, 10, 7, 11, 5, 4]
    assert list(ref.K[0, 0, :, 0]) == [8, 9, 0, 10, 0, 11, 0, 0]
