"""Mistakes planted in the oracle (on the CPU) must each fail some pin.

This checks the pins themselves: a dropped term, a wrong sign or index, a
transposed operand or an off-by-one in the mask, the grouping, the window or
the tie-break would be caught.
"""
import numpy as np
import pytest

import pins
from oracle import h2o_oracle as orc


def _fails_some(pin_list):
    for pin in pin_list:
        try:
            pin()
        except AssertionError:
            return True
    return False


def _strict_mask(n, n_q):
    m = np.zeros((n_q, n + n_q), dtype=bool)
    m[:, :n] = True
    m[:, n:] = np.tril(np.ones((n_q, n_q), dtype=bool), -1)
    m[0, n] = True            # keep row 0 non-empty
    return m


def _no_cache_mask(n, n_q):
    m = np.zeros((n_q, n + n_q), dtype=bool)
    m[:, n:] = np.tril(np.ones((n_q, n_q), dtype=bool))
    if n:
        m[:, :n - 1] = True   # drops the last cache slot
    return m


def _upper_mask(n, n_q):
    m = np.zeros((n_q, n + n_q), dtype=bool)
    m[:, :n] = True
    m[:, n:] = np.triu(np.ones((n_q, n_q), dtype=bool))   # anti-causal
    return m


ATT = [
    ("causal off by one", "visible_mask", _strict_mask),
    ("last cache slot dropped", "visible_mask", _no_cache_mask),
    ("transposed causal mask", "visible_mask", _upper_mask),
    ("interleaved grouping", "kv_head_of", lambda h, G: h % G),
]


@pytest.mark.parametrize("name,attr,fn", ATT, ids=[a[0] for a in ATT])
def test_attention_mutation_caught(monkeypatch, name, attr, fn):
    monkeypatch.setattr(orc, attr, fn)
    assert _fails_some(pins.ALL_ATTENTION_PINS), name


def _mut_attention(kind):
    real = orc.attention_one_cache

    def wrapped(q, kc, vc, n, kn, vn, scale):
        if kind == "scale dropped":
            return real(q, kc, vc, n, kn, vn, 1.0)
        O, W, lse = real(q, kc, vc, n, kn, vn, scale)
        if kind == "weights not summed over heads":
            H_q, H_kv = q.shape[1], kc.shape[0]
            W = W / (H_q // H_kv)
        if kind == "chunk weights shifted":
            C = kc.shape[1]
            W = W.copy()
            W[:, C:] = np.roll(W[:, C:], 1, axis=1)
        return O, W, lse
    return wrapped


@pytest.mark.parametrize("kind", ["scale dropped", "weights not summed over heads",
                                  "chunk weights shifted"])
def test_attention_wrapper_mutation_caught(monkeypatch, kind):
    monkeypatch.setattr(orc, "attention_one_cache", _mut_attention(kind))
    assert _fails_some(pins.ALL_ATTENTION_PINS), kind


def _mut_evict(kind):
    def evict(score, pos, n, t0, colsum32, n_q, window):
        if kind == "window off by one":
            return real(score, pos, n, t0, colsum32, n_q, window + 1)
        if kind == "score not accumulated":
            cs = colsum32.copy()
            cs[:n] = 0
            return real(score, pos, n, t0, cs, n_q, window)
        if kind == "ties to higher index":
            import builtins
            orig = builtins.sorted

            def rsorted(it, key=None, reverse=False):
                if key is not None and reverse is False:
                    items = list(it)
                    try:
                        probe = key(items[0]) if items else None
                    except Exception:
                        probe = None
                    if isinstance(probe, tuple) and len(probe) == 2:
                        return orig(items, key=lambda c: (key(c)[0], -key(c)[1]))
                return orig(it, key=key, reverse=reverse)
            builtins.sorted = rsorted
            try:
                return real(score, pos, n, t0, colsum32, n_q, window)
            finally:
                builtins.sorted = orig
        if kind == "placement reversed":
            sc, ps, pl = real(score, pos, n, t0, colsum32, n_q, window)
            if len(pl.slots) > 1:
                C = score.shape[0]
                sc, ps = score.astype(np.float32).copy(), pos.copy()
                sc[:n] = (sc[:n] + colsum32[:n]).astype(np.float32)
                pl.slots = pl.slots[::-1]
                for s, i in zip(pl.slots, pl.tokens):
                    sc[s] = colsum32[C + i]
                    ps[s] = t0 + i
            return sc, ps, pl
        raise AssertionError(kind)
    real = orc.evict_one_head
    return evict


@pytest.mark.parametrize("kind", ["window off by one", "score not accumulated",
                                  "ties to higher index", "placement reversed"])
def test_evict_mutation_caught(monkeypatch, kind):
    monkeypatch.setattr(orc, "evict_one_head", _mut_evict(kind))
    assert _fails_some(pins.ALL_EVICT_PINS + [pins.check_trajectory]), kind
