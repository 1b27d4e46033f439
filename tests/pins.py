"""Pins of the CPU oracle against things other than itself.

Each ``check_*`` function raises ``AssertionError`` when the oracle disagrees
with an independent statement of the result: a brute-force loop written
differently, a library routine (torch SDPA in fp64), a closed form, an
invariant, or a hand-worked example from ``tests/golden``.  The oracle tests
call them directly; the mutation tests plant mistakes in the oracle and check
that some pin fails.
"""
from __future__ import annotations

import json
import math
import os
from fractions import Fraction

import numpy as np
import torch

from oracle import h2o_oracle as orc

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rand_case(rng, n_q, n, C, H_q, H_kv, d):
    q = rng.standard_normal((n_q, H_q, d))
    kc = rng.standard_normal((H_kv, C, d))
    vc = rng.standard_normal((H_kv, C, d))
    kn = rng.standard_normal((n_q, H_kv, d))
    vn = rng.standard_normal((n_q, H_kv, d))
    return q, kc, vc, kn, vn


# ---------------------------------------------------------------- attention

def brute_attention(q, kc, vc, n, kn, vn, scale):
    """Per-query loops in plain Python floats.  KV head g serves the query
    heads g*G .. g*G+G-1; query i sees cache slots 0..n-1 and chunk keys 0..i."""
    n_q, H_q, d = q.shape
    H_kv, C, _ = kc.shape
    G = H_q // H_kv
    O = [[[0.0] * d for _ in range(H_q)] for _ in range(n_q)]
    W = [[0.0] * (C + n_q) for _ in range(H_kv)]
    for g in range(H_kv):
        for r in range(G):
            h = g * G + r
            for i in range(n_q):
                keys = [(s, kc[g, s], vc[g, s]) for s in range(n)]
                keys += [(C + j, kn[j, g], vn[j, g]) for j in range(i + 1)]
                logits = [scale * sum(float(q[i, h, t]) * float(k[t]) for t in range(d))
                          for _, k, _ in keys]
                mx = max(logits)
                ex = [math.exp(x - mx) for x in logits]
                Z = sum(ex)
                for (idx, _, v), e in zip(keys, ex):
                    p = e / Z
                    W[g][idx] += p
                    for t in range(d):
                        O[i][h][t] += p * float(v[t])
    return np.array(O), np.array(W)


def check_bruteforce(seed=0, cases=((3, 4, 6, 4, 2, 3), (5, 0, 4, 2, 2, 2),
                                     (4, 7, 7, 3, 1, 5), (1, 2, 3, 8, 2, 4))):
    rng = np.random.default_rng(seed)
    for (n_q, n, C, H_q, H_kv, d) in cases:
        q, kc, vc, kn, vn = _rand_case(rng, n_q, n, C, H_q, H_kv, d)
        scale = 0.7
        O, W, _ = orc.attention_one_cache(q, kc, vc, n, kn, vn, scale)
        Ob, Wb = brute_attention(q, kc, vc, n, kn, vn, scale)
        assert np.allclose(O, Ob, rtol=0, atol=1e-12), np.abs(O - Ob).max()
        assert np.allclose(W, Wb, rtol=0, atol=1e-12), np.abs(W - Wb).max()


def check_sdpa(seed=1, cases=((16, 40, 48, 8, 2, 16), (9, 0, 12, 4, 4, 8),
                              (33, 17, 64, 6, 3, 32))):
    """Output against torch's fp64 SDPA with an explicit boolean mask; the
    KV heads are expanded to query heads with repeat_interleave."""
    rng = np.random.default_rng(seed)
    for (n_q, n, C, H_q, H_kv, d) in cases:
        q, kc, vc, kn, vn = _rand_case(rng, n_q, n, C, H_q, H_kv, d)
        scale = 1.0 / math.sqrt(d)
        O, _, lse = orc.attention_one_cache(q, kc, vc, n, kn, vn, scale)
        G = H_q // H_kv
        K = torch.cat([torch.from_numpy(kc[:, :n]), torch.from_numpy(kn).transpose(0, 1)], 1)
        V = torch.cat([torch.from_numpy(vc[:, :n]), torch.from_numpy(vn).transpose(0, 1)], 1)
        K = K.repeat_interleave(G, dim=0)            # [H_q, n + n_q, d]
        V = V.repeat_interleave(G, dim=0)
        Q = torch.from_numpy(q).transpose(0, 1)      # [H_q, n_q, d]
        mask = torch.ones(n_q, n + n_q, dtype=torch.bool)
        mask[:, n:] = torch.ones(n_q, n_q, dtype=torch.bool).tril()
        ref = torch.nn.functional.scaled_dot_product_attention(
            Q, K, V, attn_mask=mask, scale=scale).transpose(0, 1).numpy()
        assert np.allclose(O, ref, rtol=0, atol=1e-12), np.abs(O - ref).max()
        logits = torch.einsum("hid,hjd->hij", Q, K) * scale
        logits = logits.masked_fill(~mask, -math.inf)
        ref_lse = torch.logsumexp(logits, dim=-1).numpy()
        assert np.allclose(lse, ref_lse, rtol=0, atol=1e-12)


def check_uniform_closed_form(n_q=7, n=5, C=9, H_q=6, H_kv=2, d=4, seed=2):
    """Q = 0 makes every visible logit equal: query i averages its n + i + 1
    visible values, slot s receives G * sum_i 1/(n+i+1) and chunk key j
    receives G * sum_{i>=j} 1/(n+i+1)."""
    rng = np.random.default_rng(seed)
    _, kc, vc, kn, vn = _rand_case(rng, n_q, n, C, H_q, H_kv, d)
    q = np.zeros((n_q, H_q, d))
    O, W, _ = orc.attention_one_cache(q, kc, vc, n, kn, vn, 1.0)
    G = H_q // H_kv
    for h in range(H_q):
        g = h // G
        for i in range(n_q):
            vis = np.concatenate([vc[g, :n], vn[:i + 1, g]])
            assert np.allclose(O[i, h], vis.mean(0), atol=1e-13)
    for g in range(H_kv):
        slot_w = G * sum(Fraction(1, n + i + 1) for i in range(n_q))
        for s in range(n):
            assert abs(W[g, s] - float(slot_w)) < 1e-13
        assert np.all(W[g, n:C] == 0.0)
        for j in range(n_q):
            wj = G * sum(Fraction(1, n + i + 1) for i in range(j, n_q))
            assert abs(W[g, C + j] - float(wj)) < 1e-13


def check_one_hot(d=8, n=6, C=8, n_q=4, H_q=4, H_kv=2):
    """A key aligned with every query at a huge logit takes all the weight."""
    rng = np.random.default_rng(3)
    _, kc, vc, kn, vn = _rand_case(rng, n_q, n, C, H_q, H_kv, d)
    kc *= 0.01
    kn *= 0.01
    q = np.zeros((n_q, H_q, d))
    q[:, :, 0] = 30.0
    kc[:, 3, :] = 0.0
    kc[:, 3, 0] = 30.0           # logit 900 against |logit| < 2 elsewhere
    O, W, _ = orc.attention_one_cache(q, kc, vc, n, kn, vn, 1.0)
    G = H_q // H_kv
    for h in range(H_q):
        assert np.allclose(O[:, h], vc[h // G, 3][None, :], atol=1e-12)
    for g in range(H_kv):
        assert abs(W[g, 3] - n_q * G) < 1e-9
        assert abs(W[g].sum() - W[g, 3]) < 1e-9


def check_single_query_empty_cache(d=5, H_q=6, H_kv=3, C=4):
    """n = 0 and one query: the only visible key is the query's own."""
    rng = np.random.default_rng(4)
    q, kc, vc, kn, vn = _rand_case(rng, 1, 0, C, H_q, H_kv, d)
    O, W, lse = orc.attention_one_cache(q, kc, vc, 0, kn, vn, 0.3)
    G = H_q // H_kv
    for h in range(H_q):
        assert np.array_equal(O[0, h], vn[0, h // G])
        assert abs(lse[h, 0] - 0.3 * float(q[0, h] @ kn[0, h // G])) < 1e-13
    expect = np.zeros((H_kv, C + 1))
    expect[:, C] = G
    assert np.array_equal(W, expect)


def check_weight_total(seed=5):
    """Every probability row sums to 1, so all weights of KV head g add up to
    n_q * G."""
    rng = np.random.default_rng(seed)
    for (n_q, n, C, H_q, H_kv, d) in ((17, 30, 32, 8, 2, 8), (6, 0, 6, 3, 1, 4)):
        q, kc, vc, kn, vn = _rand_case(rng, n_q, n, C, H_q, H_kv, d)
        _, W, _ = orc.attention_one_cache(q, kc, vc, n, kn, vn, 0.5)
        assert np.allclose(W.sum(axis=1), n_q * (H_q // H_kv), rtol=0, atol=1e-11)
        assert np.all(W >= 0)


def check_causality(seed=6, n_q=9, n=5, C=8, H_q=4, H_kv=2, d=6):
    """Changing chunk key/value j leaves the outputs of queries i < j and the
    weights of every other key seen only by them unchanged."""
    rng = np.random.default_rng(seed)
    q, kc, vc, kn, vn = _rand_case(rng, n_q, n, C, H_q, H_kv, d)
    O0, _, _ = orc.attention_one_cache(q, kc, vc, n, kn, vn, 0.4)
    for j in (0, 4, n_q - 1):
        kn2, vn2 = kn.copy(), vn.copy()
        kn2[j] += 5.0
        vn2[j] -= 3.0
        O1, _, _ = orc.attention_one_cache(q, kc, vc, n, kn2, vn2, 0.4)
        assert np.array_equal(O0[:j], O1[:j])
        assert not np.allclose(O0[j:], O1[j:])


def check_mha_reduction(seed=7, n_q=8, n=6, C=6, H=4, d=5):
    """With G = 1 each query head reads its own KV head."""
    rng = np.random.default_rng(seed)
    q, kc, vc, kn, vn = _rand_case(rng, n_q, n, C, H, H, d)
    O, _, _ = orc.attention_one_cache(q, kc, vc, n, kn, vn, 0.5)
    for h in range(H):
        Oh, _, _ = orc.attention_one_cache(q[:, h:h + 1], kc[h:h + 1], vc[h:h + 1], n,
                                           kn[:, h:h + 1], vn[:, h:h + 1], 0.5)
        assert np.allclose(O[:, h], Oh[:, 0], atol=1e-14)


def check_golden_attention():
    with open(os.path.join(GOLDEN, "attention_hand_example.json")) as f:
        gd = json.load(f)
    a = {k: np.array(v, dtype=np.float64) for k, v in gd["inputs"].items()}
    O, W, _ = orc.attention_one_cache(a["q"], a["kc"], a["vc"], gd["n"], a["kn"], a["vn"],
                                      gd["scale"])
    exp_O = np.array([[[Fraction(x) for x in row] for row in head] for head in gd["expect_O"]],
                     dtype=object).astype(np.float64)
    exp_W = np.array([[float(Fraction(x)) for x in row] for row in gd["expect_colsum"]])
    assert np.allclose(O, exp_O, atol=1e-13), (O, exp_O)
    assert np.allclose(W, exp_W, atol=1e-13), (W, exp_W)


# ----------------------------------------------------------------- eviction

def rank_count_keep(cands, k_keep):
    """Keep x iff fewer than k_keep candidates come before it, where y comes
    before x when its score is larger, or equal with a smaller index."""
    kept = set()
    for (ix, sx) in cands:
        before = sum(1 for (iy, sy) in cands if sy > sx or (sy == sx and iy < ix))
        if before < k_keep:
            kept.add(ix)
    return kept


def check_evict_rankcount(seed=8, trials=300):
    """Selection and placement against the rank-count definition, with
    quantised scores so that ties are frequent."""
    rng = np.random.default_rng(seed)
    for _ in range(trials):
        C = int(rng.integers(1, 9))
        n = int(rng.integers(0, C + 1))
        n_q = int(rng.integers(1, 7))
        W = int(rng.integers(0, C + 1))
        t0 = int(rng.integers(n, n + 20))
        score = (rng.integers(0, 4, C) / 4).astype(np.float32)
        pos = np.full(C, -1, np.int32)
        pos[:n] = rng.permutation(t0)[:n]
        colsum = (rng.integers(0, 4, C + n_q) / 4).astype(np.float32)
        colsum[n:C] = 0
        sc, ps, pl = orc.evict_one_head(score, pos, n, t0, colsum, n_q, W)
        upd = score.copy()
        upd[:n] = score[:n] + colsum[:n]
        if n + n_q <= C:
            assert pl.slots == list(range(n, n + n_q)) and pl.tokens == list(range(n_q))
            continue
        limit = t0 + n_q - W
        allc = [(s, float(upd[s]), int(pos[s])) for s in range(n)]
        allc += [(C + i, float(colsum[C + i]), t0 + i) for i in range(n_q)]
        prot = {ix for ix, _, p in allc if p >= limit}
        unprot = [(ix, s) for ix, s, p in allc if p < limit]
        kept = prot | rank_count_keep(unprot, C - len(prot))
        assert len(kept) == C
        for s in range(n):
            if s in kept:
                assert ps[s] == pos[s] and sc[s] == upd[s]
        new_kept = [ix - C for ix in sorted(kept) if ix >= C]
        free = sorted([s for s in range(n) if s not in kept] + list(range(n, C)))
        assert pl.tokens == new_kept and pl.slots == free
        for s, i in zip(free, new_kept):
            assert ps[s] == t0 + i and sc[s] == colsum[C + i]
        assert len(set(ps.tolist())) == C            # positions unique, no empty slot


def check_golden_evict():
    with open(os.path.join(GOLDEN, "evict_hand_examples.json")) as f:
        cases = json.load(f)["cases"]
    for c in cases:
        sc, ps, pl = orc.evict_one_head(
            np.array(c["score"], np.float32), np.array(c["pos"], np.int32), c["n"], c["t0"],
            np.array(c["colsum"], np.float32), c["n_q"], c["window"])
        assert sc.tolist() == c["expect_score"], (c["name"], sc.tolist())
        assert ps.tolist() == c["expect_pos"], (c["name"], ps.tolist())
        assert pl.slots == c["expect_slots"] and pl.tokens == c["expect_tokens"], c["name"]


def _is_nearest_f32(r: np.float32, a: np.float32, b: np.float32) -> bool:
    exact = Fraction(float(a)) + Fraction(float(b))
    err = abs(Fraction(float(r)) - exact)
    for nb in (np.nextafter(r, np.float32(np.inf)), np.nextafter(r, np.float32(-np.inf))):
        e2 = abs(Fraction(float(nb)) - exact)
        if e2 < err:
            return False
        if e2 == err:   # halfway: round to even significand
            if int(np.float32(r).view(np.uint32)) & 1:
                return False
    return True


def check_fp32_accumulate(seed=9, trials=2000):
    """The score update is the fp32 value nearest to the exact sum."""
    rng = np.random.default_rng(seed)
    a = (rng.random(trials) * 10.0 ** rng.integers(-3, 3, trials)).astype(np.float32)
    b = (rng.random(trials) * 10.0 ** rng.integers(-6, 1, trials)).astype(np.float32)
    for x, y in zip(a, b):
        # full cache of one slot, no window: the old slot (score x + y >= 0)
        # outranks a new token given weight -1, so its updated score survives
        sc2, _, _ = orc.evict_one_head(np.array([x], np.float32), np.array([0], np.int32), 1,
                                       1, np.array([y, -1.0], np.float32), 1, 0)
        assert _is_nearest_f32(sc2[0], x, y), (x, y, sc2[0])


# ------------------------------------------------------- multi-step trajectory

def token_centric_run(chunks, C, W, H_q, H_kv, scale):
    """Independent re-statement of the whole step for one cache: the cache is
    a set of tokens (no slots); continuous random scores make ties impossible,
    so the kept set is the top by score after the protected ones."""
    G = H_q // H_kv
    toks = [dict() for _ in range(H_kv)]   # pos -> (k, v, score)
    outs = []
    t0 = 0
    for (q, kn, vn) in chunks:
        n_q = q.shape[0]
        O = np.zeros(q.shape)
        new_w = [np.zeros(n_q) for _ in range(H_kv)]
        old_w = [{p: 0.0 for p in toks[g]} for g in range(H_kv)]
        for h in range(H_q):
            g = h // G
            plist = sorted(toks[g])
            for i in range(n_q):
                ks = [toks[g][p][0] for p in plist] + [kn[j, g] for j in range(i + 1)]
                vs = [toks[g][p][1] for p in plist] + [vn[j, g] for j in range(i + 1)]
                lg = np.array([scale * float(q[i, h] @ k) for k in ks])
                e = np.exp(lg - lg.max())
                p_ = e / e.sum()
                O[i, h] = p_ @ np.array(vs)
                for a, pp in enumerate(plist):
                    old_w[g][pp] += p_[a]
                new_w[g][:i + 1] += p_[len(plist):]
        outs.append(O)
        for g in range(H_kv):
            cur = {p: (k, v, np.float32(np.float32(s) + np.float32(old_w[g][p])))
                   for p, (k, v, s) in toks[g].items()}
            for i in range(n_q):
                cur[t0 + i] = (kn[i, g], vn[i, g], np.float32(new_w[g][i]))
            if len(cur) > C:
                limit = t0 + n_q - W
                prot = [p for p in cur if p >= limit]
                rest = sorted((p for p in cur if p < limit), key=lambda p: -cur[p][2])
                keep = set(prot) | set(rest[:C - len(prot)])
                cur = {p: cur[p] for p in keep}
            toks[g] = cur
        t0 += n_q
    return outs, toks


def check_trajectory(seed=10, C=12, W=2, H_q=4, H_kv=2, d=4, chunk_sizes=(5, 5, 3, 6, 4, 5)):
    rng = np.random.default_rng(seed)
    chunks = [(rng.standard_normal((m, H_q, d)), rng.standard_normal((m, H_kv, d)),
               rng.standard_normal((m, H_kv, d))) for m in chunk_sizes]
    scale = 0.5
    cache = orc.OracleCache(1, H_q, H_kv, d, C, W, scale=scale)
    outs_ref, toks = token_centric_run(chunks, C, W, H_q, H_kv, scale)
    for (q, kn, vn), Oref in zip(chunks, outs_ref):
        O, _ = cache.step(q[None], kn[None], vn[None])
        assert np.allclose(O[0], Oref, atol=1e-12)
    for g in range(H_kv):
        valid = cache.pos[0, g] >= 0
        assert set(cache.pos[0, g][valid].tolist()) == set(toks[g])
        for s in np.nonzero(valid)[0]:
            k, v, sc = toks[g][int(cache.pos[0, g, s])]
            assert np.array_equal(cache.K[0, g, s], k) and np.array_equal(cache.V[0, g, s], v)
            assert abs(float(cache.scores[0, g, s]) - float(sc)) <= 1e-6 * abs(float(sc))


ALL_ATTENTION_PINS = [check_bruteforce, check_sdpa, check_uniform_closed_form, check_one_hot,
                      check_single_query_empty_cache, check_weight_total, check_causality,
                      check_mha_reduction, check_golden_attention]
ALL_EVICT_PINS = [check_evict_rankcount, check_golden_evict, check_fp32_accumulate]
ALL_PINS = ALL_ATTENTION_PINS + ALL_EVICT_PINS + [check_trajectory]
