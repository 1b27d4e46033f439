"""Pins of the oracle's quantised-cache format (the Q-Hitter reading):
hand-worked rows, the defining properties of the symmetric int8 code, the
bf16 rounding against torch's, and the placement of quantised tokens over a
multi-step run (every cached row is the quantised form of the token at its
position)."""
import json
import os

import numpy as np
import torch

from oracle import h2o_oracle as orc

HERE = os.path.dirname(os.path.abspath(__file__))


def test_hand_worked_rows():
    ex = json.load(open(os.path.join(HERE, "golden", "q8_hand_examples.json")))
    for row in ex["rows"]:
        q, s = orc.quantize_row_q8(np.array(row["x"], np.float32))
        assert q.tolist() == row["q"], row["what"]
        assert np.float32(s) == np.float32(row["s"]), row["what"]
        assert orc.dequantize_q8(q, s).tolist() == row["x_hat"], row["what"]


def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.standard_normal(100000).astype(np.float32) * 10,
                        np.float32([1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -1.0 - 2 ** -8,
                                    1.0 + 2 ** -8 + 2 ** -20, 3e38, 1e-30, 0.0, -0.0])])
    ours = orc.bf16_round(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).float().numpy()
    assert np.array_equal(ours.view(np.uint32), ref.view(np.uint32))


def test_code_properties():
    rng = np.random.default_rng(1)
    for trial in range(300):
        d = int(rng.choice([8, 64, 128]))
        x = (rng.standard_normal(d) * 10 ** rng.uniform(-3, 3)).astype(np.float32)
        x = torch.from_numpy(x).to(torch.bfloat16).float().numpy()   # inputs are bf16 values
        q, s = orc.quantize_row_q8(x)
        assert q.dtype == np.int8 and np.all(np.abs(q.astype(int)) <= 127)
        j = int(np.argmax(np.abs(x)))
        assert abs(int(q[j])) == 127 and np.sign(q[j]) == np.sign(x[j])
        xh = orc.dequantize_q8(q, s)
        # code error at most half a step (plus the division's rounding), then
        # the bf16 rounding of the product
        bound = 0.5 * float(s) * (1 + 1e-5) + np.abs(xh) * 2.0 ** -8 + 1e-30
        assert np.all(np.abs(xh - x) <= bound)
        # the code is the nearest one to x / s, up to the fp32 rounding of
        # the quotient (|x / s| <= 127.00001: its rounding moves it by at most
        # 2^-17, which can tip a quotient that is almost a half-integer)
        qs = q.astype(np.float64) * float(s)
        for dq in (-1, 1):
            alt = (q.astype(np.float64) + dq) * float(s)
            assert np.all(np.abs(qs - x) <= np.abs(alt - x) + 2.0 ** -16 * float(s))


def test_quantised_cache_holds_each_token_quantised():
    """Over a run with eviction, every valid slot holds the quantised form of
    the token whose position it records (K and V), and the scores evolve
    exactly as in the unquantised cache fed the same summed weights."""
    rng = np.random.default_rng(2)
    B, Hq, Hkv, d, C, W, nq = 2, 4, 2, 16, 24, 3, 8
    q8 = orc.OracleCache(B, Hq, Hkv, d, C, W, kv_format="q8")
    ref = orc.OracleCache(B, Hq, Hkv, d, C, W)
    tokens_k, tokens_v = {}, {}
    for step in range(6):
        Kn = torch.randn(B, nq, Hkv, d).to(torch.bfloat16).double().numpy()
        Vn = torch.randn(B, nq, Hkv, d).to(torch.bfloat16).double().numpy()
        for i in range(nq):
            tokens_k[q8.t0 + i] = Kn[:, i]
            tokens_v[q8.t0 + i] = Vn[:, i]
        cs = (rng.random((B, Hkv, C + nq)) * 2).astype(np.float32)
        cs[:, :, q8.n:C] = 0
        q8.evict(cs, Kn, Vn)
        ref.evict(cs, Kn, Vn)
        assert np.array_equal(q8.pos, ref.pos) and np.array_equal(q8.scores, ref.scores)
        for b in range(B):
            for g in range(Hkv):
                for s in range(q8.n):
                    p = int(q8.pos[b, g, s])
                    qk, sk = orc.quantize_row_q8(tokens_k[p][b, g])
                    qv, sv = orc.quantize_row_q8(tokens_v[p][b, g])
                    assert np.array_equal(q8.Kq[b, g, s], qk) and q8.Ks[b, g, s] == sk
                    assert np.array_equal(q8.Vq[b, g, s], qv) and q8.Vs[b, g, s] == sv
                    assert np.array_equal(q8.K[b, g, s], orc.dequantize_q8(qk, sk))
                    assert np.array_equal(q8.V[b, g, s], orc.dequantize_q8(qv, sv))


def test_attention_reads_the_dequantised_rows():
    """The quantised cache's attention is the plain attention over the values
    bf16(q * s): built here from the codes directly, independently of the
    cache's own bookkeeping."""
    rng = np.random.default_rng(3)
    B, Hq, Hkv, d, C, n, nq = 1, 4, 2, 32, 40, 40, 6
    cache = orc.OracleCache(B, Hq, Hkv, d, C, 0, kv_format="q8")
    Kq = rng.integers(-127, 128, (B, Hkv, C, d)).astype(np.int8)
    Vq = rng.integers(-127, 128, (B, Hkv, C, d)).astype(np.int8)
    Ks = (rng.random((B, Hkv, C)) * 0.05).astype(np.float32)
    Vs = (rng.random((B, Hkv, C)) * 0.05).astype(np.float32)
    cache.load_q8(Kq, Ks, Vq, Vs, np.zeros((B, Hkv, C), np.float32),
                  np.tile(np.arange(C, dtype=np.int32), (B, Hkv, 1)), n, C)
    Q = rng.standard_normal((B, nq, Hq, d))
    Kn = rng.standard_normal((B, nq, Hkv, d))
    Vn = rng.standard_normal((B, nq, Hkv, d))
    O, cs, _ = cache.attention(Q, Kn, Vn)
    Kd = np.empty((B, Hkv, C, d))
    Vd = np.empty_like(Kd)
    for g in range(Hkv):
        for s in range(C):     # element by element, from the definition
            for e in range(d):
                Kd[0, g, s, e] = float(torch.tensor(float(np.float32(Kq[0, g, s, e]) * Ks[0, g, s]),
                                                    dtype=torch.float32).to(torch.bfloat16))
                Vd[0, g, s, e] = float(torch.tensor(float(np.float32(Vq[0, g, s, e]) * Vs[0, g, s]),
                                                    dtype=torch.float32).to(torch.bfloat16))
    O2, cs2, _ = orc.attention_one_cache(Q[0], Kd[0], Vd[0], n, Kn[0], Vn[0],
                                         1 / np.sqrt(d))
    assert np.allclose(O[0], O2, rtol=0, atol=1e-12)
    assert np.allclose(cs[0], cs2, rtol=0, atol=1e-12)
