"""Pins of the oracle's attention backward: torch fp64 autograd of the same
masked attention (a library routine), central finite differences on a tiny
case, closed forms (constant V rows: no gradient to q and k; dO = u in every
row: dV is the column sum of P times u), and zero gradient for slots that
are not valid."""
import numpy as np
import pytest
import torch

from oracle import h2o_oracle as orc


def _case(seed, n_q=5, H_q=4, H_kv=2, d=8, C=9, n=6):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((n_q, H_q, d))
    kc = rng.standard_normal((H_kv, C, d))
    vc = rng.standard_normal((H_kv, C, d))
    kc[:, n:] = 0
    vc[:, n:] = 0
    kn = rng.standard_normal((n_q, H_kv, d))
    vn = rng.standard_normal((n_q, H_kv, d))
    do = rng.standard_normal((n_q, H_q, d))
    return q, kc, vc, n, kn, vn, do, 1.0 / np.sqrt(d)


def _torch_grads(q, kc, vc, n, kn, vn, do, scale):
    """The same attention written with torch ops (fp64), differentiated by
    autograd."""
    T = {k: torch.tensor(v, dtype=torch.float64, requires_grad=True)
         for k, v in dict(q=q, kc=kc, vc=vc, kn=kn, vn=vn).items()}
    n_q, H_q, d = q.shape
    H_kv = kc.shape[0]
    G = H_q // H_kv
    mask = torch.zeros(n_q, n + n_q, dtype=torch.bool)
    mask[:, :n] = True
    mask[:, n:] = torch.tril(torch.ones(n_q, n_q, dtype=torch.bool))
    outs = []
    for h in range(H_q):
        g = h // G
        keys = torch.cat([T["kc"][g, :n], T["kn"][:, g]], 0)
        vals = torch.cat([T["vc"][g, :n], T["vn"][:, g]], 0)
        o = torch.nn.functional.scaled_dot_product_attention(
            T["q"][:, h][None, None], keys[None, None], vals[None, None],
            attn_mask=mask[None, None], scale=scale)[0, 0]
        outs.append(o)
    O = torch.stack(outs, 1)
    (O * torch.tensor(do)).sum().backward()
    return [T[k].grad.numpy() for k in ("q", "kc", "vc", "kn", "vn")]


@pytest.mark.parametrize("seed,shape", [(0, {}), (1, dict(n=0, C=3)), (2, dict(H_kv=4)),
                                        (3, dict(n_q=1)), (4, dict(H_kv=1, H_q=3))])
def test_backward_matches_torch_autograd(seed, shape):
    args = _case(seed, **shape)
    got = orc.attention_backward_one_cache(*args)
    ref = _torch_grads(*args)
    for name, a, b in zip(("dq", "dkc", "dvc", "dkn", "dvn"), got, ref):
        assert np.allclose(a, b, atol=1e-12, rtol=1e-10), name


def test_backward_matches_finite_differences():
    q, kc, vc, n, kn, vn, do, scale = _case(7, n_q=3, H_q=2, H_kv=1, d=4, C=4, n=3)
    grads = orc.attention_backward_one_cache(q, kc, vc, n, kn, vn, do, scale)

    def loss(q, kc, vc, kn, vn):
        o, _, _ = orc.attention_one_cache(q, kc, vc, n, kn, vn, scale)
        return float((o * do).sum())

    base = dict(q=q, kc=kc, vc=vc, kn=kn, vn=vn)
    rng = np.random.default_rng(0)
    eps = 1e-6
    for k, (name, g) in enumerate(zip(("q", "kc", "vc", "kn", "vn"), grads)):
        for _ in range(6):
            idx = tuple(int(rng.integers(s)) for s in base[name].shape)
            if name in ("kc", "vc") and idx[1] >= n:
                continue
            plus = {a: b.copy() for a, b in base.items()}
            minus = {a: b.copy() for a, b in base.items()}
            plus[name][idx] += eps
            minus[name][idx] -= eps
            num = (loss(**plus) - loss(**minus)) / (2 * eps)
            assert abs(num - g[idx]) < 1e-6, (name, idx, num, g[idx])


def test_constant_values_give_no_query_or_key_gradient():
    """Every visible V row equal: O is that row whatever P is, so dq = dk = 0."""
    q, kc, vc, n, kn, vn, do, scale = _case(3)
    row = np.arange(kc.shape[2], dtype=float)
    vc[:, :n] = row
    vn[:] = row
    dq, dkc, _, dkn, _ = orc.attention_backward_one_cache(q, kc, vc, n, kn, vn, do, scale)
    assert np.allclose(dq, 0, atol=1e-12)
    assert np.allclose(dkc, 0, atol=1e-12) and np.allclose(dkn, 0, atol=1e-12)


def test_uniform_output_gradient_gives_column_sums():
    """dO = u in every row of every head: dV of a key is (summed weight of the
    key over its group's heads and the queries) times u."""
    q, kc, vc, n, kn, vn, do, scale = _case(5)
    u = np.linspace(-1, 1, q.shape[2])
    do[:] = u
    _, _, dvc, _, dvn = orc.attention_backward_one_cache(q, kc, vc, n, kn, vn, do, scale)
    _, colsum, _ = orc.attention_one_cache(q, kc, vc, n, kn, vn, scale)
    C = kc.shape[1]
    for g in range(kc.shape[0]):
        assert np.allclose(dvc[g, :n], np.outer(colsum[g, :n], u), atol=1e-12)
        assert np.allclose(dvn[:, g], np.outer(colsum[g, C:], u), atol=1e-12)


def test_invalid_slots_get_no_gradient():
    q, kc, vc, n, kn, vn, do, scale = _case(9, C=12, n=5)
    _, dkc, dvc, _, _ = orc.attention_backward_one_cache(q, kc, vc, n, kn, vn, do, scale)
    assert not dkc[:, n:].any() and not dvc[:, n:].any()
