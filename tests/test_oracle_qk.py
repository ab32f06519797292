"""Pins for the oracle with different query and key lengths (Nq != Nk).

The pages only use self-attention (Nq = Nk). With Nq != Nk, causal masking is
aligned to the bottom-right corner of the score matrix -- query i sees keys
j <= i + Nk - Nq, so the last query sees every key -- which is our reading;
causal with Nq > Nk would leave rows without keys and is rejected. As in
``test_oracle.py``, nothing here reuses the oracle's formulas: a separate
pure-Python brute force with the full softmax Jacobian, central finite
differences of the forward, closed forms and identities.
"""
import math

import numpy as np
import pytest

import attn_inputs

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")


def _rand(seed, *shape):
    return attn_inputs.standard_normal(seed, int(np.prod(shape))).reshape(shape)


def brute_qk(q, k, v, dout, causal, scale):
    """Pure-Python loops for Nq x Nk scores; returns o, lse, dq, dk, dv."""
    Nq, Nk, d = len(q), len(k), len(q[0])
    allowed = [[(not causal) or j <= i + Nk - Nq for j in range(Nk)] for i in range(Nq)]
    s = [[scale * sum(q[i][c] * k[j][c] for c in range(d)) for j in range(Nk)] for i in range(Nq)]
    e = [[math.exp(s[i][j]) if allowed[i][j] else 0.0 for j in range(Nk)] for i in range(Nq)]
    z = [sum(row) for row in e]
    p = [[e[i][j] / z[i] for j in range(Nk)] for i in range(Nq)]
    o = [[sum(p[i][j] * v[j][c] for j in range(Nk)) for c in range(d)] for i in range(Nq)]
    lse = [math.log(z[i]) for i in range(Nq)]
    dp = [[sum(dout[i][c] * v[j][c] for c in range(d)) for j in range(Nk)] for i in range(Nq)]
    ds = [[sum(dp[i][kk] * p[i][kk] * ((1.0 if kk == j else 0.0) - p[i][j]) for kk in range(Nk))
           for j in range(Nk)] for i in range(Nq)]
    dq = [[scale * sum(ds[i][j] * k[j][c] for j in range(Nk)) for c in range(d)] for i in range(Nq)]
    dk = [[scale * sum(ds[i][j] * q[i][c] for i in range(Nq)) for c in range(d)] for j in range(Nk)]
    dv = [[sum(p[i][j] * dout[i][c] for i in range(Nq)) for c in range(d)] for j in range(Nk)]
    return o, lse, dq, dk, dv


SHAPES = [  # Nq, Nk, d, causal
    (3, 7, 4, False), (3, 7, 4, True), (7, 3, 4, False), (1, 5, 3, True), (5, 12, 2, True),
    (12, 5, 3, False),
]


@pytest.mark.parametrize("Nq,Nk,d,causal", SHAPES)
def test_brute_force(oracle_mod, Nq, Nk, d, causal):
    scale = 0.8
    q, do = _rand(300, Nq, d), _rand(301, Nq, d)
    k, v = _rand(302, Nk, d), _rand(303, Nk, d)
    o, lse, dq, dk, dv = brute_qk(q.tolist(), k.tolist(), v.tolist(), do.tolist(), causal, scale)
    fo, flse = oracle_mod.attention_forward(q, k, v, causal, scale)
    g = oracle_mod.attention_backward(q, k, v, do, causal, scale)
    np.testing.assert_allclose(fo, o, rtol=0, atol=1e-11)
    np.testing.assert_allclose(flse, lse, rtol=0, atol=1e-11)
    for name, ref in (("o", o), ("dq", dq), ("dk", dk), ("dv", dv)):
        np.testing.assert_allclose(g[name], ref, rtol=0, atol=1e-11, err_msg=name)
    np.testing.assert_allclose(g["lse"], lse, rtol=0, atol=1e-11)
    assert g["dq"].shape == (Nq, d) and g["dk"].shape == (Nk, d)


@pytest.mark.parametrize("causal", [False, True])
def test_finite_differences(oracle_mod, causal):
    Nq, Nk, d, scale = 4, 7, 3, 0.7
    q, do = _rand(310, Nq, d), _rand(311, Nq, d)
    k, v = _rand(312, Nk, d), _rand(313, Nk, d)
    g = oracle_mod.attention_backward(q, k, v, do, causal, scale)

    def loss(args):
        o, _ = oracle_mod.attention_forward(args["q"], args["k"], args["v"], causal, scale,
                                            nthreads=1)
        return float(np.sum(do * o))

    h = 1e-6
    for name, x, grad in (("q", q, g["dq"]), ("k", k, g["dk"]), ("v", v, g["dv"])):
        fd = np.zeros_like(x)
        for idx in np.ndindex(x.shape):
            xp, xm = x.copy(), x.copy()
            xp[idx] += h
            xm[idx] -= h
            args_p = {"q": q, "k": k, "v": v}
            args_m = dict(args_p)
            args_p[name], args_m[name] = xp, xm
            fd[idx] = (loss(args_p) - loss(args_m)) / (2 * h)
        err = np.linalg.norm(fd - grad) / max(np.linalg.norm(grad), 1e-30)
        assert err < 1e-7, (name, err)


def test_uniform_scores_bottom_right(oracle_mod):
    """Q = 0: query i averages V over the keys j <= i + Nk - Nq it sees."""
    Nq, Nk, d = 4, 9, 3
    q = np.zeros((Nq, d))
    k, v = _rand(320, Nk, d), _rand(321, Nk, d)
    o, lse = oracle_mod.attention_forward(q, k, v, True, 0.5)
    for i in range(Nq):
        n = i + Nk - Nq + 1
        np.testing.assert_allclose(o[i], v[:n].mean(axis=0), rtol=0, atol=1e-13)
        assert abs(lse[i] - math.log(n)) < 1e-13


def test_single_query_causal_sees_every_key(oracle_mod):
    k, v = _rand(330, 6, 4), _rand(331, 6, 4)
    q = _rand(332, 1, 4)
    a = oracle_mod.attention_forward(q, k, v, True, 0.6)
    b = oracle_mod.attention_forward(q, k, v, False, 0.6)
    np.testing.assert_array_equal(a[0], b[0])
    np.testing.assert_array_equal(a[1], b[1])


def test_gradient_sum_identities(oracle_mod):
    q, do = _rand(340, 5, 3), _rand(341, 5, 3)
    k, v = _rand(342, 8, 3), _rand(343, 8, 3)
    for causal in (False, True):
        g = oracle_mod.attention_backward(q, k, v, do, causal, 0.9)
        np.testing.assert_allclose(g["dk"].sum(axis=0), 0.0, atol=1e-12)
        np.testing.assert_allclose(g["dv"].sum(axis=0), do.sum(axis=0), atol=1e-12)


def test_rows_variant_agrees(oracle_mod):
    q, do = _rand(350, 20, 4), _rand(351, 20, 4)
    k, v = _rand(352, 33, 4), _rand(353, 33, 4)
    for causal in (False, True):
        g = oracle_mod.attention_backward(q, k, v, do, causal, 0.5)
        qr, kr = np.array([0, 7, 19]), np.array([0, 12, 20, 32])
        dq, dk, dv = oracle_mod.attention_backward_rows(q, k, v, do, causal, 0.5, qr, kr)
        np.testing.assert_allclose(dq, g["dq"][qr], atol=1e-12)
        np.testing.assert_allclose(dk, g["dk"][kr], atol=1e-12)
        np.testing.assert_allclose(dv, g["dv"][kr], atol=1e-12)


def test_causal_with_more_queries_than_keys_is_rejected(oracle_mod):
    q, k = _rand(360, 5, 2), _rand(361, 3, 2)
    with pytest.raises(ValueError):
        oracle_mod.attention_forward(q, k, k, True, 1.0)
    with pytest.raises(ValueError):
        oracle_mod.attention_backward(q, k, k, q, True, 1.0)
