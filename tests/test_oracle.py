"""Pins for the fp64 oracle, from what the pages and the mathematics fix.

None of these checks reuses the oracle's own formulas: the brute force below is
a separate pure-Python formulation (no max subtraction, the softmax Jacobian
written out in full, D taken as sum_k p_ik dP_ik instead of dO . O), the
gradients are also checked by central finite differences of the forward, and
the rest are closed forms and identities of softmax attention.

The pages print no worked values: the twelve-token, four-by-four-tile
simulation on the "FlashAttention (v2)" glossary page has its numbers only in an
interactive figure. Its shape (N = 12, tiles of 4) is used for the independent
online-softmax recurrence check.
"""
import math

import numpy as np
import pytest

import attn_inputs

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")


# ---------------------------------------------------------------- brute force
def brute_attention(q, k, v, dout, causal, scale):
    """Pure-Python loops; returns o, lse, dq, dk, dv as nested lists."""
    N, d = len(q), len(q[0])
    allowed = [[(not causal) or j <= i for j in range(N)] for i in range(N)]
    s = [[scale * sum(q[i][c] * k[j][c] for c in range(d)) for j in range(N)] for i in range(N)]
    e = [[math.exp(s[i][j]) if allowed[i][j] else 0.0 for j in range(N)] for i in range(N)]
    z = [sum(row) for row in e]
    p = [[e[i][j] / z[i] for j in range(N)] for i in range(N)]
    o = [[sum(p[i][j] * v[j][c] for j in range(N)) for c in range(d)] for i in range(N)]
    lse = [math.log(z[i]) for i in range(N)]
    dp = [[sum(dout[i][c] * v[j][c] for c in range(d)) for j in range(N)] for i in range(N)]
    # softmax Jacobian: d p_ik / d s_ij = p_ik (delta_jk - p_ij)
    ds = [[sum(dp[i][kk] * p[i][kk] * ((1.0 if kk == j else 0.0) - p[i][j]) for kk in range(N))
           for j in range(N)] for i in range(N)]
    dq = [[scale * sum(ds[i][j] * k[j][c] for j in range(N)) for c in range(d)] for i in range(N)]
    dk = [[scale * sum(ds[i][j] * q[i][c] for i in range(N)) for c in range(d)] for j in range(N)]
    dv = [[sum(p[i][j] * dout[i][c] for i in range(N)) for c in range(d)] for j in range(N)]
    return o, lse, dq, dk, dv


def _rand(seed, *shape):
    return attn_inputs.standard_normal(seed, int(np.prod(shape))).reshape(shape)


@pytest.mark.parametrize("N,d", [(1, 3), (5, 4), (12, 8), (16, 2)])
@pytest.mark.parametrize("causal", [False, True])
def test_brute_force(oracle_mod, N, d, causal):
    q, k, v, do = (_rand(100 + t + 10 * N + d, N, d) for t in range(4))
    scale = 1.0 / math.sqrt(d) if d > 2 else 0.9
    bo, blse, bdq, bdk, bdv = (np.array(x) for x in brute_attention(
        q.tolist(), k.tolist(), v.tolist(), do.tolist(), causal, scale))
    o, lse = oracle_mod.attention_forward(q, k, v, causal, scale)
    np.testing.assert_allclose(o, bo, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, blse, rtol=0, atol=1e-12)
    g = oracle_mod.attention_backward(q, k, v, do, causal, scale)
    np.testing.assert_allclose(g["o"], bo, rtol=0, atol=1e-12)
    np.testing.assert_allclose(g["lse"], blse, rtol=0, atol=1e-12)
    for name, ref in (("dq", bdq), ("dk", bdk), ("dv", bdv)):
        np.testing.assert_allclose(g[name], ref, rtol=0, atol=1e-11, err_msg=name)


def test_brute_force_bf16_inputs(oracle_mod):
    """bf16 bit patterns from the shared generator widen exactly to the same doubles."""
    t = attn_inputs.make_qkvdo(0, 1, 2, 9, 4)
    scale = 0.5
    o, lse = oracle_mod.attention_forward(t["q"], t["k"], t["v"], False, scale)
    for h in range(2):
        f = [attn_inputs.bf16_bits_to_f64(t[n][0, h]).tolist() for n in ("q", "k", "v", "do")]
        bo, blse, *_ = brute_attention(*f, False, scale)
        np.testing.assert_allclose(o[0, h], bo, atol=1e-12, rtol=0)
        np.testing.assert_allclose(lse[0, h], blse, atol=1e-12, rtol=0)


# ------------------------------------------------------- finite differences
@pytest.mark.parametrize("causal", [False, True])
def test_finite_differences(oracle_mod, causal):
    N, d, scale = 6, 4, 0.7
    q, k, v, do = (_rand(200 + t, N, d) for t in range(4))
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


# ---------------------------------------------------------------- invariants
@pytest.mark.parametrize("causal", [False, True])
def test_uniform_scores_give_mean_of_v(oracle_mod, causal):
    N, d = 10, 5
    q = np.zeros((N, d))
    k, v = _rand(300, N, d), _rand(301, N, d)
    o, lse = oracle_mod.attention_forward(q, k, v, causal, 0.3)
    for i in range(N):
        n = i + 1 if causal else N
        np.testing.assert_allclose(o[i], v[:n].mean(axis=0), atol=1e-14)
        assert abs(lse[i] - math.log(n)) < 1e-14


def test_causal_row_zero(oracle_mod):
    N, d, scale = 7, 6, 0.4
    q, k, v = _rand(310, N, d), _rand(311, N, d), _rand(312, N, d)
    o, lse = oracle_mod.attention_forward(q, k, v, True, scale)
    np.testing.assert_array_equal(o[0], v[0])
    assert abs(lse[0] - scale * float(q[0] @ k[0])) < 1e-14


def test_rows_of_p_sum_to_one(oracle_mod):
    """With V = I (d = N), O is P itself: non-negative rows summing to 1."""
    N = 9
    q, k = _rand(320, N, N), _rand(321, N, N)
    for causal in (False, True):
        p, _ = oracle_mod.attention_forward(q, k, np.eye(N), causal, 0.5)
        assert (p >= 0).all()
        np.testing.assert_allclose(p.sum(axis=1), 1.0, atol=1e-14)
        if causal:
            assert np.all(np.triu(p, 1) == 0.0)


def test_shift_invariance(oracle_mod):
    """Adding u to every key row keeps O and shifts LSE_i by scale * q_i . u."""
    N, d, scale = 11, 4, 0.6
    q, k, v = _rand(330, N, d), _rand(331, N, d), _rand(332, N, d)
    u = _rand(333, d)
    for causal in (False, True):
        o1, l1 = oracle_mod.attention_forward(q, k, v, causal, scale)
        o2, l2 = oracle_mod.attention_forward(q, k + u, v, causal, scale)
        np.testing.assert_allclose(o2, o1, atol=1e-13)
        np.testing.assert_allclose(l2 - l1, scale * (q @ u), atol=1e-13)


def test_permutation_equivariance(oracle_mod):
    N, d = 8, 3
    q, k, v = _rand(340, N, d), _rand(341, N, d), _rand(342, N, d)
    perm = np.random.default_rng(0).permutation(N)
    o1, l1 = oracle_mod.attention_forward(q, k, v, False, 0.8)
    o2, l2 = oracle_mod.attention_forward(q[perm], k, v, False, 0.8)
    np.testing.assert_allclose(o2, o1[perm], atol=1e-14)
    o3, l3 = oracle_mod.attention_forward(q, k[perm], v[perm], False, 0.8)
    np.testing.assert_allclose(o3, o1, atol=1e-13)
    np.testing.assert_allclose(l3, l1, atol=1e-13)


@pytest.mark.parametrize("causal", [False, True])
def test_gradient_sum_identities(oracle_mod, causal):
    """Rows of dS sum to zero and rows of P to one: sum_j dK_j = 0, sum_j dV_j = sum_i dO_i."""
    N, d = 13, 6
    q, k, v, do = (_rand(350 + t, N, d) for t in range(4))
    g = oracle_mod.attention_backward(q, k, v, do, causal, 0.45)
    np.testing.assert_allclose(g["dk"].sum(axis=0), 0.0, atol=1e-12)
    np.testing.assert_allclose(g["dv"].sum(axis=0), do.sum(axis=0), atol=1e-12)
    if causal:  # the last key is seen only by the last query row
        p_last = math.exp(0.45 * float(q[-1] @ k[-1]) - g["lse"][-1])
        np.testing.assert_allclose(g["dv"][-1], p_last * do[-1], atol=1e-13)


def test_single_token(oracle_mod):
    d, scale = 5, 0.3
    q, k, v, do = (_rand(360 + t, 1, d) for t in range(4))
    for causal in (False, True):
        g = oracle_mod.attention_backward(q, k, v, do, causal, scale)
        np.testing.assert_array_equal(g["o"], v)
        assert abs(g["lse"][0] - scale * float(q[0] @ k[0])) < 1e-15
        np.testing.assert_array_equal(g["dv"], do)
        np.testing.assert_allclose(g["dq"], 0.0, atol=1e-15)
        np.testing.assert_allclose(g["dk"], 0.0, atol=1e-15)


def test_one_dominant_key(oracle_mod):
    """A score far above the rest puts all the weight on that key (large magnitudes stay finite)."""
    N, d = 6, 4
    k = _rand(370, N, d)
    v = _rand(371, N, d)
    q = np.tile(k[3] * 200.0, (N, 1))
    o, lse = oracle_mod.attention_forward(q, k, v, False, 1.0)
    assert np.isfinite(lse).all()
    np.testing.assert_allclose(o, np.tile(v[3], (N, 1)), atol=1e-12)


# ------------------------------------- tiled online softmax (shape N=12, tile 4)
def online_softmax_tiled(q, k, v, causal, scale, tile):
    """Exact attention, key tile by key tile, with a running max and sum, rescaling
    the accumulator when the max grows and dividing by the sum once at the end
    ("FlashAttention-2" summary page, How It Works item 2)."""
    N, d = q.shape
    o = np.zeros((N, d))
    m = np.full(N, -np.inf)
    l = np.zeros(N)
    for j0 in range(0, N, tile):
        s = scale * (q @ k[j0:j0 + tile].T)
        if causal:
            cols = np.arange(j0, min(N, j0 + tile))
            s = np.where(cols[None, :] <= np.arange(N)[:, None], s, -np.inf)
        m_new = np.maximum(m, s.max(axis=1))
        alpha = np.exp(m - m_new)
        p = np.exp(s - m_new[:, None])
        l = l * alpha + p.sum(axis=1)
        o = o * alpha[:, None] + p @ v[j0:j0 + tile]
        m = m_new
    return o / l[:, None], m + np.log(l)


@pytest.mark.parametrize("causal", [False, True])
def test_tiled_online_softmax_matches(oracle_mod, causal):
    N, d = 12, 4
    q, k, v = _rand(380, N, d), _rand(381, N, d), _rand(382, N, d)
    to, tl = online_softmax_tiled(q, k, v, causal, 0.5, 4)
    o, lse = oracle_mod.attention_forward(q, k, v, causal, 0.5)
    np.testing.assert_allclose(o, to, atol=1e-12)
    np.testing.assert_allclose(lse, tl, atol=1e-12)


# ------------------------------------------------ sampled rows agree with full
@pytest.mark.parametrize("causal", [False, True])
def test_rows_variants_agree(oracle_mod, causal):
    t = attn_inputs.make_qkvdo(7, 1, 2, 40, 8)
    scale = 1 / math.sqrt(8)
    g = oracle_mod.attention_backward(t["q"], t["k"], t["v"], t["do"], causal, scale)
    rows = np.array([0, 5, 39, 17])
    o, lse = oracle_mod.attention_forward(t["q"], t["k"], t["v"], causal, scale, rows=rows)
    np.testing.assert_allclose(o, g["o"][:, :, rows], atol=1e-13)
    np.testing.assert_allclose(lse, g["lse"][:, :, rows], atol=1e-13)
    dq, dk, dv = oracle_mod.attention_backward_rows(t["q"], t["k"], t["v"], t["do"], causal, scale,
                                                    rows, rows[::-1])
    np.testing.assert_allclose(dq, g["dq"][:, :, rows], atol=1e-12)
    np.testing.assert_allclose(dk, g["dk"][:, :, rows[::-1]], atol=1e-12)
    np.testing.assert_allclose(dv, g["dv"][:, :, rows[::-1]], atol=1e-12)


def test_rejects_bad_rows(oracle_mod):
    q = np.zeros((3, 2))
    with pytest.raises(ValueError):
        oracle_mod.attention_forward(q, q, q, False, 1.0, rows=[3])


# ------------------------------------------------------------- input generator
def test_generator_is_standard_normal_and_deterministic():
    a = attn_inputs.standard_normal(12345, 200000)
    assert abs(a.mean()) < 0.01 and abs(a.std() - 1) < 0.01
    np.testing.assert_array_equal(a, attn_inputs.standard_normal(12345, 200000))
    # published SplitMix64 test vector: seed 0 -> first output 0xE220A8397B1DCDAF
    assert int(attn_inputs.splitmix64(0, 1)[0]) == 0xE220A8397B1DCDAF
    bits = attn_inputs.to_bf16_bits(np.array([1.0, -2.0, 1.00390625, 1.005859375, np.nan]))
    assert [hex(int(x)) for x in bits] == ["0x3f80", "0xc000", "0x3f80", "0x3f81", "0x7fc0"]
