"""Pins for the backward oracle (gradients of sum(dO * O)), against facts that
do not come from the backward code itself: central finite differences of the
forward oracle, closed forms, and identities that the softmax fixes."""
import numpy as np
import pytest

import oracle


def _rand(shape, seed, std=1.0):
    return np.random.default_rng(seed).standard_normal(shape) * std


def _loss(q, k, v, dout, causal, scale):
    O, _ = oracle.attention(q, k, v, causal=causal, scale=scale)
    return float(np.sum(O * dout))


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N,d", [(1, 2), (3, 2), (5, 3), (6, 4)])
def test_backward_matches_finite_differences(N, d, causal):
    q, k, v, dout = (_rand((1, 1, N, d), 80 + s) for s in range(4))
    scale = 0.7
    dq, dk, dv = oracle.attention_backward(q, k, v, dout, causal, scale)
    h = 1e-5
    for name, x, g in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        for idx in np.ndindex(N, d):
            xp, xm = x.copy(), x.copy()
            xp[0, 0][idx] += h
            xm[0, 0][idx] -= h
            args_p = {"q": q, "k": k, "v": v}
            args_m = {"q": q, "k": k, "v": v}
            args_p[name], args_m[name] = xp, xm
            fd = (_loss(args_p["q"], args_p["k"], args_p["v"], dout, causal, scale) -
                  _loss(args_m["q"], args_m["k"], args_m["v"], dout, causal, scale)) / (2 * h)
            assert abs(fd - g[0][idx]) < 1e-7 * max(1.0, abs(fd)), (name, idx, fd, g[0][idx])


def test_single_key_closed_form():
    q, k, v, dout = (_rand((1, 1, 1, 4), 90 + s) for s in range(4))
    dq, dk, dv = oracle.attention_backward(q, k, v, dout, False, 0.5)
    assert np.array_equal(dv[0], dout[0, 0])        # O = v_0 exactly
    assert np.all(dq == 0) and np.all(dk == 0)      # the softmax of one score is constant


@pytest.mark.parametrize("causal", [False, True])
def test_softmax_identities(causal):
    """Rows of P sum to 1 and rows of dS sum to 0, so sum_j dV_j = sum_i dO_i
    and sum_j dK_j = 0."""
    q, k, v, dout = (_rand((1, 2, 40, 8), 95 + s) for s in range(4))
    dq, dk, dv = oracle.attention_backward(q, k, v, dout, causal, 0.3)
    for h in range(2):
        assert np.allclose(dv[h].sum(axis=0), dout[0, h].sum(axis=0), rtol=0, atol=1e-12)
        assert np.allclose(dk[h].sum(axis=0), 0.0, rtol=0, atol=1e-12)


def test_causal_first_key_gets_no_gradient_from_its_own_row_only():
    """Causal, N = 2: row 0 sees only key 0, so key 1 receives gradient only
    from row 1; q_0 receives none (its softmax has a single entry)."""
    q, k, v, dout = (_rand((1, 1, 2, 3), 99 + s) for s in range(4))
    dq, dk, dv = oracle.attention_backward(q, k, v, dout, True, 1.0)
    assert np.all(dq[0, 0] == 0)
    O, _ = oracle.attention(q, k, v, causal=True, scale=1.0)
    p = np.exp(q[0, 0, 1] @ k[0, 0].T)
    p /= p.sum()
    assert np.allclose(dv[0, 1], p[1] * dout[0, 0, 1], rtol=0, atol=1e-14)
