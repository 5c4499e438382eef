"""Pins for the oracle's attention gradients (oracle/grad.py).

Each gradient is checked against central finite differences of the C forward
oracle (pinned separately), element by element, and against closed forms:
a single token for the linear attention, a window of one for the softmax
attention.  A dropped term of the quotient rule, a missing 1 + u factor, a
transposed score matrix or a leak outside the causal band breaks one of them.
"""
import math

import numpy as np
import pytest

import oracle
from oracle import grad


def rng(seed):
    return np.random.Generator(np.random.PCG64(seed))


def fd_grad(f, x, dy, h=1e-6):
    """d/dx of sum(f(x) * dy) by central differences, element by element."""
    g = np.zeros_like(x)
    it = np.nditer(x, flags=["multi_index"])
    for _ in it:
        idx = it.multi_index
        xp, xm = x.copy(), x.copy()
        xp[idx] += h
        xm[idx] -= h
        g[idx] = (np.sum(f(xp) * dy) - np.sum(f(xm) * dy)) / (2 * h)
    return g


@pytest.mark.parametrize("L,d,dv", [(6, 4, 3), (9, 16, 5)])
def test_linattn_grad_matches_finite_differences(L, d, dv):
    r = rng(L * 10 + d)
    q, k = r.standard_normal((1, L, d)) * 0.5, r.standard_normal((1, L, d)) * 0.5
    v, dy = r.standard_normal((1, L, dv)), r.standard_normal((1, L, dv))
    eps = 1e-6
    dq, dk, dv_ = grad.linattn_grad(q, k, v, dy, eps)
    fwd = lambda qq, kk, vv: oracle.linattn_quadratic(qq, kk, vv, eps, threads=1)
    np.testing.assert_allclose(dq, fd_grad(lambda x: fwd(x, k, v), q, dy), rtol=1e-6, atol=1e-8)
    np.testing.assert_allclose(dk, fd_grad(lambda x: fwd(q, x, v), k, dy), rtol=1e-6, atol=1e-8)
    np.testing.assert_allclose(dv_, fd_grad(lambda x: fwd(q, k, x), v, dy), rtol=1e-6, atol=1e-8)


def test_linattn_grad_single_token_closed_form():
    """L = 1: y = v w / (w + eps), w = 1 + u + u^2/2, u = q.k / sqrt(d)."""
    r = rng(3)
    d, dv, eps = 16, 4, 0.3  # a large eps makes the q, k gradients visible
    q, k = r.standard_normal((1, 1, d)), r.standard_normal((1, 1, d))
    v, dy = r.standard_normal((1, 1, dv)), r.standard_normal((1, 1, dv))
    u = float(q[0, 0] @ k[0, 0]) / math.sqrt(d)
    w = 1 + u + u * u / 2
    g = eps / (w + eps) ** 2 * (1 + u) * float(dy[0, 0] @ v[0, 0])  # dL/du
    dq, dk, dv_ = grad.linattn_grad(q, k, v, dy, eps)
    np.testing.assert_allclose(dv_[0, 0], dy[0, 0] * w / (w + eps), rtol=1e-12)
    np.testing.assert_allclose(dq[0, 0], g * k[0, 0] / math.sqrt(d), rtol=1e-12, atol=1e-15)
    np.testing.assert_allclose(dk[0, 0], g * q[0, 0] / math.sqrt(d), rtol=1e-12, atol=1e-15)


@pytest.mark.parametrize("L,dh,W", [(7, 4, 3), (10, 8, 64), (12, 4, 5)])
def test_window_grad_matches_finite_differences(L, dh, W):
    r = rng(L * 100 + W)
    q, k = r.standard_normal((1, L, dh)), r.standard_normal((1, L, dh))
    v, dy = r.standard_normal((1, L, dh)), r.standard_normal((1, L, dh))
    dq, dk, dv = grad.window_grad(q, k, v, dy, W)
    fwd = lambda qq, kk, vv: oracle.window_attn(qq, kk, vv, W, threads=1)
    np.testing.assert_allclose(dq, fd_grad(lambda x: fwd(x, k, v), q, dy), rtol=1e-6, atol=1e-8)
    np.testing.assert_allclose(dk, fd_grad(lambda x: fwd(q, x, v), k, dy), rtol=1e-6, atol=1e-8)
    np.testing.assert_allclose(dv, fd_grad(lambda x: fwd(q, k, x), v, dy), rtol=1e-6, atol=1e-8)


def test_window_grad_window_one_is_identity():
    """W = 1: y_t = v_t, so dv = dy and dq = dk = 0."""
    r = rng(9)
    q, k, v, dy = (r.standard_normal((2, 6, 4)) for _ in range(4))
    dq, dk, dv = grad.window_grad(q, k, v, dy, 1)
    np.testing.assert_array_equal(dv, dy)
    assert np.all(dq == 0) and np.all(dk == 0)


def test_grads_are_per_sequence_over_leading_dims():
    """Leading [B, H] dims are independent sequences: the batched gradient equals
    the gradient of each sequence taken alone."""
    r = rng(21)
    q, k = r.standard_normal((2, 3, 7, 16)) * 0.3, r.standard_normal((2, 3, 7, 16)) * 0.3
    v, dy = r.standard_normal((2, 3, 7, 5)), r.standard_normal((2, 3, 7, 5))
    full = grad.linattn_grad(q, k, v, dy, 1e-6)
    wq, wk, wv, wdy = (r.standard_normal((2, 3, 9, 8)) for _ in range(4))
    wfull = grad.window_grad(wq, wk, wv, wdy, 4)
    for b in range(2):
        for h in range(3):
            one = grad.linattn_grad(q[b, h], k[b, h], v[b, h], dy[b, h], 1e-6)
            wone = grad.window_grad(wq[b, h], wk[b, h], wv[b, h], wdy[b, h], 4)
            for a, e in zip(full, one):
                np.testing.assert_array_equal(a[b, h], e)
            for a, e in zip(wfull, wone):
                np.testing.assert_array_equal(a[b, h], e)
