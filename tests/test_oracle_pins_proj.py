"""Pins for the oracle's projection and BaseConv routines (test infrastructure).

The per-head projection is fixed by special cases that reduce it to a reshape
(identity and permutation weights), to a closed form (rank-one weights) and to
a library contraction (numpy einsum).  BaseConv is fixed by filters that reduce
the convolution to a product with the current or a shifted input, by a
constant input (where the causal truncation of the first K-1 positions gives
partial sums of the taps), by causality, and by a brute-force loop written
here independently.  A transposed weight, a head/position swap, a wrong tap
index or a missing causal cut breaks at least one of them.
"""
import numpy as np
import pytest

import oracle

ATOL = 1e-12


def rng(seed):
    return np.random.Generator(np.random.PCG64(seed))


# ----------------------------------------------------------------- projections

def test_proj_identity_is_head_split():
    r = rng(1)
    B, L, H, D = 2, 7, 3, 4
    x = r.standard_normal((B, L, H * D))
    y = oracle.proj_heads(x, np.eye(H * D), H)
    for b in range(B):
        for h in range(H):
            for t in range(L):
                assert np.array_equal(y[b, h, t], x[b, t, h * D:(h + 1) * D])


def test_proj_permutation_reorders_features():
    r = rng(2)
    B, L, Dm, H, D = 1, 5, 8, 2, 4
    x = r.standard_normal((B, L, Dm))
    perm = r.permutation(Dm)
    w = np.zeros((H * D, Dm))
    w[np.arange(H * D), perm] = 1.0  # output feature n reads input feature perm[n]
    y = oracle.proj_heads(x, w, H)
    for h in range(H):
        for d in range(D):
            assert np.array_equal(y[0, h, :, d], x[0, :, perm[h * D + d]])


def test_proj_rank_one_closed_form():
    r = rng(3)
    B, L, Dm, H, D = 2, 6, 10, 4, 3
    x = r.standard_normal((B, L, Dm))
    u, v = r.standard_normal(H * D), r.standard_normal(Dm)
    y = oracle.proj_heads(x, np.outer(u, v), H)
    xv = x @ v  # [B, L]
    for h in range(H):
        for d in range(D):
            np.testing.assert_allclose(y[:, h, :, d], xv * u[h * D + d], rtol=1e-12, atol=ATOL)


def test_proj_matches_einsum():
    r = rng(4)
    B, L, Dm, H, D = 3, 9, 16, 4, 8
    x = r.standard_normal((B, L, Dm))
    w = r.standard_normal((H * D, Dm))
    ref = np.einsum("blk,hdk->bhld", x, w.reshape(H, D, Dm))
    np.testing.assert_allclose(oracle.proj_heads(x, w, H), ref, rtol=1e-12, atol=1e-12)


# ----------------------------------------------------------------- BaseConv

def brute_baseconv(x, w, bias, h):
    B, L, D = x.shape
    K = h.shape[1]
    y = np.zeros((B, L, D))
    for b in range(B):
        for t in range(L):
            for c in range(D):
                lin = bias[c]
                for k in range(D):
                    lin += x[b, t, k] * w[c, k]
                conv = 0.0
                for j in range(K):
                    if t - j >= 0:
                        conv += h[c, j] * x[b, t - j, c]
                y[b, t, c] = lin * conv
    return y


def test_baseconv_brute_force():
    r = rng(5)
    B, L, D, K = 2, 7, 5, 3
    x, w = r.standard_normal((B, L, D)), r.standard_normal((D, D))
    bias, h = r.standard_normal(D), r.standard_normal((D, K))
    np.testing.assert_allclose(oracle.baseconv(x, w, bias, h), brute_baseconv(x, w, bias, h),
                               rtol=1e-12, atol=1e-12)


def test_baseconv_identity_filter_squares():
    """h = delta at tap 0, W = I, bias = 0: y = x * x."""
    r = rng(6)
    x = r.standard_normal((2, 6, 4))
    h = np.zeros((4, 3))
    h[:, 0] = 1.0
    y = oracle.baseconv(x, np.eye(4), np.zeros(4), h)
    np.testing.assert_array_equal(y, x * x)


@pytest.mark.parametrize("j", [1, 2, 3])
def test_baseconv_shift_filter(j):
    """h = delta at tap j: y[t] = linear(x[t]) * x[t-j], zero for t < j."""
    r = rng(7 + j)
    B, L, D, K = 1, 8, 3, 4
    x, w, bias = r.standard_normal((B, L, D)), r.standard_normal((D, D)), r.standard_normal(D)
    h = np.zeros((D, K))
    h[:, j] = 1.0
    y = oracle.baseconv(x, w, bias, h)
    lin = x @ w.T + bias
    assert np.all(y[:, :j] == 0.0)
    np.testing.assert_allclose(y[:, j:], lin[:, j:] * x[:, :L - j], rtol=1e-12, atol=ATOL)


def test_baseconv_constant_input_partial_tap_sums():
    """x = 1 everywhere: conv at t is the sum of taps 0..min(K-1, t)."""
    D, K, L = 3, 4, 7
    r = rng(11)
    w, bias, h = r.standard_normal((D, D)), r.standard_normal(D), r.standard_normal((D, K))
    y = oracle.baseconv(np.ones((1, L, D)), w, bias, h)
    lin = w.sum(axis=1) + bias
    for t in range(L):
        taps = h[:, :min(K - 1, t) + 1].sum(axis=1)
        np.testing.assert_allclose(y[0, t], lin * taps, rtol=1e-12, atol=ATOL)


def test_baseconv_causal():
    """Changing x at t0 leaves y before t0 unchanged, and after t0 + K - 1 too."""
    r = rng(12)
    B, L, D, K = 1, 10, 4, 3
    x, w = r.standard_normal((B, L, D)), r.standard_normal((D, D))
    bias, h = r.standard_normal(D), r.standard_normal((D, K))
    t0 = 4
    x2 = x.copy()
    x2[0, t0] += 1.0
    y1, y2 = oracle.baseconv(x, w, bias, h), oracle.baseconv(x2, w, bias, h)
    np.testing.assert_array_equal(y1[0, :t0], y2[0, :t0])
    np.testing.assert_array_equal(y1[0, t0 + K:], y2[0, t0 + K:])
    assert not np.allclose(y1[0, t0], y2[0, t0])
