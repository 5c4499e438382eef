"""Pins for the fp64 oracle, checked against things other than the oracle.

Each test fixes the oracle to an independent fact: the Taylor identity the
blog post prints (golden fixture), the closed-form kernel
w(q,k) = 1 + q.k/sqrt(d) + (q.k)^2/(2d) used without the feature map at all,
textbook softmax attention (numpy, and torch's CPU scaled_dot_product_attention
as a library routine), invariants that follow from the definition, and
agreement of the three training views (recurrent / quadratic / chunked) the
"based/train" README lists.  A dropped term, a wrong scale, sign or index in
any oracle routine breaks at least one of them.
"""
import math
import os

import numpy as np
import pytest
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
RTOL = 1e-12


def rng(seed):
    return np.random.Generator(np.random.PCG64(seed))


def kernel_w(q, k):
    """Closed form of phi(q).phi(k) (second-order expansion of exp(q.k/sqrt d))."""
    d = q.shape[-1]
    u = float(np.dot(q, k)) / math.sqrt(d)
    return 1.0 + u + 0.5 * u * u


def brute_linattn(q, k, v, eps):
    """y_t = sum_{s<=t} w(q_t,k_s) v_s / (sum_{s<=t} w(q_t,k_s) + eps), no features."""
    L, dv = v.shape
    y = np.zeros((L, dv))
    for t in range(L):
        num = np.zeros(dv)
        den = 0.0
        for s in range(t + 1):
            w = kernel_w(q[t], k[s])
            num += w * v[s]
            den += w
        y[t] = num / (den + eps)
    return y


def assert_close(a, b, rtol=RTOL, atol=0.0):
    a, b = np.asarray(a), np.asarray(b)
    scale = max(1.0, float(np.max(np.abs(b)))) if b.size else 1.0
    err = float(np.max(np.abs(a - b))) if a.size else 0.0
    assert err <= rtol * scale + atol, f"max abs err {err:.3e} (scale {scale:.3e})"


# --------------------------------------------------------------------------
# feature map
# --------------------------------------------------------------------------

def test_golden_taylor_identity():
    """phi(q).phi(k) equals the page's printed expansion at exact points."""
    path = os.path.join(GOLDEN, "taylor_identity.txt")
    rows = [l for l in open(path, encoding="utf-8") if l.strip() and not l.startswith("#")]
    assert len(rows) >= 8
    for line in rows:
        qs, ks, es = line.split("|")
        q = np.array([float(x) for x in qs.split()])
        k = np.array([float(x) for x in ks.split()])
        expect = float(es)
        got = float(np.dot(oracle.phi(q), oracle.phi(k)))
        assert abs(got - expect) <= 1e-14 * max(1.0, expect), (q, k, got, expect)


@pytest.mark.parametrize("d", [1, 2, 3, 5, 16])
def test_phi_closed_form(d):
    r = rng(11 + d)
    for _ in range(50):
        q = r.standard_normal(d) * r.uniform(0.1, 3.0)
        k = r.standard_normal(d) * r.uniform(0.1, 3.0)
        got = float(np.dot(oracle.phi(q), oracle.phi(k)))
        expect = kernel_w(q, k)
        assert abs(got - expect) <= 1e-13 * max(1.0, abs(expect))


def test_phi_structure():
    """Feature count, constant feature, rank-1 symmetric quadratic block."""
    d = 16
    assert oracle.num_features(d) == 273
    f0 = oracle.phi(np.zeros(d))
    assert f0[0] == 1.0 and np.all(f0[1:] == 0.0)
    x = rng(3).standard_normal(d)
    f = oracle.phi(x)
    lin, quad = f[1:1 + d], f[1 + d:].reshape(d, d)
    # linear block is a positive multiple of x; flipping x flips only it
    c = lin / x
    assert np.allclose(c, c[0], rtol=1e-14) and c[0] > 0
    fm = oracle.phi(-x)
    assert np.array_equal(fm[1:1 + d], -lin) and np.array_equal(fm[1 + d:], f[1 + d:])
    # quadratic block: row-major vec of a positive multiple of x x^T
    assert np.allclose(quad, quad.T, rtol=0, atol=1e-15)
    outer = np.outer(x, x)
    ratio = quad / outer
    assert np.allclose(ratio, ratio[0, 0], rtol=1e-13) and ratio[0, 0] > 0
    # with those shapes fixed, the two scales are pinned by the identity
    assert abs(np.dot(f, f) - kernel_w(x, x)) < 1e-12 * kernel_w(x, x)


# --------------------------------------------------------------------------
# causal linear attention
# --------------------------------------------------------------------------

@pytest.mark.parametrize("d,L,dv", [(16, 9, 4), (16, 24, 3), (3, 17, 5), (1, 12, 2)])
def test_linattn_brute_force(d, L, dv):
    r = rng(100 + d * L)
    q = r.standard_normal((L, d)) * 0.5
    k = r.standard_normal((L, d)) * 0.5
    v = r.standard_normal((L, dv))
    eps = 1e-6
    ref = brute_linattn(q, k, v, eps)
    assert_close(oracle.linattn_recurrent(q, k, v, eps), ref)
    assert_close(oracle.linattn_quadratic(q, k, v, eps), ref)
    assert_close(oracle.linattn_chunked(q, k, v, [0, 4, 5, L], eps), ref)


def test_linattn_eps_only_in_denominator():
    r = rng(7)
    q, k = r.standard_normal((6, 16)), r.standard_normal((6, 16))
    v = r.standard_normal((6, 3))
    big = 0.75
    assert_close(oracle.linattn_recurrent(q, k, v, big), brute_linattn(q, k, v, big))


def test_views_agree_ragged_partitions():
    """Recurrent, quadratic and chunked views over several partitions."""
    r = rng(21)
    B, H, L, d, dv = 2, 2, 200, 16, 8
    q = r.standard_normal((B, H, L, d)) * 0.4
    k = r.standard_normal((B, H, L, d)) * 0.4
    v = r.standard_normal((B, H, L, dv))
    y_rec = oracle.linattn_recurrent(q, k, v)
    y_quad = oracle.linattn_quadratic(q, k, v)
    assert_close(y_quad, y_rec)
    parts = [list(range(0, L + 1)), list(range(0, L, 7)) + [L], [0, 64, 128, 192, L], [0, L]]
    cuts = np.sort(r.choice(np.arange(1, L), size=11, replace=False))
    parts.append([0] + cuts.tolist() + [L])
    for b in parts:
        assert_close(oracle.linattn_chunked(q, k, v, b), y_rec)
    with pytest.raises(ValueError):
        oracle.linattn_chunked(q, k, v, [0, 10, 10, L])


def test_state_carry_and_export():
    """Splitting the sequence and carrying (S, z) reproduces one pass; the
    exported state reads out the closed-form kernel sums for any probe."""
    r = rng(33)
    L, d, dv = 150, 16, 6
    q = r.standard_normal((L, d)) * 0.5
    k = r.standard_normal((L, d)) * 0.5
    v = r.standard_normal((L, dv))
    y, S, z = oracle.linattn_recurrent(q, k, v, return_state=True)
    for cut in (1, 63, 64, 65, 149):
        y1, S1, z1 = oracle.linattn_recurrent(q[:cut], k[:cut], v[:cut], return_state=True)
        y2 = oracle.linattn_recurrent(q[cut:], k[cut:], v[cut:], S0=S1, z0=z1)
        assert_close(np.concatenate([y1, y2]), y)
    assert S.shape == (273, dv) and z.shape == (273,)
    assert z[0] == L
    assert_close(S[0], v.sum(0))
    for probe in r.standard_normal((5, d)):
        fp = oracle.phi(probe)
        ws = np.array([kernel_w(probe, k[s]) for s in range(L)])
        assert_close(fp @ z, ws.sum(), rtol=1e-12)
        assert_close(fp @ S, ws @ v, rtol=1e-12)


def test_invariants():
    r = rng(44)
    L, d, dv, eps = 80, 16, 5, 1e-6
    v = r.standard_normal((L, dv))
    cnt = np.arange(1, L + 1)[:, None]
    run_mean = np.cumsum(v, 0) / cnt
    # q = 0: every weight is 1, so y_t is the running mean times den/(den+eps)
    k = r.standard_normal((L, d))
    y = oracle.linattn_recurrent(np.zeros((L, d)), k, v, eps)
    assert_close(y, run_mean * cnt / (cnt + eps))
    # k = 0: likewise, for any q
    q = r.standard_normal((L, d))
    y = oracle.linattn_recurrent(q, np.zeros((L, d)), v, eps)
    assert_close(y, run_mean * cnt / (cnt + eps))
    # L = 1
    q1, k1, v1 = q[:1], k[:1], v[:1]
    w = kernel_w(q1[0], k1[0])
    assert_close(oracle.linattn_recurrent(q1, k1, v1, eps), v1 * w / (w + eps))
    # convex hull: weights are >= 1/2 > 0, so y stays within [min v, max v]
    q, k = r.standard_normal((L, d)) * 2, r.standard_normal((L, d)) * 2
    y = oracle.linattn_recurrent(q, k, v, 0.0)
    lo = np.minimum.accumulate(v, 0)
    hi = np.maximum.accumulate(v, 0)
    assert np.all(y >= lo - 1e-12) and np.all(y <= hi + 1e-12)
    # linear in v
    assert_close(oracle.linattn_recurrent(q, k, 3.0 * v - 1.0, 0.0), 3.0 * y - 1.0)


# --------------------------------------------------------------------------
# sliding-window softmax attention
# --------------------------------------------------------------------------

def brute_window(q, k, v, W):
    L, dh = q.shape
    s = q @ k.T / math.sqrt(dh)
    i, j = np.arange(L)[:, None], np.arange(L)[None, :]
    mask = (j <= i) & (j > i - W)
    s = np.where(mask, s, -np.inf)
    s = s - s.max(1, keepdims=True)
    p = np.exp(s)
    p /= p.sum(1, keepdims=True)
    return p @ v


@pytest.mark.parametrize("L,dh,W", [(1, 8, 64), (50, 16, 64), (130, 8, 64), (130, 8, 5),
                                    (40, 4, 1), (70, 16, 200)])
def test_window_brute_force(L, dh, W):
    r = rng(55 + L + W)
    q, k, v = (r.standard_normal((L, dh)) for _ in range(3))
    y = oracle.window_attn(q, k, v, W)
    assert_close(y, brute_window(q, k, v, W), rtol=1e-13)


def test_window_library_softmax():
    """torch's CPU scaled_dot_product_attention in fp64 as an independent routine."""
    r = rng(66)
    B, H, L, dh, W = 2, 3, 150, 32, 64
    q, k, v = (r.standard_normal((B, H, L, dh)) for _ in range(3))
    y = oracle.window_attn(q, k, v, W)
    i, j = torch.arange(L)[:, None], torch.arange(L)[None, :]
    mask = (j <= i) & (j > i - W)
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q), torch.from_numpy(k), torch.from_numpy(v), attn_mask=mask)
    assert_close(y, ref.numpy(), rtol=1e-12)
    # window >= L is plain causal softmax attention
    y_full = oracle.window_attn(q, k, v, L + 3)
    ref_c = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q), torch.from_numpy(k), torch.from_numpy(v), is_causal=True)
    assert_close(y_full, ref_c.numpy(), rtol=1e-12)
    # window 1 returns v itself
    assert_close(oracle.window_attn(q, k, v, 1), v, rtol=1e-15)


# --------------------------------------------------------------------------
# decode
# --------------------------------------------------------------------------

def test_decode_continues_prefill():
    """prefill(L1) then n one-token steps == one pass over L1 + n tokens, for
    both the linear state and the window ring."""
    r = rng(77)
    n_seq, L1, n, d, dv, dh, W = 3, 100, 40, 16, 8, 16, 64
    L = L1 + n
    q, k = r.standard_normal((n_seq, L, d)) * 0.5, r.standard_normal((n_seq, L, d)) * 0.5
    v = r.standard_normal((n_seq, L, dv))
    wq, wk, wv = (r.standard_normal((n_seq, L, dh)) for _ in range(3))
    y_ref = oracle.linattn_recurrent(q, k, v)
    yw_ref = oracle.window_attn(wq, wk, wv, W)
    _, S, z = oracle.linattn_recurrent(q[:, :L1], k[:, :L1], v[:, :L1], return_state=True)
    S, z = np.ascontiguousarray(S), np.ascontiguousarray(z)
    k_ring, v_ring = oracle.ring_fill(wk[:, :L1], wv[:, :L1], W)
    for t in range(L1, L):
        y = oracle.decode_linear(q[:, t], k[:, t], v[:, t], S, z)
        assert_close(y, y_ref[:, t])
        yw = oracle.decode_window(wq[:, t], wk[:, t], wv[:, t], k_ring, v_ring, t, W)
        assert_close(yw, yw_ref[:, t], rtol=1e-13)


@pytest.mark.parametrize("L1,W", [(5, 64), (63, 64), (64, 64), (65, 64), (200, 7), (9, 7)])
def test_decode_continues_short_and_wrapped_prefill(L1, W):
    """The ring handed over after prefills shorter than, equal to and longer
    than the window (wrapped slots) continues the window exactly."""
    r = rng(100 + L1 + W)
    n_seq, n, dh = 2, 12, 8
    L = L1 + n
    wq, wk, wv = (r.standard_normal((n_seq, L, dh)) for _ in range(3))
    yw_ref = oracle.window_attn(wq, wk, wv, W)
    k_ring, v_ring = oracle.ring_fill(wk[:, :L1], wv[:, :L1], W)
    for t in range(L1, L):
        yw = oracle.decode_window(wq[:, t], wk[:, t], wv[:, t], k_ring, v_ring, t, W)
        assert_close(yw, yw_ref[:, t], rtol=1e-13)


def test_ring_fill_slots():
    """Slot p mod W holds position p of the last W positions; the rest is zero."""
    k = np.arange(1.0, 11.0).reshape(1, 10, 1)
    kr, vr = oracle.ring_fill(k, -k, 4)
    # positions 6..9 -> slots 2, 3, 0, 1
    assert kr[0, :, 0].tolist() == [9.0, 10.0, 7.0, 8.0]
    assert vr[0, :, 0].tolist() == [-9.0, -10.0, -7.0, -8.0]
    kr, _ = oracle.ring_fill(k[:, :3], k[:, :3], 8)
    assert kr[0, :, 0].tolist() == [1.0, 2.0, 3.0, 0, 0, 0, 0, 0]


def test_decode_from_empty():
    """Decoding from a zero state and empty ring equals the prefill views."""
    r = rng(88)
    n_seq, L, d, dv, dh, W = 2, 70, 16, 4, 8, 64
    q, k = r.standard_normal((n_seq, L, d)), r.standard_normal((n_seq, L, d))
    v = r.standard_normal((n_seq, L, dv))
    wq, wk, wv = (r.standard_normal((n_seq, L, dh)) for _ in range(3))
    S = np.zeros((n_seq, 273, dv))
    z = np.zeros((n_seq, 273))
    kr, vr = np.zeros((n_seq, W, dh)), np.zeros((n_seq, W, dh))
    y_ref = oracle.linattn_quadratic(q, k, v)
    yw_ref = oracle.window_attn(wq, wk, wv, W)
    for t in range(L):
        assert_close(oracle.decode_linear(q[:, t], k[:, t], v[:, t], S, z), y_ref[:, t])
        assert_close(oracle.decode_window(wq[:, t], wk[:, t], wv[:, t], kr, vr, t, W),
                     yw_ref[:, t], rtol=1e-13)
