"""fp64 gradients of the two attention layers -- TEST INFRASTRUCTURE ONLY.

Only ``tests/`` may import this module (it imports nothing from the product).
The "based/train" README lists the training views of the linear attention
(quadratic, fla_parallel, linear); training needs the gradient of the forward
map those views compute.  These routines write that gradient out in plain numpy
float64, one sequence at a time, from the quadratic (masked) form:

  linear attention ("Базированная модель, часть 2", section "Что за линейное
  внимание?"): w_ts = phi(q_t).phi(k_s) = 1 + u + u^2/2 with u = q_t.k_s/sqrt(d)
  for s <= t, N_t = sum_s w_ts v_s, D_t = sum_s w_ts + eps, y_t = N_t / D_t;

  sliding-window softmax attention (Based README, introduction, item 1):
  y_t = sum_{s in [t-W+1, t]} softmax_s(q_t.k_s / sqrt(dh)) v_s.

Given dL/dy these return dL/dq, dL/dk, dL/dv.  Pinned in
``tests/test_oracle_pins_grad.py`` by central finite differences of the C
forward oracle (itself pinned) and by closed forms for L = 1 and W = 1.
"""
from __future__ import annotations

import math

import numpy as np


def _seqs(*arrs):
    """Flatten leading dims: [..., L, x] -> [n, L, x]."""
    lead = arrs[0].shape[:-2]
    n = int(np.prod(lead)) if lead else 1
    return lead, [np.asarray(a, dtype=np.float64).reshape((n,) + a.shape[-2:]) for a in arrs]


def linattn_grad(q, k, v, dy, eps: float = 1e-6):
    """Gradient of the causal Taylor linear attention: (dq, dk, dv)."""
    lead, (q, k, v, dy) = _seqs(q, k, v, dy)
    n, L, d = q.shape
    c = 1.0 / math.sqrt(d)
    mask = np.tril(np.ones((L, L)))
    dq, dk, dv = np.zeros_like(q), np.zeros_like(k), np.zeros_like(v)
    for i in range(n):
        u = (q[i] @ k[i].T) * c                          # [t, s]
        w = (1.0 + u + 0.5 * u * u) * mask
        num = w @ v[i]                                   # [t, dv]
        den = w.sum(axis=1) + eps                        # [t]
        y = num / den[:, None]
        dnum = dy[i] / den[:, None]                      # dL/dN_t
        dden = -(dy[i] * y).sum(axis=1) / den            # dL/dD_t
        dw = (dnum @ v[i].T + dden[:, None]) * mask      # dL/dw_ts
        dv[i] = w.T @ dnum
        du = dw * (1.0 + u)                              # dw/du = 1 + u
        dq[i] = (du @ k[i]) * c
        dk[i] = (du.T @ q[i]) * c
    return (dq.reshape(lead + dq.shape[-2:]), dk.reshape(lead + dk.shape[-2:]),
            dv.reshape(lead + dv.shape[-2:]))


def window_grad(q, k, v, dy, window: int = 64):
    """Gradient of the causal sliding-window softmax attention: (dq, dk, dv)."""
    lead, (q, k, v, dy) = _seqs(q, k, v, dy)
    n, L, dh = q.shape
    c = 1.0 / math.sqrt(dh)
    t_idx = np.arange(L)[:, None]
    s_idx = np.arange(L)[None, :]
    band = (s_idx <= t_idx) & (s_idx > t_idx - window)
    dq, dk, dv = np.zeros_like(q), np.zeros_like(k), np.zeros_like(v)
    for i in range(n):
        sc = np.where(band, (q[i] @ k[i].T) * c, -np.inf)
        sc = sc - sc.max(axis=1, keepdims=True)
        p = np.exp(sc)
        p /= p.sum(axis=1, keepdims=True)                # softmax over the band
        dv[i] = p.T @ dy[i]
        dp = dy[i] @ v[i].T
        ds = p * (dp - (dp * p).sum(axis=1, keepdims=True))
        dq[i] = (ds @ k[i]) * c
        dk[i] = (ds.T @ q[i]) * c
    return (dq.reshape(lead + dq.shape[-2:]), dk.reshape(lead + dk.shape[-2:]),
            dv.reshape(lead + dv.shape[-2:]))
