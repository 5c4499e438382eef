"""GPU parity of the attention gradients (based_linattn_bwd,
based_window_attn_bwd) against the fp64 gradient oracle (oracle/grad.py) on
the same seeded inputs.

fp32 inputs are computed in fp32 on CUDA cores: the per-(b, h) relative L2
error is bounded by fp32 accumulation over at most L terms, 2e-4 here.  bf16
inputs run on the tensor cores.  The linear attention's gradient takes bf16
operands for three intermediates (w, e = dw (1 + u'), dN): each rounding is at
most 2^-9 relative, a product term carries at most two of them, and the terms
of each sum are independent, so the relative L2 error of a gradient is about
2 x 2^-9 / sqrt(3) ~ 2.3e-3 for terms of random sign; 1e-2 leaves room for the
partial cancellation in dq and dk (their terms sum to nearly zero for every
query).  The window attention's gradient rounds P (for dv) and dS (for dq, dk)
to bf16, one rounding per term: about 2^-9 / sqrt(3) ~ 1.1e-3, with the same
cancellation in dq and dk (each row of dS sums to zero); the same 1e-2 bound.
"""
import numpy as np
import pytest
import torch

import linear_attention_lm_b200 as lab
from linear_attention_lm_b200 import build as lab_build
from oracle import grad

pytestmark = pytest.mark.gpu
REL = 2e-4
REL_LIN_BF16 = 1e-2  # linear attention, bf16 inputs, tensor-core path
REL_WIN_BF16 = 1e-2  # window attention, bf16 inputs, tensor-core path


def lin_rel(dtype):
    return REL_LIN_BF16 if dtype == torch.bfloat16 else REL


@pytest.fixture(scope="module", autouse=True)
def _lib():
    lab_build.build()
    lab.load_library()
    torch.cuda.set_device(0)


def head_rel_l2(y, ref):
    n = ref.shape[0] * ref.shape[1]
    a, b = y.reshape(n, -1), ref.reshape(n, -1)
    return float(np.max(np.linalg.norm(a - b, axis=1) / np.maximum(np.linalg.norm(b, axis=1), 1e-30)))


def make(seed, B, H, L, dv, dtype):
    r = np.random.Generator(np.random.PCG64(seed))
    q = r.standard_normal((B, H, L, 16)) * 0.25
    k = r.standard_normal((B, H, L, 16)) * 0.25
    v = r.standard_normal((B, H, L, dv))
    dy = r.standard_normal((B, H, L, dv))
    ts = [torch.from_numpy(a).to(dtype) for a in (q, k, v, dy)]
    return ts, [t.double().numpy() for t in ts]


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("B,H,L,dv,eps", [
    (1, 2, 100, 64, 1e-6),    # two query tiles, ragged tail
    (2, 1, 130, 128, 1e-6),   # three tiles, d_v = 128
    # a single token: q and k reach y only through eps (their gradient is
    # eps/(w+eps)^2 times O(1)), so a large eps keeps it above fp32 rounding
    (1, 1, 1, 64, 0.5),
    (1, 3, 64, 64, 1e-6),     # exactly one tile
    (1, 1, 257, 64, 1e-6),    # five tiles, one row in the last
])
def test_linattn_grad_matches_oracle(B, H, L, dv, eps, dtype):
    (q, k, v, dy), (q64, k64, v64, dy64) = make(L * 7 + dv, B, H, L, dv, dtype)
    dq, dk, dvv = lab.linattn_grad(q.cuda(), k.cuda(), v.cuda(), dy.cuda(), eps)
    torch.cuda.synchronize()
    assert lab.based_get_device_error() == 0
    rq, rk, rv = grad.linattn_grad(q64, k64, v64, dy64, eps)
    errs = [head_rel_l2(g.double().cpu().numpy(), r) for g, r in ((dq, rq), (dk, rk), (dvv, rv))]
    print(f"linattn grad {dtype} B={B} H={H} L={L} dv={dv}: rel L2 dq {errs[0]:.2e} "
          f"dk {errs[1]:.2e} dv {errs[2]:.2e}")
    assert max(errs) <= lin_rel(dtype), errs


def test_linattn_grad_layer_shape_sampled():
    """layer_360m's linear-attention shape (B=8, H=16, L=2048, d_v=64): the
    gradient is per sequence, so the oracle checks three whole sequences."""
    B, H, L, dv = 8, 16, 2048, 64
    (q, k, v, dy), _ = make(5, B, H, L, dv, torch.bfloat16)
    dq, dk, dvv = lab.linattn_grad(q.cuda(), k.cuda(), v.cuda(), dy.cuda(), 1e-6)
    torch.cuda.synchronize()
    assert lab.based_get_device_error() == 0
    for b, h in ((0, 0), (3, 7), (7, 15)):
        sl = (slice(b, b + 1), slice(h, h + 1))
        rq, rk, rv = grad.linattn_grad(*(t[sl].double().numpy() for t in (q, k, v, dy)), 1e-6)
        errs = [head_rel_l2(g[sl].double().cpu().numpy(), r)
                for g, r in ((dq, rq), (dk, rk), (dvv, rv))]
        print(f"linattn grad layer_360m ({b}, {h}): rel L2 dq {errs[0]:.2e} dk {errs[1]:.2e} "
              f"dv {errs[2]:.2e}")
        assert max(errs) <= REL_LIN_BF16, errs


# ------------------------------------------------------------------ window attention

@pytest.mark.parametrize("dtype,dh", [(torch.bfloat16, 64), (torch.float32, 64),
                                      (torch.bfloat16, 128)])
@pytest.mark.parametrize("B,H,L,W", [
    (1, 2, 100, 64),    # one query tile, ragged tail
    (2, 1, 200, 7),     # a short window
    (1, 1, 1, 64),      # a single token (dq = dk = 0)
    (1, 3, 64, 64),     # half a tile
    (1, 1, 257, 1),     # window of one: dv = dy, dq = dk = 0; three tiles
    (1, 1, 130, 33),
    (1, 2, 384, 64),    # three whole tiles: bands crossing tile edges
])
def test_window_grad_matches_oracle(B, H, L, W, dtype, dh):
    r = np.random.Generator(np.random.PCG64(L * 11 + W + dh))
    ts = [torch.from_numpy(r.standard_normal((B, H, L, dh))).to(dtype) for _ in range(4)]
    q, k, v, dy = ts
    dq, dk, dv = lab.window_grad(q.cuda(), k.cuda(), v.cuda(), dy.cuda(), W)
    torch.cuda.synchronize()
    assert lab.based_get_device_error() == 0
    rq, rk, rv = grad.window_grad(*(t.double().numpy() for t in ts), W)
    tol = REL_WIN_BF16 if dtype == torch.bfloat16 else REL
    for got, ref in ((dq, rq), (dk, rk), (dv, rv)):
        got = got.double().cpu().numpy()
        scale = max(float(np.linalg.norm(ref)), 1.0)  # dq = dk = 0 exactly for W = 1 or L = 1
        assert float(np.linalg.norm(got - ref)) <= tol * scale
        if np.linalg.norm(ref) > 0:
            assert head_rel_l2(got, ref) <= tol


def test_window_grad_layer_shape_sampled():
    """layer_360m's window shape (B=8, H=16, L=2048, d_h=64, W=64): three
    whole sequences against the oracle."""
    B, H, L = 8, 16, 2048
    r = np.random.Generator(np.random.PCG64(17))
    ts = [torch.from_numpy(r.standard_normal((B, H, L, 64))).to(torch.bfloat16) for _ in range(4)]
    dq, dk, dv = lab.window_grad(*(t.cuda() for t in ts), 64)
    torch.cuda.synchronize()
    assert lab.based_get_device_error() == 0
    for b, h in ((0, 0), (4, 9), (7, 15)):
        sl = (slice(b, b + 1), slice(h, h + 1))
        rq, rk, rv = grad.window_grad(*(t[sl].double().numpy() for t in ts), 64)
        assert head_rel_l2(dq[sl].double().cpu().numpy(), rq) <= REL_WIN_BF16
        assert head_rel_l2(dk[sl].double().cpu().numpy(), rk) <= REL_WIN_BF16
        assert head_rel_l2(dv[sl].double().cpu().numpy(), rv) <= REL_WIN_BF16
