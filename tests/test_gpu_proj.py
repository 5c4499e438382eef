"""GPU parity for the projection kernels (per-head input projection and
BaseConv) through the C ABI, against the fp64 oracle on the same seeded inputs.

Both kernels take bf16 operands, accumulate in fp32 and round once to bf16, so
each output element must match the oracle (fp64 on the same bf16 inputs) to
within one bf16 rounding: |err| <= 2^-8 |ref| + 1e-4 * rms(ref) (the absolute
term covers fp32 accumulation-order differences where the result is near 0).
"""
import numpy as np
import pytest
import torch

import linear_attention_lm_b200 as lab
import oracle
from linear_attention_lm_b200 import build as lab_build

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    lab_build.build()
    lab.load_library()
    torch.cuda.set_device(0)


def gen(seed, shape, scale=1.0):
    """Seeded N(0, scale^2) values rounded to bf16 (returned as a bf16 torch tensor)."""
    r = np.random.Generator(np.random.PCG64(seed))
    a = r.standard_normal(shape) * scale
    return torch.from_numpy(a).to(torch.bfloat16)


def f64(t):
    return t.double().cpu().numpy()


def check_close(y, ref):
    y, ref = f64(y) if torch.is_tensor(y) else y, ref
    rms = float(np.sqrt(np.mean(ref * ref))) if ref.size else 0.0
    err = np.abs(y - ref)
    bound = 2.0 ** -8 * np.abs(ref) + 1e-4 * rms
    worst = float(np.max(err - bound)) if ref.size else 0.0
    assert worst <= 0.0, f"max excess {worst:.3e} (rms {rms:.3e})"


# ------------------------------------------------------------------ projection

@pytest.mark.parametrize("B,L,d_model,H,D", [
    (1, 200, 256, 16, 16),    # one N tile, ragged M tail
    (2, 130, 1024, 16, 64),   # four N tiles, rows of two sequences in one M tile
    (1, 64, 512, 32, 8),      # D = 8, a tile shorter than 128 rows
    (3, 257, 192, 4, 64),     # three K blocks
])
def test_proj_heads_matches_oracle(B, L, d_model, H, D):
    x = gen(100 + L, (B, L, d_model))
    w = gen(200 + d_model, (H * D, d_model), 0.02)
    y = lab.proj_heads(x.cuda(), w.cuda(), H)
    torch.cuda.synchronize()
    assert lab.based_get_device_error() == 0
    check_close(y, oracle.proj_heads(f64(x), f64(w), H))


def test_proj_heads_full_size_sampled():
    """layer_360m's q/k (16 heads of 16) and v (16 heads of 64) projections,
    B=8, L=2048, d_model=1024: every token of every head on two sequences and a
    ragged time slice of the others (the projection is per token)."""
    B, L, dm, H = 8, 2048, 1024, 16
    x = gen(7, (B, L, dm))
    xd = x.cuda()
    for D, seed in ((16, 8), (64, 9)):
        w = gen(seed, (H * D, dm), 0.02)
        y = lab.proj_heads(xd, w.cuda(), H).cpu()
        torch.cuda.synchronize()
        wd = f64(w)
        for b in (0, 5):
            check_close(y[b:b + 1], oracle.proj_heads(f64(x[b:b + 1]), wd, H))
        t0, t1 = 1000, 1131
        check_close(y[:, :, t0:t1], oracle.proj_heads(f64(x[:, t0:t1]), wd, H))
    assert lab.based_get_device_error() == 0


@pytest.mark.parametrize("B,L,d_model,H,Ds", [
    (1, 100, 256, 16, (16, 16, 64, 64, 64, 64)),  # one pair tile, the odd CTA's rows all past M
    (3, 257, 192, 32, (8, 64)),                    # ragged M over several pair tiles
    (2, 300, 1024, 16, (64, 16, 64, 16)),          # projections of different widths interleaved
    (2, 384, 256, 32, (8, 32, 128)),               # rows in whole 128-row blocks of a sequence
                                                   # leave by TMA: boxes 16, 64 and 2 x 128
                                                   # bytes wide (no swizzle, 64B, 128B)
])
def test_proj_heads_multi_matches_oracle(B, L, d_model, H, Ds):
    """Every output of one multi-projection launch against the oracle's
    projection with that output's rows of the stacked weights."""
    x = gen(600 + L, (B, L, d_model))
    w = gen(700 + d_model, (H * sum(Ds), d_model), 0.02)
    ys = lab.proj_heads_multi(x.cuda(), w.cuda(), H, Ds)
    torch.cuda.synchronize()
    assert lab.based_get_device_error() == 0
    off = 0
    for D, y in zip(Ds, ys):
        check_close(y, oracle.proj_heads(f64(x), f64(w[off:off + H * D]), H))
        off += H * D


def test_proj_heads_multi_full_size_sampled():
    """layer_360m's six projections (q, k: 16 heads of 16; v and the window
    layer's q, k, v: 16 heads of 64) of x [8, 2048, 1024] in one launch, checked
    on two whole sequences and a ragged time slice of all of them."""
    B, L, dm, H = 8, 2048, 1024, 16
    Ds = (16, 16, 64, 64, 64, 64)
    x = gen(21, (B, L, dm))
    w = gen(22, (H * sum(Ds), dm), 0.02)
    ys = [y.cpu() for y in lab.proj_heads_multi(x.cuda(), w.cuda(), H, Ds)]
    torch.cuda.synchronize()
    assert lab.based_get_device_error() == 0
    off = 0
    for D, y in zip(Ds, ys):
        wd = f64(w[off:off + H * D])
        for b in (2, 7):
            check_close(y[b:b + 1], oracle.proj_heads(f64(x[b:b + 1]), wd, H))
        check_close(y[:, :, 1500:1533], oracle.proj_heads(f64(x[:, 1500:1533]), wd, H))
        off += H * D


# ------------------------------------------------------------------ BaseConv

@pytest.mark.parametrize("B,L,D,K", [
    (2, 150, 256, 3),    # ragged M, a tile holding the end and start of two sequences
    (1, 300, 512, 4),
    (3, 37, 256, 1),     # K = 1: linear(x) * h[:, 0] * x
    (1, 200, 256, 8),    # the most taps
    (4, 3, 256, 4),      # sequences shorter than the filter
])
def test_baseconv_matches_oracle(B, L, D, K):
    x = gen(300 + L, (B, L, D))
    w = gen(400 + D, (D, D), 0.03)
    r = np.random.Generator(np.random.PCG64(500 + K))
    bias = torch.from_numpy(r.standard_normal(D) * 0.1).float()
    taps = torch.from_numpy(r.standard_normal((D, K)) * 0.5).float()
    y = lab.baseconv(x.cuda(), w.cuda(), bias.cuda(), taps.cuda())
    torch.cuda.synchronize()
    assert lab.based_get_device_error() == 0
    check_close(y, oracle.baseconv(f64(x), f64(w), bias.double().numpy(), taps.double().numpy()))


def test_baseconv_full_size_sampled():
    """B=8, L=2048, D=1024, K=3 (layer_360m width): one whole sequence, and a
    time slice of every sequence (the oracle runs on the slice plus the K-1
    rows before it, whose own outputs are dropped)."""
    B, L, D, K = 8, 2048, 1024, 3
    x = gen(11, (B, L, D))
    w = gen(12, (D, D), 0.03)
    r = np.random.Generator(np.random.PCG64(13))
    bias = torch.from_numpy(r.standard_normal(D) * 0.1).float()
    taps = torch.from_numpy(r.standard_normal((D, K)) * 0.5).float()
    y = lab.baseconv(x.cuda(), w.cuda(), bias.cuda(), taps.cuda()).cpu()
    torch.cuda.synchronize()
    assert lab.based_get_device_error() == 0
    wd, bd, hd = f64(w), bias.double().numpy(), taps.double().numpy()
    check_close(y[3:4], oracle.baseconv(f64(x[3:4]), wd, bd, hd))
    t0, t1 = 777, 900
    ref = oracle.baseconv(f64(x[:, t0 - (K - 1):t1]), wd, bd, hd)[:, K - 1:]
    check_close(y[:, t0:t1], ref)
