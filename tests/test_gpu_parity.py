"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle on the
same seeded inputs.

Tolerances: bf16 inputs with fp32 accumulation -- relative L2 error <= 5e-3 per
(batch, head) and elementwise |err| <= 2e-2; fp32 inputs -- elementwise
|err| <= 1e-4.  Exported fp32 states: relative L2 <= 5e-3 per (batch, head)
for bf16 runs, 1e-5 for fp32 runs.
"""
import numpy as np
import pytest
import torch

import linear_attention_lm_b200 as lab
import oracle
from linear_attention_lm_b200 import build as lab_build
from linear_attention_lm_b200.inputs import (WORKLOADS, decode_step_inputs, prefill_inputs,
                                              to_f64)

pytestmark = pytest.mark.gpu

REL_BF16, ATOL_BF16, ATOL_F32 = 5e-3, 2e-2, 1e-4


@pytest.fixture(scope="module", autouse=True)
def _lib():
    lab_build.build()
    lab.load_library()
    torch.cuda.set_device(0)


def test_loaded_device_code_is_sm100():
    """The CUDA runtime runs the library's sm_100a device code on this GPU."""
    assert lab.based_binary_version() == 100


def head_rel_l2(y, ref):
    """max over leading (b, h) of ||y - ref|| / ||ref|| over the trailing dims."""
    n = ref.shape[0] * ref.shape[1] if ref.ndim >= 3 else 1
    a = y.reshape(n, -1)
    b = ref.reshape(n, -1)
    num = np.linalg.norm(a - b, axis=1)
    den = np.maximum(np.linalg.norm(b, axis=1), 1e-30)
    return float(np.max(num / den)) if n else 0.0


def check(y_gpu, ref, dtype, what, state=False):
    y = to_f64(y_gpu)
    assert y.shape == ref.shape, (what, y.shape, ref.shape)
    assert np.all(np.isfinite(y)), what
    if y.size == 0:
        return
    err = float(np.max(np.abs(y - ref)))
    rel = head_rel_l2(y, ref)
    if dtype == torch.float32:
        lim = 1e-5 if state else ATOL_F32
        ok = (rel <= lim) if state else (err <= lim)
    else:
        ok = rel <= REL_BF16 and (state or err <= ATOL_BF16)
    assert ok, f"{what}: max|err|={err:.3e} max head relL2={rel:.3e}"


def run_linattn(w, check_state=True):
    dev = torch.device("cuda:0")
    x = prefill_inputs(w, device=dev)
    y, S, z = lab.linattn(x["q"], x["k"], x["v"], w.eps, return_state=True)
    torch.cuda.synchronize()
    assert lab.based_get_device_error() == 0
    q, k, v = to_f64(x["q"]), to_f64(x["k"]), to_f64(x["v"])
    y_ref, S_ref, z_ref = oracle.linattn_recurrent(q, k, v, w.eps, return_state=True)
    check(y, y_ref, w.torch_dtype, f"{w.name} y")
    if check_state:
        check(S, S_ref, w.torch_dtype, f"{w.name} state_kv", state=True)
        check(z, z_ref, w.torch_dtype, f"{w.name} state_k", state=True)


def run_window(w):
    dev = torch.device("cuda:0")
    x = prefill_inputs(w, device=dev)
    y = lab.window_attn(x["wq"], x["wk"], x["wv"], w.window)
    torch.cuda.synchronize()
    ref = oracle.window_attn(to_f64(x["wq"]), to_f64(x["wk"]), to_f64(x["wv"]), w.window)
    check(y, ref, w.torch_dtype, f"{w.name} window")


# --------------------------------------------------------------------------
# linear attention prefill
# --------------------------------------------------------------------------

def test_linattn_tiny_fp32():
    run_linattn(WORKLOADS["tiny_fp32"])


@pytest.mark.parametrize("L", [1, 31, 63, 64, 65, 129, 200])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_linattn_ragged_lengths(L, dtype):
    w = WORKLOADS["long_16k"].with_(B=2, H=2, L=L, dtype=dtype, name=f"ragged{L}")
    run_linattn(w)


@pytest.mark.parametrize("dv", [64, 128])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_linattn_head_dims(dv, dtype):
    w = WORKLOADS["layer_1b3"].with_(B=2, H=3, L=333, dv=dv, dtype=dtype, name=f"dv{dv}")
    run_linattn(w)


@pytest.mark.parametrize("L", [3000, 1025])
def test_linattn_split_segments(L):
    """Few sequences, long L: the prefill splits each sequence into segments
    (state-only pass, running sums of the partials, seeded main pass); ragged
    last chunk, state export."""
    w = WORKLOADS["long_16k"].with_(B=1, H=2, L=L, name=f"split{L}")
    assert lab.based_linattn_workspace_bytes(1, 2, L, 16, 64, lab.BASED_BF16) > 0
    run_linattn(w)


@pytest.mark.parametrize("H,L,dv", [(64, 1024, 64), (20, 1500, 64), (5, 900, 128)])
def test_linattn_split_segment_counts(H, L, dv):
    """Two segments (one partial: no running sum), several segments, and d_v =
    128 split into 64-column slices that are split into segments themselves."""
    w = WORKLOADS["long_16k"].with_(B=1, H=H, L=L, dv=dv, name=f"seg{H}_{L}_{dv}")
    assert lab.based_linattn_workspace_bytes(1, H, L, 16, dv, lab.BASED_BF16) > 0
    run_linattn(w)


def test_linattn_empty_and_state_only():
    dev = torch.device("cuda:0")
    q = torch.empty((2, 2, 0, 16), dtype=torch.bfloat16, device=dev)
    v = torch.empty((2, 2, 0, 64), dtype=torch.bfloat16, device=dev)
    y, S, z = lab.linattn(q, q, v, return_state=True)
    torch.cuda.synchronize()
    assert y.numel() == 0
    assert torch.count_nonzero(S).item() == 0 and torch.count_nonzero(z).item() == 0


@pytest.mark.parametrize("name", ["layer_360m", "layer_1b3", "long_16k"])
def test_linattn_full_workloads(name):
    run_linattn(WORKLOADS[name])


# --------------------------------------------------------------------------
# sliding-window attention prefill
# --------------------------------------------------------------------------

def test_window_tiny_fp32():
    run_window(WORKLOADS["tiny_fp32"])


@pytest.mark.parametrize("L,W", [(1, 64), (40, 64), (64, 64), (65, 64), (200, 64), (200, 7),
                                 (130, 1)])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_window_ragged(L, W, dtype):
    w = WORKLOADS["long_16k"].with_(B=2, Hw=2, L=L, window=W, dtype=dtype, name=f"win{L}_{W}")
    run_window(w)


@pytest.mark.parametrize("dh", [64, 128])
def test_window_head_dims(dh):
    w = WORKLOADS["layer_1b3"].with_(B=1, Hw=3, L=333, dh=dh, name=f"windh{dh}")
    run_window(w)


@pytest.mark.parametrize("dh", [64, 128])
def test_window_fp32_large_blocks(dh):
    """fp32 window on a problem with two 64-query blocks per SM (the small
    fp32 cases above run 16-query blocks); ragged last block."""
    w = WORKLOADS["layer_1b3"].with_(B=2, Hw=16, L=1000, dh=dh, dtype="f32",
                                     name=f"winf32_{dh}")
    run_window(w)


@pytest.mark.parametrize("name", ["layer_360m", "layer_1b3", "long_16k"])
def test_window_full_workloads(name):
    run_window(WORKLOADS[name])


# --------------------------------------------------------------------------
# decode: prefill -> state export + ring fill -> recurrent steps
# --------------------------------------------------------------------------

def run_decode(w, steps, sample):
    dev = torch.device("cuda:0")
    x = prefill_inputs(w, device=dev)
    _, S, z = lab.linattn(x["q"], x["k"], x["v"], w.eps, return_state=True)
    k_ring, v_ring = lab.window_ring_fill(x["wk"], x["wv"], w.window)
    torch.cuda.synchronize()
    # oracle on a sample of sequences (flat (b, h) indices)
    g = np.random.Generator(np.random.PCG64(5))
    lin_idx = np.sort(g.choice(w.B * w.H, size=min(sample, w.B * w.H), replace=False))
    win_idx = np.sort(g.choice(w.B * w.Hw, size=min(sample, w.B * w.Hw), replace=False))

    def pick(t, idx):
        a = to_f64(t)
        return np.ascontiguousarray(a.reshape((-1,) + a.shape[2:])[idx])

    _, S_o, z_o = oracle.linattn_recurrent(pick(x["q"], lin_idx), pick(x["k"], lin_idx),
                                           pick(x["v"], lin_idx), w.eps, return_state=True)
    S_o, z_o = np.ascontiguousarray(S_o), np.ascontiguousarray(z_o)
    check(torch.from_numpy(pick(S, lin_idx)), S_o, torch.bfloat16, "prefill state_kv", state=True)
    # the oracle's ring comes from the prefill inputs, never from the GPU's ring
    kr_o, vr_o = oracle.ring_fill(pick(x["wk"], win_idx), pick(x["wv"], win_idx), w.window)
    out = torch.empty((w.B, w.H, w.dv), dtype=w.torch_dtype, device=dev)
    wout = torch.empty((w.B, w.Hw, w.dh), dtype=w.torch_dtype, device=dev)
    for step in range(steps):
        d = decode_step_inputs(w, step, device=dev)
        lab.based_decode_step(d["q"], d["k"], d["v"], S, z, out, d["wq"], d["wk"], d["wv"],
                              k_ring, v_ring, wout, pos=w.L + step, window=w.window, eps=w.eps)
        o_ref = oracle.decode_linear(pick(d["q"], lin_idx), pick(d["k"], lin_idx),
                                     pick(d["v"], lin_idx), S_o, z_o, w.eps)
        ow_ref = oracle.decode_window(pick(d["wq"], win_idx), pick(d["wk"], win_idx),
                                      pick(d["wv"], win_idx), kr_o, vr_o, w.L + step, w.window)
        check(torch.from_numpy(pick(out, lin_idx)[:, None]), o_ref[:, None], w.torch_dtype,
              f"decode step {step}")
        check(torch.from_numpy(pick(wout, win_idx)[:, None]), ow_ref[:, None], w.torch_dtype,
              f"decode window step {step}")
    assert lab.based_get_device_error() == 0
    check(torch.from_numpy(pick(S, lin_idx)), S_o, torch.bfloat16, "final state_kv", state=True)
    check(torch.from_numpy(pick(z, lin_idx)), z_o, torch.bfloat16, "final state_k", state=True)


@pytest.mark.parametrize("L", [5, 63, 64, 65, 512])
@pytest.mark.parametrize("W", [7, 64])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_ring_fill_bit_exact(L, W, dtype):
    """based_window_ring_fill against the oracle's ring (slot p mod W holds
    position p): bit-exact in the written slots; the other slots keep what the
    caller put there."""
    dev = torch.device("cuda:0")
    w = WORKLOADS["long_16k"].with_(B=2, Hw=3, L=L, window=W, dtype=dtype, name=f"ring{L}_{W}")
    x = prefill_inputs(w, device=dev)
    sentinel = 3.5
    k_ring = torch.full((w.B, w.Hw, W, w.dh), sentinel, dtype=w.torch_dtype, device=dev)
    v_ring = torch.full_like(k_ring, sentinel)
    lab.based_window_ring_fill(x["wk"], x["wv"], k_ring, v_ring, W)
    torch.cuda.synchronize()
    assert lab.based_get_device_error() == 0
    kr_o, vr_o = oracle.ring_fill(to_f64(x["wk"]), to_f64(x["wv"]), W)
    written = sorted({p % W for p in range(max(0, L - W), L)})
    untouched = [s for s in range(W) if s not in written]
    for got, ref in ((k_ring, kr_o), (v_ring, vr_o)):
        g = to_f64(got)
        assert np.array_equal(g[:, :, written], ref[:, :, written])
        assert np.all(g[:, :, untouched] == sentinel)


def test_decode_small_from_short_prefill():
    """Prefill shorter than the window: the ring is partly empty at first."""
    w = WORKLOADS["decode_b128"].with_(B=3, H=2, Hw=2, L=5, steps=80, name="dec_small")
    run_decode(w, steps=80, sample=6)


def test_decode_dv128_fp32():
    w = WORKLOADS["decode_b128"].with_(B=2, H=2, Hw=2, L=70, dv=128, dh=128, dtype="f32",
                                       name="dec_f32")
    run_decode(w, steps=20, sample=4)


def test_decode_full_workload():
    """B=128 x 16 heads, 512-token prefill, 1024 steps; oracle on 32 sampled
    sequences of each part, every step compared."""
    w = WORKLOADS["decode_b128"]
    run_decode(w, steps=w.steps, sample=32)


def test_decode_zero_state_matches_prefill():
    """Decoding from an all-zero state and empty ring reproduces prefill."""
    dev = torch.device("cuda:0")
    w = WORKLOADS["long_16k"].with_(B=2, H=2, Hw=2, L=70, name="dec_zero")
    x = prefill_inputs(w, device=dev)
    y = lab.linattn(x["q"], x["k"], x["v"], w.eps)
    yw = lab.window_attn(x["wq"], x["wk"], x["wv"], w.window)
    S = torch.zeros((2, 2, 273, 64), dtype=torch.float32, device=dev)
    z = torch.zeros((2, 2, 273), dtype=torch.float32, device=dev)
    kr = torch.zeros((2, 2, 64, 64), dtype=torch.bfloat16, device=dev)
    vr = torch.zeros_like(kr)
    ys, yws = [], []
    for t in range(w.L):
        o = torch.empty((2, 2, 64), dtype=torch.bfloat16, device=dev)
        ow = torch.empty_like(o)
        lab.based_decode_step(x["q"][:, :, t].contiguous(), x["k"][:, :, t].contiguous(),
                              x["v"][:, :, t].contiguous(), S, z, o, x["wq"][:, :, t].contiguous(),
                              x["wk"][:, :, t].contiguous(), x["wv"][:, :, t].contiguous(), kr, vr,
                              ow, pos=t, window=w.window, eps=w.eps)
        ys.append(o)
        yws.append(ow)
    torch.cuda.synchronize()
    check(torch.stack(ys, 2), to_f64(y), torch.bfloat16, "decode vs prefill")
    check(torch.stack(yws, 2), to_f64(yw), torch.bfloat16, "decode window vs prefill")


# --------------------------------------------------------------------------
# decode with per-sequence positions (prompts of different lengths)
# --------------------------------------------------------------------------

@pytest.mark.parametrize("W", [64, 7])
def test_decode_per_sequence_positions(W):
    """Window decode for a batch whose sequences start at different positions
    (prefill lengths 5, 63, 64 and 200): each sequence's ring is built by the
    oracle from its own prefill, every step is compared with the oracle
    stepping that sequence at its own position."""
    dev = torch.device("cuda:0")
    lens = [5, 63, 64, 200]
    B, Hw, dh, steps = len(lens), 2, 64, 70
    w = WORKLOADS["decode_b128"].with_(B=B, H=2, Hw=Hw, L=max(lens), window=W, name="dec_ragged")
    x = prefill_inputs(w, device=dev)
    wk, wv = to_f64(x["wk"]), to_f64(x["wv"])
    kr_o = np.zeros((B, Hw, W, dh))
    vr_o = np.zeros_like(kr_o)
    for b, Lb in enumerate(lens):
        kr_o[b], vr_o[b] = oracle.ring_fill(wk[b, :, :Lb], wv[b, :, :Lb], W)
    k_ring = torch.from_numpy(kr_o).to(torch.bfloat16).to(dev)
    v_ring = torch.from_numpy(vr_o).to(torch.bfloat16).to(dev)
    wout = torch.empty((B, Hw, dh), dtype=torch.bfloat16, device=dev)
    for step in range(steps):
        d = decode_step_inputs(w, step, device=dev)
        pos = torch.tensor([Lb + step for Lb in lens], dtype=torch.int64, device=dev)
        lab.based_decode_step(None, None, None, None, None, None, d["wq"], d["wk"], d["wv"],
                              k_ring, v_ring, wout, pos=pos, window=W)
        ref = np.stack([oracle.decode_window(to_f64(d["wq"])[b], to_f64(d["wk"])[b],
                                             to_f64(d["wv"])[b], kr_o[b], vr_o[b],
                                             lens[b] + step, W) for b in range(B)])
        check(wout, ref, torch.bfloat16, f"per-sequence decode step {step}")
    assert lab.based_get_device_error() == 0


def test_decode_positions_equal_match_scalar_entry_point():
    """All positions equal: based_decode_step_at and based_decode_step give
    bit-identical outputs and rings."""
    dev = torch.device("cuda:0")
    w = WORKLOADS["decode_b128"].with_(B=3, H=2, Hw=2, L=90, name="dec_eq")
    x = prefill_inputs(w, device=dev)
    _, S, z = lab.linattn(x["q"], x["k"], x["v"], w.eps, return_state=True)
    kr, vr = lab.window_ring_fill(x["wk"], x["wv"], w.window)
    state = [(S.clone(), z.clone(), kr.clone(), vr.clone()) for _ in range(2)]
    outs = []
    for use_array, (S_, z_, kr_, vr_) in zip((False, True), state):
        o = torch.empty((3, 2, 64), dtype=torch.bfloat16, device=dev)
        wo = torch.empty_like(o)
        for step in range(5):
            d = decode_step_inputs(w, step, device=dev)
            pos = w.L + step
            if use_array:
                pos = torch.full((3,), pos, dtype=torch.int64, device=dev)
            lab.based_decode_step(d["q"], d["k"], d["v"], S_, z_, o, d["wq"], d["wk"], d["wv"],
                                  kr_, vr_, wo, pos=pos, window=w.window, eps=w.eps)
        torch.cuda.synchronize()
        outs.append((o, wo, S_, kr_, vr_))
    for a, b in zip(*outs):
        assert torch.equal(a, b)


def test_decode_negative_position_is_refused_on_the_device():
    dev = torch.device("cuda:0")
    B, Hw, W, dh = 2, 2, 64, 64
    ring = torch.randn(B, Hw, W, dh, device=dev).to(torch.bfloat16)
    k_ring, v_ring = ring.clone(), ring.clone()
    wq = torch.randn(B, Hw, dh, device=dev).to(torch.bfloat16)
    wout = torch.full((B, Hw, dh), 7.0, dtype=torch.bfloat16, device=dev)
    pos = torch.tensor([100, -3], dtype=torch.int64, device=dev)
    lab.based_decode_step(None, None, None, None, None, None, wq, wq, wq, k_ring, v_ring, wout,
                          pos=pos, window=W)
    assert lab.based_get_device_error() == 1  # BASED_ERR_INVALID_ARG
    assert torch.equal(k_ring[1], ring[1]) and torch.equal(v_ring[1], ring[1])
    assert torch.all(wout[1] == 7.0)
    assert not torch.equal(k_ring[0], ring[0])  # sequence 0 was served
