"""The failure path of the bounded waits, run on the GPU without a fault.

Every mbarrier wait in the tensor-core kernels gives up after a time limit;
the kernel then records BASED_ERR_TIMEOUT in the library's status word, waits
(again bounded) for its own loads and stores in flight, releases its tensor
memory and returns.  The test hook based_debug_stall makes the first CTA of
one kernel leave one input load out and shortens the limit to 1 ms, so that
exactly this path runs: nothing faults, traps or hangs.  Each test first
checks a clean call, then the stalled call (BASED_ERR_TIMEOUT reported), then
a clean call again (status OK, same output as before, parity with the
oracle), so the context stays usable after the timeout.
"""
import numpy as np
import pytest
import torch

import linear_attention_lm_b200 as lab
import oracle
from linear_attention_lm_b200 import build as lab_build
from linear_attention_lm_b200.inputs import WORKLOADS, prefill_inputs, to_f64

pytestmark = pytest.mark.gpu

LIMIT_NS = 1_000_000      # 1 ms
DEFAULT_NS = 2_000_000_000
TIMEOUT = 4


@pytest.fixture(scope="module", autouse=True)
def _lib():
    lab_build.build()
    lab.load_library()
    torch.cuda.set_device(0)
    yield
    lab.based_debug_stall(lab.STALL_NONE, DEFAULT_NS)


def rel_l2(a, b):
    n = b.shape[0] * b.shape[1]
    a2, b2 = a.reshape(n, -1), b.reshape(n, -1)
    return float(np.max(np.linalg.norm(a2 - b2, axis=1) / np.linalg.norm(b2, axis=1)))


def stalled(which, fn):
    lab.based_debug_stall(which, LIMIT_NS)
    try:
        out = fn()
        status = lab.based_get_device_error()
    finally:
        lab.based_debug_stall(lab.STALL_NONE, DEFAULT_NS)
    return out, status


def test_linattn_wait_runs_out_then_recovers():
    dev = torch.device("cuda:0")
    # 128 sequences: one CTA each (no split), four 128-token chunks per CTA
    w = WORKLOADS["layer_360m"].with_(L=512, name="stall_lin")
    x = prefill_inputs(w, device=dev)

    def run():
        y, S, z = lab.linattn(x["q"], x["k"], x["v"], w.eps, return_state=True)
        torch.cuda.synchronize()
        return y

    y_clean = run()
    assert lab.based_get_device_error() == 0
    _, status = stalled(lab.STALL_LINATTN_V, run)
    assert status == TIMEOUT
    assert lab.based_get_device_error() == 0  # read and cleared
    y_again = run()
    assert lab.based_get_device_error() == 0
    assert torch.equal(y_again, y_clean)
    idx = slice(0, 4)  # the oracle on the first four sequences (those of the stalled CTA)
    ref = oracle.linattn_recurrent(to_f64(x["q"])[0, idx], to_f64(x["k"])[0, idx],
                                   to_f64(x["v"])[0, idx], w.eps)
    assert rel_l2(to_f64(y_again)[0, idx][None], ref[None]) <= 5e-3


def test_window_wait_runs_out_then_recovers():
    dev = torch.device("cuda:0")
    w = WORKLOADS["layer_360m"].with_(L=512, name="stall_win")
    x = prefill_inputs(w, device=dev)

    def run():
        y = lab.window_attn(x["wq"], x["wk"], x["wv"], w.window)
        torch.cuda.synchronize()
        return y

    y_clean = run()
    assert lab.based_get_device_error() == 0
    _, status = stalled(lab.STALL_WINDOW_V, run)
    assert status == TIMEOUT
    assert lab.based_get_device_error() == 0
    y_again = run()
    assert lab.based_get_device_error() == 0
    assert torch.equal(y_again, y_clean)
    idx = slice(0, 4)
    ref = oracle.window_attn(to_f64(x["wq"])[0, idx], to_f64(x["wk"])[0, idx],
                             to_f64(x["wv"])[0, idx], w.window)
    assert rel_l2(to_f64(y_again)[0, idx][None], ref[None]) <= 5e-3


def test_stall_hook_rejects_bad_arguments():
    with pytest.raises(lab.BasedError):
        lab.based_debug_stall(7, LIMIT_NS)
    with pytest.raises(lab.BasedError):
        lab.based_debug_stall(lab.STALL_NONE, 0)
