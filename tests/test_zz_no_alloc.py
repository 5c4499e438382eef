"""The allocation-free linear-attention prefill, based_linattn_fwd_noalloc.

Some callers cannot allocate device memory at all -- a plugin whose host
framework owns every allocation, or a latency-critical loop that cannot
afford cudaMalloc's device synchronisation -- so they cannot hand
based_linattn_fwd the workspace it asks for when it splits long sequences
across CTAs.  The no-alloc entry point takes its scratch from a fixed array
inside the library instead.  This test calls it through the C ABI on problems
that do need scratch and checks it against based_linattn_fwd with a
workspace, on two calls in a row (the second reuses the array the first left
behind).  It lives in its own file so that pytest collects it last, and it
sets up everything it needs so that it also passes alone in a fresh process.
"""
import numpy as np
import pytest
import torch

import linear_attention_lm_b200 as lab
from linear_attention_lm_b200 import build as lab_build
from linear_attention_lm_b200.inputs import WORKLOADS, prefill_inputs, to_f64

pytestmark = pytest.mark.gpu

REL_BF16, ATOL_BF16 = 5e-3, 2e-2


def head_rel_l2(a, b):
    n = b.shape[0] * b.shape[1]
    a2, b2 = a.reshape(n, -1), b.reshape(n, -1)
    return float(np.max(np.linalg.norm(a2 - b2, axis=1) /
                        np.maximum(np.linalg.norm(b2, axis=1), 1e-30)))


def test_noalloc_matches_workspace_entry_point():
    lab_build.build()
    lab.load_library()
    torch.cuda.set_device(0)
    dev = torch.device("cuda:0")
    # calls in a row with different problems; all split into segments, the
    # last one with d_v = 128 (the other tensor-core layout)
    cases = [WORKLOADS["long_16k"].with_(B=1, H=2, L=3000, name="noalloc_a"),
             WORKLOADS["long_16k"].with_(B=2, H=1, L=2100, wid=7, name="noalloc_b"),
             WORKLOADS["long_16k"].with_(B=1, H=3, L=2500, dv=128, wid=8, name="noalloc_c")]
    for w in cases:
        need = lab.based_linattn_workspace_bytes(w.B, w.H, w.L, w.d, w.dv, lab.BASED_BF16)
        assert need > 0, "the case must exercise the scratch path"
        x = prefill_inputs(w, device=dev)
        shape_s = (w.B, w.H, lab.NUM_FEATURES, w.dv)
        y_ref = torch.empty_like(x["v"])
        S_ref = torch.empty(shape_s, dtype=torch.float32, device=dev)
        z_ref = torch.empty(shape_s[:3], dtype=torch.float32, device=dev)
        ws = torch.empty(need, dtype=torch.uint8, device=dev)
        lab.based_linattn_fwd(x["q"], x["k"], x["v"], y_ref, w.eps, S_ref, z_ref, workspace=ws)
        y = torch.full_like(x["v"], float("nan"))
        S = torch.full(shape_s, float("nan"), dtype=torch.float32, device=dev)
        z = torch.full(shape_s[:3], float("nan"), dtype=torch.float32, device=dev)
        lab.based_linattn_fwd_noalloc(x["q"], x["k"], x["v"], y, w.eps, S, z)
        torch.cuda.synchronize()
        assert lab.based_get_device_error() == 0
        a, b = to_f64(y), to_f64(y_ref)
        assert np.all(np.isfinite(a))
        assert head_rel_l2(a, b) <= REL_BF16 and float(np.max(np.abs(a - b))) <= ATOL_BF16
        for got, ref in ((S, S_ref), (z, z_ref)):
            g, r = to_f64(got), to_f64(ref)
            assert np.all(np.isfinite(g)) and head_rel_l2(g, r) <= REL_BF16


def test_noalloc_scratch_covers_every_split():
    """The scratch array (16 MiB) covers the largest workspace any problem
    asks for on this GPU: the split keeps (segments - 1) x sequences at most
    one per SM, so the need peaks near SMs x 160 x 80 x 4 bytes (every d_v runs
    as 64-column slices).
    Sizes beyond the array would be refused with BASED_ERR_WORKSPACE before
    any launch; none is reachable here."""
    lab_build.build()
    lab.load_library()
    torch.cuda.set_device(0)
    worst = 0
    for dv in (64, 128):
        for BH in (1, 2, 3, 5, 16, 37, 74):
            for L in (1024, 4096, 65536, 1 << 20):
                worst = max(worst, lab.based_linattn_workspace_bytes(1, BH, L, 16, dv,
                                                                     lab.BASED_BF16))
    assert 0 < worst <= 16 << 20
