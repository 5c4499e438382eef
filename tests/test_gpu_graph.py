"""The prefill calls captured in a CUDA graph (as bench.py times them) give
bit-identical results to the same calls launched one by one: the kernels'
programmatic dependent launches keep their ordering inside a graph."""
import pytest
import torch

import linear_attention_lm_b200 as lab
from linear_attention_lm_b200.inputs import WORKLOADS, prefill_inputs

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name,kw", [
    ("bf16", dict(B=2, H=4, Hw=4, L=1000)),
    ("split", dict(B=1, H=2, Hw=2, L=3000)),
    ("f32", dict(B=1, H=2, Hw=2, L=300, dtype="f32")),
])
def test_graph_replay_matches_direct_calls(name, kw):
    dev = torch.device("cuda:0")
    w = WORKLOADS["long_16k"].with_(name=f"graph_{name}", **kw)
    x = prefill_inputs(w, device=dev)
    dt = lab.BASED_BF16 if w.dtype == "bf16" else lab.BASED_F32
    ws_bytes = lab.based_linattn_workspace_bytes(w.B, w.H, w.L, w.d, w.dv, dt)
    ws = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device=dev)

    def outputs():
        return {"y": torch.empty_like(x["v"]), "yw": torch.empty_like(x["wq"]),
                "S": torch.empty((w.B, w.H, 273, w.dv), dtype=torch.float32, device=dev),
                "z": torch.empty((w.B, w.H, 273), dtype=torch.float32, device=dev)}

    def step(o):
        lab.based_linattn_fwd(x["q"], x["k"], x["v"], o["y"], w.eps, o["S"], o["z"],
                              workspace=ws[:ws_bytes] if ws_bytes else None)
        lab.based_window_attn_fwd(x["wq"], x["wk"], x["wv"], o["yw"], w.window)

    direct = outputs()
    step(direct)
    torch.cuda.synchronize()
    replayed = outputs()
    cap = torch.cuda.Stream(device=dev)
    cap.wait_stream(torch.cuda.current_stream(dev))
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=cap):
        step(replayed)
        step(replayed)  # a second step right behind the first, as in the bench
    graph.replay()
    torch.cuda.synchronize()
    assert lab.based_get_device_error() == 0
    for key in direct:
        assert torch.equal(direct[key], replayed[key]), key
