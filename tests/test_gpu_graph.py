"""The layer inside a CUDA graph: lc_moe_forward and lc_moe_bias_update only enqueue work on the
caller's stream (no host synchronisation, no allocation, all state in caller-owned buffers), so
one control step can be captured once and replayed. Replays must give, bit for bit, what the same
sequence of eager calls gives (the routing and the bias update are deterministic, the combine
sums in a fixed order)."""
import pytest
import torch

from mixture_experts_zero_b200 import binding as B

from tests.gpu_util import make

pytestmark = pytest.mark.gpu


def steps(d, bias, counts, out, ws, n, stream=None):
    w = d["w"]
    outs = []
    for _ in range(n):
        B.lc_moe_forward(d["x"], d["wr"], bias, d["w13"], d["w2"], w.K, out=out, counts=counts, ws=ws,
                         stream=stream)
        B.lc_moe_bias_update(bias, counts, w.T, w.N, w.Z, w.K, w.K_e, 0.05, reset_counts=True,
                             stream=stream)
        outs.append(out.clone())
    return outs


@pytest.mark.parametrize("name", ["tiny", "small"])
def test_captured_control_step_replays_like_eager_calls(cuda_device, name):
    d = make(name)
    w = d["w"]
    s = B.Shape(w.T, w.d, w.N, w.Z, w.K, w.I)
    bias0 = d["bias"].clone()

    # eager reference: three control steps
    bias_e = bias0.clone()
    counts_e = torch.zeros(w.E, dtype=torch.int32, device="cuda")
    out_e = torch.empty(w.T, w.d, dtype=torch.bfloat16, device="cuda")
    ws_e = B.new_workspace(s)
    ref = steps(d, bias_e, counts_e, out_e, ws_e, 3)

    # captured: one control step in a graph, replayed three times
    bias_g = bias0.clone()
    counts_g = torch.zeros(w.E, dtype=torch.int32, device="cuda")
    out_g = torch.empty(w.T, w.d, dtype=torch.bfloat16, device="cuda")
    ws_g = B.new_workspace(s)
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):  # first use (library setup) outside the capture, then restore
        steps(d, bias_g, counts_g, out_g, ws_g, 1, stream=side)
    torch.cuda.current_stream().wait_stream(side)
    bias_g.copy_(bias0)
    counts_g.zero_()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        stream = torch.cuda.current_stream()
        B.lc_moe_forward(d["x"], d["wr"], bias_g, d["w13"], d["w2"], w.K, out=out_g, counts=counts_g,
                         ws=ws_g, stream=stream)
        B.lc_moe_bias_update(bias_g, counts_g, w.T, w.N, w.Z, w.K, w.K_e, 0.05, reset_counts=True,
                             stream=stream)
    got = []
    for _ in range(3):
        graph.replay()
        got.append(out_g.clone())
    torch.cuda.synchronize()
    assert B.lc_moe_read_status(ws_g) == 0
    for a, b in zip(got, ref):
        assert torch.equal(a, b)
    assert torch.equal(bias_g, bias_e)
    assert not torch.equal(bias_g, bias0)  # the control moved the biases between replays
    del graph
