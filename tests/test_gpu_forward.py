"""GPU parity of the whole layer (lc_moe_forward) against the oracle, the pins the pages fix on
the GPU (all-zero-expert picks return x exactly), determinism, and the full-size workloads in the
launch configuration the benchmark times (outputs checked on sampled tokens)."""
import numpy as np
import pytest
import torch

import oracle
from mixture_experts_zero_b200 import binding as B

from tests.gpu_util import assert_out_close, make, np_bits, oracle_tokens

pytestmark = pytest.mark.gpu


def forward(d, **kw):
    w = d["w"]
    idx = torch.empty(w.T, w.K, dtype=torch.int32, device="cuda")
    gate = torch.empty(w.T, w.K, dtype=torch.float32, device="cuda")
    counts = torch.zeros(w.E, dtype=torch.int32, device="cuda")
    s = B.Shape(w.T, w.d, w.N, w.Z, w.K, w.I)
    ws = kw.pop("ws", None)
    if ws is None:
        ws = B.new_workspace(s)
    out = B.lc_moe_forward(d["x"], d["wr"], d["bias"], d["w13"], d["w2"], w.K, idx=idx, gate=gate,
                           counts=counts, ws=ws, **kw)
    assert B.lc_moe_read_status(ws) == 0
    return out, idx, gate, counts, ws


@pytest.mark.parametrize("name", ["tiny", "small"])
def test_forward_end_to_end_grid_inputs(cuda_device, name):
    """Grid inputs make the router logits exact, so the GPU's routing must equal the oracle's
    own routing bit for bit, and the output must match the oracle's MoE equation."""
    d = make(name, grid=True)
    w = d["w"]
    out, idx, gate, counts, _ = forward(d)
    ref = oracle.forward(np_bits(d["x"]), np_bits(d["wr"]), d["bias"].cpu().numpy(),
                         np_bits(d["w13"]), np_bits(d["w2"]), w.N, w.Z, w.K)
    np.testing.assert_array_equal(idx.cpu().numpy(), ref["idx"])
    np.testing.assert_array_equal(gate.cpu().numpy().view(np.uint32), ref["gate"].view(np.uint32))
    np.testing.assert_array_equal(counts.cpu().numpy(), ref["counts"])
    assert_out_close(np_bits(out), ref["out_exact"], what="out")


def test_forward_general_inputs_small(cuda_device):
    """N(0,1) activations: routing checked stage-wise (oracle routing of the GPU's logits), the
    output against the oracle's layer evaluated on the GPU's routing."""
    d = make("small")
    w = d["w"]
    out, idx, gate, counts, _ = forward(d)
    logits = B.lc_moe_router_logits(d["x"], d["wr"])
    r_idx, r_gate, r_counts, _ = oracle.route(logits.cpu().numpy(), d["bias"].cpu().numpy(), w.K)
    np.testing.assert_array_equal(idx.cpu().numpy(), r_idx)
    np.testing.assert_array_equal(gate.cpu().numpy().view(np.uint32), r_gate.view(np.uint32))
    np.testing.assert_array_equal(counts.cpu().numpy(), r_counts)
    tokens = np.arange(0, w.T, 7)
    ref = oracle_tokens(np_bits(d["x"]), tokens, r_idx, r_gate, w.N, d["w13"], d["w2"])
    assert_out_close(np_bits(out)[tokens], ref, what="out")


def test_all_zero_expert_picks_return_x_exactly(cuda_device):
    d = make("tiny")
    w = d["w"]
    assert w.Z >= w.K
    d["bias"][w.N:] = 10.0
    out, idx, gate, counts, _ = forward(d)
    assert bool((idx >= w.N).all())
    assert torch.equal(out, d["x"])
    assert int(counts[: w.N].sum()) == 0


def test_gates_sum_to_one(cuda_device):
    d = make("small", experts=False)
    w = d["w"]
    idx, gate = B.lc_moe_route(d["x"], d["wr"], d["bias"], w.K, w.N)
    s = gate.double().sum(1)
    assert float((s - 1).abs().max()) <= w.K * 2.0 ** -24 + 2.0 ** -24


def test_forward_is_deterministic(cuda_device):
    d = make("small")
    a = forward(d)
    b = forward(d, ws=a[4])
    for u, v in zip(a[:4], b[:4]):
        assert torch.equal(u, v)


def test_forward_ragged_token_counts(cuda_device):
    """Token counts that are not multiples of the 128-row tile or the 256-token block."""
    for T in [1, 3, 129, 300]:
        d = make("small", T=T, grid=True)
        w = d["w"]
        out, idx, gate, counts, _ = forward(d)
        ref = oracle.forward(np_bits(d["x"]), np_bits(d["wr"]), d["bias"].cpu().numpy(),
                             np_bits(d["w13"]), np_bits(d["w2"]), w.N, w.Z, w.K)
        np.testing.assert_array_equal(idx.cpu().numpy(), ref["idx"])
        assert_out_close(np_bits(out), ref["out_exact"], what=f"out T={T}")


@pytest.mark.parametrize("name,n_tok", [("decode", 12), ("prefill", 10)])
def test_forward_full_shape_sampled_tokens(cuda_device, name, n_tok):
    """LongCat-Flash shape, grid activations (exact logits): routing of every token equals the
    oracle's routing of the exact logits; sampled tokens' outputs equal the oracle's layer."""
    d = make(name, grid=True)
    w = d["w"]
    out, idx, gate, counts, _ = forward(d)
    logits = B.lc_moe_router_logits(d["x"], d["wr"]).cpu().numpy()
    r_idx, r_gate, r_counts, _ = oracle.route(logits, d["bias"].cpu().numpy(), w.K)
    np.testing.assert_array_equal(idx.cpu().numpy(), r_idx)
    np.testing.assert_array_equal(gate.cpu().numpy().view(np.uint32), r_gate.view(np.uint32))
    np.testing.assert_array_equal(counts.cpu().numpy(), r_counts)
    rng = np.random.default_rng(6)
    tokens = np.sort(rng.choice(w.T, n_tok, replace=False))
    # the sampled tokens' logits are exact: recompute them with the oracle
    z_s = oracle.router_logits(np.ascontiguousarray(np_bits(d["x"])[tokens]), np_bits(d["wr"]))
    np.testing.assert_array_equal(z_s, logits[tokens])
    ref = oracle_tokens(np_bits(d["x"]), tokens, r_idx, r_gate, w.N, d["w13"], d["w2"])
    assert_out_close(np_bits(out)[tokens], ref, what="out")
