"""GPU parity of the routing steps: router GEMM (tcgen05), softmax + biased top-K, histogram.

Routing indices, gates and counts are compared bit for bit with the oracle fed the same fp32
logits (the method's decisions are integers decided in fp32). Logits are compared exactly on
integer-grid inputs (every summation order is exact) and within an fp32 accumulation bound on
general inputs."""
import numpy as np
import pytest
import torch

import oracle
from mixture_experts_zero_b200 import binding as B
from mixture_experts_zero_b200 import inputs

from tests.gpu_util import make, np_bits

pytestmark = pytest.mark.gpu

SMALL = ["tiny", "small"]


def exact_grid_logits(x: torch.Tensor, wr: torch.Tensor) -> np.ndarray:
    k = np.rint(oracle.bf16_bits_to_f64(np_bits(x)) * 16).astype(np.int64)
    j = np.rint(oracle.bf16_bits_to_f64(np_bits(wr)) * 64).astype(np.int64)
    return ((k @ j.T).astype(np.float64) * 2.0 ** -10).astype(np.float32)


@pytest.mark.parametrize("name", SMALL)
def test_router_logits_exact_on_grid(cuda_device, name):
    d = make(name, grid=True, experts=False)
    z = B.lc_moe_router_logits(d["x"], d["wr"])
    torch.cuda.synchronize()
    np.testing.assert_array_equal(z.cpu().numpy(), exact_grid_logits(d["x"], d["wr"]))


@pytest.mark.parametrize("name,rows", [("decode", None), ("prefill", 48), ("bias_loop", 32)])
def test_router_logits_full_shape(cuda_device, name, rows):
    """LongCat-Flash shape (d=6144, E=768): grid inputs are exact for every row; general N(0,1)
    inputs are checked on sampled rows against the oracle's double-precision dot products."""
    d = make(name, grid=True, experts=False)
    z = B.lc_moe_router_logits(d["x"], d["wr"])
    T = d["x"].shape[0]
    sel = np.arange(T) if rows is None else np.random.default_rng(0).choice(T, rows, replace=False)
    exact = exact_grid_logits(d["x"][torch.as_tensor(sel, device=d["x"].device)], d["wr"])
    np.testing.assert_array_equal(z.cpu().numpy()[sel], exact)
    g = make(name, grid=False, experts=False)
    z = B.lc_moe_router_logits(g["x"], g["wr"]).cpu().numpy()
    xs = np_bits(g["x"])[sel]
    ref = oracle.router_logits(np.ascontiguousarray(xs), np_bits(g["wr"]))
    bound = (np.abs(oracle.bf16_bits_to_f64(xs)) @ np.abs(oracle.bf16_bits_to_f64(np_bits(g["wr"]))).T)
    err = np.abs(z[sel].astype(np.float64) - ref.astype(np.float64))
    assert np.all(err <= bound * 2.0 ** -20 + 1e-6), float(np.max(err / (bound + 1e-30)))


@pytest.mark.parametrize("name", ["tiny", "small", "decode", "prefill"])
def test_topk_bit_exact_from_the_same_logits(cuda_device, name):
    d = make(name, grid=False, experts=False)
    w = d["w"]
    z = B.lc_moe_router_logits(d["x"], d["wr"])
    counts = torch.zeros(w.E, dtype=torch.int32, device="cuda")
    idx, gate = B.lc_moe_topk(z, d["bias"], w.K, w.N, counts=counts)
    r_idx, r_gate, r_counts, bad = oracle.route(z.cpu().numpy(), d["bias"].cpu().numpy(), w.K)
    assert bad == 0
    np.testing.assert_array_equal(idx.cpu().numpy(), r_idx)
    np.testing.assert_array_equal(gate.cpu().numpy().view(np.uint32), r_gate.view(np.uint32))
    np.testing.assert_array_equal(counts.cpu().numpy(), r_counts)


def test_topk_ties_and_ragged_expert_counts(cuda_device):
    """Integer logits make exact score ties common; expert counts that are not multiples of 32
    leave lanes without values."""
    rng = np.random.default_rng(1)
    for (T, E, K) in [(37, 12, 3), (100, 33, 5), (64, 65, 32), (5, 2048, 12), (300, 96, 6), (1, 1, 1)]:
        z = rng.integers(-2, 3, (T, E)).astype(np.float32)
        b = (rng.integers(-1, 2, E) * 2.0 ** -6).astype(np.float32)
        N = max(1, E // 2)
        zt = torch.from_numpy(z).cuda()
        bt = torch.from_numpy(b).cuda()
        counts = torch.zeros(E, dtype=torch.int32, device="cuda")
        idx, gate = B.lc_moe_topk(zt, bt, K, N, counts=counts)
        r_idx, r_gate, r_counts, _ = oracle.route(z, b, K)
        np.testing.assert_array_equal(idx.cpu().numpy(), r_idx)
        np.testing.assert_array_equal(gate.cpu().numpy().view(np.uint32), r_gate.view(np.uint32))
        np.testing.assert_array_equal(counts.cpu().numpy(), r_counts)


@pytest.mark.parametrize("name", SMALL)
def test_route_entry_point_grid_inputs_end_to_end(cuda_device, name):
    """lc_moe_route on grid inputs equals the oracle's own router logits + routing, end to end."""
    d = make(name, grid=True, experts=False)
    w = d["w"]
    counts = torch.zeros(w.E, dtype=torch.int32, device="cuda")
    logits = torch.empty(w.T, w.E, dtype=torch.float32, device="cuda")
    idx, gate = B.lc_moe_route(d["x"], d["wr"], d["bias"], w.K, w.N, counts=counts, logits=logits)
    z_ref = oracle.router_logits(np_bits(d["x"]), np_bits(d["wr"]))
    np.testing.assert_array_equal(logits.cpu().numpy(), z_ref)
    r_idx, r_gate, r_counts, _ = oracle.route(z_ref, d["bias"].cpu().numpy(), w.K)
    np.testing.assert_array_equal(idx.cpu().numpy(), r_idx)
    np.testing.assert_array_equal(gate.cpu().numpy().view(np.uint32), r_gate.view(np.uint32))
    np.testing.assert_array_equal(counts.cpu().numpy(), r_counts)


def test_histogram_kernel(cuda_device):
    rng = np.random.default_rng(2)
    for n, bins in [(0, 5), (1, 1), (7, 3), (1000003, 768), (196608, 768)]:
        v = rng.integers(0, bins, n).astype(np.int32)
        t = torch.from_numpy(v).cuda()
        c = B.lc_moe_expert_hist(t, bins)
        np.testing.assert_array_equal(c.cpu().numpy(), np.bincount(v, minlength=bins))
    # out-of-range entries are skipped and reported
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    t = torch.tensor([0, 1, 5, -1, 2, 9, 1, 1], dtype=torch.int32, device="cuda")
    c = B.lc_moe_expert_hist(t, 3, ws=ws)
    assert c.cpu().tolist() == [1, 3, 1]
    assert B.lc_moe_read_status(ws, raise_on_error=False) & B.DEV_IDX_RANGE


def test_nan_logits_set_the_device_status(cuda_device):
    z = torch.zeros(4, 16, device="cuda")
    z[2, 3] = float("nan")
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    idx, gate = B.lc_moe_topk(z, torch.zeros(16, device="cuda"), 3, 8, ws=ws)
    status = B.lc_moe_read_status(ws, raise_on_error=False)
    assert status & B.DEV_NAN_KEY
    assert idx[2].cpu().tolist() == [0, 1, 2] and torch.isnan(gate[2]).all()
    assert B.lc_moe_read_status(ws) == 0  # cleared


# (T, d, E, K): expert counts below, at and between multiples of the router GEMM's 256-wide N
# tile and of 32 (the top-K kernel's lane stride), ragged token counts past a 128-row M tile,
# K = 1 and K = 16, with frequent exact ties (small d, integer-grid inputs)
ROUTE_SHAPES = [(64, 128, 12, 3), (257, 64, 96, 6), (1, 64, 300, 12), (300, 128, 512, 16),
                (513, 64, 700, 12), (1000, 256, 768, 12), (129, 64, 768, 1), (70, 64, 33, 16),
                (8192, 64, 768, 12), (5000, 64, 2000, 8)]  # the last two: 192-column router tiles


@pytest.mark.parametrize("shape", ROUTE_SHAPES, ids=[str(s) for s in ROUTE_SHAPES])
def test_route_without_logits_buffer_bit_exact_on_grid_inputs(cuda_device, shape):
    """lc_moe_route with the logits kept in its workspace: on grid inputs its picks, gates and
    counts equal the oracle's routing of the exact logits."""
    T, d, E, K = shape
    g = torch.Generator(device="cuda").manual_seed(T * 7 + E)
    x = inputs.to_grid(torch.randn(T, d, generator=g, device="cuda") * 2)
    wr = (torch.randint(-4, 5, (E, d), generator=g, device="cuda").float() * 2.0 ** -6).to(torch.bfloat16)
    bias = (torch.randint(-2, 3, (E,), generator=g, device="cuda").float() * 2.0 ** -9)
    N = max(1, (2 * E) // 3)
    counts = torch.zeros(E, dtype=torch.int32, device="cuda")
    ws = B.new_workspace(B.Shape(T, d, N, E - N, K, 64), B.OP_ROUTE)
    idx, gate = B.lc_moe_route(x, wr, bias, K, N, counts=counts, ws=ws)
    assert B.lc_moe_read_status(ws) == 0
    z = oracle.router_logits(np_bits(x), np_bits(wr))
    np.testing.assert_array_equal(z, exact_grid_logits(x, wr))
    r_idx, r_gate, r_counts, bad = oracle.route(z, bias.cpu().numpy(), K)
    assert bad == 0
    np.testing.assert_array_equal(idx.cpu().numpy(), r_idx)
    np.testing.assert_array_equal(gate.cpu().numpy().view(np.uint32), r_gate.view(np.uint32))
    np.testing.assert_array_equal(counts.cpu().numpy(), r_counts)


@pytest.mark.parametrize("name", ["decode", "prefill"])
def test_route_full_shape_grid_inputs(cuda_device, name):
    """LongCat-Flash shape on grid activations: the router logits are exact in any summation order
    (checked against an int64 product on sampled rows), so lc_moe_route's routing of every token
    must equal the oracle's routing of those exact logits, bit for bit."""
    d = make(name, grid=True, experts=False)
    w = d["w"]
    counts = torch.zeros(w.E, dtype=torch.int32, device="cuda")
    idx, gate = B.lc_moe_route(d["x"], d["wr"], d["bias"], w.K, w.N, counts=counts)
    z = B.lc_moe_router_logits(d["x"], d["wr"])
    rows = np.arange(0, w.T, max(1, w.T // 16))
    np.testing.assert_array_equal(z.cpu().numpy()[rows], exact_grid_logits(d["x"][rows], d["wr"]))
    r_idx, r_gate, r_counts, bad = oracle.route(z.cpu().numpy(), d["bias"].cpu().numpy(), w.K)
    assert bad == 0
    np.testing.assert_array_equal(idx.cpu().numpy(), r_idx)
    np.testing.assert_array_equal(gate.cpu().numpy().view(np.uint32), r_gate.view(np.uint32))
    np.testing.assert_array_equal(counts.cpu().numpy(), r_counts)
