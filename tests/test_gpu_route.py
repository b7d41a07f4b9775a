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
