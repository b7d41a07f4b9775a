"""GPU parity of the whole layer at the degenerate and extreme shapes the method and the C ABI
allow: a single FFN expert, no zero-computation experts, one pick per token, the largest K (32)
and the largest expert count (N + Z = 2048), the smallest widths (d = I = 64), ragged token
counts for the FP8 layer, and the register-copy fallback of the row gather (rows above 25 KB).
Grid activations make the router logits exact, so routing is compared bit for bit and the
output with the layer's tolerance (2e-2 x RMS plus half a bf16 step)."""
import numpy as np
import pytest
import torch

import oracle
from mixture_experts_zero_b200 import binding as B

from tests.gpu_util import assert_out_close, make, np_bits

pytestmark = pytest.mark.gpu

# (T, d, N, Z, K, I)
SHAPES = [
    (5, 64, 1, 0, 1, 64),        # one FFN expert, no zero experts, one pick
    (70, 64, 3, 0, 3, 64),       # no zero experts, every expert picked by every token
    (33, 128, 4, 28, 32, 64),    # K = 32, the largest pick count
    (40, 64, 1500, 548, 8, 64),  # N + Z = 2048, the largest expert count
    (257, 64, 9, 3, 4, 64),      # the smallest widths, T past a 256-token block
]


def run_forward(d, f8_weights=None):
    w = d["w"]
    idx = torch.empty(w.T, w.K, dtype=torch.int32, device="cuda")
    gate = torch.empty(w.T, w.K, dtype=torch.float32, device="cuda")
    counts = torch.zeros(w.E, dtype=torch.int32, device="cuda")
    s = B.Shape(w.T, w.d, w.N, w.Z, w.K, w.I)
    if f8_weights is None:
        ws = B.new_workspace(s)
        out = B.lc_moe_forward(d["x"], d["wr"], d["bias"], d["w13"], d["w2"], w.K, idx=idx, gate=gate,
                               counts=counts, ws=ws)
    else:
        ws = B.new_workspace(s, B.OP_FORWARD_FP8)
        out = B.lc_moe_forward_fp8(d["x"], d["wr"], d["bias"], *f8_weights, w.K, idx=idx, gate=gate,
                                   counts=counts, ws=ws)
    assert B.lc_moe_read_status(ws) == 0
    return out, idx, gate, counts


def check_against(ref, out, idx, gate, counts, what):
    np.testing.assert_array_equal(idx.cpu().numpy(), ref["idx"])
    np.testing.assert_array_equal(gate.cpu().numpy().view(np.uint32), ref["gate"].view(np.uint32))
    np.testing.assert_array_equal(counts.cpu().numpy(), ref["counts"])
    assert_out_close(np_bits(out), ref["out_exact"], what=what)


@pytest.mark.parametrize("shape", SHAPES, ids=[str(s) for s in SHAPES])
def test_forward_degenerate_and_extreme_shapes(cuda_device, shape):
    T, d_, N, Z, K, I = shape
    d = make("tiny", grid=True, T=T, d=d_, N=N, Z=Z, K=K, K_e=min(K, N), I=I)
    w = d["w"]
    out, idx, gate, counts = run_forward(d)
    ref = oracle.forward(np_bits(d["x"]), np_bits(d["wr"]), d["bias"].cpu().numpy(), np_bits(d["w13"]),
                         np_bits(d["w2"]), w.N, w.Z, w.K)
    check_against(ref, out, idx, gate, counts, f"out {shape}")
    if Z == 0:
        assert int(counts.sum()) == T * K  # every pick is an FFN expert


# FP8 needs d and I multiples of 128
FP8_SHAPES = [(1, 128, 4, 2, 3, 128), (129, 128, 1, 0, 1, 128), (300, 256, 6, 3, 4, 128)]


@pytest.mark.parametrize("shape", FP8_SHAPES, ids=[str(s) for s in FP8_SHAPES])
def test_forward_fp8_ragged_and_degenerate(cuda_device, shape):
    T, d_, N, Z, K, I = shape
    d = make("tiny", grid=True, T=T, d=d_, N=N, Z=Z, K=K, K_e=min(K, N), I=I)
    w = d["w"]
    wq, wsc = oracle.quantize_rows_e4m3(np_bits(d["w13"]).reshape(N * 2 * I, d_))
    w2q, w2s = oracle.quantize_rows_e4m3(np_bits(d["w2"]).reshape(N * d_, I))
    host = (wq.reshape(N, 2 * I, d_), wsc.reshape(N, 2 * I), w2q.reshape(N, d_, I), w2s.reshape(N, d_))
    out, idx, gate, counts = run_forward(d, tuple(torch.from_numpy(a).cuda() for a in host))
    ref = oracle.forward_fp8(np_bits(d["x"]), np_bits(d["wr"]), d["bias"].cpu().numpy(), *host, N, Z, K)
    check_against(ref, out, idx, gate, counts, f"fp8 out {shape}")


def test_fp8_rejects_widths_that_are_not_multiples_of_128(cuda_device):
    s = B.Shape(16, 192, 4, 2, 3, 128)
    assert B.lc_moe_workspace_bytes(s, B.OP_FORWARD_FP8) == 0
    s = B.Shape(16, 128, 4, 2, 3, 64)
    assert B.lc_moe_workspace_bytes(s, B.OP_FORWARD_FP8) == 0


def test_row_gather_register_fallback_for_wide_rows(cuda_device):
    """Rows of d = 12864 bf16 (25.7 KB) exceed the bulk-copy gather's shared-memory slots and take
    the register-copy kernel; the grouped rows must still be the token rows, bit for bit."""
    rng = np.random.default_rng(8)
    T, K, N, E, d = 300, 3, 8, 12, 12864
    idx = np.stack([rng.permutation(E)[:K] for _ in range(T)]).astype(np.int32)
    x = torch.randn(T, d, device="cuda").to(torch.bfloat16)
    offsets, row_token, pair_row, x_perm = B.lc_moe_permute(torch.from_numpy(idx).cuda(), N, E, x=x)
    r_off, r_rt, r_pr = oracle.permute(idx, N)
    M = int(r_off[-1])
    np.testing.assert_array_equal(offsets.cpu().numpy(), r_off)
    assert torch.equal(x_perm[:M], x[torch.from_numpy(r_rt.astype(np.int64)).cuda()])
