"""GPU parity of the FP8 (E4M3) expert path against the oracle.

The quantiser is integer-valued work decided in fp32 on both sides (amax, one IEEE division for
the scale, one per element, then round-to-nearest-even to E4M3): codes and scales must match the
oracle bit for bit. The layer's output is checked with the same rule as the bf16 layer
(2e-2 x RMS plus half a bf16 step against the oracle's double sums): both sides multiply the
same E4M3 codes and scales, so they differ by fp32 accumulation order, the bf16 roundings of H
and Y, and the E4M3 rounding of an H element that lands next to a rounding boundary. The oracle
always quantises from the bf16 weights itself; no code or scale it uses comes from the GPU.
E4M3 K-steps are 128 elements, so the FP8 workloads take I a multiple of 128 (the tiny
workload's I = 64 is raised to 128).
"""
import numpy as np
import pytest
import torch

import oracle
from mixture_experts_zero_b200 import binding as B

from tests.gpu_util import assert_out_close, make, np_bits

pytestmark = pytest.mark.gpu


def bf16_rows(rng, shape, scales):
    v = rng.standard_normal(shape).astype(np.float32) * scales
    return torch.from_numpy(v).to(torch.bfloat16)


def test_quantize_matches_oracle_bit_for_bit(cuda_device):
    rng = np.random.default_rng(3)
    R, C = 300, 1024
    row_scale = np.exp(rng.uniform(-30, 20, (R, 1))).astype(np.float32)
    x = bf16_rows(rng, (R, C), row_scale)
    x[5] = 0.0                                  # all-zero row: scale 1, codes 0
    x[6, :] = 0.0
    x[6, 17] = -3.0                             # one non-zero: +-448 there, zeros elsewhere
    x[7] = x[7] * 1e-3
    x[7, 0] = 1.0                               # most values underflow to (signed) zero codes
    xg = x.cuda()
    q, s = B.lc_moe_quantize_e4m3(xg)
    rq, rs = oracle.quantize_rows_e4m3(np_bits(x))
    np.testing.assert_array_equal(s.cpu().numpy().view(np.uint32), rs.view(np.uint32))
    np.testing.assert_array_equal(q.cpu().numpy(), rq)
    assert rq[6, 17] == 0xFE and np.all(np.delete(rq[6], 17) == 0) and rs[5] == 1.0


@pytest.mark.parametrize("R,C", [(1, 8), (33, 136), (1000, 6144)])
def test_quantize_ragged_shapes(cuda_device, R, C):
    rng = np.random.default_rng(R + C)
    x = bf16_rows(rng, (R, C), np.float32(0.7))
    q, s = B.lc_moe_quantize_e4m3(x.cuda())
    rq, rs = oracle.quantize_rows_e4m3(np_bits(x))
    np.testing.assert_array_equal(s.cpu().numpy().view(np.uint32), rs.view(np.uint32))
    np.testing.assert_array_equal(q.cpu().numpy(), rq)


FP8_CHANGES = {"tiny": {"I": 128}, "small": {}}


def oracle_weights(d):
    """Oracle quantisation of W13 and W2 (from the bf16 weights): host arrays and their uploads."""
    w = d["w"]
    wq, wsc = oracle.quantize_rows_e4m3(np_bits(d["w13"]).reshape(w.N * 2 * w.I, w.d))
    w2q, w2s = oracle.quantize_rows_e4m3(np_bits(d["w2"]).reshape(w.N * w.d, w.I))
    host = (wq.reshape(w.N, 2 * w.I, w.d), wsc.reshape(w.N, 2 * w.I), w2q.reshape(w.N, w.d, w.I),
            w2s.reshape(w.N, w.d))
    return host, tuple(torch.from_numpy(a).cuda() for a in host)


def forward_fp8(d, qw):
    w = d["w"]
    idx = torch.empty(w.T, w.K, dtype=torch.int32, device="cuda")
    gate = torch.empty(w.T, w.K, dtype=torch.float32, device="cuda")
    counts = torch.zeros(w.E, dtype=torch.int32, device="cuda")
    ws = B.new_workspace(B.Shape(w.T, w.d, w.N, w.Z, w.K, w.I), B.OP_FORWARD_FP8)
    out = B.lc_moe_forward_fp8(d["x"], d["wr"], d["bias"], *qw, w.K, idx=idx, gate=gate,
                               counts=counts, ws=ws)
    assert B.lc_moe_read_status(ws) == 0
    return out, idx, gate, counts


@pytest.mark.parametrize("name", ["tiny", "small"])
def test_forward_fp8_grid_inputs(cuda_device, name):
    d = make(name, grid=True, **FP8_CHANGES[name])
    w = d["w"]
    host, dev = oracle_weights(d)
    out, idx, gate, counts = forward_fp8(d, dev)
    ref = oracle.forward_fp8(np_bits(d["x"]), np_bits(d["wr"]), d["bias"].cpu().numpy(), *host,
                             w.N, w.Z, w.K)
    np.testing.assert_array_equal(idx.cpu().numpy(), ref["idx"])
    np.testing.assert_array_equal(gate.cpu().numpy().view(np.uint32), ref["gate"].view(np.uint32))
    np.testing.assert_array_equal(counts.cpu().numpy(), ref["counts"])
    assert_out_close(np_bits(out), ref["out_exact"], what="out")


def test_forward_fp8_differs_from_bf16_by_fp8_rounding_only(cuda_device):
    """The FP8 layer and the bf16 layer route identically; their outputs differ by the E4M3
    rounding of the expert operands (a few per cent of the expert terms), not more."""
    d = make("small", grid=True)
    w = d["w"]
    _, dev = oracle_weights(d)
    out8, idx8, _, _ = forward_fp8(d, dev)
    out = B.lc_moe_forward(d["x"], d["wr"], d["bias"], d["w13"], d["w2"], w.K)
    ref_idx = torch.empty_like(idx8)
    B.lc_moe_forward(d["x"], d["wr"], d["bias"], d["w13"], d["w2"], w.K, idx=ref_idx)
    assert torch.equal(idx8, ref_idx)
    a, b = out8.float(), out.float()
    rms = b.pow(2).mean().sqrt()
    diff = (a - b).abs()
    assert diff.max() > 0
    assert diff.pow(2).mean().sqrt() < 0.05 * rms


def oracle_tokens_fp8(x_bits, tokens, idx, gate, N, w13, w2):
    """Oracle FP8-layer output of the given tokens for the given routing: token rows and the
    touched experts' W13 and W2 quantised by the oracle, one expert at a time."""
    K = idx.shape[1]
    d = x_bits.shape[1]
    I = w2.shape[2]
    xq, sx = oracle.quantize_rows_e4m3(np.ascontiguousarray(x_bits[tokens]))
    pairs = [(j, r) for j in range(len(tokens)) for r in range(K) if idx[tokens[j], r] < N]
    Y = np.zeros((len(pairs), d), np.uint16)
    experts = np.array([idx[tokens[j], r] for j, r in pairs], np.int64)
    for e in np.unique(experts):
        sel = np.nonzero(experts == e)[0]
        wq, wsc = oracle.quantize_rows_e4m3(np_bits(w13[int(e)]).reshape(2 * I, d))
        w2q, w2s = oracle.quantize_rows_e4m3(np_bits(w2[int(e)]).reshape(d, I))
        rows = np.array([pairs[i][0] for i in sel])
        _, y = oracle.expert_rows_fp8(np.ascontiguousarray(xq[rows]), np.ascontiguousarray(sx[rows]),
                                      np.zeros(sel.size, np.int32), wq.reshape(1, 2 * I, d),
                                      wsc.reshape(1, 2 * I), w2q.reshape(1, d, I), w2s.reshape(1, d),
                                      want_h=False)
        Y[sel] = y
    pr = np.full((len(tokens), K), -1, np.int32)
    for i, (j, r) in enumerate(pairs):
        pr[j, r] = i
    _, exact = oracle.combine(np.ascontiguousarray(x_bits[tokens]), Y, np.ascontiguousarray(idx[tokens]),
                              np.ascontiguousarray(gate[tokens]), pr, N, want_exact=True)
    return exact


@pytest.mark.parametrize("name", ["prefill", "decode"])
def test_forward_fp8_full_size_sampled(cuda_device, name):
    """The benchmark's FP8 launch configuration at full size (W13 and W2 quantised on the GPU, as
    the benchmark does), checked on sampled tokens against the oracle's own quantisation."""
    d = make(name)
    w = d["w"]
    w13q, w13s = B.lc_moe_quantize_e4m3(d["w13"])
    w2q, w2s = B.lc_moe_quantize_e4m3(d["w2"])
    out, idx, gate, _ = forward_fp8(d, (w13q, w13s, w2q, w2s))
    del w13q, w13s, w2q, w2s
    rng = np.random.default_rng(17)
    tokens = np.sort(rng.choice(w.T, size=6, replace=False))
    idx_h, gate_h = idx.cpu().numpy(), gate.cpu().numpy()
    ref = oracle_tokens_fp8(np_bits(d["x"]), tokens, idx_h, gate_h, w.N, d["w13"], d["w2"])
    assert_out_close(np_bits(out)[tokens], ref, what="out")
