"""GPU parity of the grouped SwiGLU expert GEMMs (tcgen05 + TMEM + TMA) and of the combine.

Stage by stage, each against the oracle fed the GPU's own inputs to that stage:
H = bf16(silu(X Wg^T) * (X Wu^T)) from the GPU's grouped rows X, and Y = bf16(H Wd^T) from the
GPU's H, must each be within one bf16 rounding step of the oracle (which computes in double and
rounds once); the combine output must be within one step of the oracle's double sum of the GPU's
Y rows, and within 2e-2 * RMS of it overall."""
import numpy as np
import pytest
import torch

import oracle
from mixture_experts_zero_b200 import binding as B

from tests.gpu_util import (assert_out_close, assert_within_ulp, expert_down_sampled,
                            expert_rows_sampled, make, np_bits)

pytestmark = pytest.mark.gpu


def run_grouped(x_rows: torch.Tensor, sizes, w13, w2, T: int, K: int):
    """Place rows grouped by expert (group e has sizes[e] rows) into a [T*K, d] buffer and run
    the grouped GEMMs."""
    N = w13.shape[0]
    d = x_rows.shape[1]
    offsets = np.concatenate([[0], np.cumsum(sizes)]).astype(np.int32)
    M = int(offsets[-1])
    assert M <= T * K
    xp = torch.zeros(T * K, d, dtype=torch.bfloat16, device="cuda")
    xp[:M] = x_rows[:M]
    h, y = B.lc_moe_expert_ffn(xp, torch.from_numpy(offsets).cuda(), w13, w2, T, K)
    return offsets, xp, h, y


@pytest.mark.parametrize("name", ["tiny", "small"])
def test_grouped_gemms_all_rows(cuda_device, name):
    d = make(name)
    w = d["w"]
    idx, _ = B.lc_moe_route(d["x"], d["wr"], d["bias"], w.K, w.N)
    offsets, row_token, pair_row, x_perm = B.lc_moe_permute(idx, w.N, w.E, x=d["x"])
    h, y = B.lc_moe_expert_ffn(x_perm, offsets, d["w13"], d["w2"], w.T, w.K)
    off = offsets.cpu().numpy()
    M = int(off[-1])
    experts = np.repeat(np.arange(w.N), np.diff(off)).astype(np.int32)
    H, _ = oracle.expert_rows(np_bits(x_perm[:M]), experts, np_bits(d["w13"]), np_bits(d["w2"]))
    same_h = assert_within_ulp(np_bits(h[:M]), H, what="H")
    Y = oracle.expert_down(np_bits(h[:M]), experts, np_bits(d["w2"]))
    same_y = assert_within_ulp(np_bits(y[:M]), Y, what="Y")
    # the rounding steps differ only near rounding boundaries
    assert same_h > 0.95 and same_y > 0.95, (same_h, same_y)


def test_grouped_gemms_ragged_group_sizes(cuda_device):
    """Group sizes around the 128-row tile (0, 1, 127, 128, 129, 255, 256, 257, ...), gate/up
    width I = 128 and I = 64 (a half tile), d = 256 and 192 (down tile of 64); and gate/up widths
    whose row tiles span both accumulators (I a multiple of 256: I = 512 and 768, with d = 1024
    and 1536), with group sizes on both sides of every tile rule (cold below 128 / 256 rows, a
    padded 128..255-row remainder, leftover rows below 128 after full 256-row tiles)."""
    rng = np.random.default_rng(4)
    for (d, I, sizes) in [(256, 128, [0, 1, 127, 128, 129, 0, 255, 256, 257, 3]),
                          (192, 64, [5, 0, 0, 300, 1, 64]),
                          (128, 192, [130, 2, 0, 77]),
                          (1024, 512, [0, 1, 64, 127, 128, 129, 255, 256, 257, 383, 384, 511, 512, 640, 1000]),
                          (1536, 768, [300, 3, 0, 513, 128, 70])]:
        N = len(sizes)
        M = int(np.sum(sizes))
        T, K = M, 1
        x = (torch.randn(M, d, device="cuda")).to(torch.bfloat16)
        w13 = (torch.randn(N, 2 * I, d, device="cuda") / d ** 0.5).to(torch.bfloat16)
        w2 = (torch.randn(N, d, I, device="cuda") / I ** 0.5).to(torch.bfloat16)
        offsets, xp, h, y = run_grouped(x, sizes, w13, w2, T, K)
        experts = np.repeat(np.arange(N), sizes).astype(np.int32)
        H, _ = oracle.expert_rows(np_bits(x), experts, np_bits(w13), np_bits(w2))
        assert_within_ulp(np_bits(h[:M]), H, what=f"H d={d} I={I}")
        Y = oracle.expert_down(np_bits(h[:M]), experts, np_bits(w2))
        assert_within_ulp(np_bits(y[:M]), Y, what=f"Y d={d} I={I}")


@pytest.mark.parametrize("name,n_rows", [("decode", 24), ("prefill", 24)])
def test_grouped_gemms_full_shape_sampled_rows(cuda_device, name, n_rows):
    """LongCat-Flash shape (d=6144, I=2048, 512 experts): every row of the GPU's grouped GEMMs is
    computed; sampled rows (first/last rows of groups and tile boundaries) are checked."""
    d = make(name)
    w = d["w"]
    idx, _ = B.lc_moe_route(d["x"], d["wr"], d["bias"], w.K, w.N)
    offsets, row_token, pair_row, x_perm = B.lc_moe_permute(idx, w.N, w.E, x=d["x"])
    h, y = B.lc_moe_expert_ffn(x_perm, offsets, d["w13"], d["w2"], w.T, w.K)
    off = offsets.cpu().numpy()
    M = int(off[-1])
    experts = np.repeat(np.arange(w.N), np.diff(off))
    rng = np.random.default_rng(5)
    big = int(np.argmax(np.diff(off)))
    cand = [off[big], off[big] + 127, off[big] + 128, off[big + 1] - 1, 0, M - 1]
    cand += list(rng.choice(M, n_rows - len(cand), replace=False))
    rows = np.unique(np.clip(np.array(cand), 0, M - 1))
    H, _ = expert_rows_sampled(np_bits(x_perm)[rows], experts[rows], d["w13"], d["w2"])
    assert_within_ulp(np_bits(h)[rows], H, what="H")
    Y = expert_down_sampled(np_bits(h)[rows], experts[rows], d["w2"])
    assert_within_ulp(np_bits(y)[rows], Y, what="Y")


@pytest.mark.parametrize("name", ["tiny", "small", "decode"])
def test_combine_matches_oracle(cuda_device, name):
    d = make(name, experts=False)
    w = d["w"]
    idx, gate = B.lc_moe_route(d["x"], d["wr"], d["bias"], w.K, w.N)
    offsets, row_token, pair_row, _ = B.lc_moe_permute(idx, w.N, w.E)
    M = int(offsets[-1])
    y = torch.randn(w.T * w.K, w.d, device="cuda").to(torch.bfloat16)
    out = B.lc_moe_combine(d["x"], y, gate, pair_row)
    ref, exact = oracle.combine(np_bits(d["x"]), np_bits(y), idx.cpu().numpy(), gate.cpu().numpy(),
                                pair_row.cpu().numpy(), w.N, want_exact=True)
    got = np_bits(out)
    assert_out_close(got, exact, what="combine")
    # fp32 accumulation vs double: equal after bf16 rounding except near rounding boundaries
    assert assert_within_ulp(got, ref, what="combine") > 0.97


def test_clock_probe_reports_each_gemms_sm_clock(cuda_device):
    """With the clock probe set, each grouped GEMM launch records CTA 0's start and end (global
    timer and cycle counter); the ratio is a plausible SM clock, and unsetting the probe stops the
    writes."""
    d = make("small")
    w = d["w"]
    idx, _ = B.lc_moe_route(d["x"], d["wr"], d["bias"], w.K, w.N)
    offsets, _, _, x_perm = B.lc_moe_permute(idx, w.N, w.E, x=d["x"])
    probe = torch.zeros(8, dtype=torch.int64, device="cuda")
    B.lc_moe_set_clock_probe(probe)
    try:
        B.lc_moe_expert_ffn(x_perm, offsets, d["w13"], d["w2"], w.T, w.K)
        torch.cuda.synchronize()
    finally:
        B.lc_moe_set_clock_probe(None)
    p = probe.cpu().tolist()
    for o in (0, 4):
        assert p[o + 2] > p[o] > 0 and p[o + 3] > p[o + 1]
        mhz = (p[o + 3] - p[o + 1]) / (p[o + 2] - p[o]) * 1e3
        assert 300.0 < mhz < 2500.0, mhz
    probe.zero_()
    B.lc_moe_expert_ffn(x_perm, offsets, d["w13"], d["w2"], w.T, w.K)
    torch.cuda.synchronize()
    assert int(probe.abs().sum()) == 0
