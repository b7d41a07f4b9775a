"""Pins of the oracle's FP8 (E4M3) expert path against facts fixed outside it.

The FP8 path is a reading of the LongCat-Flash llm-wiki entity page, section 5 (inference and
deployment: FP8/BF16 quantisation, an FP8 deployment on one node); the scaling scheme (one fp32
scale per weight row and per token row, amax / 448) is this library's. What pins it:
  - the E4M3 code table and its rounding against PyTorch's float8_e4m3fn conversion (a library
    routine written from the OCP 8-bit floating point definition), plus the format's fixed
    points (largest finite 448, smallest subnormal 2^-9, saturation, ties to even);
  - row quantisation: the largest element of a row maps to +-448, every element is within half
    a code step of x / s;
  - each FP8 projection reduces exactly to the pinned bf16 oracle when its inputs are E4M3
    values times power-of-two scales (then quantisation is exact): gate/up give the bf16 H bit
    for bit, the down projection the bf16 Y; the FP8 layer is the MoE-equation combine of its
    FP8 experts with the bf16 layer's routing.
"""
import numpy as np
import pytest
import torch

import oracle


def torch_e4m3_bits(v: np.ndarray) -> np.ndarray:
    return torch.from_numpy(np.asarray(v, np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def test_code_table_matches_the_format_definition():
    codes = np.arange(256, dtype=np.uint8)
    ours = oracle.e4m3_to_f64(codes)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    nan = np.isnan(ref)
    assert list(codes[nan]) == [0x7F, 0xFF]
    assert np.array_equal(np.isnan(ours), nan)
    np.testing.assert_array_equal(ours[~nan], ref[~nan])
    # fixed points of the format
    assert ours[0x7E] == 448.0 and ours[0x01] == 2.0 ** -9 and ours[0x08] == 2.0 ** -6
    assert ours[0x38] == 1.0 and ours[0x80] == 0.0 and np.signbit(ours[0x80])


def test_every_finite_code_round_trips():
    codes = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], dtype=np.uint8)
    vals = oracle.e4m3_to_f64(codes).astype(np.float32)
    np.testing.assert_array_equal(oracle.f32_to_e4m3(vals), codes)


def test_rounding_matches_pytorch_within_range():
    rng = np.random.default_rng(11)
    v = np.concatenate([
        rng.uniform(-448, 448, 20000),
        rng.standard_normal(20000) * 3,
        rng.standard_normal(5000) * 2.0 ** -7,          # subnormal range
    ]).astype(np.float32)
    np.testing.assert_array_equal(oracle.f32_to_e4m3(v), torch_e4m3_bits(v))


def test_ties_go_to_the_even_code_and_large_values_saturate():
    codes = np.array([c for c in range(0x7E)], dtype=np.uint8)   # positive finite codes, ascending
    vals = oracle.e4m3_to_f64(codes)
    mids = ((vals[:-1] + vals[1:]) / 2).astype(np.float32)
    assert np.array_equal(mids.astype(np.float64), (vals[:-1] + vals[1:]) / 2)   # exact in fp32
    got = oracle.f32_to_e4m3(mids)
    want = np.where(codes[:-1] % 2 == 0, codes[:-1], codes[1:])
    np.testing.assert_array_equal(got, want)
    np.testing.assert_array_equal(oracle.f32_to_e4m3(-mids), want | 0x80)
    big = np.array([448.0, 449.0, 464.0, 500.0, 1e30, np.inf], np.float32)
    np.testing.assert_array_equal(oracle.f32_to_e4m3(big), np.full(6, 0x7E, np.uint8))
    np.testing.assert_array_equal(oracle.f32_to_e4m3(-big), np.full(6, 0xFE, np.uint8))
    assert oracle.f32_to_e4m3(np.array([np.nan], np.float32))[0] == 0x7F


def bf16_bits(a) -> np.ndarray:
    return torch.from_numpy(np.asarray(a, np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def test_row_quantisation_scale_and_error_bound():
    rng = np.random.default_rng(5)
    x = rng.standard_normal((64, 512)).astype(np.float32) * np.exp(rng.uniform(-6, 3, (64, 1)))
    x[3] = 0.0
    xb = bf16_bits(x)
    q, s = oracle.quantize_rows_e4m3(xb)
    xv = oracle.bf16_bits_to_f64(xb)
    amax = np.abs(xv).max(axis=1).astype(np.float32)
    want_s = np.where(amax > 0, amax / np.float32(448.0), np.float32(1.0)).astype(np.float32)
    np.testing.assert_array_equal(s, want_s)
    assert np.all(q[3] == 0) and s[3] == 1.0
    # the largest element of every non-zero row is +-448
    for r in range(64):
        if r == 3:
            continue
        k = int(np.argmax(np.abs(xv[r])))
        assert q[r, k] & 0x7F == 0x7E
    # |x/s - q| is at most half the spacing of the codes around x/s
    deq = oracle.e4m3_to_f64(q)
    u = xv / s[:, None].astype(np.float64)
    spacing = np.where(np.abs(u) < 2.0 ** -6, 2.0 ** -9, 2.0 ** (np.floor(np.log2(np.maximum(np.abs(u), 1e-300))) - 3))
    assert np.all(np.abs(u - deq) <= spacing / 2 * (1 + 1e-6))


def exact_fp8_matrix(rng, rows, cols, row_exp):
    """Rows of E4M3 values times 2^row_exp[r], each row holding one +-448 entry, so that the row
    quantisation is exact: scale 2^row_exp[r], codes = the chosen values."""
    codes = rng.integers(0, 0x7E, size=(rows, cols)).astype(np.uint8) | (rng.integers(0, 2, (rows, cols)).astype(np.uint8) << 7)
    codes[np.arange(rows), rng.integers(0, cols, rows)] = 0x7E | (rng.integers(0, 2, rows).astype(np.uint8) << 7)
    vals = oracle.e4m3_to_f64(codes) * np.exp2(row_exp)[:, None]
    return codes, vals


def test_fp8_experts_reduce_to_the_bf16_oracle_on_exact_inputs():
    """Gate/up operands that quantise exactly give the bf16 oracle's H bit for bit; Y is then the
    FP8 down projection of that H."""
    rng = np.random.default_rng(9)
    n, d, I, M = 3, 64, 32, 10
    x_codes, xv = exact_fp8_matrix(rng, M, d, rng.integers(-9, -5, M).astype(np.float64))
    w_exp = rng.integers(-14, -10, n * 2 * I).astype(np.float64)   # gate and up rows differ
    w_codes, wv = exact_fp8_matrix(rng, n * 2 * I, d, w_exp)
    xb, wb = bf16_bits(xv), bf16_bits(wv).reshape(n, 2 * I, d)
    assert np.array_equal(oracle.bf16_bits_to_f64(xb), xv)          # exact in bf16 too
    w2 = bf16_bits(rng.standard_normal((n, d, I)) * 0.05)
    row_expert = rng.integers(0, n, M).astype(np.int32)
    xq, sx = oracle.quantize_rows_e4m3(xb)
    wq, sw = oracle.quantize_rows_e4m3(wb.reshape(n * 2 * I, d))
    w2q, w2s = oracle.quantize_rows_e4m3(w2.reshape(n * d, I))
    np.testing.assert_array_equal(xq, x_codes)
    np.testing.assert_array_equal(wq, w_codes)
    h8, y8 = oracle.expert_rows_fp8(xq, sx, row_expert, wq.reshape(n, 2 * I, d), sw.reshape(n, 2 * I),
                                    w2q.reshape(n, d, I), w2s.reshape(n, d))
    h, _ = oracle.expert_rows(xb, row_expert, wb, w2)
    np.testing.assert_array_equal(h8, h)
    np.testing.assert_array_equal(y8, oracle.expert_down_fp8(h, row_expert, w2q.reshape(n, d, I), w2s.reshape(n, d)))


def test_fp8_down_projection_reduces_to_the_bf16_one_on_exact_inputs():
    """H rows and W2 rows that quantise exactly: the FP8 down projection is the bf16 one."""
    rng = np.random.default_rng(12)
    n, d, I, M = 2, 48, 64, 9
    _, hv = exact_fp8_matrix(rng, M, I, rng.integers(-6, -2, M).astype(np.float64))
    _, w2v = exact_fp8_matrix(rng, n * d, I, rng.integers(-16, -12, n * d).astype(np.float64))
    hb, w2b = bf16_bits(hv), bf16_bits(w2v).reshape(n, d, I)
    row_expert = rng.integers(0, n, M).astype(np.int32)
    w2q, w2s = oracle.quantize_rows_e4m3(w2b.reshape(n * d, I))
    y8 = oracle.expert_down_fp8(hb, row_expert, w2q.reshape(n, d, I), w2s.reshape(n, d))
    np.testing.assert_array_equal(y8, oracle.expert_down(hb, row_expert, w2b))


def test_fp8_down_projection_quantises_each_h_row():
    """General H rows: Y is the bf16 rounding of the scaled E4M3 product of the row-quantised H
    and W2 (recomputed here with a float64 matrix product, so allow one bf16 step for a different
    summation order at a rounding boundary), and differs from the unquantised bf16 Y."""
    rng = np.random.default_rng(21)
    n, d, I, M = 2, 40, 128, 16
    hb = bf16_bits(rng.standard_normal((M, I)) * 0.3)
    w2b = bf16_bits(rng.standard_normal((n, d, I)) / np.sqrt(I))
    row_expert = rng.integers(0, n, M).astype(np.int32)
    w2q, w2s = oracle.quantize_rows_e4m3(w2b.reshape(n * d, I))
    w2q, w2s = w2q.reshape(n, d, I), w2s.reshape(n, d)
    y8 = oracle.bf16_bits_to_f64(oracle.expert_down_fp8(hb, row_expert, w2q, w2s))
    hq, sh = oracle.quantize_rows_e4m3(hb)
    hdq = oracle.e4m3_to_f64(hq) * sh[:, None].astype(np.float64)
    wdq = oracle.e4m3_to_f64(w2q) * w2s[:, :, None].astype(np.float64)
    want = np.stack([wdq[row_expert[r]] @ hdq[r] for r in range(M)])
    step = 2.0 ** (np.floor(np.log2(np.maximum(np.abs(want), 2.0 ** -126))) - 7)
    assert np.all(np.abs(y8 - want) <= step)
    y16 = oracle.bf16_bits_to_f64(oracle.expert_down(hb, row_expert, w2b))
    assert np.mean(np.abs(y8 - y16) > step) > 0.1


def test_fp8_layer_is_the_combine_of_its_fp8_experts():
    """The FP8 layer routes like the bf16 layer (routing never sees FP8) and its output is the
    MoE-equation combine of the FP8 experts' rows and the zero-expert identity term."""
    rng = np.random.default_rng(4)
    T, d, N, Z, K, I = 12, 64, 4, 2, 3, 32
    xb = bf16_bits(rng.standard_normal((T, d)))
    w13 = bf16_bits(rng.standard_normal((N, 2 * I, d)) / np.sqrt(d))
    w2 = bf16_bits(rng.standard_normal((N, d, I)) / np.sqrt(I))
    wr = bf16_bits(rng.integers(-4, 5, (N + Z, d)) * 2.0 ** -6)
    bias = np.zeros(N + Z, np.float32)
    wq, sw = oracle.quantize_rows_e4m3(w13.reshape(N * 2 * I, d))
    w2q, w2s = oracle.quantize_rows_e4m3(w2.reshape(N * d, I))
    wq, sw, w2q, w2s = wq.reshape(N, 2 * I, d), sw.reshape(N, 2 * I), w2q.reshape(N, d, I), w2s.reshape(N, d)
    f8 = oracle.forward_fp8(xb, wr, bias, wq, sw, w2q, w2s, N, Z, K)
    ref = oracle.forward(xb, wr, bias, w13, w2, N, Z, K)
    for k in ("idx", "gate", "counts", "logits"):
        np.testing.assert_array_equal(f8[k], ref[k], err_msg=k)
    offsets, row_token, pair_row = oracle.permute(f8["idx"], N)
    row_expert = np.repeat(np.arange(N, dtype=np.int32), np.diff(offsets))
    xq, sx = oracle.quantize_rows_e4m3(xb)
    _, y = oracle.expert_rows_fp8(np.ascontiguousarray(xq[row_token]), np.ascontiguousarray(sx[row_token]),
                                  row_expert, wq, sw, w2q, w2s, want_h=False)
    out, exact = oracle.combine(xb, y, f8["idx"], f8["gate"], pair_row, N, want_exact=True)
    np.testing.assert_array_equal(f8["out"], out)
    np.testing.assert_array_equal(f8["out_exact"], exact)


def test_fp8_layer_on_general_inputs_is_close_to_but_not_the_bf16_layer():
    rng = np.random.default_rng(8)
    T, d, N, Z, K, I = 16, 128, 4, 2, 3, 64
    xb = bf16_bits(rng.standard_normal((T, d)))
    w13 = bf16_bits(rng.standard_normal((N, 2 * I, d)) / np.sqrt(d))
    w2 = bf16_bits(rng.standard_normal((N, d, I)) / np.sqrt(I))
    wr = bf16_bits(rng.integers(-4, 5, (N + Z, d)) * 2.0 ** -6)
    bias = np.zeros(N + Z, np.float32)
    wq, sw = oracle.quantize_rows_e4m3(w13.reshape(N * 2 * I, d))
    w2q, w2s = oracle.quantize_rows_e4m3(w2.reshape(N * d, I))
    f8 = oracle.forward_fp8(xb, wr, bias, wq.reshape(N, 2 * I, d), sw.reshape(N, 2 * I),
                            w2q.reshape(N, d, I), w2s.reshape(N, d), N, Z, K)
    ref = oracle.forward(xb, wr, bias, w13, w2, N, Z, K)
    np.testing.assert_array_equal(f8["idx"], ref["idx"])          # routing does not see FP8
    diff = np.abs(f8["out_exact"] - ref["out_exact"])
    rms = np.sqrt(np.mean(ref["out_exact"] ** 2))
    assert diff.max() > 0                                          # the quantisation acts
    # and stays at FP8 accuracy: E4M3 keeps 3 mantissa bits (relative rounding error <= 2^-4 per
    # operand), so the expert terms carry errors of a few per cent of their size
    assert np.sqrt(np.mean(diff ** 2)) < 0.05 * rms
    assert diff.max() < 0.25 * rms
