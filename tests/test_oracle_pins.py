"""Pins for the CPU oracle: what the pages and the mathematics fix, checked without a GPU.

Each test ties one step of the oracle to something other than itself: a closed form, an exact
integer computation, a library routine (numpy / scipy / torch), brute-force enumeration, or a
special case the LongCat-Flash llm-wiki entity page states (section 2.1: zero-computation
experts return their input; the bias update and its fixed point).
"""
import fractions
import itertools
import math
import pathlib

import numpy as np
import pytest
import scipy.special
import torch

import oracle
from mixture_experts_zero_b200 import inputs

GOLDEN = pathlib.Path(__file__).resolve().parent / "golden"


def bf16(a) -> np.ndarray:
    """float values -> bf16 bits through torch (library rounding, float32 -> bf16)."""
    t = torch.as_tensor(np.asarray(a, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def f64(bits) -> np.ndarray:
    return oracle.bf16_bits_to_f64(bits)


def rand_layer(rng, T, d, N, Z, I, w_std=0.1, grid=False):
    E = N + Z
    if grid:
        x = np.clip(np.round(rng.standard_normal((T, d)) * 16), -128, 128) / 16
        wr = rng.integers(-4, 5, (E, d)) / 64.0
    else:
        x = rng.standard_normal((T, d))
        wr = rng.standard_normal((E, d)) * 0.5
    w13 = rng.standard_normal((N, 2 * I, d)) * w_std
    w2 = rng.standard_normal((N, d, I)) * w_std
    return bf16(x), bf16(wr), bf16(w13), bf16(w2)


# ----------------------------------------------------------------------------- bf16 rounding

def test_bf16_rounding_matches_library_on_fp32_values():
    rng = np.random.default_rng(0)
    vals = np.concatenate([
        rng.standard_normal(20000).astype(np.float32) * np.float32(10.0) ** rng.integers(-30, 30, 20000).astype(np.float32),
        np.array([0.0, -0.0, 1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, 1.0 + 2 ** -9, 1.0 + 3 * 2 ** -9,
                  2.0 ** -130, 2.0 ** -133, 3 * 2.0 ** -134, 3.3e38, 3.4e38, -3.39e38], dtype=np.float32),
    ]).astype(np.float32)
    vals = vals[np.isfinite(vals)]
    mine = oracle.f64_to_bf16_bits(vals.astype(np.float64))
    ref = bf16(vals)
    np.testing.assert_array_equal(mine, ref)


# ------------------------------------------------------------------------------ router logits

def test_router_logits_exact_on_grid_inputs():
    """Grid inputs: every product is a multiple of 2^-10, so the exact dot product is an integer
    times 2^-10 and fits fp32 exactly; compare with an int64 computation."""
    rng = np.random.default_rng(1)
    T, d, E = 37, 256, 19
    k = rng.integers(-128, 129, (T, d))
    j = rng.integers(-4, 5, (E, d))
    x = bf16(k / 16.0)
    wr = bf16(j / 64.0)
    z = oracle.router_logits(x, wr)
    exact = (k.astype(np.int64) @ j.astype(np.int64).T).astype(np.float64) * 2.0 ** -10
    np.testing.assert_array_equal(z, exact.astype(np.float32))


def test_router_logits_general_inputs_close_to_float64_matmul():
    rng = np.random.default_rng(2)
    x = bf16(rng.standard_normal((16, 384)))
    wr = bf16(rng.standard_normal((24, 384)))
    z = oracle.router_logits(x, wr)
    ref = f64(x) @ f64(wr).T
    np.testing.assert_allclose(z, ref, rtol=1e-6, atol=1e-5)


# ---------------------------------------------------------------------------- exp and sum spec

def _ulp32(v: float) -> float:
    return float(np.spacing(np.float32(abs(v))))


def test_exp_spec_within_two_ulp_of_exp():
    us = np.concatenate([np.linspace(-86.0, 0.0, 40001), -np.abs(np.random.default_rng(3).standard_normal(20000)) * 10,
                         np.array([0.0, -1e-30, -1e-7, -0.5 * math.log(2), -math.log(2), -85.9999])])
    us = us.astype(np.float32)
    worst = 0.0
    for u in us:
        got = oracle.exp_spec(float(u))
        ref = math.exp(float(u))
        worst = max(worst, abs(got - ref) / _ulp32(ref))
    assert worst <= 2.0, worst
    assert oracle.exp_spec(0.0) == 1.0
    assert oracle.exp_spec(-86.5) == 0.0
    assert oracle.exp_spec(float("-inf")) == 0.0
    assert math.isnan(oracle.exp_spec(float("nan")))


def test_sum_spec_error_bound_and_small_cases():
    rng = np.random.default_rng(4)
    for E in [1, 2, 12, 31, 32, 33, 96, 768, 2048]:
        v = rng.random(E).astype(np.float32)
        got = oracle.sum_spec(v)
        exact = math.fsum(float(a) for a in v)
        # every value is >= 0: relative error of any summation tree is below (depth) * eps
        depth = math.ceil(E / 32) + 5
        assert abs(got - exact) <= depth * 2.0 ** -24 * exact * 1.0001 + 1e-45, (E, got, exact)
    # order-free cases: exact sums of small integers
    assert oracle.sum_spec(np.ones(768, np.float32)) == 768.0
    assert oracle.sum_spec(np.arange(100, dtype=np.float32)) == 4950.0


# -------------------------------------------------------------------------------- routing

def _keys(scores, bias):
    return (scores.astype(np.float32) + bias.astype(np.float32)).astype(np.float32)


def test_scores_are_the_softmax_over_all_experts():
    rng = np.random.default_rng(5)
    z = (rng.standard_normal((64, 96)) * 4).astype(np.float32)
    b = np.zeros(96, np.float32)
    *_, scores = oracle.route(z, b, 6, want_scores=True)
    ref = scipy.special.softmax(z.astype(np.float64), axis=1)
    np.testing.assert_allclose(scores, ref, rtol=2e-6, atol=1e-30)


def test_topk_matches_brute_force_subset_enumeration():
    """The chosen set maximises the exact sum of keys; among maximal sets it is the
    lexicographically smallest index set (ties to the lower index). Keys are drawn on a coarse
    grid so that ties are frequent."""
    rng = np.random.default_rng(6)
    for trial in range(60):
        E = int(rng.integers(3, 11))
        K = int(rng.integers(1, E + 1))
        z = np.round(rng.standard_normal((1, E)) * 2).astype(np.float32)
        b = (np.round(rng.standard_normal(E) * 4) / 64).astype(np.float32)
        idx, gate, cnt, bad, s = oracle.route(z, b, K, want_scores=True)
        assert bad == 0
        key = _keys(s[0], b)
        best = None
        for sub in itertools.combinations(range(E), K):
            tot = sum(fractions.Fraction(float(key[i])) for i in sub)
            if best is None or tot > best[0]:
                best = (tot, sub)
        assert tuple(sorted(idx[0].tolist())) == best[1], (trial, key, idx)
        # rank order: descending key, equal keys by ascending index (a stable sort)
        order = sorted(range(E), key=lambda i: (-float(key[i]), i))[:K]
        assert idx[0].tolist() == order


def test_ties_go_to_the_lower_index():
    z = np.zeros((1, 8), np.float32)          # all scores equal
    b = np.zeros(8, np.float32)
    idx, *_ = oracle.route(z, b, 3)
    assert idx[0].tolist() == [0, 1, 2]
    b[5] = 1.0                                # one clear winner, the rest tied
    idx, *_ = oracle.route(z, b, 3)
    assert idx[0].tolist() == [5, 0, 1]


def test_gates_are_unbiased_scores_renormalised_over_the_chosen():
    rng = np.random.default_rng(7)
    T, E, K = 200, 48, 5
    z = (rng.standard_normal((T, E)) * 3).astype(np.float32)
    b = (rng.standard_normal(E) * 0.05).astype(np.float32)
    idx, gate, cnt, bad = oracle.route(z, b, K)
    assert bad == 0
    # softmax over the chosen logits (a library routine), the same thing in exact arithmetic
    chosen = np.take_along_axis(z, idx, axis=1).astype(np.float64)
    ref = scipy.special.softmax(chosen, axis=1)
    np.testing.assert_allclose(gate, ref, rtol=4e-6)
    # gate sum within K * 2^-24 of one
    assert np.max(np.abs(gate.astype(np.float64).sum(1) - 1.0)) <= K * 2.0 ** -24 + 2.0 ** -24
    # the bias steers selection only: the same picks with a zero bias give the same gates
    idx0, gate0, _, _ = oracle.route(z, np.zeros(E, np.float32), K)
    same = np.all(np.sort(idx0, 1) == np.sort(idx, 1), axis=1)
    assert same.any()
    for t in np.nonzero(same)[0]:
        np.testing.assert_array_equal(np.sort(gate0[t]), np.sort(gate[t]))


def test_bias_is_added_to_scores_with_the_right_sign():
    rng = np.random.default_rng(8)
    T, E, K = 100, 24, 4
    z = rng.standard_normal((T, E)).astype(np.float32)
    b = np.zeros(E, np.float32)
    b[7] = 2.0      # larger than any score: always picked, first
    b[3] = -2.0     # never picked
    idx, *_ = oracle.route(z, b, K)
    assert np.all(idx[:, 0] == 7)
    assert not np.any(idx == 3)


def test_counts_are_the_histogram_of_picks_and_accumulate():
    rng = np.random.default_rng(9)
    z = rng.standard_normal((300, 40)).astype(np.float32)
    b = np.zeros(40, np.float32)
    idx, gate, cnt, _ = oracle.route(z, b, 7)
    np.testing.assert_array_equal(cnt, np.bincount(idx.ravel(), minlength=40))
    idx2, _, cnt2, _ = oracle.route(z, b, 7, counts=cnt.copy())
    np.testing.assert_array_equal(cnt2, 2 * np.bincount(idx.ravel(), minlength=40))


def test_nan_logit_is_reported():
    z = np.zeros((3, 10), np.float32)
    z[1, 4] = np.nan
    idx, gate, cnt, bad = oracle.route(z, np.zeros(10, np.float32), 2)
    assert bad == 1


# -------------------------------------------------------------------------------- permutation

def test_permute_is_a_stable_sort_of_ffn_picks_by_expert():
    rng = np.random.default_rng(10)
    T, N, Z, K = 513, 20, 9, 5
    z = rng.standard_normal((T, N + Z)).astype(np.float32)
    idx, *_ = oracle.route(z, np.zeros(N + Z, np.float32), K)
    offsets, row_token, pair_row = oracle.permute(idx, N)
    flat = idx.ravel()
    ffn = np.nonzero(flat < N)[0]
    order = ffn[np.argsort(flat[ffn], kind="stable")]      # library stable sort
    np.testing.assert_array_equal(row_token, order // K)
    expect_pair_row = np.full(T * K, -1, np.int32)
    expect_pair_row[order] = np.arange(order.size)
    np.testing.assert_array_equal(pair_row.ravel(), expect_pair_row)
    np.testing.assert_array_equal(offsets, np.concatenate([[0], np.cumsum(np.bincount(flat[ffn], minlength=N))]))


def test_permute_all_zero_picks_gives_no_rows():
    idx = np.array([[5, 6], [6, 7]], np.int32)
    offsets, row_token, pair_row = oracle.permute(idx, 4)
    assert offsets.tolist() == [0, 0, 0, 0, 0] and row_token.size == 0
    assert np.all(pair_row == -1)


# ------------------------------------------------------------------------------------ experts

def _swiglu_ref(xb, w13b, w2b, e):
    """Textbook SwiGLU with library matmuls in float64 and torch's bf16 rounding of H and Y."""
    I = w2b.shape[2]
    x = f64(xb)
    wg, wu = f64(w13b[e, :I]), f64(w13b[e, I:])
    g = x @ wg.T
    u = x @ wu.T
    h = torch.from_numpy(g * scipy.special.expit(g) * u).to(torch.bfloat16).to(torch.float64).numpy()
    y = torch.from_numpy(h @ f64(w2b[e]).T).to(torch.bfloat16).to(torch.float64).numpy()
    return h, y


def test_expert_rows_match_textbook_swiglu():
    rng = np.random.default_rng(11)
    M, d, N, I = 40, 64, 3, 32
    x, _, w13, w2 = rand_layer(rng, M, d, N, 1, I, w_std=0.3)
    re = rng.integers(0, N, M).astype(np.int32)
    h, y = oracle.expert_rows(x, re, w13, w2)
    for r in range(M):
        hr, yr = _swiglu_ref(x[r:r + 1], w13, w2, re[r])
        # H: same value up to one bf16 step (the reference rounds twice: double->float->bf16)
        np.testing.assert_allclose(f64(h[r]), hr[0], rtol=2 ** -7, atol=1e-6)
        np.testing.assert_allclose(f64(y[r]), yr[0], rtol=2 ** -7, atol=2 ** -8 * np.abs(yr).max())


def test_expert_down_matches_textbook_and_the_full_expert():
    rng = np.random.default_rng(19)
    M, d, N, I = 30, 48, 3, 64
    h = bf16(rng.standard_normal((M, I)))
    w2 = bf16(rng.standard_normal((N, d, I)) * 0.2)
    re = rng.integers(0, N, M).astype(np.int32)
    y = oracle.expert_down(h, re, w2)
    for r in range(M):
        ref = torch.from_numpy(f64(h[r]) @ f64(w2[re[r]]).T).to(torch.bfloat16).to(torch.float64).numpy()
        np.testing.assert_allclose(f64(y[r]), ref, rtol=2 ** -7, atol=1e-6)
    # the down projection of the full expert's own H reproduces its Y bit for bit
    x, _, w13, w2b = rand_layer(rng, M, d, N, 1, I, w_std=0.3)
    H, Y = oracle.expert_rows(x, re, w13, w2b)
    np.testing.assert_array_equal(oracle.expert_down(H, re, w2b), Y)


# ------------------------------------------------------------------------------- whole layer

def test_all_zero_expert_picks_return_the_input_exactly():
    """Zero-computation experts return their input; with every pick a zero expert the output is
    (sum of gates) * x = x, exactly after bf16 rounding."""
    rng = np.random.default_rng(12)
    T, d, N, Z, K, I = 50, 64, 6, 4, 3, 32
    x, wr, w13, w2 = rand_layer(rng, T, d, N, Z, I)
    b = np.zeros(N + Z, np.float32)
    b[N:] = 10.0
    res = oracle.forward(x, wr, b, w13, w2, N, Z, K)
    assert np.all(res["idx"] >= N)
    np.testing.assert_array_equal(res["out"], x)


def test_single_ffn_expert_brute_force():
    """N=1, Z=3, K=2, d=8, I=4: out = g0 * SwiGLU(x) + (1 - g0) * x when the FFN expert is
    picked (g0 its gate), and out = x otherwise."""
    rng = np.random.default_rng(13)
    T, d, N, Z, K, I = 256, 8, 1, 3, 2, 4
    x, wr, w13, w2 = rand_layer(rng, T, d, N, Z, I, w_std=0.5)
    b = (rng.standard_normal(N + Z) * 0.1).astype(np.float32)
    res = oracle.forward(x, wr, b, w13, w2, N, Z, K)
    xf, wrf = f64(x), f64(wr)
    s = scipy.special.softmax(xf @ wrf.T, axis=1)
    key = s + b
    picked = 0
    for t in range(T):
        order = sorted(range(N + Z), key=lambda i: (-key[t, i], i))[:K]
        if sorted(order) != sorted(res["idx"][t].tolist()):
            # a selection flip is only acceptable at a near-tie of the keys
            k_sorted = np.sort(key[t])[::-1]
            assert abs(k_sorted[K - 1] - k_sorted[K]) < 1e-6
            continue
        if 0 in order:
            picked += 1
            g0 = s[t, 0] / sum(s[t, i] for i in order)
            _, y = _swiglu_ref(x[t:t + 1], w13, w2, 0)
            ref = g0 * y[0] + (1 - g0) * xf[t]
        else:
            ref = xf[t]
        np.testing.assert_allclose(f64(res["out"][t]), ref, rtol=2 ** -7, atol=2 ** -9 * np.abs(ref).max())
    assert 20 < picked < T - 20     # both branches exercised


def test_no_zero_experts_reduces_to_textbook_topk_moe():
    """Z = 0: a plain softmax top-K MoE with renormalised gates, written with torch ops."""
    rng = np.random.default_rng(14)
    T, d, N, K, I = 48, 32, 6, 2, 16
    x, wr, w13, w2 = rand_layer(rng, T, d, N, 0, I, w_std=0.4)
    res = oracle.forward(x, wr, np.zeros(N, np.float32), w13, w2, N, 0, K)
    xt = torch.from_numpy(f64(x))
    probs = torch.softmax(xt @ torch.from_numpy(f64(wr)).T, dim=1)
    top_p, top_i = torch.topk(probs, K, dim=1)
    gates = top_p / top_p.sum(1, keepdim=True)
    out = torch.zeros_like(xt)
    for t in range(T):
        for r in range(K):
            e = int(top_i[t, r])
            _, y = _swiglu_ref(x[t:t + 1], w13, w2, e)
            out[t] += gates[t, r] * torch.from_numpy(y[0])
    np.testing.assert_allclose(f64(res["out"]), out.numpy(), rtol=2 ** -6, atol=3e-3)


def test_combine_weights_rows_and_identity_terms():
    rng = np.random.default_rng(15)
    T, d, N, Z, K = 20, 16, 4, 3, 3
    x = bf16(rng.standard_normal((T, d)))
    z = rng.standard_normal((T, N + Z)).astype(np.float32)
    idx, gate, _, _ = oracle.route(z, np.zeros(N + Z, np.float32), K)
    offsets, row_token, pair_row = oracle.permute(idx, N)
    y = bf16(rng.standard_normal((row_token.size, d)))
    out = oracle.combine(x, y, idx, gate, pair_row, N)
    ref = np.zeros((T, d))
    for t in range(T):
        for r in range(K):
            v = f64(y[pair_row[t, r]]) if idx[t, r] < N else f64(x[t])
            ref[t] += float(gate[t, r]) * v
    np.testing.assert_array_equal(out, oracle.f64_to_bf16_bits(ref))


# ------------------------------------------------------------------------------- bias update

def test_bias_update_is_zero_at_the_target_load():
    """If every expert's share T_i/(K T_all) equals K_e/(K N), the update is exactly zero.
    With E K_e = K N (true for every LongCat-shaped workload) that is T_i = K T_all / E."""
    for (N, Z, K, K_e, T_all) in [(512, 256, 12, 8, 8192), (64, 32, 6, 4, 4096), (8, 4, 3, 2, 64)]:
        E = N + Z
        assert E * K_e == K * N
        counts = np.full(E, K * T_all // E, np.int32)
        b0 = np.random.default_rng(16).standard_normal(E).astype(np.float32)
        b1 = oracle.bias_update(b0, counts, T_all, N, Z, K, K_e, 1e-3)
        np.testing.assert_array_equal(b1, b0)


def test_bias_update_matches_exact_rational_value_and_sign():
    rng = np.random.default_rng(17)
    N, Z, K, K_e, T_all, mu = 512, 256, 12, 8, 8192, 1e-3
    E = N + Z
    counts = rng.multinomial(K * T_all, np.ones(E) / E).astype(np.int32)
    b0 = np.zeros(E, np.float32)
    b1 = oracle.bias_update(b0, counts, T_all, N, Z, K, K_e, mu)
    mu32 = float(np.float32(mu))
    for i in range(E):
        exact = mu32 * (fractions.Fraction(K_e, K * N) - fractions.Fraction(int(counts[i]), K * T_all))
        # four fp32 roundings on terms of size <= K_e/(K N): a few ulps of that scale
        assert abs(float(b1[i]) - float(exact)) <= 4 * mu32 * 2 ** -24 * (K_e / (K * N)) * 4
        target = K * T_all / E
        if counts[i] > target:
            assert b1[i] < 0
        elif counts[i] < target:
            assert b1[i] > 0
    # the rule moves the bias vector along a zero-sum direction when sum T_i = K T_all
    assert abs(float(np.sum(b1.astype(np.float64)))) < E * 8 * mu32 * 2 ** -24 * (K_e / (K * N)) * 4


def test_bias_control_loop_drives_ffn_count_towards_target():
    """Start with the zero experts favoured (b = +offset on them): the mean number of FFN
    experts per token starts below K_e and the update rule moves it toward K_e."""
    rng = np.random.default_rng(18)
    N, Z, K, K_e, d, T = 16, 8, 6, 4, 64, 512
    E = N + Z
    assert E * K_e == K * N
    wr = bf16(rng.standard_normal((E, d)) * 0.05)
    b = np.zeros(E, np.float32)
    b[N:] = 2.0 / E
    mu = 3e-2
    history = []
    for step in range(200):
        x = bf16(rng.standard_normal((T, d)))
        z = oracle.router_logits(x, wr)
        idx, gate, counts, bad = oracle.route(z, b, K)
        history.append(float(np.mean(np.sum(idx < N, axis=1))))
        b = oracle.bias_update(b, counts, T, N, Z, K, K_e, mu)
    start = abs(np.mean(history[:5]) - K_e)
    end = abs(np.mean(history[-50:]) - K_e)
    assert history[0] < K_e - 0.5
    assert end < 0.05 * start
    assert end < 0.15


# ------------------------------------------------------------------ constants from the pages

def _golden():
    vals = {}
    for line in (GOLDEN / "longcat_flash_config.txt").read_text().splitlines():
        if line.strip() and not line.startswith("#"):
            k, v = line.split()
            vals[k] = float(v)
    return vals


def test_activated_parameter_range_pins_swiglu_experts_and_k_e():
    """The spread of activated parameters (max - min) is what the K picks add when all of them
    are FFN experts rather than zero experts: K * layers * (parameters of one expert). With three
    hidden x width matrices per expert (SwiGLU) this reproduces the printed spread to 0.2 %;
    two matrices would give 2/3 of it. The printed mean then gives K_e = 8 FFN experts."""
    g = _golden()
    per_expert = 3 * g["hidden"] * g["ffn_expert_width"]
    spread = g["experts_per_token"] * g["layers"] * per_expert / 1e9
    printed = g["activated_max_billion"] - g["activated_min_billion"]
    assert abs(spread - printed) / printed < 0.005
    k_e = (g["activated_mean_billion"] - g["activated_min_billion"]) / printed * g["experts_per_token"]
    assert round(k_e) == 8
    w = inputs.WORKLOADS["prefill"]
    assert (w.d, w.I, w.N, w.Z, w.K, w.K_e) == (g["hidden"], g["ffn_expert_width"], g["ffn_experts"],
                                                g["zero_experts"], g["experts_per_token"], 8)
    # the routed experts hold most of the 560B total
    assert g["ffn_experts"] * g["layers"] * per_expert / 1e9 < g["total_params_billion"]
