"""Helpers shared by the GPU parity tests: workload tensors on the device, host copies for the
oracle, and oracle evaluation of selected rows with expert weights fetched one expert at a time
(the full-size expert weights are 38.6 GB)."""
from __future__ import annotations

import numpy as np
import torch

import oracle
from mixture_experts_zero_b200 import inputs

# Output tolerance: |gpu - oracle| <= 2e-2 * RMS(oracle) + half a bf16 step of the oracle value,
# elementwise, with the oracle's output taken before its final rounding to bf16. The half step
# is the representation error of the bf16 output itself: beyond ~10 x RMS it alone exceeds
# 2e-2 * RMS, so a correctly rounded output could not meet the bound without it.
REL_RMS_TOL = 2e-2
# Intermediates H and Y: one bf16 step, plus an absolute allowance for fp32 accumulation error
# where a dot product nearly cancels (relative error is large there although the absolute error
# is ~1e-6 of the RMS).
ACC_ABS_TOL = 2.0 ** -14


def np_bits(t: torch.Tensor) -> np.ndarray:
    return inputs.bits(t)


def f64(bits: np.ndarray) -> np.ndarray:
    return oracle.bf16_bits_to_f64(bits)


def bf16_ulp(v: np.ndarray) -> np.ndarray:
    """Spacing of bf16 values at magnitude |v| (8 significant bits)."""
    a = np.maximum(np.abs(np.asarray(v, np.float64)), 2.0 ** -126)
    return 2.0 ** (np.floor(np.log2(a)) - 7)


def assert_within_ulp(got_bits: np.ndarray, ref_bits: np.ndarray, n_ulp: float = 1.0, what="",
                      abs_tol: float = ACC_ABS_TOL):
    """Elementwise |gpu - oracle| <= n_ulp bf16 steps + abs_tol * RMS(oracle): both round a value
    computed from the same inputs (fp32 on the GPU, double in the oracle), so they differ by one
    rounding step plus the fp32 accumulation error. Returns the fraction of bit-identical
    elements."""
    got, ref = f64(got_bits), f64(ref_bits)
    rms = float(np.sqrt(np.mean(ref ** 2))) if ref.size else 0.0
    lim = n_ulp * bf16_ulp(np.maximum(np.abs(got), np.abs(ref))) + abs_tol * rms
    bad = np.abs(got - ref) > lim
    if bad.any():
        i = np.argwhere(bad)[0]
        raise AssertionError(f"{what}: {int(bad.sum())} elements beyond {n_ulp} bf16 step(s); "
                             f"first at {tuple(i)}: gpu {got[tuple(i)]} oracle {ref[tuple(i)]}")
    return float(np.mean(np.asarray(got_bits) == np.asarray(ref_bits)))


def assert_out_close(got_bits: np.ndarray, exact: np.ndarray, tol: float = REL_RMS_TOL, what=""):
    """Output check against the oracle's double-precision value: elementwise
    |gpu - exact| <= tol * RMS(exact) + half a bf16 step at |exact|. Returns (max error beyond the
    half step, RMS)."""
    got = f64(got_bits)
    if not exact.size:
        return 0.0, 0.0
    rms = float(np.sqrt(np.mean(exact ** 2)))
    beyond = np.abs(got - exact) - 0.5 * bf16_ulp(exact)
    err = float(np.max(beyond))
    assert err <= tol * rms + 1e-30, (
        f"{what}: max abs err beyond the bf16 half step {err:.3e} > {tol} * rms {rms:.3e}")
    return err, rms


def expert_rows_sampled(x_rows_bits: np.ndarray, experts: np.ndarray, w13: torch.Tensor,
                        w2: torch.Tensor):
    """Oracle H and Y of rows ``x_rows_bits`` (uint16 [m, d]) routed to ``experts`` (int [m]),
    copying each distinct expert's weights to the host once."""
    m, d = x_rows_bits.shape
    I = w2.shape[2]
    H = np.empty((m, I), np.uint16)
    Y = np.empty((m, d), np.uint16)
    for e in np.unique(experts):
        sel = np.nonzero(experts == e)[0]
        w13e = np_bits(w13[int(e)]).reshape(1, 2 * I, d)
        w2e = np_bits(w2[int(e)]).reshape(1, d, I)
        h, y = oracle.expert_rows(np.ascontiguousarray(x_rows_bits[sel]), np.zeros(sel.size, np.int32),
                                  w13e, w2e)
        H[sel] = h
        Y[sel] = y
    return H, Y


def expert_down_sampled(h_bits: np.ndarray, experts: np.ndarray, w2: torch.Tensor) -> np.ndarray:
    """Oracle down projection Y = bf16(H Wd^T) of given bf16 rows H, one expert at a time."""
    m, I = h_bits.shape
    d = w2.shape[1]
    Y = np.empty((m, d), np.uint16)
    for e in np.unique(experts):
        sel = np.nonzero(experts == e)[0]
        w2e = np_bits(w2[int(e)]).reshape(1, d, I)
        Y[sel] = oracle.expert_down(np.ascontiguousarray(h_bits[sel]), np.zeros(sel.size, np.int32), w2e)
    return Y


def oracle_tokens(x_bits: np.ndarray, tokens: np.ndarray, idx: np.ndarray, gate: np.ndarray, N: int,
                  w13: torch.Tensor, w2: torch.Tensor) -> np.ndarray:
    """Oracle layer output of the given tokens for the given routing (idx/gate [T, K]), as the
    double sums before rounding to bf16."""
    K = idx.shape[1]
    d = x_bits.shape[1]
    pairs = [(t, r) for t in tokens for r in range(K) if idx[t, r] < N]
    rows = np.array([x_bits[t] for t, _ in pairs], np.uint16).reshape(len(pairs), d)
    experts = np.array([idx[t, r] for t, r in pairs], np.int64)
    _, Y = expert_rows_sampled(rows, experts, w13, w2) if pairs else (None, np.zeros((0, d), np.uint16))
    # pair_row into the sampled Y
    pr = np.full((len(tokens), K), -1, np.int32)
    for j, (t, r) in enumerate(pairs):
        pr[list(tokens).index(t), r] = j
    xs = np.ascontiguousarray(x_bits[tokens])
    _, exact = oracle.combine(xs, Y, np.ascontiguousarray(idx[tokens]), np.ascontiguousarray(gate[tokens]),
                              pr, N, want_exact=True)
    return exact


def make(name: str, grid: bool = False, experts: bool = True, **changes):
    w = inputs.WORKLOADS[name]
    if changes:
        w = inputs.scaled(w, **changes)
    d = inputs.make(w, device="cuda", grid=grid, experts=experts)
    d["w"] = w
    return d
