"""CPU oracle for the zero-computation-expert MoE layer and its expert-bias update.

TEST INFRASTRUCTURE. Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU
baseline leg may import this package. It never imports the CUDA package and the CUDA package
never imports it; the two share no code.

Every function is a thin numpy wrapper around ``moe_oracle.c`` (plain C, double accumulation,
explicitly specified fp32 steps), which follows the LongCat-Flash llm-wiki entity page:
section 2.1 (the MoE equation with zero-computation experts E_i(x)=x, and the bias-update
equation of the dynamic computation-budget control), section 2.3.2 (softmax gating) and the
core-parameter table of section 1. bf16 tensors are passed as ``uint16`` arrays of raw bits.
"""
from __future__ import annotations

import ctypes
import numpy as np

from . import build as _build

_LIB = None


def configure(L: ctypes.CDLL) -> ctypes.CDLL:
    """Declare the argument and result types of the oracle's C entry points on a loaded library."""
    P = ctypes.c_void_p
    I64 = ctypes.c_int64
    L.oracle_abi_version.restype = ctypes.c_int
    L.oracle_num_threads.restype = ctypes.c_int
    L.oracle_double_to_bf16.argtypes = [ctypes.c_double]
    L.oracle_double_to_bf16.restype = ctypes.c_uint16
    L.oracle_bf16_to_double.argtypes = [ctypes.c_uint16]
    L.oracle_bf16_to_double.restype = ctypes.c_double
    L.oracle_router_logits.argtypes = [P, P, I64, I64, I64, P]
    L.oracle_exp_spec.argtypes = [ctypes.c_float]
    L.oracle_exp_spec.restype = ctypes.c_float
    L.oracle_sum_spec.argtypes = [P, I64]
    L.oracle_sum_spec.restype = ctypes.c_float
    L.oracle_route.argtypes = [P, P, I64, I64, I64, P, P, P, P]
    L.oracle_route.restype = I64
    L.oracle_permute.argtypes = [P, I64, I64, I64, P, P, P]
    L.oracle_permute.restype = I64
    L.oracle_expert_rows.argtypes = [P, P, I64, I64, I64, P, P, P, P]
    L.oracle_expert_down.argtypes = [P, P, I64, I64, I64, P, P]
    L.oracle_combine.argtypes = [P, P, P, P, P, I64, I64, I64, I64, P, P]
    L.oracle_forward.argtypes = [P, P, P, P, P, I64, I64, I64, I64, I64, I64, P, P, P, P, P, P]
    L.oracle_forward.restype = I64
    L.oracle_bias_update.argtypes = [P, P, I64, I64, I64, I64, I64, ctypes.c_float]
    L.oracle_e4m3_to_double.argtypes = [ctypes.c_uint8]
    L.oracle_e4m3_to_double.restype = ctypes.c_double
    L.oracle_float_to_e4m3.argtypes = [ctypes.c_float]
    L.oracle_float_to_e4m3.restype = ctypes.c_uint8
    L.oracle_quantize_rows_e4m3.argtypes = [P, I64, I64, P, P]
    L.oracle_expert_rows_fp8.argtypes = [P, P, P, I64, I64, I64, P, P, P, P, P, P]
    L.oracle_expert_down_fp8.argtypes = [P, P, I64, I64, I64, P, P, P]
    L.oracle_forward_fp8.argtypes = [P, P, P, P, P, P, P, I64, I64, I64, I64, I64, I64, P, P, P, P, P, P]
    L.oracle_forward_fp8.restype = I64
    return L


def lib() -> ctypes.CDLL:
    global _LIB
    if _LIB is None:
        _LIB = configure(ctypes.CDLL(str(_build.build())))
    return _LIB


def _c(a: np.ndarray, dtype) -> np.ndarray:
    a = np.ascontiguousarray(a)
    if a.dtype != dtype:
        raise TypeError(f"expected {np.dtype(dtype)}, got {a.dtype}")
    return a


def _p(a: np.ndarray | None):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def num_threads() -> int:
    return lib().oracle_num_threads()


# ----------------------------------------------------------------------------------- bf16 --

def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """Raw bf16 bits (uint16) -> float64 values (exact)."""
    u = np.ascontiguousarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return u.view(np.float32).astype(np.float64)


def f64_to_bf16_bits(v) -> np.ndarray:
    """float64 -> nearest bf16 (ties to even), one rounding, as uint16 bits."""
    L = lib()
    flat = np.asarray(v, dtype=np.float64).ravel()
    out = np.fromiter((L.oracle_double_to_bf16(float(a)) for a in flat), dtype=np.uint16,
                      count=flat.size)
    return out.reshape(np.shape(v))


# ------------------------------------------------------------------------------ the steps --

def router_logits(x: np.ndarray, wr: np.ndarray) -> np.ndarray:
    """z[t,i] = sum_j x[t,j] Wr[i,j], accumulated in double and rounded once to fp32."""
    x = _c(x, np.uint16); wr = _c(wr, np.uint16)
    T, d = x.shape
    E = wr.shape[0]
    assert wr.shape == (E, d)
    z = np.empty((T, E), dtype=np.float32)
    lib().oracle_router_logits(_p(x), _p(wr), T, d, E, _p(z))
    return z


def exp_spec(u: float) -> float:
    """The project-specified fp32 exp used by the softmax (Cody-Waite + degree-7 Taylor)."""
    return lib().oracle_exp_spec(ctypes.c_float(u))


def sum_spec(v: np.ndarray) -> float:
    """The project-specified fp32 sum (32 strided partial sums, then an xor butterfly)."""
    v = _c(np.asarray(v, dtype=np.float32), np.float32)
    return lib().oracle_sum_spec(_p(v), v.size)


def route(z: np.ndarray, bias: np.ndarray, K: int, counts: np.ndarray | None = None,
          want_scores: bool = False):
    """Softmax over all experts, top-K of (score + bias), gates renormalised over the K.

    Returns (idx[T,K] int32, gate[T,K] float32, counts[E] int32, n_nan_tokens[, scores]).
    ``counts`` is added to when given (a fresh zero array otherwise)."""
    z = _c(z, np.float32); bias = _c(bias, np.float32)
    T, E = z.shape
    assert bias.shape == (E,) and 0 < K <= E
    idx = np.empty((T, K), dtype=np.int32)
    gate = np.empty((T, K), dtype=np.float32)
    cnt = np.zeros(E, dtype=np.int32) if counts is None else _c(counts, np.int32)
    scores = np.empty((T, E), dtype=np.float32) if want_scores else None
    bad = lib().oracle_route(_p(z), _p(bias), T, E, K, _p(idx), _p(gate), _p(cnt), _p(scores))
    if want_scores:
        return idx, gate, cnt, int(bad), scores
    return idx, gate, cnt, int(bad)


def permute(idx: np.ndarray, N: int):
    """Rows of FFN picks ordered by expert, then token. Returns (offsets[N+1], row_token[M],
    pair_row[T,K]) with pair_row = -1 for zero-computation picks."""
    idx = _c(idx, np.int32)
    T, K = idx.shape
    offsets = np.empty(N + 1, dtype=np.int32)
    row_token = np.empty(T * K, dtype=np.int32)
    pair_row = np.empty((T, K), dtype=np.int32)
    M = lib().oracle_permute(_p(idx), T, K, N, _p(offsets), _p(row_token), _p(pair_row))
    return offsets, row_token[:M].copy(), pair_row


def expert_rows(xrows: np.ndarray, row_expert: np.ndarray, w13: np.ndarray, w2: np.ndarray,
                want_h: bool = True):
    """SwiGLU expert of each row: H = bf16(silu(x Wg^T) * (x Wu^T)), Y = bf16(H Wd^T).

    w13 is [N, 2I, d] (gate rows then up rows), w2 is [N, d, I]. Returns (H[M,I], Y[M,d]) as
    bf16 bits (H is None when ``want_h`` is false)."""
    xrows = _c(xrows, np.uint16); row_expert = _c(row_expert, np.int32)
    w13 = _c(w13, np.uint16); w2 = _c(w2, np.uint16)
    M, d = xrows.shape
    n, two_i, d2 = w13.shape
    I = two_i // 2
    assert d2 == d and w2.shape == (n, d, I) and row_expert.shape == (M,)
    if M and (row_expert.min() < 0 or row_expert.max() >= n):
        raise ValueError("row_expert out of range")
    h = np.empty((M, I), dtype=np.uint16) if want_h else None
    y = np.empty((M, d), dtype=np.uint16)
    lib().oracle_expert_rows(_p(xrows), _p(row_expert), M, d, I, _p(w13), _p(w2), _p(h), _p(y))
    return h, y


def expert_down(h: np.ndarray, row_expert: np.ndarray, w2: np.ndarray) -> np.ndarray:
    """The down projection alone: Y = bf16(H Wd[e]^T) for given bf16 rows H [M, I]."""
    h = _c(h, np.uint16); row_expert = _c(row_expert, np.int32); w2 = _c(w2, np.uint16)
    M, I = h.shape
    n, d, I2 = w2.shape
    assert I2 == I and row_expert.shape == (M,)
    if M and (row_expert.min() < 0 or row_expert.max() >= n):
        raise ValueError("row_expert out of range")
    y = np.empty((M, d), dtype=np.uint16)
    lib().oracle_expert_down(_p(h), _p(row_expert), M, d, I, _p(w2), _p(y))
    return y


def combine(x: np.ndarray, y: np.ndarray, idx: np.ndarray, gate: np.ndarray,
            pair_row: np.ndarray, N: int, want_exact: bool = False):
    """out_t = bf16(sum_r g_r * (Y[pair_row] if FFN pick else x_t)), double, rank order.
    With ``want_exact`` returns (out, the double sums before rounding)."""
    x = _c(x, np.uint16); y = _c(y, np.uint16); idx = _c(idx, np.int32)
    gate = _c(gate, np.float32); pair_row = _c(pair_row, np.int32)
    T, d = x.shape
    K = idx.shape[1]
    out = np.empty((T, d), dtype=np.uint16)
    acc = np.empty((T, d), dtype=np.float64) if want_exact else None
    lib().oracle_combine(_p(x), _p(y), _p(idx), _p(gate), _p(pair_row), T, d, K, N, _p(out), _p(acc))
    return (out, acc) if want_exact else out


def forward(x, wr, bias, w13, w2, N: int, Z: int, K: int, counts: np.ndarray | None = None):
    """The whole layer from the MoE equation. Returns dict(out, out_exact, logits, idx, gate,
    counts, bad); out_exact holds the double sums before their rounding to bf16."""
    x = _c(x, np.uint16); wr = _c(wr, np.uint16); bias = _c(bias, np.float32)
    w13 = _c(w13, np.uint16); w2 = _c(w2, np.uint16)
    T, d = x.shape
    E = N + Z
    I = w2.shape[2]
    assert wr.shape == (E, d) and w13.shape == (N, 2 * I, d) and w2.shape == (N, d, I)
    out = np.empty((T, d), dtype=np.uint16)
    logits = np.empty((T, E), dtype=np.float32)
    idx = np.empty((T, K), dtype=np.int32)
    gate = np.empty((T, K), dtype=np.float32)
    cnt = np.zeros(E, dtype=np.int32) if counts is None else _c(counts, np.int32)
    acc = np.empty((T, d), dtype=np.float64)
    bad = lib().oracle_forward(_p(x), _p(wr), _p(bias), _p(w13), _p(w2), T, d, N, Z, K, I,
                               _p(out), _p(logits), _p(idx), _p(gate), _p(cnt), _p(acc))
    return dict(out=out, out_exact=acc, logits=logits, idx=idx, gate=gate, counts=cnt, bad=int(bad))


def bias_update(bias: np.ndarray, counts: np.ndarray, T_all: int, N: int, Z: int, K: int,
                K_e: int, mu: float) -> np.ndarray:
    """b_i + mu*(K_e/(K N) - T_i/(K T_all)) in fp32, for all N+Z experts (returns a new array)."""
    b = np.array(bias, dtype=np.float32, copy=True)
    counts = _c(counts, np.int32)
    assert b.shape == (N + Z,) and counts.shape == (N + Z,)
    lib().oracle_bias_update(_p(b), _p(counts), T_all, N, Z, K, K_e, ctypes.c_float(mu))
    return b


# ------------------------------------------------------------------------------ FP8 experts --

def e4m3_to_f64(codes) -> np.ndarray:
    """E4M3 codes (uint8) -> float64 values (NaN for the NaN codes)."""
    L = lib()
    table = np.array([L.oracle_e4m3_to_double(c) for c in range(256)], dtype=np.float64)
    return table[np.asarray(codes, dtype=np.uint8)]


def f32_to_e4m3(v) -> np.ndarray:
    """float32 -> nearest E4M3 code, ties to even, saturating at 448 (one rounding)."""
    L = lib()
    flat = np.asarray(v, dtype=np.float32).ravel()
    out = np.fromiter((L.oracle_float_to_e4m3(float(a)) for a in flat), dtype=np.uint8,
                      count=flat.size)
    return out.reshape(np.shape(v))


def quantize_rows_e4m3(src: np.ndarray):
    """Row-wise E4M3 quantisation of bf16 bits [R, C]: s = amax/448 (fp32), q = E4M3(x / s).
    Returns (q uint8 [R, C], s float32 [R])."""
    src = _c(src, np.uint16)
    R, C = src.shape
    q = np.empty((R, C), dtype=np.uint8)
    s = np.empty(R, dtype=np.float32)
    lib().oracle_quantize_rows_e4m3(_p(src), R, C, _p(q), _p(s))
    return q, s


def expert_rows_fp8(xq: np.ndarray, sx: np.ndarray, row_expert: np.ndarray, w13q: np.ndarray,
                    w13_scale: np.ndarray, w2q: np.ndarray, w2_scale: np.ndarray,
                    want_h: bool = True):
    """FP8 SwiGLU expert of each row: gate/up from E4M3 codes with row scales, H rounded to bf16,
    then H quantised per row and the down projection from E4M3 codes. w13q [N, 2I, d] uint8 with
    w13_scale [N, 2I]; w2q [N, d, I] uint8 with w2_scale [N, d]. Returns (H, Y) bf16 bits."""
    xq = _c(xq, np.uint8); sx = _c(sx, np.float32); row_expert = _c(row_expert, np.int32)
    w13q = _c(w13q, np.uint8); w13_scale = _c(w13_scale, np.float32)
    w2q = _c(w2q, np.uint8); w2_scale = _c(w2_scale, np.float32)
    M, d = xq.shape
    n, two_i, d2 = w13q.shape
    I = two_i // 2
    assert d2 == d and w2q.shape == (n, d, I) and w13_scale.shape == (n, two_i)
    assert w2_scale.shape == (n, d) and sx.shape == (M,) and row_expert.shape == (M,)
    if M and (row_expert.min() < 0 or row_expert.max() >= n):
        raise ValueError("row_expert out of range")
    h = np.empty((M, I), dtype=np.uint16) if want_h else None
    y = np.empty((M, d), dtype=np.uint16)
    lib().oracle_expert_rows_fp8(_p(xq), _p(sx), _p(row_expert), M, d, I, _p(w13q), _p(w13_scale),
                                 _p(w2q), _p(w2_scale), _p(h), _p(y))
    return h, y


def expert_down_fp8(h: np.ndarray, row_expert: np.ndarray, w2q: np.ndarray, w2_scale: np.ndarray):
    """The FP8 down projection alone: each bf16 row of H quantised per row, Y = bf16 of the
    scaled E4M3 product with W2 codes w2q [N, d, I] and scales w2_scale [N, d]."""
    h = _c(h, np.uint16); row_expert = _c(row_expert, np.int32)
    w2q = _c(w2q, np.uint8); w2_scale = _c(w2_scale, np.float32)
    M, I = h.shape
    n, d, I2 = w2q.shape
    assert I2 == I and w2_scale.shape == (n, d) and row_expert.shape == (M,)
    if M and (row_expert.min() < 0 or row_expert.max() >= n):
        raise ValueError("row_expert out of range")
    y = np.empty((M, d), dtype=np.uint16)
    lib().oracle_expert_down_fp8(_p(h), _p(row_expert), M, d, I, _p(w2q), _p(w2_scale), _p(y))
    return y


def forward_fp8(x, wr, bias, w13q, w13_scale, w2q, w2_scale, N: int, Z: int, K: int,
                counts: np.ndarray | None = None):
    """The layer with FP8 experts (token rows and H rows quantised per row). Same return value
    as ``forward``."""
    x = _c(x, np.uint16); wr = _c(wr, np.uint16); bias = _c(bias, np.float32)
    w13q = _c(w13q, np.uint8); w13_scale = _c(w13_scale, np.float32)
    w2q = _c(w2q, np.uint8); w2_scale = _c(w2_scale, np.float32)
    T, d = x.shape
    E = N + Z
    I = w2q.shape[2]
    assert wr.shape == (E, d) and w13q.shape == (N, 2 * I, d) and w2q.shape == (N, d, I)
    assert w13_scale.shape == (N, 2 * I) and w2_scale.shape == (N, d)
    out = np.empty((T, d), dtype=np.uint16)
    logits = np.empty((T, E), dtype=np.float32)
    idx = np.empty((T, K), dtype=np.int32)
    gate = np.empty((T, K), dtype=np.float32)
    cnt = np.zeros(E, dtype=np.int32) if counts is None else _c(counts, np.int32)
    acc = np.empty((T, d), dtype=np.float64)
    bad = lib().oracle_forward_fp8(_p(x), _p(wr), _p(bias), _p(w13q), _p(w13_scale), _p(w2q),
                                   _p(w2_scale), T, d, N, Z, K, I, _p(out), _p(logits), _p(idx),
                                   _p(gate), _p(cnt), _p(acc))
    return dict(out=out, out_exact=acc, logits=logits, idx=idx, gate=gate, counts=cnt, bad=int(bad))
