"""ctypes binding of ``libmoezero.so``: the C entry points of ``include/lc_moe.h`` under the same
names, taking torch tensors. Argument marshalling only (shapes, dtypes, data pointers, the current
CUDA stream); every step of the layer runs in the library's CUDA kernels.

The library is loaded on first use. If it has not been built, or the device is not a B200
(sm_100), calls raise: there is no other code path.
"""
from __future__ import annotations

import ctypes
import pathlib
import threading

import torch

_PKG = pathlib.Path(__file__).resolve().parent
LIB_PATH = _PKG / "libmoezero.so"

# return codes and device status bits (include/lc_moe.h)
OK = 0
ERR_INVALID_ARG, ERR_UNSUPPORTED_SHAPE, ERR_WORKSPACE_TOO_SMALL, ERR_NOT_SM100 = 1, 2, 3, 4
ERR_CUDA, ERR_DEVICE_STATUS, ERR_TIMEOUT, ERR_MISALIGNED = 5, 6, 7, 8
DEV_IDX_RANGE, DEV_NAN_KEY, DEV_WAIT_TIMEOUT, DEV_DUP_PICK = 0x1, 0x2, 0x4, 0x8
OP_FORWARD, OP_ROUTE, OP_PERMUTE, OP_STATUS, OP_FORWARD_FP8 = 0, 1, 2, 3, 4
NUM_STAGES = 7
STAGE_NAMES = ("router_gemm", "topk", "permute", "gather", "gemm1_swiglu", "gemm2_down", "combine")

EXPORTED = (
    "lc_moe_abi_version", "lc_moe_strerror", "lc_moe_workspace_bytes", "lc_moe_set_wait_limit_ns",
    "lc_moe_forward", "lc_moe_forward_timed", "lc_moe_route", "lc_moe_bias_update",
    "lc_moe_read_status", "lc_moe_router_logits", "lc_moe_topk", "lc_moe_expert_hist",
    "lc_moe_permute", "lc_moe_expert_ffn", "lc_moe_combine", "lc_moe_permute_noalloc",
    "lc_moe_quantize_e4m3", "lc_moe_forward_fp8", "lc_moe_forward_fp8_timed",
    "lc_moe_check_wait_timeout", "lc_moe_ep_regroup_plan", "lc_moe_copy_rows", "lc_moe_set_clock_probe",
)


class Shape(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int32), ("d", ctypes.c_int32), ("N", ctypes.c_int32),
                ("Z", ctypes.c_int32), ("K", ctypes.c_int32), ("I", ctypes.c_int32)]


class LcMoeError(RuntimeError):
    def __init__(self, code: int, what: str = ""):
        self.code = code
        msg = _lib().lc_moe_strerror(code).decode()
        super().__init__(f"{what}: {msg} (code {code})" if what else f"{msg} (code {code})")


_LIB = None
_LOCK = threading.Lock()


def _lib() -> ctypes.CDLL:
    global _LIB
    if _LIB is None:
        with _LOCK:
            if _LIB is None:
                if not LIB_PATH.exists():
                    raise RuntimeError(
                        f"{LIB_PATH} is not built; run `python -m mixture_experts_zero_b200.build`")
                _LIB = _configure(ctypes.CDLL(str(LIB_PATH)))
    return _LIB


def _configure(L: ctypes.CDLL) -> ctypes.CDLL:
    P, I32, I64, SZ = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
    SP = ctypes.POINTER(Shape)
    L.lc_moe_abi_version.restype = I32
    L.lc_moe_strerror.argtypes = [ctypes.c_int]
    L.lc_moe_strerror.restype = ctypes.c_char_p
    L.lc_moe_workspace_bytes.argtypes = [SP, ctypes.c_int]
    L.lc_moe_workspace_bytes.restype = SZ
    L.lc_moe_set_wait_limit_ns.argtypes = [ctypes.c_uint64]
    L.lc_moe_set_wait_limit_ns.restype = None
    L.lc_moe_set_clock_probe.argtypes = [P]
    L.lc_moe_set_clock_probe.restype = None
    fwd = [SP, P, P, P, P, P, P, P, P, P, P, SZ, P]
    L.lc_moe_forward.argtypes = fwd
    L.lc_moe_forward_timed.argtypes = fwd + [ctypes.POINTER(P)]
    L.lc_moe_route.argtypes = [SP, P, P, P, P, P, P, P, P, SZ, P]
    L.lc_moe_bias_update.argtypes = [P, P, I64, I32, I32, I32, I32, ctypes.c_float, I32, P]
    L.lc_moe_read_status.argtypes = [P, ctypes.POINTER(ctypes.c_uint32), P]
    L.lc_moe_router_logits.argtypes = [SP, P, P, P, P, SZ, P]
    L.lc_moe_topk.argtypes = [SP, P, P, P, P, P, P, SZ, P]
    L.lc_moe_expert_hist.argtypes = [P, I64, I32, P, P, SZ, P]
    L.lc_moe_permute.argtypes = [SP, P, P, P, P, P, P, P, SZ, P]
    L.lc_moe_expert_ffn.argtypes = [SP, P, P, P, P, P, P, P, SZ, P]
    L.lc_moe_combine.argtypes = [SP, P, P, P, P, P, P, SZ, P]
    L.lc_moe_permute_noalloc.argtypes = [SP, P, P, P, P, P, P, P, P]
    L.lc_moe_quantize_e4m3.argtypes = [P, I64, I32, P, P, P]
    fwd8 = [SP, P, P, P, P, P, P, P, P, P, P, P, P, SZ, P]
    L.lc_moe_forward_fp8.argtypes = fwd8
    L.lc_moe_forward_fp8_timed.argtypes = fwd8 + [ctypes.POINTER(P)]
    L.lc_moe_check_wait_timeout.argtypes = [P, SZ, P]
    L.lc_moe_ep_regroup_plan.argtypes = [P, I32, I32, P, I64, P, P, SZ, P]
    L.lc_moe_copy_rows.argtypes = [P, P, P, I64, I32, I32, P, SZ, P]
    return L


def library() -> ctypes.CDLL:
    """The loaded ``libmoezero.so`` (raises if it is not built)."""
    return _lib()


# ------------------------------------------------------------------------------- helpers --

def _ptr(t: torch.Tensor | None):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _need(t: torch.Tensor, dtype, shape, name):
    if t.dtype != dtype:
        raise TypeError(f"{name}: expected {dtype}, got {t.dtype}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: expected shape {tuple(shape)}, got {tuple(t.shape)}")
    if not t.is_cuda or not t.is_contiguous():
        raise ValueError(f"{name}: expected a contiguous CUDA tensor")


def _check(rc: int, what: str):
    if rc != OK:
        raise LcMoeError(rc, what)


def shape_of(T: int, d: int, N: int, Z: int, K: int, I: int) -> Shape:
    return Shape(T, d, N, Z, K, I)


def lc_moe_workspace_bytes(shape: Shape, op: int = OP_FORWARD) -> int:
    return int(_lib().lc_moe_workspace_bytes(ctypes.byref(shape), op))


def new_workspace(shape: Shape, op: int = OP_FORWARD, device=None) -> torch.Tensor:
    """A zero-filled workspace (uint8 CUDA tensor) for entry point ``op`` and ``shape``."""
    n = lc_moe_workspace_bytes(shape, op)
    if n == 0:
        raise LcMoeError(ERR_UNSUPPORTED_SHAPE, "lc_moe_workspace_bytes")
    return torch.zeros(n, dtype=torch.uint8, device=device or "cuda")


def lc_moe_set_wait_limit_ns(limit_ns: int) -> None:
    _lib().lc_moe_set_wait_limit_ns(int(limit_ns))


def lc_moe_set_clock_probe(probe) -> None:
    """probe: int64 device tensor of 8 elements (GEMM 1: start ns, start cycles, end ns, end
    cycles of CTA 0; GEMM 2 the same), or None to stop."""
    if probe is not None:
        assert probe.is_cuda and probe.dtype == torch.int64 and probe.numel() >= 8 and probe.is_contiguous()
    _lib().lc_moe_set_clock_probe(None if probe is None else _ptr(probe))


def _dims(x, wr, w13=None, w2=None, K=None):
    T, d = x.shape
    E = wr.shape[0]
    if w13 is not None:
        N, two_i, _ = w13.shape
        I = two_i // 2
    else:
        N, I = None, None
    return T, d, E, N, I


# ---------------------------------------------------------------------------- entry points --

def lc_moe_forward(x, wr, bias, w13, w2, K: int, out=None, idx=None, gate=None, counts=None,
                   ws=None, stream=None, events=None):
    """MoE(x) with N = w13.shape[0] FFN experts and Z = wr.shape[0] - N zero experts.
    Returns ``out`` [T, d] bf16. ``counts`` (int32 [E]) is added to when given."""
    T, d, E, N, I = _dims(x, wr, w13)
    Z = E - N
    _need(x, torch.bfloat16, (T, d), "x")
    _need(wr, torch.bfloat16, (E, d), "wr")
    _need(bias, torch.float32, (E,), "bias")
    _need(w13, torch.bfloat16, (N, 2 * I, d), "w13")
    _need(w2, torch.bfloat16, (N, d, I), "w2")
    if out is None:
        out = torch.empty(T, d, dtype=torch.bfloat16, device=x.device)
    _need(out, torch.bfloat16, (T, d), "out")
    if idx is not None:
        _need(idx, torch.int32, (T, K), "idx")
    if gate is not None:
        _need(gate, torch.float32, (T, K), "gate")
    if counts is not None:
        _need(counts, torch.int32, (E,), "counts")
    s = Shape(T, d, N, Z, K, I)
    if ws is None:
        ws = new_workspace(s, OP_FORWARD, x.device)
    args = [ctypes.byref(s), _ptr(x), _ptr(wr), _ptr(bias), _ptr(w13), _ptr(w2), _ptr(out),
            _ptr(idx), _ptr(gate), _ptr(counts), _ptr(ws), ws.numel(), _stream(stream)]
    if events is None:
        _check(_lib().lc_moe_forward(*args), "lc_moe_forward")
    else:
        _check(_lib().lc_moe_forward_timed(*args, _event_array(events)), "lc_moe_forward_timed")
    return out


def _event_array(events):
    if len(events) != NUM_STAGES + 1:
        raise ValueError(f"events: need {NUM_STAGES + 1} CUDA events")
    for e in events:
        if not e.cuda_event:  # torch creates the CUDA event lazily, on its first record
            e.record()
    return (ctypes.c_void_p * len(events))(*[ctypes.c_void_p(e.cuda_event) for e in events])


def lc_moe_quantize_e4m3(src, dst=None, scale=None, stream=None):
    """Row-wise E4M3 quantisation of a bf16 matrix [R, C] (any leading shape, rows = all but the
    last dimension). Returns (codes uint8, same shape; scale float32 [R...])."""
    if src.dtype != torch.bfloat16 or not src.is_cuda or not src.is_contiguous():
        raise ValueError("src: expected a contiguous bf16 CUDA tensor")
    C = src.shape[-1]
    R = src.numel() // C if C else 0
    if dst is None:
        dst = torch.empty(src.shape, dtype=torch.uint8, device=src.device)
    if scale is None:
        scale = torch.empty(src.shape[:-1], dtype=torch.float32, device=src.device)
    _need(dst, torch.uint8, tuple(src.shape), "dst")
    _need(scale, torch.float32, tuple(src.shape[:-1]), "scale")
    _check(_lib().lc_moe_quantize_e4m3(_ptr(src), R, C, _ptr(dst), _ptr(scale), _stream(stream)),
           "lc_moe_quantize_e4m3")
    return dst, scale


def lc_moe_forward_fp8(x, wr, bias, w13q, w13_scale, w2q, w2_scale, K: int, out=None, idx=None,
                       gate=None, counts=None, ws=None, stream=None, events=None):
    """MoE(x) with E4M3 experts: w13q [N, 2I, d] / w2q [N, d, I] uint8 codes with row scales
    w13_scale [N, 2I] / w2_scale [N, d] float32 (from lc_moe_quantize_e4m3). Returns ``out``
    [T, d] bf16."""
    T, d = x.shape
    E = wr.shape[0]
    N, two_i, _ = w13q.shape
    I = two_i // 2
    _need(x, torch.bfloat16, (T, d), "x")
    _need(wr, torch.bfloat16, (E, d), "wr")
    _need(bias, torch.float32, (E,), "bias")
    _need(w13q, torch.uint8, (N, 2 * I, d), "w13q")
    _need(w13_scale, torch.float32, (N, 2 * I), "w13_scale")
    _need(w2q, torch.uint8, (N, d, I), "w2q")
    _need(w2_scale, torch.float32, (N, d), "w2_scale")
    if out is None:
        out = torch.empty(T, d, dtype=torch.bfloat16, device=x.device)
    _need(out, torch.bfloat16, (T, d), "out")
    if idx is not None:
        _need(idx, torch.int32, (T, K), "idx")
    if gate is not None:
        _need(gate, torch.float32, (T, K), "gate")
    if counts is not None:
        _need(counts, torch.int32, (E,), "counts")
    s = Shape(T, d, N, E - N, K, I)
    if ws is None:
        ws = new_workspace(s, OP_FORWARD_FP8, x.device)
    args = [ctypes.byref(s), _ptr(x), _ptr(wr), _ptr(bias), _ptr(w13q), _ptr(w13_scale), _ptr(w2q),
            _ptr(w2_scale), _ptr(out), _ptr(idx), _ptr(gate), _ptr(counts), _ptr(ws), ws.numel(),
            _stream(stream)]
    if events is None:
        _check(_lib().lc_moe_forward_fp8(*args), "lc_moe_forward_fp8")
    else:
        _check(_lib().lc_moe_forward_fp8_timed(*args, _event_array(events)), "lc_moe_forward_fp8_timed")
    return out


def lc_moe_route(x, wr, bias, K: int, N: int, idx=None, gate=None, counts=None, logits=None,
                 ws=None, stream=None):
    """Router GEMM + softmax + biased top-K (+ histogram). Returns (idx, gate)."""
    T, d = x.shape
    E = wr.shape[0]
    _need(x, torch.bfloat16, (T, d), "x")
    _need(wr, torch.bfloat16, (E, d), "wr")
    _need(bias, torch.float32, (E,), "bias")
    if idx is None:
        idx = torch.empty(T, K, dtype=torch.int32, device=x.device)
    if gate is None:
        gate = torch.empty(T, K, dtype=torch.float32, device=x.device)
    _need(idx, torch.int32, (T, K), "idx")
    _need(gate, torch.float32, (T, K), "gate")
    if counts is not None:
        _need(counts, torch.int32, (E,), "counts")
    if logits is not None:
        _need(logits, torch.float32, (T, E), "logits")
    s = Shape(T, d, N, E - N, K, 64)
    if ws is None:
        ws = new_workspace(s, OP_ROUTE, x.device)
    _check(_lib().lc_moe_route(ctypes.byref(s), _ptr(x), _ptr(wr), _ptr(bias), _ptr(idx), _ptr(gate),
                               _ptr(counts), _ptr(logits), _ptr(ws), ws.numel(), _stream(stream)),
           "lc_moe_route")
    return idx, gate


def lc_moe_bias_update(bias, counts, T_all: int, N: int, Z: int, K: int, K_e: int, mu: float,
                       reset_counts: bool = False, stream=None):
    """b_i += mu * (K_e/(K N) - T_i/(K T_all)) in place on the device (all N + Z experts)."""
    _need(bias, torch.float32, (N + Z,), "bias")
    _need(counts, torch.int32, (N + Z,), "counts")
    _check(_lib().lc_moe_bias_update(_ptr(bias), _ptr(counts), int(T_all), N, Z, K, K_e,
                                     ctypes.c_float(mu), int(bool(reset_counts)), _stream(stream)),
           "lc_moe_bias_update")
    return bias


def lc_moe_check_wait_timeout(ws=None, stream=None):
    """Enqueue the device check of the bounded waits (gives up after the current wait limit and
    sets LC_MOE_DEV_WAIT_TIMEOUT in ws's status word). Returns the workspace."""
    if ws is None:
        ws = new_workspace(Shape(1, 64, 1, 0, 1, 64), OP_STATUS)
    _check(_lib().lc_moe_check_wait_timeout(_ptr(ws), ws.numel(), _stream(stream)),
           "lc_moe_check_wait_timeout")
    return ws


def lc_moe_read_status(ws, stream=None, raise_on_error: bool = True) -> int:
    """Synchronise, read and clear the workspace's device status word; return its bits."""
    v = ctypes.c_uint32(0)
    rc = _lib().lc_moe_read_status(_ptr(ws), ctypes.byref(v), _stream(stream))
    if raise_on_error and rc != OK:
        raise LcMoeError(rc, f"device status 0x{v.value:x}")
    return int(v.value)


def lc_moe_router_logits(x, wr, logits=None, ws=None, stream=None):
    T, d = x.shape
    E = wr.shape[0]
    _need(x, torch.bfloat16, (T, d), "x")
    _need(wr, torch.bfloat16, (E, d), "wr")
    if logits is None:
        logits = torch.empty(T, E, dtype=torch.float32, device=x.device)
    _need(logits, torch.float32, (T, E), "logits")
    s = Shape(T, d, E, 0, 1, 64)
    if ws is None:
        ws = new_workspace(s, OP_STATUS, x.device)
    _check(_lib().lc_moe_router_logits(ctypes.byref(s), _ptr(x), _ptr(wr), _ptr(logits), _ptr(ws),
                                       ws.numel(), _stream(stream)), "lc_moe_router_logits")
    return logits


def lc_moe_topk(logits, bias, K: int, N: int, idx=None, gate=None, counts=None, ws=None,
                stream=None):
    T, E = logits.shape
    _need(logits, torch.float32, (T, E), "logits")
    _need(bias, torch.float32, (E,), "bias")
    if idx is None:
        idx = torch.empty(T, K, dtype=torch.int32, device=logits.device)
    if gate is None:
        gate = torch.empty(T, K, dtype=torch.float32, device=logits.device)
    _need(idx, torch.int32, (T, K), "idx")
    _need(gate, torch.float32, (T, K), "gate")
    if counts is not None:
        _need(counts, torch.int32, (E,), "counts")
    s = Shape(T, 64, N, E - N, K, 64)
    if ws is None:
        ws = new_workspace(s, OP_STATUS, logits.device)
    _check(_lib().lc_moe_topk(ctypes.byref(s), _ptr(logits), _ptr(bias), _ptr(idx), _ptr(gate),
                              _ptr(counts), _ptr(ws), ws.numel(), _stream(stream)), "lc_moe_topk")
    return idx, gate


def lc_moe_expert_hist(idx, n_bins: int, counts=None, ws=None, stream=None):
    if idx.dtype != torch.int32 or not idx.is_cuda or not idx.is_contiguous():
        raise ValueError("idx: expected a contiguous int32 CUDA tensor")
    if counts is None:
        counts = torch.zeros(n_bins, dtype=torch.int32, device=idx.device)
    _need(counts, torch.int32, (n_bins,), "counts")
    if ws is None:
        ws = torch.zeros(256, dtype=torch.uint8, device=idx.device)
    _check(_lib().lc_moe_expert_hist(_ptr(idx), idx.numel(), n_bins, _ptr(counts), _ptr(ws),
                                     ws.numel(), _stream(stream)), "lc_moe_expert_hist")
    return counts


def lc_moe_permute(idx, N: int, E: int, x=None, d: int = 64, want_rows: bool = True, ws=None,
                   stream=None):
    """Group FFN picks by expert. Returns (offsets[N+1], row_token[T*K], pair_row[T,K], x_perm or None)."""
    T, K = idx.shape
    _need(idx, torch.int32, (T, K), "idx")
    dev = idx.device
    if x is not None:
        d = x.shape[1]
        _need(x, torch.bfloat16, (T, d), "x")
    offsets = torch.empty(N + 1, dtype=torch.int32, device=dev)
    row_token = torch.empty(T * K, dtype=torch.int32, device=dev)
    pair_row = torch.empty(T, K, dtype=torch.int32, device=dev)
    x_perm = torch.empty(T * K, d, dtype=torch.bfloat16, device=dev) if (x is not None and want_rows) else None
    s = Shape(T, d, N, E - N, K, 64)
    if ws is None:
        ws = new_workspace(s, OP_PERMUTE, dev)
    _check(_lib().lc_moe_permute(ctypes.byref(s), _ptr(idx), _ptr(x), _ptr(offsets), _ptr(row_token),
                                 _ptr(pair_row), _ptr(x_perm), _ptr(ws), ws.numel(), _stream(stream)),
           "lc_moe_permute")
    return offsets, row_token, pair_row, x_perm


def lc_moe_expert_ffn(x_perm, offsets, w13, w2, T: int, K: int, h=None, y=None, ws=None,
                      stream=None):
    """Grouped SwiGLU experts over rows grouped by lc_moe_permute. Returns (h, y)."""
    N, two_i, d = w13.shape
    I = two_i // 2
    rows = T * K
    _need(x_perm, torch.bfloat16, (rows, d), "x_perm")
    _need(offsets, torch.int32, (N + 1,), "offsets")
    _need(w13, torch.bfloat16, (N, 2 * I, d), "w13")
    _need(w2, torch.bfloat16, (N, d, I), "w2")
    if h is None:
        h = torch.empty(rows, I, dtype=torch.bfloat16, device=x_perm.device)
    if y is None:
        y = torch.empty(rows, d, dtype=torch.bfloat16, device=x_perm.device)
    _need(h, torch.bfloat16, (rows, I), "h")
    _need(y, torch.bfloat16, (rows, d), "y")
    s = Shape(T, d, N, max(0, K - N), K, I)
    if ws is None:
        ws = new_workspace(s, OP_STATUS, x_perm.device)
    _check(_lib().lc_moe_expert_ffn(ctypes.byref(s), _ptr(x_perm), _ptr(offsets), _ptr(w13), _ptr(w2),
                                    _ptr(h), _ptr(y), _ptr(ws), ws.numel(), _stream(stream)),
           "lc_moe_expert_ffn")
    return h, y


def lc_moe_combine(x, y, gate, pair_row, out=None, ws=None, stream=None):
    T, d = x.shape
    K = gate.shape[1]
    _need(x, torch.bfloat16, (T, d), "x")
    _need(gate, torch.float32, (T, K), "gate")
    _need(pair_row, torch.int32, (T, K), "pair_row")
    if y.dtype != torch.bfloat16 or y.dim() != 2 or y.shape[1] != d or not y.is_contiguous():
        raise ValueError("y: expected a contiguous bf16 [rows, d] tensor")
    if out is None:
        out = torch.empty(T, d, dtype=torch.bfloat16, device=x.device)
    _need(out, torch.bfloat16, (T, d), "out")
    s = Shape(T, d, 1, K, K, 64)
    if ws is None:
        ws = new_workspace(s, OP_STATUS, x.device)
    _check(_lib().lc_moe_combine(ctypes.byref(s), _ptr(x), _ptr(y), _ptr(gate), _ptr(pair_row),
                                 _ptr(out), _ptr(ws), ws.numel(), _stream(stream)), "lc_moe_combine")
    return out


def lc_moe_permute_noalloc(idx, N: int, E: int, x=None, d: int = 64, want_rows: bool = True,
                           status=None, stream=None):
    """lc_moe_permute without a workspace (the library's own fixed-size tables; see the header).
    Returns (offsets[N+1], row_token[T*K], pair_row[T,K], x_perm or None). ``status`` is an
    optional int32 CUDA tensor of one element that receives device status bits."""
    T, K = idx.shape
    _need(idx, torch.int32, (T, K), "idx")
    dev = idx.device
    if x is not None:
        d = x.shape[1]
        _need(x, torch.bfloat16, (T, d), "x")
    if status is not None:
        _need(status, torch.int32, (1,), "status")
    offsets = torch.empty(N + 1, dtype=torch.int32, device=dev)
    row_token = torch.empty(T * K, dtype=torch.int32, device=dev)
    pair_row = torch.empty(T, K, dtype=torch.int32, device=dev)
    x_perm = torch.empty(T * K, d, dtype=torch.bfloat16, device=dev) if (x is not None and want_rows) else None
    s = Shape(T, d, N, E - N, K, 64)
    _check(_lib().lc_moe_permute_noalloc(ctypes.byref(s), _ptr(idx), _ptr(x), _ptr(offsets),
                                         _ptr(row_token), _ptr(pair_row), _ptr(x_perm), _ptr(status),
                                         _stream(stream)), "lc_moe_permute_noalloc")
    return offsets, row_token, pair_row, x_perm


# ------------------------------------------------------------------- expert parallelism --

def _status_ws(device):
    return new_workspace(Shape(1, 64, 1, 0, 1, 64), OP_STATUS, device)


def lc_moe_ep_regroup_plan(cnt, m_cap: int | None = None, perm=None, offsets=None, ws=None, stream=None):
    """Expert-major order of rows received source-major. ``cnt`` int32 [G, n_local] (device):
    rows source s sent for local expert e. Returns (perm [M] int32, offsets [n_local + 1] int32)
    with M = cnt.sum() (m_cap, when given, is the length of ``perm``)."""
    if cnt.dtype != torch.int32 or cnt.dim() != 2 or not cnt.is_cuda or not cnt.is_contiguous():
        raise ValueError("cnt: expected a contiguous int32 CUDA tensor [G, n_local]")
    G, n_local = cnt.shape
    if m_cap is None:
        m_cap = int(cnt.sum().item())
    if perm is None:
        perm = torch.empty(max(m_cap, 1), dtype=torch.int32, device=cnt.device)
    if offsets is None:
        offsets = torch.empty(n_local + 1, dtype=torch.int32, device=cnt.device)
    _need(offsets, torch.int32, (n_local + 1,), "offsets")
    if ws is None:
        ws = _status_ws(cnt.device)
    _check(_lib().lc_moe_ep_regroup_plan(_ptr(cnt), G, n_local, _ptr(perm), int(m_cap), _ptr(offsets),
                                         _ptr(ws), ws.numel(), _stream(stream)), "lc_moe_ep_regroup_plan")
    return perm[:m_cap], offsets


def lc_moe_copy_rows(src, index, scatter: bool = False, out=None, ws=None, stream=None):
    """Rows of ``src`` [n, ...] moved through the permutation ``index`` [n] int32:
    out[i] = src[index[i]] (gather) or out[index[i]] = src[i] (scatter)."""
    n = index.shape[0]
    if src.shape[0] < n or not src.is_cuda or not src.is_contiguous():
        raise ValueError("src: expected a contiguous CUDA tensor with at least len(index) rows")
    _need(index, torch.int32, (n,), "index")
    row_bytes = src[0].numel() * src.element_size() if src.shape[0] else 16
    if out is None:
        out = torch.empty((n,) + tuple(src.shape[1:]), dtype=src.dtype, device=src.device)
    if ws is None:
        ws = _status_ws(src.device)
    _check(_lib().lc_moe_copy_rows(_ptr(src), _ptr(out), _ptr(index), n, row_bytes, 1 if scatter else 0,
                                   _ptr(ws), ws.numel(), _stream(stream)), "lc_moe_copy_rows")
    return out
