"""The C-ABI library without a GPU: it loads, exports every entry point include/lc_moe.h declares,
and its host-side checks reject bad arguments before any CUDA call."""
import ctypes
import pathlib
import re

import pytest

from mixture_experts_zero_b200 import binding, build

HEADER = pathlib.Path(__file__).resolve().parent.parent / "include" / "lc_moe.h"


@pytest.fixture(scope="module")
def lib():
    build.build()
    return binding.library()


def declared_functions():
    text = HEADER.read_text()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(lc_moe_\w+)\s*\(", text)))


def test_header_declares_the_documented_entry_points():
    names = declared_functions()
    for must in ["lc_moe_route", "lc_moe_forward", "lc_moe_bias_update", "lc_moe_read_status",
                 "lc_moe_workspace_bytes", "lc_moe_strerror"]:
        assert must in names
    assert set(names) == set(binding.EXPORTED)


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name
    assert lib.lc_moe_abi_version() == 1


def test_strerror_covers_codes(lib):
    for code in range(0, 9):
        assert lib.lc_moe_strerror(code).decode() != "unknown error code"
    assert lib.lc_moe_strerror(99).decode() == "unknown error code"


def ws_bytes(T, d, N, Z, K, I, op=binding.OP_FORWARD):
    return binding.lc_moe_workspace_bytes(binding.Shape(T, d, N, Z, K, I), op)


def test_workspace_sizes(lib):
    # LongCat-Flash prefill shape: logits, routing records, grouping tables and 3 row buffers
    T, d, N, Z, K, I = 16384, 6144, 512, 256, 12, 2048
    fwd = ws_bytes(T, d, N, Z, K, I)
    rows = T * K
    assert fwd >= T * (N + Z) * 4 + rows * (2 * d + I) * 2
    assert fwd < T * (N + Z) * 4 + rows * (2 * d + I) * 2 + 64 * 2 ** 20
    assert ws_bytes(T, d, N, Z, K, I, binding.OP_ROUTE) >= 256 + T * (N + Z) * 4
    assert ws_bytes(T, d, N, Z, K, I, binding.OP_STATUS) == 256
    assert ws_bytes(T, d, N, Z, K, I, binding.OP_PERMUTE) >= 256 + 2 * (T // 256) * N * 4
    # rows are capped by the number of FFN experts when N < K
    small_n = ws_bytes(64, 128, 2, 10, 8, 64)
    assert small_n < ws_bytes(64, 128, 8, 4, 8, 64)


@pytest.mark.parametrize("shape", [
    (16, 100, 8, 4, 3, 64),    # d not a multiple of 64
    (16, 128, 8, 4, 3, 96),    # I not a multiple of 64
    (16, 128, 8, 4, 33, 64),   # K > 32
    (16, 128, 2, 0, 3, 64),    # K > N + Z
    (16, 128, 2000, 100, 3, 64),  # N + Z > 2048
    (-1, 128, 8, 4, 3, 64),    # T < 0
    (16, 128, 0, 4, 3, 64),    # no FFN expert
])
def test_unsupported_shapes_are_rejected_on_the_host(lib, shape):
    s = binding.Shape(*shape)
    assert lib.lc_moe_workspace_bytes(ctypes.byref(s), 0) == 0
    p = ctypes.c_void_p(256)
    rc = lib.lc_moe_forward(ctypes.byref(s), p, p, p, p, p, p, None, None, None, p, 1 << 40, None)
    assert rc == binding.ERR_UNSUPPORTED_SHAPE


def test_argument_checks_precede_any_cuda_call(lib):
    s = binding.Shape(16, 128, 8, 4, 3, 64)
    p = ctypes.c_void_p(256)
    need = lib.lc_moe_workspace_bytes(ctypes.byref(s), 0)
    # null required buffer
    assert lib.lc_moe_forward(ctypes.byref(s), None, p, p, p, p, p, None, None, None, p, need, None) == binding.ERR_INVALID_ARG
    # workspace too small
    assert lib.lc_moe_forward(ctypes.byref(s), p, p, p, p, p, p, None, None, None, p, need - 1, None) == binding.ERR_WORKSPACE_TOO_SMALL
    # misaligned pointer
    q = ctypes.c_void_p(264)
    assert lib.lc_moe_forward(ctypes.byref(s), q, p, p, p, p, p, None, None, None, p, need, None) == binding.ERR_MISALIGNED
    # T = 0 is a no-op that needs no device
    s0 = binding.Shape(0, 128, 8, 4, 3, 64)
    assert lib.lc_moe_forward(ctypes.byref(s0), p, p, p, p, p, p, None, None, None, p, 1 << 20, None) == 0
    # bias update scalars
    assert lib.lc_moe_bias_update(p, p, 0, 8, 4, 3, 2, ctypes.c_float(1e-3), 0, None) == binding.ERR_INVALID_ARG
    assert lib.lc_moe_bias_update(p, p, 64, 8, 4, 3, 4, ctypes.c_float(1e-3), 0, None) == binding.ERR_INVALID_ARG
    assert lib.lc_moe_bias_update(p, p, 64, 8, 4, 3, 2, ctypes.c_float(float("nan")), 0, None) == binding.ERR_INVALID_ARG
    assert lib.lc_moe_expert_hist(p, 10, 0, p, p, 256, None) == binding.ERR_INVALID_ARG
    assert lib.lc_moe_read_status(None, None, None) == binding.ERR_INVALID_ARG
    assert lib.lc_moe_check_wait_timeout(None, 256, None) == binding.ERR_INVALID_ARG
    assert lib.lc_moe_check_wait_timeout(p, 255, None) == binding.ERR_WORKSPACE_TOO_SMALL
    assert lib.lc_moe_check_wait_timeout(q, 256, None) == binding.ERR_MISALIGNED


def test_valid_call_without_a_device_reports_a_cuda_error(lib):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a device is present")
    s = binding.Shape(16, 128, 8, 4, 3, 64)
    p = ctypes.c_void_p(256)
    need = lib.lc_moe_workspace_bytes(ctypes.byref(s), 0)
    assert lib.lc_moe_forward(ctypes.byref(s), p, p, p, p, p, p, None, None, None, p, need, None) == binding.ERR_CUDA
    assert lib.lc_moe_check_wait_timeout(p, 256, None) == binding.ERR_CUDA


def test_the_cuda_package_never_imports_the_oracle():
    pkg = pathlib.Path(binding.__file__).resolve().parent
    for f in list(pkg.rglob("*.py")) + list(pkg.rglob("*.cu")) + list(pkg.rglob("*.cuh")):
        text = f.read_text()
        assert "import oracle" not in text and "from oracle" not in text, f
        assert "moe_oracle" not in text, f


def test_clock_probe_setting_needs_no_device_and_checks_its_buffer(lib):
    """The probe is a process-wide pointer the library stores (no CUDA call): setting and clearing
    it works without a GPU, and the binding refuses a buffer that is not 8 int64 on the device."""
    import torch
    binding.lc_moe_set_clock_probe(None)
    with pytest.raises(AssertionError):
        binding.lc_moe_set_clock_probe(torch.zeros(8, dtype=torch.int64))  # host memory
    lib.lc_moe_set_clock_probe(ctypes.c_void_p(0x1000))
    lib.lc_moe_set_clock_probe(None)
