"""The allocation-free grouping entry point, lc_moe_permute_noalloc, against lc_moe_permute and
against the CPU oracle's grouping.

Some callers cannot allocate device memory: an engine whose memory planner hands out all device
memory up front and refuses later requests, or a caller with no workspace of its own to pass.
For them lc_moe_permute_noalloc keeps the grouping tables in a fixed-size array inside the
library. Its results must equal lc_moe_permute's bit for bit (integer tables and row copies are
exact), on two calls in a row with different shapes, so the second call cannot depend on what the
first one left in the shared array. Its integer tables must also equal the oracle's grouping
(FFN picks ordered by expert, then by token), which shares no code with either GPU path.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from mixture_experts_zero_b200 import binding as B
from mixture_experts_zero_b200 import inputs

pytestmark = pytest.mark.gpu


def _cases():
    # 1) the small workload, routed by the library itself
    w = inputs.WORKLOADS["small"]
    d = inputs.make(w, device="cuda", experts=False)
    idx, _ = B.lc_moe_route(d["x"], d["wr"], d["bias"], w.K, w.N)
    yield idx, w.N, w.E, d["x"]
    # 2) the LongCat-Flash routing width with a ragged token count: distinct random picks
    T, N, E, K, dm = 1000, 512, 768, 12, 256
    g = torch.Generator(device="cuda")
    g.manual_seed(11)
    idx = torch.rand(T, E, generator=g, device="cuda").argsort(dim=1)[:, :K].to(torch.int32).contiguous()
    x = torch.randn(T, dm, generator=g, device="cuda").to(torch.bfloat16)
    yield idx, N, E, x


def test_noalloc_grouping_equals_workspace_grouping_on_two_calls(cuda_device):
    for idx, N, E, x in _cases():
        status = torch.zeros(1, dtype=torch.int32, device="cuda")
        got = B.lc_moe_permute_noalloc(idx, N, E, x=x, status=status)
        want = B.lc_moe_permute(idx, N, E, x=x)
        torch.cuda.synchronize()
        M = int(want[0][-1])
        assert torch.equal(got[0], want[0])                    # offsets
        assert torch.equal(got[1][:M], want[1][:M])            # row -> token
        assert torch.equal(got[2], want[2])                    # pick -> row
        assert torch.equal(got[3][:M], want[3][:M])            # grouped rows
        assert int(status.item()) == 0
        assert 0 < M < idx.numel()
        # the oracle's grouping of the same picks: offsets, row -> token, pick -> row
        o_off, o_row_token, o_pair_row = oracle.permute(idx.cpu().numpy(), N)
        assert np.array_equal(got[0].cpu().numpy(), o_off)
        assert np.array_equal(got[1][:M].cpu().numpy(), o_row_token)
        assert np.array_equal(got[2].cpu().numpy(), o_pair_row)
        # grouped rows are the token rows named by the oracle's row -> token table
        xb = inputs.bits(x)
        assert np.array_equal(inputs.bits(got[3][:M]), xb[o_row_token])


def test_noalloc_grouping_rejects_shapes_beyond_its_capacity(cuda_device):
    L = B.library()
    # ceil(70000 / 256) * 512 = 140288 table entries > 131072
    s = B.Shape(70000, 64, 512, 256, 12, 64)
    p = ctypes.c_void_p(256)
    rc = L.lc_moe_permute_noalloc(ctypes.byref(s), p, None, p, p, p, None, None, None)
    assert rc == B.ERR_UNSUPPORTED_SHAPE
