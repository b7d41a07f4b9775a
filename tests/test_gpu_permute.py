"""GPU parity of the grouping step (counting sort of FFN picks by expert) and the row gather:
offsets, row->token map and pick->row map are compared bit for bit with the oracle."""
import numpy as np
import pytest
import torch

import oracle
from mixture_experts_zero_b200 import binding as B

from tests.gpu_util import make, np_bits

pytestmark = pytest.mark.gpu


def check_permute(idx_np: np.ndarray, N: int, E: int, x: torch.Tensor | None = None):
    idx = torch.from_numpy(np.ascontiguousarray(idx_np)).cuda()
    offsets, row_token, pair_row, x_perm = B.lc_moe_permute(idx, N, E, x=x)
    r_off, r_rt, r_pr = oracle.permute(idx_np, N)
    M = int(r_off[-1])
    np.testing.assert_array_equal(offsets.cpu().numpy(), r_off)
    np.testing.assert_array_equal(row_token.cpu().numpy()[:M], r_rt)
    np.testing.assert_array_equal(pair_row.cpu().numpy(), r_pr)
    if x is not None:
        rows = torch.from_numpy(r_rt.astype(np.int64)).cuda()
        assert torch.equal(x_perm[:M], x[rows])
    return M


@pytest.mark.parametrize("name", ["tiny", "small", "decode", "prefill"])
def test_permute_matches_oracle_on_routed_workloads(cuda_device, name):
    d = make(name, experts=False)
    w = d["w"]
    idx, _ = B.lc_moe_route(d["x"], d["wr"], d["bias"], w.K, w.N)
    M = check_permute(idx.cpu().numpy(), w.N, w.E, x=d["x"])
    assert 0 < M < w.T * w.K


def test_permute_edge_cases(cuda_device):
    rng = np.random.default_rng(3)
    # all picks are zero-computation experts: no rows
    idx = np.tile(np.array([[8, 9, 10]], np.int32), (70, 1))
    assert check_permute(idx, 8, 12) == 0
    # every token picks the same FFN expert first (one big group) with ragged T
    for T in [1, 255, 256, 257, 1000]:
        idx = np.stack([rng.permutation(12)[:3] for _ in range(T)]).astype(np.int32)
        idx[:, 0] = 5
        idx[:, 1:] = np.where(idx[:, 1:] == 5, 11, idx[:, 1:])
        check_permute(idx, 8, 12, x=torch.randn(T, 64, device="cuda").to(torch.bfloat16))
    # K = 1 and many experts
    idx = rng.integers(0, 2048, (3000, 1)).astype(np.int32)
    check_permute(idx, 1500, 2048)


def test_out_of_range_pick_is_reported(cuda_device):
    idx = torch.tensor([[0, 1], [2, 99]], dtype=torch.int32, device="cuda")
    s = B.Shape(2, 64, 4, 2, 2, 64)
    ws = B.new_workspace(s, B.OP_PERMUTE)
    B.lc_moe_permute(idx, 4, 6, ws=ws)
    assert B.lc_moe_read_status(ws, raise_on_error=False) & B.DEV_IDX_RANGE
