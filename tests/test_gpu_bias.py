"""GPU parity of the expert-bias update (LongCat-Flash llm-wiki entity page, section 2.1, dynamic
computation-budget control) and of the bias-control loop at LongCat-Flash shape: every step's
counts and biases are bit-exact with the oracle, and the loop drives the mean number of FFN
experts per token toward K_e."""
import numpy as np
import pytest
import torch

import oracle
from mixture_experts_zero_b200 import binding as B
from mixture_experts_zero_b200 import inputs

pytestmark = pytest.mark.gpu


def test_bias_update_bit_exact(cuda_device):
    rng = np.random.default_rng(7)
    for (N, Z, K, K_e, T_all, mu) in [(512, 256, 12, 8, 8192, 1e-3), (64, 32, 6, 4, 4096, 3e-3),
                                      (8, 4, 3, 2, 64, 0.1), (512, 256, 12, 8, 10 ** 9 + 7, 1e-3)]:
        E = N + Z
        counts = rng.integers(0, 3 * K * min(T_all, 10 ** 6) // E + 1, E).astype(np.int32)
        b = rng.standard_normal(E).astype(np.float32) * 0.01
        bt = torch.from_numpy(b.copy()).cuda()
        ct = torch.from_numpy(counts).cuda()
        B.lc_moe_bias_update(bt, ct, T_all, N, Z, K, K_e, mu, reset_counts=True)
        ref = oracle.bias_update(b, counts, T_all, N, Z, K, K_e, mu)
        np.testing.assert_array_equal(bt.cpu().numpy().view(np.uint32), ref.view(np.uint32))
        assert int(ct.abs().sum()) == 0


@pytest.mark.parametrize("grid,mu", [(True, 1e-3), (False, 1e-1)])
def test_bias_control_loop_full_shape(cuda_device, grid, mu):
    """30 steps of the bias-control loop at LongCat-Flash shape (T=8192, d=6144, 512 FFN + 256
    zero experts, K=12, K_e=8), from a start that favours the zero experts (b = +2/E on them).
    Each step: route on the GPU, compare counts with the oracle's routing of the GPU logits,
    update the biases on the GPU and compare them bit for bit with the oracle's update. At the
    workload's mu = 1e-3 the pages' convergence takes ~20B tokens, far beyond 30 steps; the run
    with mu = 0.1 shows the direction of the control within the 30 steps."""
    w = inputs.WORKLOADS["bias_loop"]
    g = inputs.generator(w.seed, "cuda")
    wr = inputs.draw_router(w, g, "cuda")
    bias = torch.zeros(w.E, dtype=torch.float32, device="cuda")
    bias[w.N:] = 2.0 / w.E
    b_ref = bias.cpu().numpy().copy()
    counts = torch.zeros(w.E, dtype=torch.int32, device="cuda")
    logits = torch.empty(w.T, w.E, dtype=torch.float32, device="cuda")
    s = B.Shape(w.T, w.d, w.N, w.Z, w.K, w.I)
    ws = B.new_workspace(s, B.OP_ROUTE)
    mean_ffn = []
    for step in range(30):
        x = inputs.draw_x(w, g, "cuda", grid=grid)
        idx, gate = B.lc_moe_route(x, wr, bias, w.K, w.N, counts=counts, logits=logits, ws=ws)
        r_idx, r_gate, r_counts, bad = oracle.route(logits.cpu().numpy(), b_ref, w.K)
        assert bad == 0
        np.testing.assert_array_equal(counts.cpu().numpy(), r_counts)
        if step % 10 == 0:
            np.testing.assert_array_equal(idx.cpu().numpy(), r_idx)
        mean_ffn.append(float(r_counts[: w.N].sum()) / w.T)
        B.lc_moe_bias_update(bias, counts, w.T, w.N, w.Z, w.K, w.K_e, mu, reset_counts=True)
        b_ref = oracle.bias_update(b_ref, r_counts, w.T, w.N, w.Z, w.K, w.K_e, mu)
        np.testing.assert_array_equal(bias.cpu().numpy().view(np.uint32), b_ref.view(np.uint32))
    assert B.lc_moe_read_status(ws) == 0
    assert mean_ffn[0] < w.K_e
    if mu >= 0.1:
        # the mean number of FFN experts per token moves toward K_e
        assert abs(np.mean(mean_ffn[-5:]) - w.K_e) < abs(np.mean(mean_ffn[:5]) - w.K_e) - 0.1
