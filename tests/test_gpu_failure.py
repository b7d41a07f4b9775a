"""Failure detection on the device. Every pipeline wait of the GEMMs and the row gather is bounded:
when it runs out it records LC_MOE_DEV_WAIT_TIMEOUT in the workspace's status word and raises its
CTA's abort flag, and the kernel returns instead of hanging the context. lc_moe_check_wait_timeout
runs that same bounded wait on a two-role pipeline whose first barrier phase nothing completes
(role 0 waits on it with the limit; role 1 waits, with four times the limit, on the phase role 0
would have released). The test sets a short limit, checks the status the host reads, checks from
the kernel's device time that role 1 left through role 0's abort flag (about one limit, not four),
and then runs the layer on the same context."""
import pytest
import torch

from mixture_experts_zero_b200 import binding as B

from tests.gpu_util import make

pytestmark = pytest.mark.gpu

LIMIT_NS = 20_000_000  # 20 ms per wait
DEFAULT_LIMIT_NS = 2_000_000_000


def test_a_wait_that_runs_out_is_reported_and_the_context_stays_usable(cuda_device):
    ws = B.new_workspace(B.Shape(1, 64, 1, 0, 1, 64), B.OP_STATUS)
    stream = torch.cuda.current_stream()
    B.lc_moe_set_wait_limit_ns(LIMIT_NS)
    try:
        times = []
        for _ in range(3):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            B.lc_moe_check_wait_timeout(ws, stream=stream)
            e1.record(stream)
            torch.cuda.synchronize()
            times.append(e0.elapsed_time(e1))
            with pytest.raises(B.LcMoeError) as err:
                B.lc_moe_read_status(ws)
            assert err.value.code == B.ERR_TIMEOUT
            assert B.lc_moe_read_status(ws) == 0  # the read cleared the word
    finally:
        B.lc_moe_set_wait_limit_ns(DEFAULT_LIMIT_NS)
    limit_ms = LIMIT_NS / 1e6
    for ms in times:
        assert 0.9 * limit_ms <= ms < 2.5 * limit_ms, times

    # the same context runs the layer afterwards, with a clean status word
    d = make("tiny")
    w = d["w"]
    s = B.Shape(w.T, w.d, w.N, w.Z, w.K, w.I)
    fws = B.new_workspace(s)
    out = B.lc_moe_forward(d["x"], d["wr"], d["bias"], d["w13"], d["w2"], w.K, ws=fws)
    torch.cuda.synchronize()
    assert B.lc_moe_read_status(fws) == 0
    assert torch.isfinite(out.float()).all()


def test_grouped_gemm_abort_drains_and_frees_tmem(cuda_device, monkeypatch):
    """The grouped GEMMs' own abort path, on a small grouped case (< 1 MB of operands): with the
    test switch set, each launch's MMA issuers give up at their fourth k-step as if a wait had run
    out. The host must read LC_MOE_ERR_TIMEOUT; each launch takes about one wait limit (the peer
    CTA's epilogues leave by their own bounded waits); and the next launches on
    the same context, switch unset, must give the oracle's results, which they could not if TMEM had
    not been freed or a barrier had been left mid-phase."""
    import numpy as np

    import oracle
    from tests.gpu_util import assert_within_ulp, np_bits

    d, I, sizes = 256, 128, [300, 5, 128, 40]
    N, M = len(sizes), sum(sizes)
    g = torch.Generator(device="cuda").manual_seed(9)
    x = torch.randn(M, d, generator=g, device="cuda").to(torch.bfloat16)
    w13 = (torch.randn(N, 2 * I, d, generator=g, device="cuda") / d ** 0.5).to(torch.bfloat16)
    w2 = (torch.randn(N, d, I, generator=g, device="cuda") / I ** 0.5).to(torch.bfloat16)
    offsets = torch.tensor(np.concatenate([[0], np.cumsum(sizes)]), dtype=torch.int32, device="cuda")
    ws = B.new_workspace(B.Shape(M, d, N, 0, 1, I), B.OP_STATUS)
    stream = torch.cuda.current_stream()
    B.lc_moe_set_wait_limit_ns(LIMIT_NS)
    try:
        monkeypatch.setenv("LC_MOE_DEBUG_GEMM_ABORT_KSTEP", "3")
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        B.lc_moe_expert_ffn(x, offsets, w13, w2, M, 1, ws=ws)  # both GEMM launches give up
        e1.record(stream)
        torch.cuda.synchronize()
        ms = e0.elapsed_time(e1)
        with pytest.raises(B.LcMoeError) as err:
            B.lc_moe_read_status(ws)
        assert err.value.code == B.ERR_TIMEOUT
        monkeypatch.delenv("LC_MOE_DEBUG_GEMM_ABORT_KSTEP")
        h, y = B.lc_moe_expert_ffn(x, offsets, w13, w2, M, 1, ws=ws)
        torch.cuda.synchronize()
        assert B.lc_moe_read_status(ws) == 0
    finally:
        B.lc_moe_set_wait_limit_ns(DEFAULT_LIMIT_NS)
    limit_ms = LIMIT_NS / 1e6
    # about one limit: the peer CTAs' epilogues leave by their own bounded waits (not the 2 s
    # default limit, and not at once)
    assert 0.8 * limit_ms <= ms < 8 * limit_ms, ms
    experts = np.repeat(np.arange(N), sizes).astype(np.int32)
    H, _ = oracle.expert_rows(np_bits(x), experts, np_bits(w13), np_bits(w2))
    assert_within_ulp(np_bits(h[:M]), H, what="H after the aborted launches")
    Y = oracle.expert_down(np_bits(h[:M]), experts, np_bits(w2))
    assert_within_ulp(np_bits(y[:M]), Y, what="Y after the aborted launches")
