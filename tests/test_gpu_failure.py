"""Failure detection on the GPU without faulting or hanging it.

Every wait in the expert-FFN kernels is bounded: when it runs out the kernel
reports MOE_DEV_TIMEOUT in the status word and returns. These tests make such
a wait run out (on an mbarrier that nothing arrives on) and check that the
status is reported, the call returns, and the context keeps working.
Host-detected errors are covered by tests/test_abi.py.
"""
import time

import pytest
import torch

from routed_experts_b200 import configs as C
from routed_experts_b200 import moe as M

from .gpu_helpers import check_full_small

pytestmark = pytest.mark.gpu

SMALL = C.LayerConfig("small_bf16", T=512, d=256, E=8, K=2, F=256, R=4, tile=128, budget=2, zipf_s=1.0)


@pytest.fixture(scope="module", autouse=True)
def _built():
    from routed_experts_b200 import build
    build.build()


@pytest.mark.parametrize("budget", [0, 2_000_000, 50_000_000])
def test_bounded_wait_reports_timeout(budget):
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    t0 = time.perf_counter()
    M.moe_probe_bounded_wait(status, budget)
    torch.cuda.synchronize()
    assert time.perf_counter() - t0 < 5.0
    assert int(status.item()) & M.DEV_TIMEOUT


def test_status_bits_accumulate_without_clearing_others():
    status = torch.full((1,), M.DEV_PLAN_INEXACT, dtype=torch.int32, device="cuda")
    M.moe_probe_bounded_wait(status, 1000)
    torch.cuda.synchronize()
    assert int(status.item()) == M.DEV_PLAN_INEXACT | M.DEV_TIMEOUT


def test_context_usable_after_timeout():
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    M.moe_probe_bounded_wait(status, 1000)
    torch.cuda.synchronize()
    g, _, _ = check_full_small(SMALL, 0)
    assert g["status"] & M.DEV_TIMEOUT == 0


def test_probe_rejects_bad_budget():
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    with pytest.raises(M.MoeError):
        M.moe_probe_bounded_wait(status, -1)
    with pytest.raises(M.MoeError):
        M.moe_probe_bounded_wait(status, 1 << 40)


# The real GEMM's abort path: moe_expert_ffn with every device-side wait of
# its tensor-core kernels cut to a few clock cycles. Waits run out while
# copies and MMAs are in flight; both CTAs of every pair must stop, drain what
# they issued, free tensor memory and return, and the next calls on the same
# workspace must give the right result (queues back at zero).
MED = C.LayerConfig("abort_med", T=1024, d=512, E=16, K=4, F=384, R=4, tile=128, budget=2, zipf_s=1.2)


@pytest.mark.parametrize("budget", [1, 300, 3000])
def test_expert_ffn_timeout_path_returns_and_recovers(budget):
    from routed_experts_b200 import inputs as I
    from .gpu_helpers import run_path
    inp = I.make_inputs(MED, 7, "cuda")
    ref = run_path(MED, inp, "staged")
    assert ref["status"] & M.DEV_TIMEOUT == 0
    h = torch.zeros_like(ref["h"])
    y = torch.zeros_like(ref["yp"])
    t0 = time.perf_counter()
    for _ in range(3):
        M.moe_probe_expert_ffn_timeout(MED, ref["xp"], inp["w_gate_up"], inp["w_down"], h, y, ref["ws"], budget)
    status = M.moe_read_status(ref["ws"])
    assert time.perf_counter() - t0 < 60.0
    if budget == 1:
        assert status & M.DEV_TIMEOUT
    # a new plan clears the status; the normal FFN on the same workspace is right again
    M.moe_plan(MED, inp["logits"], ref["idx"], ref["w"], ref["counts"], ref["ws"])
    M.moe_expert_ffn(MED, ref["xp"], inp["w_gate_up"], inp["w_down"], h, y, ref["ws"])
    assert M.moe_read_status(ref["ws"]) & ~M.DEV_PLAN_INEXACT == 0
    valid = torch.as_tensor((ref["plan"]["src_of"].numpy() >= 0).nonzero()[0], device="cuda")
    assert torch.equal(h[valid], ref["h"][valid])
    assert torch.equal(y[valid], ref["yp"][valid])


def test_expert_ffn_timeout_probe_rejects_bad_arguments():
    ws = M.alloc_workspace(SMALL)
    x = torch.zeros(16, device="cuda", dtype=torch.bfloat16)
    for budget in (0, 1 << 40):
        with pytest.raises(M.MoeError):
            M.moe_probe_expert_ffn_timeout(SMALL, x, x, x, x, x, ws, budget)
    with pytest.raises(M.MoeError):
        M.moe_probe_expert_ffn_timeout(C.TINY, x, x, x, x, x, ws, 100)


@pytest.mark.parametrize("budget", [1, 300, 3000])
def test_fc1_gather_timeout_path_returns_and_recovers(budget):
    """The FC1 that reads x (row-gather and signal warps besides the TMA and
    MMA threads) with every wait cut short: it stops, drains its row copies
    and stage signals, and the next call on the same workspace is right."""
    from routed_experts_b200 import inputs as I
    from .gpu_helpers import run_path
    inp = I.make_inputs(MED, 8, "cuda")
    ref = run_path(MED, inp, "fc1_gather")
    assert ref["status"] & M.DEV_TIMEOUT == 0
    h = torch.zeros_like(ref["h"])
    t0 = time.perf_counter()
    for _ in range(3):
        M.moe_probe_fc1_gather_timeout(MED, inp["x"], inp["w_gate_up"], h, ref["ws"], budget)
    status = M.moe_read_status(ref["ws"])
    assert time.perf_counter() - t0 < 60.0
    if budget == 1:
        assert status & M.DEV_TIMEOUT
    M.moe_plan(MED, inp["logits"], ref["idx"], ref["w"], ref["counts"], ref["ws"])
    M.moe_expert_fc1_gather(MED, inp["x"], inp["w_gate_up"], h, ref["ws"])
    assert M.moe_read_status(ref["ws"]) & ~M.DEV_PLAN_INEXACT == 0
    valid = torch.as_tensor((ref["plan"]["src_of"].numpy() >= 0).nonzero()[0], device="cuda")
    assert torch.equal(h[valid], ref["h"][valid])
