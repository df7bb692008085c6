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
