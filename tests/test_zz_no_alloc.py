"""moe_plan_noalloc against moe_plan, through the C ABI.

moe_plan_noalloc serves callers that cannot allocate device memory: they are
handed only their input and output buffers (a plugin inside another
framework's engine that offers no workspace, or a serving loop whose memory
is reserved up front by its own pool, where cudaMalloc can fail or stall the
device). Its scratch is a static array inside the library, shared by every
call, so two calls in a row must each give the same result as moe_plan with
a workspace of its own, whatever the previous call left behind.

This file runs last in the suite (its name sorts last) and also passes on
its own in a fresh process.
"""
import numpy as np
import pytest
import torch

from routed_experts_b200 import configs as C
from routed_experts_b200 import inputs as I

pytestmark = pytest.mark.gpu

W_ATOL = 1e-6   # the gating-weight tolerance of the parity tests


@pytest.fixture(scope="module")
def M():
    from routed_experts_b200 import build
    build.build()
    from routed_experts_b200 import moe
    moe.lib()
    return moe


def _with_workspace(M, cfg, inp):
    dev = inp["logits"].device
    idx = torch.empty(cfg.T, cfg.K, dtype=torch.int32, device=dev)
    w = torch.empty(cfg.T, cfg.K, dtype=torch.float32, device=dev)
    counts = torch.empty(cfg.E, dtype=torch.int32, device=dev)
    ws = M.alloc_workspace(cfg, M.WS_PLAN, dev)
    M.moe_plan(cfg, inp["logits"], idx, w, counts, ws)
    torch.cuda.synchronize()
    v = M.moe_plan_view(cfg)
    raw = ws.cpu()
    header = raw[v["header"]: v["header"] + 32].view(torch.int32).clone()
    row_of = raw[v["row_of"]: v["row_of"] + 4 * cfg.T * cfg.K].view(torch.int32).clone()
    return idx.cpu(), w.cpu(), counts.cpu(), row_of, header


def _no_alloc(M, cfg, inp):
    dev = inp["logits"].device
    idx = torch.full((cfg.T, cfg.K), -7, dtype=torch.int32, device=dev)
    w = torch.full((cfg.T, cfg.K), -7.0, dtype=torch.float32, device=dev)
    counts = torch.full((cfg.E,), -7, dtype=torch.int32, device=dev)
    row_of = torch.full((cfg.T * cfg.K,), -7, dtype=torch.int32, device=dev)
    header = torch.full((8,), -7, dtype=torch.int32, device=dev)
    M.moe_plan_noalloc(cfg, inp["logits"], idx, w, counts, row_of, header)
    torch.cuda.synchronize()
    return idx.cpu(), w.cpu(), counts.cpu(), row_of.cpu(), header.cpu()


def _compare(got, ref):
    g_idx, g_w, g_counts, g_row, g_hdr = got
    r_idx, r_w, r_counts, r_row, r_hdr = ref
    assert torch.equal(g_idx, r_idx)
    np.testing.assert_allclose(g_w.numpy(), r_w.numpy(), rtol=0, atol=W_ATOL)
    assert torch.equal(g_counts, r_counts)
    assert torch.equal(g_row, r_row)
    assert torch.equal(g_hdr, r_hdr)


def test_no_alloc_plan_matches_plan_on_two_calls_in_a_row(M):
    # two different layers back to back: the second call must not be
    # disturbed by what the first left in the shared static scratch
    first = C.OLMOE
    second = C.DSV3.replace(T=2048)
    in1 = I.make_inputs(first, 0, "cuda", weights=False)
    in2 = I.make_inputs(second, 1, "cuda", weights=False)
    ref1 = _with_workspace(M, first, in1)
    ref2 = _with_workspace(M, second, in2)
    _compare(_no_alloc(M, first, in1), ref1)
    _compare(_no_alloc(M, second, in2), ref2)
    # and the same layer twice
    _compare(_no_alloc(M, second, in2), ref2)


def test_no_alloc_block_planner_header(M):
    # MegaFlux's block-granular planner fills header words 6 and 7 (tau and
    # the winning candidate); they must match moe_plan's too
    cfg = C.OLMOE.replace(plan_mode=C.PLAN_BLOCKS)
    inp = I.make_inputs(cfg, 2, "cuda", weights=False)
    ref = _with_workspace(M, cfg, inp)
    assert int(ref[4][6]) > 0
    _compare(_no_alloc(M, cfg, inp), ref)
    _compare(_no_alloc(M, cfg, inp), ref)


def test_no_alloc_rejects_shapes_beyond_the_static_scratch(M):
    import ctypes
    big = C.EXTREME.replace(T=32768 * 8)
    assert M.moe_workspace_size(big, M.WS_PLAN) > 4 << 20
    fake = ctypes.c_void_p(1 << 20)
    code = M.lib().moe_plan_noalloc(ctypes.byref(M.config(big)), fake, fake, fake, fake, fake, fake, None)
    assert code == M.MOE_ERR_WORKSPACE
