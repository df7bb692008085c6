"""The C ABI library without a GPU: it builds, loads, exports every function
include/moe.h declares, and rejects bad arguments on the host before any
CUDA call."""
import ctypes
import os
import re

import pytest

from routed_experts_b200 import build
from routed_experts_b200 import configs as C

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def M():
    build.build()
    from routed_experts_b200 import moe
    moe.lib()
    return moe


def declared_functions():
    src = open(os.path.join(ROOT, "include", "moe.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(moe_[a-z0-9_]+)\s*\(", src)))


def test_exports_every_declared_function(M):
    names = declared_functions()
    assert "moe_plan" in names and "moe_layer_fwd" in names and len(names) >= 16
    lib = ctypes.CDLL(M.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), n


def test_status_strings(M):
    assert M.status_string(0) == "MOE_OK"
    assert M.status_string(3) == "MOE_ERR_WORKSPACE"


@pytest.mark.parametrize("cfg", list(C.NAMED.values()), ids=lambda c: c.name)
def test_sizes_of_named_configs(M, cfg):
    from oracle import oracle as O
    cap = M.moe_rows_capacity(cfg)
    assert cap == O.rows_capacity(cfg.N, cfg.E, cfg.R, cfg.budget, cfg.tile)
    plan_b = M.moe_workspace_size(cfg, M.WS_PLAN)
    layer_b = M.moe_workspace_size(cfg, M.WS_LAYER)
    host_b = M.moe_workspace_size(cfg, M.WS_LAYER_HOST)
    eb = cfg.elem_bytes
    assert plan_b < layer_b < host_b
    assert layer_b - plan_b >= eb * cap * ((2 if cfg.dtype == C.FP32 else 1) * cfg.d + cfg.F)
    v = M.moe_plan_view(cfg)
    assert v["rows_cap"] == cap and v["max_pieces"] == cfg.E + cfg.R * cfg.budget
    offs = [v[k] for k in ("header", "pieces", "blocks", "rank_load", "rank_replicas", "rank_row0",
                           "row_of", "src_of")]
    assert all(o % 16 == 0 for o in offs) and max(offs) < plan_b


def _code(fn, *args):
    return fn(*args)


def test_invalid_configs(M):
    L = M.lib()
    n = ctypes.c_size_t()
    bad = [
        dict(T=0), dict(R=3), dict(K=9, E=8), dict(E=6, R=4), dict(budget=-1), dict(dtype=7),
        dict(gating=5), dict(plan_mode=2),
    ]
    for kw in bad:
        cfg = C.TINY.replace(**kw)
        assert L.moe_workspace_size(ctypes.byref(M.config(cfg)), 0, ctypes.byref(n)) == M.MOE_ERR_INVALID_ARG, kw
    unsupported = [
        C.OLMOE.replace(tile=64), C.OLMOE.replace(F=1000), C.OLMOE.replace(d=2048 + 64),
        C.TINY.replace(tile=8), C.TINY.replace(K=17, E=32), C.TINY.replace(E=2048, R=4),
        C.TINY.replace(E=1024, R=32, T=256, plan_mode=C.PLAN_BLOCKS),
        C.TINY.replace(T=32768 * 16, R=4, plan_mode=C.PLAN_BLOCKS),
    ]
    for cfg in unsupported:
        assert L.moe_workspace_size(ctypes.byref(M.config(cfg)), 0, ctypes.byref(n)) == M.MOE_ERR_UNSUPPORTED, cfg
    assert L.moe_workspace_size(None, 0, ctypes.byref(n)) == M.MOE_ERR_INVALID_ARG
    assert L.moe_workspace_size(ctypes.byref(M.config(C.TINY)), 9, ctypes.byref(n)) == M.MOE_ERR_INVALID_ARG


def test_calls_reject_bad_pointers_and_small_workspace(M):
    L = M.lib()
    cfg = ctypes.byref(M.config(C.TINY))
    fake = ctypes.c_void_p(1 << 20)      # never dereferenced: every check below fails first
    odd = ctypes.c_void_p((1 << 20) + 4)
    need = M.moe_workspace_size(C.TINY, M.WS_PLAN)
    s = ctypes.c_size_t
    assert L.moe_plan(cfg, None, fake, fake, fake, fake, s(need), None) == M.MOE_ERR_INVALID_ARG
    assert L.moe_plan(cfg, odd, fake, fake, fake, fake, s(need), None) == M.MOE_ERR_INVALID_ARG
    assert L.moe_plan(cfg, fake, fake, fake, fake, fake, s(need - 1), None) == M.MOE_ERR_WORKSPACE
    assert L.moe_plan(cfg, fake, fake, fake, fake, None, s(need), None) == M.MOE_ERR_INVALID_ARG
    assert L.moe_dispatch(cfg, fake, None, fake, s(need), None) == M.MOE_ERR_INVALID_ARG
    assert L.moe_expert_ffn(cfg, fake, fake, fake, fake, odd, fake, s(need), None) == M.MOE_ERR_INVALID_ARG
    assert L.moe_combine(cfg, fake, fake, fake, fake, s(16), None) == M.MOE_ERR_WORKSPACE
    layer_need = M.moe_workspace_size(C.TINY, M.WS_LAYER)
    assert L.moe_layer_fwd(cfg, fake, fake, fake, fake, fake, fake, s(layer_need - 1), None) == M.MOE_ERR_WORKSPACE
    host_need = M.moe_workspace_size(C.TINY, M.WS_LAYER_HOST)
    assert L.moe_layer_fwd_host(cfg, fake, fake, fake, fake, fake, fake, s(host_need - 1), None) == \
        M.MOE_ERR_WORKSPACE
    v = ctypes.c_uint32()
    assert L.moe_read_status(None, None, ctypes.byref(v)) == M.MOE_ERR_INVALID_ARG


def test_backward_rejects_unsupported_shapes_bad_pointers_and_small_workspace(M):
    L = M.lib()
    fake = ctypes.c_void_p(1 << 20)      # never dereferenced: every check below fails first
    odd = ctypes.c_void_p((1 << 20) + 4)
    s = ctypes.c_size_t
    bf = C.TINY.replace(dtype=C.BF16, tile=128, d=256, F=256)
    cfg = ctypes.byref(M.config(bf))
    need = M.moe_workspace_size(bf, M.WS_LAYER_TRAIN)
    assert need > M.moe_workspace_size(bf, M.WS_LAYER_HOST)
    args = [fake] * 8
    assert L.moe_layer_bwd(cfg, *args, fake, s(need - 1), None) == M.MOE_ERR_WORKSPACE
    assert L.moe_layer_bwd(cfg, None, *args[1:], fake, s(need), None) == M.MOE_ERR_INVALID_ARG
    assert L.moe_layer_bwd(cfg, *args[:4], odd, *args[5:], fake, s(need), None) == M.MOE_ERR_INVALID_ARG
    assert L.moe_layer_fwd_train(cfg, *args[:5], fake, s(need - 1), None) == M.MOE_ERR_WORKSPACE
    assert L.moe_layer_fwd_train(cfg, *args[:4], None, fake, s(need), None) == M.MOE_ERR_INVALID_ARG
    # fp32 layers and F not a multiple of 256 have no backward kernels
    for c in (C.TINY, bf.replace(F=384)):
        n = M.moe_workspace_size(c, M.WS_LAYER_TRAIN)
        assert L.moe_layer_bwd(ctypes.byref(M.config(c)), *args, fake, s(n), None) == M.MOE_ERR_UNSUPPORTED
        assert L.moe_layer_fwd_train(ctypes.byref(M.config(c)), *args[:5], fake, s(n), None) == \
            M.MOE_ERR_UNSUPPORTED


def test_fused_ffn_checks_its_arguments(M):
    L = M.lib()
    fake = ctypes.c_void_p(1 << 20)      # never dereferenced: every check below fails first
    s = ctypes.c_size_t
    bf = C.TINY.replace(dtype=C.BF16, tile=128, d=256, F=256)
    need = M.moe_workspace_size(bf, M.WS_PLAN)
    cfg = ctypes.byref(M.config(bf))
    assert L.moe_expert_ffn_fused(cfg, fake, fake, fake, fake, fake, fake, s(need - 1), None) == M.MOE_ERR_WORKSPACE
    assert L.moe_expert_ffn_fused(cfg, fake, fake, None, fake, fake, fake, s(need), None) == M.MOE_ERR_INVALID_ARG
    n = M.moe_workspace_size(C.TINY, M.WS_PLAN)
    assert L.moe_expert_ffn_fused(ctypes.byref(M.config(C.TINY)), fake, fake, fake, fake, fake, fake, s(n),
                                  None) == M.MOE_ERR_UNSUPPORTED
    g = L.moe_expert_ffn_fused_gather
    assert g(cfg, fake, fake, fake, fake, fake, fake, s(need - 1), None) == M.MOE_ERR_WORKSPACE
    assert g(cfg, None, fake, fake, fake, fake, fake, s(need), None) == M.MOE_ERR_INVALID_ARG
    odd = ctypes.c_void_p((1 << 20) + 4)
    assert g(cfg, fake, fake, fake, odd, fake, fake, s(need), None) == M.MOE_ERR_INVALID_ARG
    assert g(ctypes.byref(M.config(C.TINY)), fake, fake, fake, fake, fake, fake, s(n), None) == \
        M.MOE_ERR_UNSUPPORTED


def test_mx_buffer_sizes(M):
    cfg = C.OLMOE
    cap = M.moe_rows_capacity(cfg)
    E, d, F = cfg.E, cfg.d, cfg.F

    def scale_bytes(rows, K):
        return -(-rows // 128) * (K // 128) * 512

    assert M.moe_mx_buffer_bytes(cfg, M.MX_XQ) == cap * d
    assert M.moe_mx_buffer_bytes(cfg, M.MX_XS) == scale_bytes(cap, d)
    assert M.moe_mx_buffer_bytes(cfg, M.MX_HQ) == cap * F
    assert M.moe_mx_buffer_bytes(cfg, M.MX_HS) == scale_bytes(cap, F)
    assert M.moe_mx_buffer_bytes(cfg, M.MX_W1Q) == E * 2 * F * d
    assert M.moe_mx_buffer_bytes(cfg, M.MX_W1S) == E * 2 * F * d // 32
    assert M.moe_mx_buffer_bytes(cfg, M.MX_W2Q) == E * d * F
    assert M.moe_mx_buffer_bytes(cfg, M.MX_W2S) == E * d * F // 32
    # MXFP4 weights: two codes per byte, the same scales, activations unchanged
    assert M.moe_mx_buffer_bytes(cfg, M.MX_W1Q, M.MX_W_E2M1) == E * 2 * F * d // 2
    assert M.moe_mx_buffer_bytes(cfg, M.MX_W2Q, M.MX_W_E2M1) == E * d * F // 2
    assert M.moe_mx_buffer_bytes(cfg, M.MX_W1S, M.MX_W_E2M1) == E * 2 * F * d // 32
    assert M.moe_mx_buffer_bytes(cfg, M.MX_XQ, M.MX_W_E2M1) == cap * d
    L = M.lib()
    n = ctypes.c_size_t(0)
    assert L.moe_mx_buffer_bytes(ctypes.byref(M.config(cfg)), 8, 0, ctypes.byref(n)) == M.MOE_ERR_INVALID_ARG
    assert L.moe_mx_buffer_bytes(ctypes.byref(M.config(cfg)), 0, 2, ctypes.byref(n)) == M.MOE_ERR_INVALID_ARG
    # fp32 layers and widths the MX GEMM does not tile are unsupported
    for bad in (C.TINY, cfg.replace(F=1000), cfg.replace(d=2176)):
        assert L.moe_mx_buffer_bytes(ctypes.byref(M.config(bad)), 0, 0, ctypes.byref(n)) in \
            (M.MOE_ERR_UNSUPPORTED, M.MOE_ERR_INVALID_ARG), bad


def test_mx_calls_check_their_arguments(M):
    L = M.lib()
    fake = ctypes.c_void_p(1 << 20)      # never dereferenced: every check below fails first
    odd = ctypes.c_void_p((1 << 20) + 8)
    s = ctypes.c_size_t
    bf = C.TINY.replace(dtype=C.BF16, tile=128, d=256, F=256)
    cfg = ctypes.byref(M.config(bf))
    plan_need = M.moe_workspace_size(bf, M.WS_PLAN)
    layer_need = M.moe_workspace_size(bf, M.WS_LAYER)
    # weights: a null or misaligned pointer, or an unsupported shape (the call has no workspace to check)
    assert L.moe_mx_quantize_weights(cfg, fake, fake, 0, fake, None, fake, fake, None) == M.MOE_ERR_INVALID_ARG
    assert L.moe_mx_quantize_weights(cfg, fake, odd, 0, fake, fake, fake, fake, None) == M.MOE_ERR_INVALID_ARG
    assert L.moe_mx_quantize_weights(cfg, fake, fake, 7, fake, fake, fake, fake, None) == M.MOE_ERR_INVALID_ARG
    tiny = ctypes.byref(M.config(C.TINY))
    assert L.moe_mx_quantize_weights(tiny, fake, fake, 0, fake, fake, fake, fake, None) == M.MOE_ERR_UNSUPPORTED
    assert L.moe_dispatch_mx(cfg, fake, fake, fake, fake, s(plan_need - 1), None) == M.MOE_ERR_WORKSPACE
    assert L.moe_dispatch_mx(cfg, fake, None, fake, fake, s(plan_need), None) == M.MOE_ERR_INVALID_ARG
    assert L.moe_expert_fc1_mx(cfg, fake, fake, fake, fake, 0, fake, fake, fake, s(plan_need - 1), None) == \
        M.MOE_ERR_WORKSPACE
    assert L.moe_expert_fc1_mx(cfg, fake, odd, fake, fake, 0, fake, fake, fake, s(plan_need), None) == \
        M.MOE_ERR_INVALID_ARG
    assert L.moe_expert_fc1_mx(cfg, fake, fake, fake, fake, 3, fake, fake, fake, s(plan_need), None) == \
        M.MOE_ERR_INVALID_ARG
    assert L.moe_expert_fc2_mx(cfg, fake, fake, fake, fake, 1, fake, fake, s(plan_need - 1), None) == \
        M.MOE_ERR_WORKSPACE
    assert L.moe_expert_fc2_mx(cfg, fake, fake, fake, None, 1, fake, fake, s(plan_need), None) == \
        M.MOE_ERR_INVALID_ARG
    assert L.moe_layer_fwd_mx(cfg, fake, fake, fake, fake, fake, fake, 0, fake, fake, s(layer_need - 1), None) == \
        M.MOE_ERR_WORKSPACE
    assert L.moe_layer_fwd_mx(cfg, fake, fake, fake, fake, fake, fake, 0, None, fake, s(layer_need), None) == \
        M.MOE_ERR_INVALID_ARG
    assert L.moe_layer_fwd_mx(cfg, fake, fake, fake, fake, fake, fake, -1, fake, fake, s(layer_need), None) == \
        M.MOE_ERR_INVALID_ARG
    assert L.moe_layer_fwd_mx(tiny, fake, fake, fake, fake, fake, fake, 0, fake, fake, s(layer_need), None) == \
        M.MOE_ERR_UNSUPPORTED


def test_binding_refuses_to_run_without_library(tmp_path, monkeypatch):
    from routed_experts_b200 import moe
    monkeypatch.setattr(moe, "_lib", None)
    monkeypatch.setattr(moe, "LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(RuntimeError, match="missing"):
        moe.lib()


@pytest.mark.parametrize("cfg", list(C.NAMED.values()), ids=lambda c: c.name)
def test_layer_path_of_named_configs(M, cfg):
    """moe_layer_fwd reads FC1's rows straight from x for bf16 layers whose x
    takes at most 64 MiB (OLMoE and Qwen3 here), through the dispatch otherwise."""
    small_x = cfg.T * cfg.d * cfg.elem_bytes <= 64 << 20
    want = M.PATH_GATHER_FC1 if cfg.dtype == C.BF16 and small_x else M.PATH_DISPATCH
    assert M.moe_layer_path(cfg) == want
    assert {"olmoe": M.PATH_GATHER_FC1, "qwen3": M.PATH_GATHER_FC1, "extreme": M.PATH_DISPATCH,
            "dsv3": M.PATH_DISPATCH}.get(cfg.name, want) == want
