"""Pins of the oracle's expert FFN and combine against the plain definition."""
import numpy as np
import pytest
import torch

from routed_experts_b200 import configs as C
from routed_experts_b200 import inputs as I


def _run(orc, inp, K, R, tile, budget, gating, dtype, round_mode=None):
    return orc.layer(inp["logits"], inp["x"], inp["w_gate_up"], inp["w_down"], K=K, R=R,
                     tile=tile, budget=budget, gating=gating, dtype=dtype, round_mode=round_mode)


def _np_inputs(cfg, seed):
    return {k: I.to_numpy_bits(v) for k, v in I.make_inputs(cfg, seed).items()}


def test_bf16_rounding_hand_cases(orc):
    # bf16 spacing at 1 is 2**-7: halfway cases go to the even mantissa
    assert orc.double_to_bf16(1.0 + 2.0 ** -8) == 0x3F80
    assert orc.double_to_bf16(1.0 + 3 * 2.0 ** -8) == 0x3F82
    assert orc.double_to_bf16(1.0 + 2.0 ** -8 + 2.0 ** -30) == 0x3F81
    assert orc.double_to_bf16(-2.0) == 0xC000
    assert orc.double_to_bf16(-0.0) == 0x8000


def test_bf16_rounding_matches_library_on_fp32_values(orc):
    rng = np.random.default_rng(11)
    v = (rng.standard_normal(2000) * 10.0 ** rng.integers(-20, 20, 2000)).astype(np.float32)
    ref = torch.from_numpy(v).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = np.array([orc.double_to_bf16(float(a)) for a in v], np.uint16)
    assert np.array_equal(got, ref)


def _random_tiny(rng):
    R = int(rng.integers(1, 4))
    E = R * int(rng.integers(1, 4))
    K = int(rng.integers(1, min(E, 3) + 1))
    T = R * int(rng.integers(1, 9))
    d = int(rng.choice([8, 16, 24]))
    F = int(rng.choice([8, 16, 32]))
    cfg = C.TINY.replace(T=T, d=d, E=E, K=K, F=F, R=R, tile=int(rng.choice([1, 2, 4, 8])),
                         budget=int(rng.integers(0, 3)), zipf_s=float(rng.uniform(0, 2)),
                         gating=int(rng.integers(0, 2)))
    return cfg


def test_sparse_layer_equals_dense_definition(orc):
    """Unrounded sparse path (plan + permute + FFN + combine) vs every expert on
    every token then masked: the plan must not change the result."""
    rng = np.random.default_rng(2024)
    for it in range(60):
        cfg = _random_tiny(rng)
        inp = _np_inputs(cfg, it)
        r = _run(orc, inp, cfg.K, cfg.R, cfg.tile, cfg.budget, cfg.gating, C.FP32,
                 round_mode=orc.ROUND_NONE)
        # round-mode NONE stores into fp32 arrays; compare the fp64 token path too
        toks = np.arange(cfg.T)
        tok = orc.token_out(toks, inp["x"], r["idx"], r["w"], inp["w_gate_up"], inp["w_down"],
                            C.FP32, orc.ROUND_NONE)
        dense = orc.dense_layer(inp["logits"], inp["x"], inp["w_gate_up"], inp["w_down"], cfg.K,
                                cfg.gating)
        scale = np.abs(dense).max() + 1e-30
        # the gating weights are stored as fp32 (relative 6e-8)
        assert np.abs(tok - dense).max() <= 2e-7 * scale, cfg
        assert np.abs(r["out"] - dense).max() <= 3e-7 * scale, cfg


def test_token_path_equals_permuted_path(orc):
    cfg = C.TINY
    inp = _np_inputs(cfg, 0)
    r = _run(orc, inp, cfg.K, cfg.R, cfg.tile, cfg.budget, cfg.gating, cfg.dtype)
    tok = orc.token_out(np.arange(cfg.T), inp["x"], r["idx"], r["w"], inp["w_gate_up"],
                        inp["w_down"], cfg.dtype, orc.ROUND_F32)
    assert np.array_equal(tok.astype(np.float32), r["out"])


def test_single_expert_is_a_swiglu_mlp(orc):
    """E = 1, K = 1: the layer reduces to one SwiGLU MLP (library ops, fp64)."""
    cfg = C.TINY.replace(T=12, d=16, E=1, K=1, F=24, R=1, tile=4, budget=0, zipf_s=0.0)
    inp = _np_inputs(cfg, 3)
    r = _run(orc, inp, 1, 1, 4, 0, cfg.gating, C.FP32, round_mode=orc.ROUND_NONE)
    x = torch.from_numpy(inp["x"]).double()
    wg = torch.from_numpy(inp["w_gate_up"][0, :cfg.F]).double()
    wu = torch.from_numpy(inp["w_gate_up"][0, cfg.F:]).double()
    wd = torch.from_numpy(inp["w_down"][0]).double()
    ref = (torch.nn.functional.silu(x @ wg.T) * (x @ wu.T)) @ wd.T
    assert np.array_equal(r["w"], np.ones((cfg.T, 1), np.float32))
    np.testing.assert_allclose(r["out"], ref.numpy(), rtol=1e-6, atol=1e-9)


def test_bf16_rounding_points(orc):
    cfg = C.TINY.replace(T=32, d=64, E=4, K=2, F=64, R=2, tile=8, budget=1, dtype=C.BF16)
    inp = _np_inputs(cfg, 5)
    r = _run(orc, inp, cfg.K, cfg.R, cfg.tile, cfg.budget, cfg.gating, C.BF16)
    dense = orc.dense_layer(orc.to_f64(inp["logits"], C.FP32), orc.to_f64(inp["x"], C.BF16),
                            orc.to_f64(inp["w_gate_up"], C.BF16), orc.to_f64(inp["w_down"], C.BF16),
                            cfg.K, cfg.gating)
    out = orc.to_f64(r["out"], C.BF16)
    # out, H and Yp are bf16 values; out is within bf16 error of the exact layer
    assert r["out"].dtype == np.uint16 and r["h"].dtype == np.uint16
    err = np.abs(out - dense)
    assert np.all(err <= 2e-2 + 1e-2 * np.abs(dense))
    assert np.linalg.norm(out - dense) <= 1e-2 * np.linalg.norm(dense)
    # padding rows of H and Yp are zero
    valid = r["src_of"] >= 0
    assert not r["h"][:r["plan"]["total_rows"]][~valid[:r["plan"]["total_rows"]]].any()


def test_output_is_invariant_to_plan_parameters(orc):
    cfg = C.TINY
    inp = _np_inputs(cfg, 1)
    base = _run(orc, inp, cfg.K, cfg.R, cfg.tile, cfg.budget, cfg.gating, cfg.dtype)
    for R, tile, budget in ((1, 16, 0), (2, 8, 1), (4, 32, 2), (8, 16, 3), (4, 16, 0)):
        r = _run(orc, inp, cfg.K, R, tile, budget, cfg.gating, cfg.dtype)
        assert np.array_equal(r["out"], base["out"]), (R, tile, budget)


def test_output_is_the_same_under_both_planners(orc):
    """The exact-S*K greedy and the block-granular search place entries
    differently ([MoonEP] "The greedy balance, step by step"; [MegaFlux] §3.1
    "Bounded greedy search"), but every entry goes through the same arithmetic
    wherever it lands, so the layer output must not change a bit."""
    for cfg, seed in ((C.TINY, 2), (C.TINY.replace(dtype=C.BF16, tile=32, budget=2), 3)):
        inp = _np_inputs(cfg, seed)
        outs = [orc.layer(inp["logits"], inp["x"], inp["w_gate_up"], inp["w_down"], K=cfg.K, R=cfg.R,
                          tile=cfg.tile, budget=cfg.budget, gating=cfg.gating, dtype=cfg.dtype,
                          plan_mode=mode) for mode in (orc.PLAN_EXACT, orc.PLAN_BLOCKS)]
        assert outs[0]["plan"]["pieces"].tolist() != outs[1]["plan"]["pieces"].tolist(), "plans should differ"
        assert np.array_equal(outs[0]["out"], outs[1]["out"])


def test_combine_weights_select_rows(orc):
    yp = np.arange(12, dtype=np.float32).reshape(4, 3)
    row_of = np.array([2, 0, 3, 1], np.int32)
    w = np.array([[0.25, 0.75], [1.0, 0.0]], np.float32)
    out = orc.combine(yp, row_of, w, C.FP32, orc.ROUND_F32)
    np.testing.assert_array_equal(out, [[0.25 * yp[2] + 0.75 * yp[0]][0], yp[3]])
