"""GPU parity: the CUDA path through the C ABI against the CPU oracle.

Bit-exact: top-k indices, counts, plan (pieces, blocks, rank loads,
replicas, rows), row maps and the dispatched rows. Within tolerance (fp32
accumulation on the GPU against fp64 in the oracle, same rounding points):
gating weights, h, yp and the layer output.
"""
import numpy as np
import pytest
import torch

from oracle import oracle as O
from routed_experts_b200 import configs as C
from routed_experts_b200 import inputs as I
from routed_experts_b200 import moe as M

from .gpu_helpers import check_full_size, check_full_small, run_stages, to_f64

pytestmark = pytest.mark.gpu

# Small layers the oracle finishes in seconds; several tiles per expert and
# ragged last tiles.
SMALL_BF16 = C.LayerConfig("small_bf16", T=512, d=256, E=8, K=2, F=256, R=4, tile=128, budget=2,
                           zipf_s=1.0)
MED_BF16 = C.LayerConfig("med_bf16", T=1024, d=512, E=16, K=4, F=384, R=4, tile=128, budget=2,
                         zipf_s=1.2, gating=C.GATE_SIGMOID_TOPK, logits="normal")
WIDE_BF16 = C.LayerConfig("wide_bf16", T=256, d=768, E=32, K=8, F=128, R=8, tile=128, budget=4,
                          zipf_s=1.5)
TINY_TILES = [C.TINY.replace(name=f"tiny_t{t}", tile=t) for t in (16, 32, 64, 128)]


@pytest.fixture(scope="module", autouse=True)
def _built():
    from routed_experts_b200 import build
    build.build()
    O.build()


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_tiny_fp32_layer(seed):
    check_full_small(C.TINY, seed)


@pytest.mark.parametrize("cfg", TINY_TILES, ids=lambda c: c.name)
def test_fp32_tile_sizes(cfg):
    check_full_small(cfg, 3)


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_small_bf16_layer(seed):
    check_full_small(SMALL_BF16, seed)


@pytest.mark.parametrize("cfg", [MED_BF16, WIDE_BF16], ids=lambda c: c.name)
def test_medium_bf16_layers(cfg):
    check_full_small(cfg, 0)


# Degenerate and edge shapes: ragged chunks and tiles (T not a multiple of
# 32, S*K not a multiple of 128), every expert chosen by every token (K = E),
# one expert per rank, one token per rank, one hot expert in every token,
# the widest top-k path (E = 1024, K = 16) with most experts nearly empty.
EDGE = [
    C.LayerConfig("ragged", T=500, d=256, E=8, K=2, F=256, R=4, tile=128, budget=2, zipf_s=1.0),
    C.LayerConfig("k_eq_e", T=256, d=256, E=4, K=4, F=128, R=2, tile=128, budget=1),
    C.LayerConfig("e_eq_r", T=512, d=256, E=4, K=2, F=128, R=4, tile=128, budget=2, zipf_s=2.0),
    C.LayerConfig("s_eq_1", T=8, d=256, E=8, K=2, F=128, R=8, tile=128, budget=1),
    C.LayerConfig("hot", T=512, d=256, E=16, K=2, F=128, R=4, tile=128, budget=2, hot_bias=30.0),
    C.LayerConfig("wide_e", T=256, d=256, E=1024, K=16, F=128, R=8, tile=128, budget=4, zipf_s=1.0,
                  gating=C.GATE_SIGMOID_TOPK),
    C.TINY.replace(name="tiny_fp32_ragged", T=100, R=4, tile=16),
]


@pytest.mark.parametrize("cfg", EDGE, ids=lambda c: c.name)
def test_edge_shapes(cfg):
    check_full_small(cfg, 1)


def test_budget_zero_is_flagged_and_still_correct():
    cfg = SMALL_BF16.replace(name="nobudget", budget=0, zipf_s=2.0)
    g, ref, _ = check_full_small(cfg, 1)
    assert ref["plan"]["status"] == O.PLAN_INEXACT
    assert g["status"] & M.DEV_PLAN_INEXACT


def test_single_rank_identity_plan():
    cfg = SMALL_BF16.replace(name="r1", R=1, budget=0)
    g, ref, _ = check_full_small(cfg, 2)
    assert ref["plan"]["moves"] == 0 and g["plan"]["moves"] == 0


def test_output_bitwise_invariant_to_plan():
    """Only the plan changes with (R, budget); each token's rows go through the
    same arithmetic wherever they sit, so the output must not change a bit."""
    base = None
    for R, B in ((1, 0), (2, 1), (4, 2), (8, 3), (4, 0)):
        cfg = SMALL_BF16.replace(R=R, budget=B)
        inp = I.make_inputs(SMALL_BF16, 4, "cuda")
        out = run_stages(cfg, inp)["out"].cpu()
        if base is None:
            base = out
        else:
            assert torch.equal(out, base), (R, B)


@pytest.mark.parametrize("cfg", [C.TINY, SMALL_BF16], ids=lambda c: c.name)
def test_layer_call_matches_staged_calls(cfg):
    inp = I.make_inputs(cfg, 5, "cuda")
    staged = run_stages(cfg, inp)["out"]
    layer = M.Layer(cfg)
    out = layer.forward(inp["logits"], inp["x"], inp["w_gate_up"], inp["w_down"])
    assert layer.status() & ~M.DEV_PLAN_INEXACT == 0
    assert torch.equal(out, staged)
    host = M.Layer(cfg, host_io=True)
    lg = inp["logits"].cpu().pin_memory()
    x = inp["x"].cpu().pin_memory()
    out_h = torch.empty(cfg.T, cfg.d, dtype=M.act_dtype(cfg)).pin_memory()
    host.forward_host(lg, x, inp["w_gate_up"], inp["w_down"], out_h)
    torch.cuda.synchronize()
    assert torch.equal(out_h, staged.cpu())


@pytest.mark.parametrize("cfg", [SMALL_BF16, MED_BF16, WIDE_BF16, C.OLMOE, C.DSV3], ids=lambda c: c.name)
def test_gathered_fc1_matches_dispatch_then_fc1(cfg):
    """FC1 reading x through the row map gives bit-identical h (padding rows
    zero in both) to dispatch + FC1, and the whole-layer call gives
    bit-identical output to the staged calls."""
    inp = I.make_inputs(cfg, 2, "cuda")
    g = run_stages(cfg, inp)
    h2 = torch.empty_like(g["h"])
    M.moe_expert_fc1_gather(cfg, inp["x"], inp["w_gate_up"], h2, g["ws"])
    total = g["plan"]["total_rows"]
    assert torch.equal(h2[:total], g["h"][:total])
    layer = M.Layer(cfg)
    out = layer.forward(inp["logits"], inp["x"], inp["w_gate_up"], inp["w_down"])
    assert layer.status() & ~M.DEV_PLAN_INEXACT == 0
    assert torch.equal(out, g["out"])
    del layer, g, inp
    torch.cuda.empty_cache()


def test_gathered_fc1_is_bf16_only():
    cfg = C.TINY
    ws = M.alloc_workspace(cfg)
    x = torch.zeros(cfg.T, cfg.d, device="cuda")
    with pytest.raises(M.MoeError):
        M.moe_expert_fc1_gather(cfg, x, x, x, ws)


def test_repeated_calls_are_deterministic():
    cfg = MED_BF16
    inp = I.make_inputs(cfg, 1, "cuda")
    layer = M.Layer(cfg)
    a = layer.forward(inp["logits"], inp["x"], inp["w_gate_up"], inp["w_down"]).clone()
    for _ in range(3):
        b = layer.forward(inp["logits"], inp["x"], inp["w_gate_up"], inp["w_down"])
        assert torch.equal(a, b)


# MegaFlux's block-granular planner (plan mode 1): the same downstream
# kernels, a different plan; bit-exact against the oracle's planner.
BLOCK_SMALL = [c.replace(name=c.name + "_blocks", plan_mode=C.PLAN_BLOCKS)
               for c in (C.TINY, SMALL_BF16, MED_BF16, WIDE_BF16)] + \
              [c.replace(name=c.name + "_blocks", plan_mode=C.PLAN_BLOCKS) for c in EDGE if c.E * c.R <= 16384]


@pytest.mark.parametrize("cfg", BLOCK_SMALL, ids=lambda c: c.name)
def test_block_planner_small_layers(cfg):
    check_full_small(cfg, 0)


@pytest.mark.parametrize("cfg", [C.OLMOE, C.QWEN3, C.EXTREME, C.DSV3], ids=lambda c: c.name)
def test_block_planner_full_size(cfg):
    check_full_size(cfg.replace(name=cfg.name + "_blocks", plan_mode=C.PLAN_BLOCKS), 0, n_tokens=4, n_rows=16)
    torch.cuda.empty_cache()


FULL = [C.OLMOE, C.QWEN3, C.EXTREME, C.DSV3]


@pytest.mark.parametrize("cfg", FULL, ids=lambda c: c.name)
def test_full_size_layer(cfg):
    check_full_size(cfg, 0)
    torch.cuda.empty_cache()


@pytest.mark.parametrize("cfg", C.QWEN3_SWEEP, ids=lambda c: c.name)
def test_qwen3_skew_sweep_plans(cfg):
    # routing, plan, row maps and dispatch at full size for every skew level
    check_full_size(cfg, 1, n_tokens=2, n_rows=8)
    torch.cuda.empty_cache()


@pytest.mark.parametrize("cfg", [SMALL_BF16, MED_BF16, WIDE_BF16, C.OLMOE, C.DSV3], ids=lambda c: c.name)
def test_fused_ffn_matches_the_staged_launches(cfg):
    """FC1 and FC2 in one launch, FC2 tiles released per block pair by the
    readiness counts, give the same bits as the separate launches, with FC1
    reading xp or gathering x through the row map; a second call without a
    new plan does too (the counts start from zero again)."""
    inp = I.make_inputs(cfg, 3, "cuda")
    g = run_stages(cfg, inp)
    for _ in range(2):
        h2 = torch.full_like(g["h"], float("nan"))
        y2 = torch.full_like(g["yp"], float("nan"))
        M.moe_expert_ffn_fused(cfg, g["xp"], inp["w_gate_up"], inp["w_down"], h2, y2, g["ws"])
        assert M.moe_read_status(g["ws"]) & ~M.DEV_PLAN_INEXACT == 0
        total = g["plan"]["total_rows"]
        assert torch.equal(h2[:total], g["h"][:total])
        assert torch.equal(y2[:total], g["yp"][:total])
        # dispatch, FC1 and FC2 in one launch: FC1 reads x through the row map
        h3 = torch.full_like(g["h"], float("nan"))
        y3 = torch.full_like(g["yp"], float("nan"))
        M.moe_expert_ffn_fused_gather(cfg, inp["x"], inp["w_gate_up"], inp["w_down"], h3, y3, g["ws"])
        assert M.moe_read_status(g["ws"]) & ~M.DEV_PLAN_INEXACT == 0
        assert torch.equal(h3[:total], g["h"][:total])
        assert torch.equal(y3[:total], g["yp"][:total])
    del g, inp
    torch.cuda.empty_cache()
