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

from .gpu_helpers import check_full_size, check_full_small, check_routing_full_size, run_path, run_stages, to_f64

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
# Large enough that every cluster of CTA pairs takes several work items of
# FC1 and of FC2 (about 300 each over 74 pairs), the operand ring wraps
# inside every item (16 or 8 k-steps against 6 stages) and both TMEM
# accumulators alternate; small enough for the oracle on a few cores.
RING_BF16 = C.LayerConfig("ring_bf16", T=4096, d=1024, E=16, K=4, F=512, R=8, tile=128, budget=2,
                          zipf_s=1.0)


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
    check_full_size(cfg.replace(name=cfg.name + "_blocks", plan_mode=C.PLAN_BLOCKS), 0, n_tokens=32)
    torch.cuda.empty_cache()


# The extreme-skew shape's second reading of its hot expert: the +30 bias
# on half of the tokens only (the expert still takes the largest share).
EXTREME_HOT50 = C.EXTREME.replace(name="extreme_hot50", hot_frac=0.5)
FULL = [C.OLMOE, C.QWEN3, C.EXTREME, C.DSV3, EXTREME_HOT50]


@pytest.mark.parametrize("cfg", FULL, ids=lambda c: c.name)
def test_full_size_layer(cfg):
    check_full_size(cfg, 0)
    torch.cuda.empty_cache()


@pytest.mark.parametrize("seed", [1, 2])
@pytest.mark.parametrize("cfg", FULL + list(C.QWEN3_SWEEP), ids=lambda c: c.name)
def test_full_size_routing_other_seeds(cfg, seed):
    # routing, gating, counts, plan and row maps for the other realizations
    check_routing_full_size(cfg, seed)
    torch.cuda.empty_cache()


@pytest.mark.parametrize("seed", [1, 2])
@pytest.mark.parametrize("cfg", [C.OLMOE, C.DSV3], ids=lambda c: c.name)
def test_full_size_layer_other_seeds(cfg, seed):
    check_full_size(cfg, seed, n_tokens=32)
    torch.cuda.empty_cache()


@pytest.mark.parametrize("cfg", C.QWEN3_SWEEP, ids=lambda c: c.name)
def test_qwen3_skew_sweep(cfg):
    # every skew level at full size: the plan bit-exact, every block sampled
    check_full_size(cfg, 1, n_tokens=32)
    torch.cuda.empty_cache()


FUSED_PATHS = ["fused", "fused_gather", "fc1_gather", "fc2_combine", "layer"]


@pytest.mark.parametrize("path", ["layer", "fc1_gather"])
def test_full_size_qwen3_layer_reading_x(path):
    """The Qwen3-shaped layer's x takes exactly 64 MiB: moe_layer_fwd reads
    FC1's rows from x there too."""
    assert M.moe_layer_path(C.QWEN3) == M.PATH_GATHER_FC1
    check_full_size(C.QWEN3, 3, path=path, n_tokens=32)
    torch.cuda.empty_cache()


@pytest.mark.parametrize("path", FUSED_PATHS)
@pytest.mark.parametrize("cfg", [C.OLMOE, C.DSV3], ids=lambda c: c.name)
def test_full_size_other_paths(cfg, path):
    """The fused launches, FC1 with the dispatch folded in, and the whole-layer
    entry against the oracle and the fp64 reference at full size."""
    check_full_size(cfg, 3, path=path, n_tokens=32)
    torch.cuda.empty_cache()


@pytest.mark.parametrize("path", ["staged", "fused", "fused_gather", "fc1_gather", "fc2_combine"])
def test_every_element_of_a_layer_whose_clusters_take_several_items(path):
    check_full_small(RING_BF16, 0, path=path, threads=True)
    torch.cuda.empty_cache()


@pytest.mark.parametrize("cfg", [SMALL_BF16, MED_BF16, WIDE_BF16], ids=lambda c: c.name)
@pytest.mark.parametrize("path", ["fused", "fused_gather", "fc1_gather", "fc2_combine"])
def test_small_layers_other_paths(cfg, path):
    check_full_small(cfg, 3, path=path)


# The combine folded into FC2: one row per token (K = 1), K = 16 (two
# batches of eight rows in the summing lanes), one token per rank.
FOLD_EDGE = [SMALL_BF16.replace(name="k1", K=1), EDGE[5], EDGE[3], EDGE[0]]


@pytest.mark.parametrize("cfg", FOLD_EDGE, ids=lambda c: c.name)
def test_fc2_combine_edge_shapes(cfg):
    check_full_small(cfg, 2, path="fc2_combine")


# FC1 reading x (the layer's path for bf16 layers whose x is at most 64 MiB)
# on the edge shapes: ragged chunks, K = E, E = R, one token per rank, a hot
# expert, E = 1024 with K = 16.
EDGE_BF16 = [c for c in EDGE if c.dtype == C.BF16]


@pytest.mark.parametrize("cfg", EDGE_BF16, ids=lambda c: c.name)
def test_fc1_gather_edge_shapes(cfg):
    check_full_small(cfg, 2, path="fc1_gather")


@pytest.mark.parametrize("cfg", EDGE_BF16, ids=lambda c: c.name)
def test_layer_matches_staged_calls_on_edge_shapes(cfg):
    assert M.moe_layer_path(cfg) == M.PATH_GATHER_FC1
    inp = I.make_inputs(cfg, 4, "cuda")
    staged = run_stages(cfg, inp)["out"]
    layer = M.Layer(cfg)
    out = layer.forward(inp["logits"], inp["x"], inp["w_gate_up"], inp["w_down"])
    assert layer.status() & ~M.DEV_PLAN_INEXACT == 0
    assert torch.equal(out, staged)


@pytest.mark.parametrize("cfg", [SMALL_BF16, MED_BF16, WIDE_BF16, RING_BF16, C.OLMOE, C.DSV3],
                         ids=lambda c: c.name)
def test_fc2_combine_is_bit_identical_to_fc2_then_combine(cfg):
    """FC2 with the combine folded in stores the same yp bits as moe_expert_fc2
    and the same out bits as moe_combine (the same fixed k order, fp32 sum
    and rounding), and a second call on the same workspace gives them again."""
    inp = I.make_inputs(cfg, 6, "cuda")
    a = run_path(cfg, inp, "staged")
    b = run_path(cfg, inp, "fc2_combine")
    assert b["status"] & ~M.DEV_PLAN_INEXACT == 0
    valid = torch.as_tensor(np.nonzero(a["plan"]["src_of"].numpy() >= 0)[0], device="cuda")
    assert torch.equal(b["yp"][valid], a["yp"][valid])
    assert torch.equal(b["out"], a["out"])
    out2 = torch.full_like(b["out"], float("nan"))
    M.moe_expert_fc2_combine(cfg, b["h"], inp["w_down"], b["w"], b["yp"], out2, b["ws"])
    assert M.moe_read_status(b["ws"]) & ~M.DEV_PLAN_INEXACT == 0
    assert torch.equal(out2, a["out"])
    del a, b, inp
    torch.cuda.empty_cache()


def test_fc2_combine_needs_a_layer_workspace_and_bf16():
    cfg = SMALL_BF16
    ws = M.alloc_workspace(cfg, M.WS_PLAN)
    z = torch.zeros(16, dtype=torch.bfloat16, device="cuda")
    w = torch.zeros(16, dtype=torch.float32, device="cuda")
    with pytest.raises(M.MoeError) as e:
        M.moe_expert_fc2_combine(cfg, z, z, w, z, z, ws)
    assert e.value.code == M.MOE_ERR_WORKSPACE
    with pytest.raises(M.MoeError) as e:
        M.moe_expert_fc2_combine(C.TINY, z, z, w, z, z, M.alloc_workspace(C.TINY, M.WS_LAYER))
    assert e.value.code == M.MOE_ERR_UNSUPPORTED


@pytest.mark.parametrize("cfg", [MED_BF16, C.OLMOE], ids=lambda c: c.name)
def test_layer_clears_what_an_earlier_call_left(cfg):
    """moe_layer_fwd on a workspace whose layer part holds garbage (as after a
    call that stopped at a timeout) gives the bits of the staged launches:
    every word it reads there is written earlier in the same call."""
    inp = I.make_inputs(cfg, 7, "cuda")
    staged = run_stages(cfg, inp)["out"]
    layer = M.Layer(cfg)
    for fill in (255, 1):
        layer.ws[M.moe_workspace_size(cfg, M.WS_PLAN):].fill_(fill)
        out = layer.forward(inp["logits"], inp["x"], inp["w_gate_up"], inp["w_down"])
        assert layer.status() & ~M.DEV_PLAN_INEXACT == 0
        assert torch.equal(out, staged), fill
    del layer, inp
    torch.cuda.empty_cache()


@pytest.mark.parametrize("cfg", [SMALL_BF16, MED_BF16, C.OLMOE], ids=lambda c: c.name)
@pytest.mark.parametrize("path", ["fused", "fused_gather"])
def test_fused_ffn_is_repeatable(cfg, path):
    """A second fused call on the same workspace, without a new plan, gives
    the same bits (its readiness counts and queues start from zero again)."""
    inp = I.make_inputs(cfg, 3, "cuda")
    a = run_path(cfg, inp, path)
    h2, y2 = torch.empty_like(a["h"]), torch.empty_like(a["yp"])
    if path == "fused":
        M.moe_expert_ffn_fused(cfg, a["xp"], inp["w_gate_up"], inp["w_down"], h2, y2, a["ws"])
    else:
        M.moe_expert_ffn_fused_gather(cfg, inp["x"], inp["w_gate_up"], inp["w_down"], h2, y2, a["ws"])
    assert M.moe_read_status(a["ws"]) & ~M.DEV_PLAN_INEXACT == 0
    valid = torch.as_tensor(np.nonzero(a["plan"]["src_of"].numpy() >= 0)[0], device="cuda")
    assert torch.equal(h2[valid], a["h"][valid])
    assert torch.equal(y2[valid], a["yp"][valid])
    del a, inp
    torch.cuda.empty_cache()
