"""GPU parity of the MXFP8 forward ([MegaFlux] §2.1 'Persistent MoE
execution': block-scaled MX MMA; §4.1 'Setup': the forward on MX operands,
fp32 accumulation, bf16 outputs) against the oracle, through the C ABI.

Weights and dispatched token rows are compared bit for bit (codes and
scales); h, formed in fp32 on the GPU and fp64 in the oracle before its
rounding to bf16 and MXFP8, within one E4M3 step with differing codes rare;
yp and out within the bf16 output tolerance."""
import numpy as np
import pytest
import torch

from routed_experts_b200 import configs as C
from routed_experts_b200 import moe as M

from .gpu_helpers import check_mx_full_size, check_mx_small

pytestmark = pytest.mark.gpu

# Small MX layers: 128-row blocks (tile 128), d % 256 == 0, F % 128 == 0.
MX_SMALL = C.LayerConfig("mx_small", T=512, d=256, E=8, K=2, F=256, R=4, tile=128, budget=2, zipf_s=1.0)
MX_SKEW = C.LayerConfig("mx_skew", T=1024, d=512, E=16, K=4, F=384, R=4, tile=128, budget=2, zipf_s=1.5,
                        hot_bias=3.0, hot_frac=0.5)
MX_SIGMOID = C.LayerConfig("mx_sigmoid", T=768, d=768, E=12, K=3, F=128, R=4, tile=128, budget=1,
                           gating=C.GATE_SIGMOID_TOPK, zipf_s=0.8)


FMTS = [M.MX_W_E4M3, M.MX_W_E2M1]
FMT_IDS = ["mxfp8_w", "mxfp4_w"]


@pytest.mark.parametrize("wfmt", FMTS, ids=FMT_IDS)
@pytest.mark.parametrize("cfg", [MX_SMALL, MX_SKEW, MX_SIGMOID], ids=lambda c: c.name)
def test_mx_layer_small(cfg, wfmt):
    check_mx_small(cfg, 0, wfmt=wfmt)


@pytest.mark.parametrize("wfmt", FMTS, ids=FMT_IDS)
def test_mx_layer_second_seed_and_block_planner(wfmt):
    check_mx_small(MX_SKEW.replace(name="mx_skew_blocks", plan_mode=C.PLAN_BLOCKS), 3, wfmt=wfmt)


def test_mx_layer_entry_matches_the_stages():
    """moe_layer_fwd_mx gives the same bits as the staged MX calls."""
    from routed_experts_b200 import inputs as I
    cfg = MX_SKEW
    from .gpu_helpers import run_mx_stages
    inp = I.make_inputs(cfg, 1, "cuda")
    g = run_mx_stages(cfg, inp, M.MX_W_E2M1)
    layer = M.Layer(cfg, "cuda")
    out = layer.forward_mx(inp["logits"], inp["x"], g["mxw"])
    torch.cuda.synchronize()
    assert torch.equal(out, g["out"])
    out2 = layer.forward_mx(inp["logits"], inp["x"], g["mxw"]).clone()
    assert torch.equal(out2, out), "the MX layer is deterministic"


@pytest.mark.parametrize("wfmt,bound", [(M.MX_W_E4M3, 0.08), (M.MX_W_E2M1, 0.3)], ids=FMT_IDS)
def test_mx_layer_is_close_to_the_bf16_layer(wfmt, bound):
    """MX operands move the output by about their rounding (E4M3: 2^-4
    relative per element; E2M1 weights: up to 1/6 relative), not more: a
    check of scale handling at size."""
    from routed_experts_b200 import inputs as I
    cfg = MX_SKEW
    inp = I.make_inputs(cfg, 2, "cuda")
    layer = M.Layer(cfg, "cuda")
    ref = layer.forward(inp["logits"], inp["x"], inp["w_gate_up"], inp["w_down"]).float().clone()
    mxw = M.MxWeights(cfg, inp["w_gate_up"], inp["w_down"], wfmt=wfmt)
    out = layer.forward_mx(inp["logits"], inp["x"], mxw).float()
    rel = (torch.linalg.norm(out - ref) / torch.linalg.norm(ref)).item()
    assert rel < bound, rel
    assert rel > 1e-4, "the MX layer should not be the bf16 layer"


@pytest.mark.parametrize("wfmt", FMTS, ids=FMT_IDS)
@pytest.mark.parametrize("name", ["olmoe", "dsv3"])
def test_mx_layer_full_size(name, wfmt):
    # one row of h and yp in every planned block, 32 tokens of out
    check_mx_full_size(C.NAMED[name], 0, n_tokens=32, wfmt=wfmt)
    torch.cuda.empty_cache()
