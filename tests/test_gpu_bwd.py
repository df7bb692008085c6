"""GPU parity of the layer's backward ([MegaFlux] §3.2 "Backward") against
the CPU oracle's backward, through the C ABI.

dx is compared element by element at the bf16 tolerance; the fp32 weight
gradients and the logits' gradient, sums of many rounded products whose
accumulation order differs (fp32 in the tensor cores, fp64 in the oracle),
elementwise against their own scale and in norm.
"""
import numpy as np
import pytest
import torch

from oracle import oracle as O
from routed_experts_b200 import configs as C
from routed_experts_b200 import inputs as I
from routed_experts_b200 import moe as M

from .gpu_helpers import assert_close, assert_grad_close, check_bwd_small, run_bwd, to_f64

pytestmark = pytest.mark.gpu

SMALL = C.LayerConfig("bwd_small", T=512, d=256, E=8, K=2, F=256, R=4, tile=128, budget=2, zipf_s=1.0)
MED = C.LayerConfig("bwd_med", T=1024, d=512, E=16, K=4, F=512, R=4, tile=128, budget=2, zipf_s=1.2,
                    gating=C.GATE_SIGMOID_TOPK, logits="normal")
WIDE = C.LayerConfig("bwd_wide", T=256, d=768, E=32, K=8, F=256, R=8, tile=128, budget=4, zipf_s=1.5)
# an expert nobody chooses (zero gradient) and experts with odd block counts
SPARSE = C.LayerConfig("bwd_sparse", T=384, d=256, E=16, K=2, F=256, R=4, tile=128, budget=1, hot_bias=30.0)


@pytest.fixture(scope="module", autouse=True)
def _built():
    from routed_experts_b200 import build
    build.build()
    O.build()


@pytest.mark.parametrize("cfg", [SMALL, MED, WIDE, SPARSE], ids=lambda c: c.name)
def test_backward_small_layers(cfg):
    check_bwd_small(cfg, 0)


def test_backward_block_planner():
    check_bwd_small(SMALL.replace(name="bwd_small_blocks", plan_mode=C.PLAN_BLOCKS), 1)


def test_backward_is_deterministic_and_plan_invariant():
    """Repeated calls give identical bits. Another plan moves rows between
    blocks: dx and the logits' gradient are per-entry arithmetic and keep
    every bit; the weight gradients change only by fp32 summation order."""
    inp, d_out, layer, g0 = run_bwd(SMALL, 3)
    g1 = layer.backward(inp["logits"], inp["w_gate_up"], inp["w_down"], d_out)
    for a, b in zip(g0, g1):
        assert torch.equal(a, b)
    other = SMALL.replace(R=8, budget=3)
    layer2 = M.Layer(other, train=True)
    layer2.forward(inp["logits"], inp["x"], inp["w_gate_up"], inp["w_down"])
    g2 = layer2.backward(inp["logits"], inp["w_gate_up"], inp["w_down"], d_out)
    assert torch.equal(g0[0], g2[0]) and torch.equal(g0[3], g2[3])
    for a, b, n in ((g0[1], g2[1], "dw_gate_up"), (g0[2], g2[2], "dw_down")):
        assert_grad_close(b.cpu().numpy(), a.cpu().numpy(), n, rel=1e-5)


def test_training_forward_gives_the_inference_output():
    for cfg in (SMALL, WIDE):
        inp = I.make_inputs(cfg, 6, "cuda")
        train, infer = M.Layer(cfg, train=True), M.Layer(cfg)
        a = train.forward(inp["logits"], inp["x"], inp["w_gate_up"], inp["w_down"])
        b = infer.forward(inp["logits"], inp["x"], inp["w_gate_up"], inp["w_down"])
        assert torch.equal(a, b)


def test_backward_leaves_the_forward_output_alone():
    inp, d_out, layer, _ = run_bwd(SMALL, 4)
    before = layer.out.clone()
    layer.backward(inp["logits"], inp["w_gate_up"], inp["w_down"], d_out)
    assert torch.equal(layer.out, before)


@pytest.mark.parametrize("cfg", [C.OLMOE, C.DSV3], ids=lambda c: c.name)
def test_backward_full_size_sampled(cfg):
    """Full-size layers: sampled tokens' dx, dw-driven logit gradients, and
    sampled weight-gradient elements of two experts, against the oracle."""
    inp, d_out, layer, (dx, dwgu, dwdn, dl) = run_bwd(cfg, 0)
    hl = I.to_numpy_bits(inp["logits"])
    idx, w = O.topk_gate(hl, cfg.K, cfg.gating)
    rng = np.random.default_rng(1)
    toks = rng.choice(cfg.T, size=4, replace=False)
    hx = I.to_numpy_bits(inp["x"])
    hgu = I.to_numpy_bits(inp["w_gate_up"])
    hdn = I.to_numpy_bits(inp["w_down"])
    hdo = I.to_numpy_bits(d_out)
    rdx, _, rdl = O.bwd_tokens(toks, hl, idx, w, hx, hgu, hdn, hdo, gating=cfg.gating, dtype=cfg.dtype,
                               round_mode=O.ROUND_BF16)
    t_dev = torch.as_tensor(toks, device="cuda")
    assert_close(to_f64(dx[t_dev]), rdx, cfg.dtype, "sampled dx rows")
    assert_grad_close(dl[t_dev].cpu().numpy(), rdl, "sampled dlogits rows")
    counts = np.bincount(idx.ravel(), minlength=cfg.E)
    # the least and the median loaded of the chosen experts (the oracle's sum
    # over an expert's entries runs in seconds for those)
    used = np.nonzero(counts)[0]
    by_load = used[np.argsort(counts[used], kind="stable")]
    for e in (int(by_load[0]), int(by_load[len(by_load) // 2])):
        n = 24
        which = rng.integers(0, 3, n)
        r = np.where(which == 2, rng.integers(0, cfg.d, n), rng.integers(0, cfg.F, n))
        c = np.where(which == 2, rng.integers(0, cfg.F, n), rng.integers(0, cfg.d, n))
        ref = O.bwd_wgrad_elems(e, which, r, c, idx, w, hx, hgu, hdn, hdo, dtype=cfg.dtype,
                                round_mode=O.ROUND_BF16)
        gu = dwgu[e].cpu().numpy()
        dn = dwdn[e].cpu().numpy()
        got = np.where(which == 0, gu[r % cfg.F, c % cfg.d], 0.0)
        got = np.where(which == 1, gu[cfg.F + r % cfg.F, c % cfg.d], got)
        got = np.where(which == 2, dn[r % cfg.d, c % cfg.F], got)
        # elementwise at the scale of the whole gradient of this expert
        scale = np.sqrt(np.mean(np.concatenate([gu.ravel(), dn.ravel()]).astype(np.float64) ** 2))
        err = np.abs(got - ref)
        assert (err <= 1e-2 * (2 * scale + np.abs(ref))).all(), (e, err.max(), scale)
    del layer
    torch.cuda.empty_cache()
