"""Pins of the oracle's backward ([MegaFlux] §3.2 "Backward").

The oracle states the backward step by step (DGrad through W2 then W1,
the SwiGLU derivative, WGrad per expert, the gating Jacobian). It is pinned
to two things outside itself: torch's autograd of a plain dense fp64
implementation of the layer's forward, and central differences of the
oracle's own forward (token_out) on sampled coordinates.
"""
import numpy as np
import pytest
import torch

from oracle import oracle as O
from routed_experts_b200 import configs as C
from routed_experts_b200 import inputs as I


def _case(T, d, E, K, F, gating, seed):
    """fp32 inputs with distinct logits (no top-k ties), weights of the usual scale."""
    rng = np.random.default_rng(seed)
    logits = rng.standard_normal((T, E)).astype(np.float32)
    x = rng.standard_normal((T, d)).astype(np.float32)
    w_gu = (0.3 * rng.standard_normal((E, 2 * F, d))).astype(np.float32)
    w_down = (0.3 * rng.standard_normal((E, d, F))).astype(np.float32)
    d_out = rng.standard_normal((T, d)).astype(np.float32)
    idx, w = O.topk_gate(logits, K, gating)
    return dict(logits=logits, x=x, w_gu=w_gu, w_down=w_down, d_out=d_out, idx=idx, w=w, gating=gating, K=K)


def _torch_grads(c):
    """Autograd of the dense definition: top-k by torch.topk, gating over the
    chosen logits, every chosen expert's SwiGLU FFN, weighted sum."""
    l = torch.tensor(c["logits"], dtype=torch.float64, requires_grad=True)
    x = torch.tensor(c["x"], dtype=torch.float64, requires_grad=True)
    wgu = torch.tensor(c["w_gu"], dtype=torch.float64, requires_grad=True)
    wdn = torch.tensor(c["w_down"], dtype=torch.float64, requires_grad=True)
    F = wdn.shape[2]
    vals, ids = torch.topk(l, c["K"], dim=1)
    if c["gating"] == C.GATE_SOFTMAX_TOPK:
        wk = torch.softmax(vals, dim=1)
    else:
        s = torch.sigmoid(vals)
        wk = s / s.sum(dim=1, keepdim=True)
    g_all = torch.einsum("td,tkfd->tkf", x, wgu[ids])          # [T, K, 2F]
    a, g = g_all[..., :F], g_all[..., F:]
    h = torch.nn.functional.silu(a) * g
    y = torch.einsum("tkf,tkdf->tkd", h, wdn[ids])
    out = (wk[..., None] * y).sum(dim=1)
    (out * torch.tensor(c["d_out"], dtype=torch.float64)).sum().backward()
    return ids.numpy(), {"dx": x.grad.numpy(), "dw_gate_up": wgu.grad.numpy(), "dw_down": wdn.grad.numpy(),
                         "dlogits": l.grad.numpy()}


def _oracle_bwd(c, dtype=C.FP32, round_mode=O.ROUND_NONE):
    return O.layer_bwd(c["logits"], c["idx"], c["w"], c["x"], c["w_gu"], c["w_down"], c["d_out"],
                       gating=c["gating"], dtype=dtype, round_mode=round_mode)


def _rel(a, b):
    return np.linalg.norm(np.asarray(a, np.float64) - b) / max(np.linalg.norm(b), 1e-300)


@pytest.mark.parametrize("gating", [C.GATE_SOFTMAX_TOPK, C.GATE_SIGMOID_TOPK], ids=["softmax", "sigmoid"])
@pytest.mark.parametrize("shape", [(6, 8, 4, 2, 6), (5, 16, 6, 3, 8), (4, 8, 1, 1, 5), (7, 12, 5, 5, 4)],
                         ids=["base", "k3", "e1k1", "k_eq_e"])
def test_backward_matches_autograd(orc, gating, shape):
    T, d, E, K, F = shape
    c = _case(T, d, E, K, F, gating, seed=sum(shape) + gating)
    ids, ref = _torch_grads(c)
    assert np.array_equal(ids, c["idx"])
    got = _oracle_bwd(c)
    # fp32 routing weights on the oracle's side (as stored by the layer) against
    # fp64 ones in torch: agreement to a few fp32 ulps, nothing looser
    for key in ("dx", "dw_gate_up", "dw_down", "dlogits"):
        assert _rel(got[key], ref[key]) < 1e-6, key
    # unchosen experts get no logit gradient, chosen ones do
    mask = np.zeros_like(ref["dlogits"], bool)
    np.put_along_axis(mask, c["idx"], True, axis=1)
    assert not got["dlogits"][~mask].any()


def test_e1_k1_softmax_has_no_logit_gradient(orc):
    c = _case(5, 8, 1, 1, 6, C.GATE_SOFTMAX_TOPK, seed=3)
    got = _oracle_bwd(c)
    # one expert, weight 1 whatever the logit: the layer is a plain SwiGLU MLP
    assert not got["dlogits"].any()
    assert np.allclose(c["w"], 1.0)


def test_backward_matches_central_differences(orc):
    """d(sum(out * d_out))/d(theta) from the oracle's own forward, by central
    differences in fp64 on sampled coordinates of x and both weights."""
    T, d, E, K, F = 5, 8, 4, 2, 6
    c = _case(T, d, E, K, F, C.GATE_SOFTMAX_TOPK, seed=7)
    got = _oracle_bwd(c)
    tokens = np.arange(T)

    def loss(x, wgu, wdn):
        out = O.token_out(tokens, x.astype(np.float32), c["idx"], c["w"], wgu.astype(np.float32),
                          wdn.astype(np.float32), C.FP32, O.ROUND_NONE)
        return float((out * c["d_out"]).sum())

    rng = np.random.default_rng(0)
    base = {"x": c["x"], "w_gu": c["w_gu"], "w_down": c["w_down"]}
    grads = {"x": got["dx"], "w_gu": got["dw_gate_up"], "w_down": got["dw_down"]}
    for name in ("x", "w_gu", "w_down"):
        for _ in range(6):
            pos = tuple(rng.integers(0, n) for n in base[name].shape)
            h = 2.0 ** -8   # exact in fp32, so the perturbed inputs are what the forward reads
            args = {k: v.copy() for k, v in base.items()}
            args[name][pos] += h
            up = loss(args["x"], args["w_gu"], args["w_down"])
            args[name][pos] -= 2 * h
            dn = loss(args["x"], args["w_gu"], args["w_down"])
            fd = (up - dn) / (2 * h)
            assert abs(fd - grads[name][pos]) <= 1e-4 * max(1.0, abs(fd)), (name, pos, fd, grads[name][pos])


def test_token_and_element_samplers_agree_with_the_full_backward(orc):
    cfg = C.TINY.replace(dtype=C.BF16, T=64, d=64, F=64)
    inp = {k: I.to_numpy_bits(v) for k, v in I.make_inputs(cfg, 1).items()}
    idx, w = O.topk_gate(inp["logits"], cfg.K, cfg.gating)
    rng = np.random.default_rng(5)
    d_out = I.to_numpy_bits(torch.tensor(rng.standard_normal((cfg.T, cfg.d)), dtype=torch.float32).to(torch.bfloat16))
    full = O.layer_bwd(inp["logits"], idx, w, inp["x"], inp["w_gate_up"], inp["w_down"], d_out,
                       gating=cfg.gating, dtype=cfg.dtype, round_mode=O.ROUND_BF16)
    toks = np.array([0, 17, 63])
    dx, dw, dl = O.bwd_tokens(toks, inp["logits"], idx, w, inp["x"], inp["w_gate_up"], inp["w_down"], d_out,
                              gating=cfg.gating, dtype=cfg.dtype, round_mode=O.ROUND_BF16)
    assert np.array_equal(dx, O.to_f64(full["dx"][toks], cfg.dtype))
    assert np.array_equal(dw, full["dw"][toks]) and np.array_equal(dl, full["dlogits"][toks])
    for e in range(cfg.E):
        which = rng.integers(0, 3, 20)
        r = np.where(which == 2, rng.integers(0, cfg.d, 20), rng.integers(0, cfg.F, 20))
        cc = np.where(which == 2, rng.integers(0, cfg.F, 20), rng.integers(0, cfg.d, 20))
        got = O.bwd_wgrad_elems(e, which, r, cc, idx, w, inp["x"], inp["w_gate_up"], inp["w_down"], d_out,
                                dtype=cfg.dtype, round_mode=O.ROUND_BF16)
        ref = np.where(which == 0, full["dw_gate_up"][e, r % cfg.F, cc % cfg.d], 0.0)
        ref = np.where(which == 1, full["dw_gate_up"][e, cfg.F + r % cfg.F, cc % cfg.d], ref)
        ref = np.where(which == 2, full["dw_down"][e, r % cfg.d, cc % cfg.F], ref)
        np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-300)


def test_bf16_rounding_points_stay_close_to_fp64(orc):
    """The bf16 mode differs from pure fp64 only by its roundings: a few
    tenths of a percent in norm, never a different order of magnitude."""
    c = _case(8, 16, 4, 2, 8, C.GATE_SOFTMAX_TOPK, seed=11)
    bits = {k: I.to_numpy_bits(torch.tensor(c[k]).to(torch.bfloat16)) for k in ("x", "w_gu", "w_down", "d_out")}
    cb = dict(c, **bits)
    exact = _oracle_bwd(dict(c, **{k: O.bf16_bits_to_f64(v).astype(np.float32) for k, v in bits.items()}))
    rounded = _oracle_bwd(cb, dtype=C.BF16, round_mode=O.ROUND_BF16)
    assert _rel(O.bf16_bits_to_f64(rounded["dx"]), exact["dx"]) < 2e-2
    for key in ("dw_gate_up", "dw_down", "dlogits"):
        assert _rel(rounded[key], exact[key]) < 2e-2, key
