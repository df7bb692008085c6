"""Pins of the oracle's top-k, gating and histogram (not against itself)."""
import numpy as np
import pytest
import scipy.special

from routed_experts_b200 import configs as C
from routed_experts_b200 import inputs as I


def test_gating_golden_cases(orc, golden):
    for case in golden["gating_cases"]:
        lg = np.array([case["logits"]], np.float32)
        for gating, key in ((C.GATE_SOFTMAX_TOPK, "softmax_topk_w"), (C.GATE_SIGMOID_TOPK, "sigmoid_topk_w")):
            idx, w = orc.topk_gate(lg, case["K"], gating)
            assert idx[0].tolist() == case["idx"], case["name"]
            np.testing.assert_allclose(w[0], case[key], rtol=0, atol=1e-7)


def _lexsort_topk(lg: np.ndarray, K: int) -> np.ndarray:
    # library route: sort each row by (-logit, expert id)
    T, E = lg.shape
    ids = np.broadcast_to(np.arange(E), (T, E))
    order = np.lexsort((ids, -lg.astype(np.float64)), axis=1)
    return order[:, :K].astype(np.int32)


@pytest.mark.parametrize("T,E,K", [(64, 8, 2), (33, 64, 8), (17, 256, 8), (40, 128, 8), (9, 5, 5)])
def test_topk_matches_library_sort(orc, T, E, K):
    rng = np.random.default_rng(T * 1000 + E)
    lg = rng.standard_normal((T, E)).astype(np.float32)
    # force ties: duplicate some columns and quantise a few rows
    lg[:, E // 2] = lg[:, 0]
    lg[::3] = np.round(lg[::3] * 2) / 2
    idx, _ = orc.topk_gate(lg, K, C.GATE_SOFTMAX_TOPK)
    assert np.array_equal(idx, _lexsort_topk(lg, K))
    assert all(len(set(r)) == K for r in idx.tolist())   # k distinct experts


@pytest.mark.parametrize("gating", [C.GATE_SOFTMAX_TOPK, C.GATE_SIGMOID_TOPK])
def test_gating_matches_library_closed_forms(orc, gating):
    rng = np.random.default_rng(5 + gating)
    T, E, K = 200, 32, 4
    lg = (rng.standard_normal((T, E)) * 3).astype(np.float32)
    idx, w = orc.topk_gate(lg, K, gating)
    l64 = lg.astype(np.float64)
    if gating == C.GATE_SOFTMAX_TOPK:
        p = scipy.special.softmax(l64, axis=1)      # full softmax, then renormalise over top-k
    else:
        p = scipy.special.expit(l64)
    sel = np.take_along_axis(p, idx.astype(np.int64), axis=1)
    ref = sel / sel.sum(axis=1, keepdims=True)
    np.testing.assert_allclose(w, ref, rtol=0, atol=2e-7)
    np.testing.assert_allclose(w.astype(np.float64).sum(axis=1), 1.0, atol=1e-6)
    assert np.all(np.diff(w, axis=1) <= 0) or gating == C.GATE_SIGMOID_TOPK


def test_histogram_matches_bincount(orc):
    rng = np.random.default_rng(1)
    idx = rng.integers(0, 37, size=(300, 6)).astype(np.int32)
    assert np.array_equal(orc.histogram(idx, 37), np.bincount(idx.ravel(), minlength=37))


@pytest.mark.parametrize("cfg", [C.TINY, C.OLMOE.replace(T=1024), C.DSV3.replace(T=512, d=64)],
                         ids=lambda c: c.name)
def test_generated_routing_properties(orc, cfg):
    inp = I.make_inputs(cfg, 0, weights=False)
    lg = inp["logits"].numpy()
    idx, w = orc.topk_gate(lg, cfg.K, cfg.gating)
    counts = orc.histogram(idx, cfg.E)
    assert counts.sum() == cfg.T * cfg.K
    assert counts.max() <= cfg.T                      # distinct experts cap one expert at T
    assert np.array_equal(idx, _lexsort_topk(lg, cfg.K))
