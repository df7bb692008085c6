"""Pins of the oracle's row maps and dispatch."""
import numpy as np
import pytest

from routed_experts_b200 import configs as C
from routed_experts_b200 import inputs as I


def test_golden_row_maps(orc, golden):
    cases = {c["name"]: c for c in golden["cases"]}
    for rm in golden["row_map_cases"]:
        pc = cases[rm["plan_case"]]
        idx = np.array(rm["idx"], np.int32)
        counts = orc.histogram(idx, pc["E"])
        assert counts.tolist() == pc["counts"]
        pl = orc.plan(pc["T"], pc["E"], pc["K"], pc["R"], pc["tile"], pc["budget"], counts)
        row_of, src_of = orc.row_maps(idx, pc["E"], pl["pieces"], rm["rows"])
        assert row_of.tolist() == rm["row_of"]
        assert src_of.tolist() == rm["src_of"]


def _library_positions(idx: np.ndarray, E: int) -> np.ndarray:
    """pos(t,k) by a stable library sort: the rank of entry (t,k) among the
    entries of its expert, in (t,k) order."""
    flat = idx.ravel()
    order = np.argsort(flat, kind="stable")
    starts = np.concatenate([[0], np.cumsum(np.bincount(flat, minlength=E))[:-1]])
    pos = np.empty_like(flat)
    pos[order] = np.arange(flat.size) - starts[flat[order]]
    return pos


@pytest.mark.parametrize("cfg", [C.TINY, C.OLMOE.replace(T=2048), C.DSV3.replace(T=1024, d=64),
                                 C.EXTREME.replace(T=2048, d=64)], ids=lambda c: c.name)
def test_row_maps_properties(orc, cfg):
    lg = I.make_inputs(cfg, 1, weights=False)["logits"].numpy()
    idx, _ = orc.topk_gate(lg, cfg.K, cfg.gating)
    counts = orc.histogram(idx, cfg.E)
    pl = orc.plan(cfg.T, cfg.E, cfg.K, cfg.R, cfg.tile, cfg.budget, counts)
    cap = orc.rows_capacity(cfg.N, cfg.E, cfg.R, cfg.budget, cfg.tile)
    assert pl["total_rows"] <= cap
    row_of, src_of = orc.row_maps(idx, cfg.E, pl["pieces"], cap)
    # row = row0 + pos - start of the piece holding pos (pos from a library sort)
    pos = _library_positions(idx, cfg.E)
    flat = idx.ravel()
    for i in range(flat.size):
        e, p = flat[i], pos[i]
        pc = [q for q in pl["pieces"] if q[0] == e and q[2] <= p < q[2] + q[3]]
        assert len(pc) == 1
        assert row_of[i] == pc[0][4] + p - pc[0][2]
    # bijection between entries and valid rows; padding rows are -1
    assert len(set(row_of.tolist())) == flat.size
    assert np.array_equal(src_of[row_of], np.repeat(np.arange(cfg.T), cfg.K))
    valid = np.zeros(cap, bool)
    for b in pl["blocks"]:
        valid[b[1]:b[1] + b[2]] = True
    assert np.array_equal(src_of >= 0, valid)
    # every valid row sits in a block of its entry's expert
    blk_expert = np.full(cap, -1)
    for b in pl["blocks"]:
        blk_expert[b[1]:b[1] + cfg.tile] = b[0]
    assert np.array_equal(blk_expert[row_of], flat)


@pytest.mark.parametrize("dtype", [C.BF16, C.FP32])
def test_dispatch_is_an_exact_copy(orc, dtype):
    rng = np.random.default_rng(3)
    T, d = 50, 64
    if dtype == C.BF16:
        x = rng.integers(0, 1 << 16, size=(T, d)).astype(np.uint16)
    else:
        x = rng.standard_normal((T, d)).astype(np.float32)
    src = rng.integers(-1, T, size=97).astype(np.int32)
    xp = orc.dispatch(x, src, dtype)
    for r, s in enumerate(src):
        if s < 0:
            assert not xp[r].any()
        else:
            assert xp[r].tobytes() == x[s].tobytes()
