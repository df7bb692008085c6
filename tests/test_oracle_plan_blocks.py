"""Pins of the oracle's block-granular planner (MegaFlux's four-candidate
search with pruning and refinement): hand-derived cases, invariants every
plan must meet, and brute force over tiny layers for the best achievable
maximum load (the greedy is a heuristic: its gap is reported, not failed)."""
import itertools
import json
import os

import numpy as np
import pytest

from routed_experts_b200 import configs as C
from routed_experts_b200 import inputs as I

from .conftest import GOLDEN


def check_block_plan(pl, T, E, K, R, tile, budget, counts):
    per = E // R
    pieces = pl["pieces"]
    counts = np.asarray(counts, np.int64)
    b = -(-counts // tile)
    tau = -(-int(b.sum()) // R)
    assert pl["info"][0] == tau and pl["status"] == 0
    for e in range(E):
        segs = sorted((int(p[2]), int(p[3])) for p in pieces if p[0] == e)
        pos = 0
        for s_, ln in segs:
            assert ln > 0 and s_ == pos and s_ % tile == 0
            assert ln % tile == 0 or s_ + ln == counts[e], "only an expert's last block may be partial"
            pos += ln
        assert pos == counts[e]
    keys = [(int(p[1]), int(p[0])) for p in pieces]
    assert len(keys) == len(set(keys)) and keys == sorted(keys)
    reps = np.zeros(R, np.int64)
    lb = np.zeros(R, np.int64)
    for p in pieces:
        e, r = int(p[0]), int(p[1])
        reps[r] += e // per != r
        lb[r] += -(-int(p[3]) // tile)
    assert np.array_equal(reps, pl["rank_replicas"]) and reps.max(initial=0) <= budget
    assert pl["info"][3] == reps.sum()
    assert np.array_equal(np.diff(pl["rank_row0"]), lb * tile)
    init = b.reshape(R, per).sum(axis=1)
    assert lb.max() == pl["info"][2]
    assert tau <= lb.max() <= init.max()
    row = 0
    blocks = []
    for p in pieces:
        assert int(p[4]) == row
        for i in range(-(-int(p[3]) // tile)):
            blocks.append([int(p[0]), row + i * tile, min(tile, int(p[3]) - i * tile), int(p[1])])
        row += -(-int(p[3]) // tile) * tile
    assert pl["blocks"].tolist() == blocks
    return int(lb.max())


def test_golden_block_plans(orc):
    with open(os.path.join(GOLDEN, "plan_blocks_cases.json")) as f:
        cases = json.load(f)["cases"]
    for c in cases:
        pl = orc.plan(c["T"], c["E"], c["K"], c["R"], c["tile"], c["budget"], np.array(c["counts"]),
                      mode=orc.PLAN_BLOCKS)
        n = c["name"]
        assert pl["pieces"].tolist() == c["pieces"], n
        assert pl["rank_load"].tolist() == c["rank_load"], n
        assert pl["rank_replicas"].tolist() == c["rank_replicas"], n
        assert pl["rank_row0"].tolist() == c["rank_row0"], n
        assert pl["moves"] == c["moves"], n
        assert pl["info"].tolist() == c["info"], n
        check_block_plan(pl, c["T"], c["E"], c["K"], c["R"], c["tile"], c["budget"], c["counts"])


def _best_max_load(b, R, per, budget):
    """Smallest possible maximum block load: every split of every expert's
    blocks over ranks with at most `budget` foreign experts per rank."""
    E = len(b)
    splits = []
    for e in range(E):
        opts = []
        for comp in itertools.product(range(b[e] + 1), repeat=R):
            if sum(comp) == b[e]:
                opts.append(comp)
        splits.append(opts)
    best = None
    for choice in itertools.product(*splits):
        load = [0] * R
        reps = [0] * R
        for e, comp in enumerate(choice):
            for r in range(R):
                load[r] += comp[r]
                reps[r] += comp[r] > 0 and e // per != r
        if max(reps) <= budget:
            m = max(load)
            best = m if best is None else min(best, m)
    return best


@pytest.mark.parametrize("R,E,tile", [(2, 2, 1), (2, 4, 1), (3, 3, 1), (2, 4, 2)])
def test_brute_force_tiny_block_plans(orc, R, E, tile):
    per = E // R
    gaps = 0
    n = 0
    for counts in itertools.product(range(0, 5), repeat=E):
        T = sum(counts)
        if T == 0 or T % R:
            continue
        for budget in (0, 1, 2):
            pl = orc.plan(T, E, 1, R, tile, budget, np.array(counts), mode=orc.PLAN_BLOCKS)
            got = check_block_plan(pl, T, E, 1, R, tile, budget, counts)
            b = [-(-c // tile) for c in counts]
            opt = _best_max_load(b, R, per, budget)
            assert got >= opt
            gaps += got > opt
            n += 1
    print(f"R={R} E={E} tile={tile}: {n} plans, {gaps} above the best achievable maximum load")


def test_enough_budget_reaches_tau(orc):
    rng = np.random.default_rng(11)
    for it in range(200):
        R = int(rng.integers(1, 7))
        E = R * int(rng.integers(1, 4))
        tile = int(rng.choice([1, 2, 4, 8]))
        T = R * int(rng.integers(1, 30))
        counts = rng.multinomial(T * 2, rng.dirichlet(np.ones(E) * 0.3)).astype(np.int32)
        pl = orc.plan(T, E, 2, R, tile, E, counts, mode=orc.PLAN_BLOCKS)
        m = check_block_plan(pl, T, E, 2, R, tile, E, counts)
        assert m == pl["info"][0], (R, E, tile, counts.tolist())


@pytest.mark.parametrize("cfg", list(C.NAMED.values()), ids=lambda c: c.name)
def test_named_configs_block_plans(orc, cfg):
    for seed in (0, 1):
        lg = I.make_inputs(cfg, seed, weights=False)["logits"].numpy()
        idx, _ = orc.topk_gate(lg, cfg.K, cfg.gating)
        counts = orc.histogram(idx, cfg.E)
        pl = orc.plan(cfg.T, cfg.E, cfg.K, cfg.R, cfg.tile, cfg.budget, counts, mode=orc.PLAN_BLOCKS)
        check_block_plan(pl, cfg.T, cfg.E, cfg.K, cfg.R, cfg.tile, cfg.budget, counts)
        # the same entries reach the same layer output through either plan
        cap = orc.rows_capacity(cfg.N, cfg.E, cfg.R, cfg.budget, cfg.tile)
        assert pl["total_rows"] <= cap
        row_of, src_of = orc.row_maps(idx, cfg.E, pl["pieces"], cap)
        assert np.array_equal(src_of[row_of], np.repeat(np.arange(cfg.T), cfg.K))
