"""The seeded input generator: published SplitMix64 outputs, distributions, recipes."""
import math

import numpy as np
import pytest
import torch

from routed_experts_b200 import configs as C
from routed_experts_b200 import inputs as I


def test_splitmix64_published_outputs():
    # First outputs of SplitMix64 seeded with 1234567, as listed with the
    # generator's reference implementation (Vigna's splitmix64.c test values).
    got = [int(v) & ((1 << 64) - 1) for v in I.splitmix64(1234567, 0, 5)]
    assert got == [6457827717110365317, 3203168211198807973, 9817491932198370423,
                   4593380528125082431, 16408922859458223821]


def test_splitmix64_matches_python_int_arithmetic():
    key = I.stream_key(7, 3)
    got = [int(v) & ((1 << 64) - 1) for v in I.splitmix64(key, 1000, 16)]
    g, m = 0x9E3779B97F4A7C15, (1 << 64) - 1
    ref = []
    for i in range(1000, 1016):
        z = (key + (i + 1) * g) & m
        z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & m
        z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & m
        ref.append(z ^ (z >> 31))
    assert got == ref


def test_uniform_and_normal_moments():
    u = I.uniform(I.stream_key(0, 99), 0, 1 << 20)
    assert float(u.min()) >= 0.0 and float(u.max()) < 1.0
    assert abs(float(u.mean()) - 0.5) < 2e-3
    n = I.normal(I.stream_key(0, 98), 1 << 20)
    assert abs(float(n.mean())) < 5e-3
    assert abs(float(n.std()) - 1.0) < 5e-3
    # chunk boundaries do not change the stream
    a = I.normal(I.stream_key(1, 5), 1001)
    b = torch.cat([I.normal(I.stream_key(1, 5), 1001)[:500], I.normal(I.stream_key(1, 5), 1001)[500:]])
    assert torch.equal(a, b)


def test_normal_is_chunk_invariant(monkeypatch):
    full = I.normal(I.stream_key(3, 4), 5003)
    monkeypatch.setattr(I, "_CHUNK", 1000)
    assert torch.equal(I.normal(I.stream_key(3, 4), 5003), full)
    monkeypatch.setattr(I, "_CHUNK", 777)
    assert torch.equal(I.normal(I.stream_key(3, 4), 5003), full)


def test_bf16_storage_rounds_fp32_values():
    v64 = I.normal(I.stream_key(2, 1), 4096)
    vb = I.normal(I.stream_key(2, 1), 4096, out_dtype=torch.bfloat16)
    assert torch.equal(v64.to(torch.float32).to(torch.bfloat16), vb)


def test_inputs_deterministic_and_seeded():
    cfg = C.TINY
    a = I.make_inputs(cfg, 0)
    b = I.make_inputs(cfg, 0)
    c = I.make_inputs(cfg, 1)
    for k in a:
        assert torch.equal(a[k], b[k])
    assert not torch.equal(a["x"], c["x"])
    assert a["logits"].shape == (cfg.T, cfg.E) and a["logits"].dtype == torch.float32
    assert a["w_gate_up"].shape == (cfg.E, 2 * cfg.F, cfg.d)
    assert a["w_down"].shape == (cfg.E, cfg.d, cfg.F)


def test_zipf_bias_is_a_permuted_zipf_ladder():
    cfg = C.OLMOE
    b = I.router_bias(cfg, 0).numpy()
    ranks = np.sort(np.exp(-b / cfg.zipf_s))
    assert np.allclose(ranks, np.arange(1, cfg.E + 1))


def test_hot_expert_recipe_puts_hot_expert_in_every_token():
    cfg = C.EXTREME.replace(T=512, d=64)
    inp = I.make_inputs(cfg, 0, weights=False)
    h = I.hot_expert(cfg, 0)
    lg = inp["logits"]
    assert bool((lg.argmax(dim=1) == h).all())


@pytest.mark.parametrize("cfg", list(C.NAMED.values()), ids=lambda c: c.name)
def test_named_configs_are_consistent(cfg):
    assert cfg.E % cfg.R == 0 and cfg.T % cfg.R == 0
    assert cfg.K <= cfg.E
    assert (cfg.S * cfg.K) % cfg.tile == 0
    assert cfg.d % 64 == 0 and cfg.F % 64 == 0
    if cfg.dtype == C.BF16:
        assert cfg.tile == 128


def test_expert_weights_match_slices_of_the_full_tensors(monkeypatch):
    # odd offsets and a chunk boundary inside an expert's range
    monkeypatch.setattr(I, "_CHUNK", 1000)
    cfg = C.LayerConfig("ew", T=16, d=64, E=5, K=2, F=48, R=1, tile=16, budget=0)
    full = I.make_inputs(cfg, 3)
    wgu, wdn = I.expert_weights(cfg, 3, [4, 1, 2])
    assert torch.equal(wgu, full["w_gate_up"][[4, 1, 2]])
    assert torch.equal(wdn, full["w_down"][[4, 1, 2]])


def test_normal_with_an_offset_is_a_slice():
    key = I.stream_key(9, 1)
    ref = I.normal(key, 101)
    for start in (0, 1, 2, 37, 64):
        assert torch.equal(I.normal(key, 101 - start, start=start), ref[start:])
