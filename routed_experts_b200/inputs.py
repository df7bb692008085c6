"""Seeded synthetic inputs for the routed-expert MoE layer.

This module only draws random tensors. It holds none of the layer's
arithmetic (no top-k, gating, planning, permutation, FFN or combine), so
both the CUDA path's tests and the CPU oracle's tests may take their
inputs from it.

Generator (counter-based, so any element can be drawn on any device):
  * SplitMix64 (Steele, Lea, Flood, "Fast splittable pseudorandom number
    generators", OOPSLA 2014): output i of a stream whose state starts at
    ``key`` is mix64(key + (i+1)*0x9E3779B97F4A7C15), with
    mix64(z) = z ^= z>>30; z *= 0xBF58476D1CE4E5B9; z ^= z>>27;
               z *= 0x94D049BB133111EB; z ^= z>>31.
  * stream key of (seed, tensor id) = first output of a SplitMix64 stream
    whose state starts at seed * 2**16 + tensor_id.
  * uniform in [0,1): top 53 bits * 2**-53.
  * normal: Box-Muller on consecutive uniform pairs (u0, u1):
    r = sqrt(-2 ln(1-u0)); n0 = r cos(2 pi u1), n1 = r sin(2 pi u1).
  * bf16 tensors: fp64 -> fp32 (round to nearest even) -> bf16 (round to
    nearest even).

Recipe per layer (input workloads of the MegaFlux paper, §4.1 "Routing
workload construction": balanced routes and Zipf-skewed expert popularity
with expert loads permuted across fixed owners):
  * x ~ N(0,1), [T, d].
  * router weights Wr ~ N(0, w_std^2), [d, E]; expert weights
    w_gate_up [E, 2F, d] and w_down [E, d, F] ~ N(0, w_std^2).
  * logits = fp32(x @ Wr + bias) in fp64 ("xwr"), or fp32(N(0,1) + bias)
    ("normal").
  * Zipf bias: bias_e = -s * ln(rank_e), rank_e = 1 + position of expert e
    in a seeded permutation of the experts (the stable argsort of E uniform
    draws).
  * hot expert: a seeded expert gets +hot_bias on a seeded hot_frac of the
    tokens.

The integer part is bit-identical on every device. The Box-Muller and the
router matmul use the device's fp64 libm/BLAS, so tensors drawn on two
devices can differ in the last fp64 bit; a test always hands the oracle the
very tensors the GPU path received.
"""
from __future__ import annotations

import math

import numpy as np
import torch

from .configs import BF16, LayerConfig

_GAMMA = 0x9E3779B97F4A7C15
_M1 = 0xBF58476D1CE4E5B9
_M2 = 0x94D049BB133111EB
_MASK64 = (1 << 64) - 1

TID_X, TID_WR, TID_WGU, TID_WDOWN, TID_LOGITS, TID_PERM, TID_HOT, TID_HOTTOK, TID_DOUT = 1, 2, 3, 4, 5, 6, 7, 8, 9

_CHUNK = 1 << 24


def _s64(c: int) -> int:
    """A uint64 constant as the int64 with the same bits."""
    c &= _MASK64
    return c - (1 << 64) if c >= (1 << 63) else c


def _lsr(z: torch.Tensor, s: int) -> torch.Tensor:
    """Logical right shift of int64 bit patterns."""
    return (z >> s) & ((1 << (64 - s)) - 1)


def _mix64(z: torch.Tensor) -> torch.Tensor:
    z = (z ^ _lsr(z, 30)) * _s64(_M1)
    z = (z ^ _lsr(z, 27)) * _s64(_M2)
    return z ^ _lsr(z, 31)


def _mix64_int(z: int) -> int:
    z &= _MASK64
    z = ((z ^ (z >> 30)) * _M1) & _MASK64
    z = ((z ^ (z >> 27)) * _M2) & _MASK64
    return z ^ (z >> 31)


def stream_key(seed: int, tid: int) -> int:
    return _mix64_int(seed * (1 << 16) + tid + _GAMMA)


def splitmix64(key: int, start: int, n: int, device="cpu") -> torch.Tensor:
    """Outputs start..start+n-1 of the SplitMix64 stream with state ``key``, as int64 bits."""
    i = torch.arange(start + 1, start + n + 1, dtype=torch.int64, device=device)
    z = _s64(key) + i * _s64(_GAMMA)
    return _mix64(z)


def uniform(key: int, start: int, n: int, device="cpu") -> torch.Tensor:
    z = splitmix64(key, start, n, device)
    return _lsr(z, 11).to(torch.float64) * (2.0 ** -53)


def normal(key: int, n: int, device="cpu", out_dtype=torch.float64, std: float = 1.0,
           start: int = 0) -> torch.Tensor:
    """Normals start..start+n-1 (times std) of stream ``key``, drawn in chunks, stored as out_dtype."""
    out = torch.empty(n, dtype=out_dtype, device=device)
    pos = 0
    while pos < n:
        m = min(_CHUNK, n - pos)
        # element j of the stream is the cos (j even) or sin (j odd) output of
        # pair j//2, which uses uniforms 2*(j//2) and 2*(j//2)+1
        a = start + pos
        p0 = a // 2
        npairs = (a + m - 1) // 2 - p0 + 1
        u = uniform(key, 2 * p0, 2 * npairs, device).view(-1, 2)
        r = torch.sqrt(-2.0 * torch.log1p(-u[:, 0]))
        th = (2.0 * math.pi) * u[:, 1]
        v = torch.stack((r * torch.cos(th), r * torch.sin(th)), dim=1).reshape(-1)
        v = v[a - 2 * p0: a - 2 * p0 + m]
        if std != 1.0:
            v = v * std
        if out_dtype == torch.bfloat16:
            v = v.to(torch.float32).to(torch.bfloat16)
        else:
            v = v.to(out_dtype)
        out[pos:pos + m] = v
        pos += m
    return out


def expert_permutation(seed: int, E: int) -> torch.Tensor:
    """A seeded permutation of experts: perm[j] is the expert whose draw is j-th smallest."""
    u = uniform(stream_key(seed, TID_PERM), 0, E)
    return torch.sort(u, stable=True).indices


def router_bias(cfg: LayerConfig, seed: int) -> torch.Tensor:
    """Per-expert bias [E] (fp64) and, for the hot-expert recipe, a per-token mask."""
    bias = torch.zeros(cfg.E, dtype=torch.float64)
    if cfg.zipf_s != 0.0:
        perm = expert_permutation(seed, cfg.E)
        rank = torch.empty(cfg.E, dtype=torch.float64)
        rank[perm] = torch.arange(1, cfg.E + 1, dtype=torch.float64)
        bias -= cfg.zipf_s * torch.log(rank)
    return bias


def hot_expert(cfg: LayerConfig, seed: int) -> int:
    u = float(uniform(stream_key(seed, TID_HOT), 0, 1)[0])
    return min(int(u * cfg.E), cfg.E - 1)


def make_inputs(cfg: LayerConfig, seed: int = 0, device="cpu", weights: bool = True) -> dict:
    """All layer inputs for ``cfg`` and ``seed`` on ``device``.

    Returns logits fp32 [T,E], x [T,d], w_gate_up [E,2F,d], w_down [E,d,F]
    (bf16 or fp32 per cfg.dtype). Rows 0..F-1 of w_gate_up[e] are the gate
    projection, rows F..2F-1 the up projection; both weight tensors are
    stored K-major (the contraction index is the last one). With
    ``weights=False`` the expert weights are left out (routing-only checks).
    """
    dt = torch.bfloat16 if cfg.dtype == BF16 else torch.float32
    T, d, E, F = cfg.T, cfg.d, cfg.E, cfg.F
    x = normal(stream_key(seed, TID_X), T * d, device, dt).view(T, d)
    out = {}
    if weights:
        out["w_gate_up"] = normal(stream_key(seed, TID_WGU), E * 2 * F * d, device, dt,
                                  cfg.w_std).view(E, 2 * F, d)
        out["w_down"] = normal(stream_key(seed, TID_WDOWN), E * d * F, device, dt,
                               cfg.w_std).view(E, d, F)
    bias = router_bias(cfg, seed).to(device)
    if cfg.logits == "xwr":
        wr = normal(stream_key(seed, TID_WR), d * E, device, dt, cfg.w_std).view(d, E)
        lg = x.to(torch.float64) @ wr.to(torch.float64)
    elif cfg.logits == "normal":
        lg = normal(stream_key(seed, TID_LOGITS), T * E, device, torch.float64).view(T, E)
    else:
        raise ValueError(f"unknown router recipe {cfg.logits!r}")
    lg = lg + bias
    if cfg.hot_bias != 0.0:
        h = hot_expert(cfg, seed)
        if cfg.hot_frac >= 1.0:
            lg[:, h] += cfg.hot_bias
        else:
            ut = uniform(stream_key(seed, TID_HOTTOK), 0, T, device)
            lg[:, h] += torch.where(ut < cfg.hot_frac, cfg.hot_bias, 0.0)
    out["logits"] = lg.to(torch.float32).contiguous()
    out["x"] = x.contiguous()
    return out


def expert_weights(cfg: LayerConfig, seed: int, experts, device="cpu"):
    """The expert weights of ``make_inputs`` for the listed experts only:
    (w_gate_up [n, 2F, d], w_down [n, d, F]), bit-identical to those experts'
    slices of the full tensors (the streams are counter-based, so each
    expert's elements are drawn from their own positions)."""
    dt = torch.bfloat16 if cfg.dtype == BF16 else torch.float32
    d, F = cfg.d, cfg.F
    es = [int(e) for e in experts]
    wgu = torch.empty(len(es), 2 * F, d, dtype=dt, device=device)
    wdn = torch.empty(len(es), d, F, dtype=dt, device=device)
    for i, e in enumerate(es):
        wgu[i] = normal(stream_key(seed, TID_WGU), 2 * F * d, device, dt, cfg.w_std,
                        start=e * 2 * F * d).view(2 * F, d)
        wdn[i] = normal(stream_key(seed, TID_WDOWN), d * F, device, dt, cfg.w_std,
                        start=e * d * F).view(d, F)
    return wgu, wdn


def make_grad_out(cfg: LayerConfig, seed: int = 0, device="cpu") -> torch.Tensor:
    """A seeded upstream gradient dL/dout [T, d] for the backward, N(0, 1) in
    the layer's activation type."""
    dt = torch.bfloat16 if cfg.dtype == BF16 else torch.float32
    return normal(stream_key(seed, TID_DOUT), cfg.T * cfg.d, device, dt).view(cfg.T, cfg.d).contiguous()


def to_numpy_bits(t: torch.Tensor) -> np.ndarray:
    """A host numpy view of a tensor: bf16 as uint16 bit patterns, others as-is."""
    t = t.detach().cpu().contiguous()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    return t.numpy()
