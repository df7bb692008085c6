"""Helpers for the GPU parity tests: run the layer through the C ABI stage by
stage, and compare every stage with the CPU oracle on the same inputs."""
from __future__ import annotations

import concurrent.futures
import os

import numpy as np
import torch

from oracle import oracle as O
from routed_experts_b200 import configs as C
from routed_experts_b200 import inputs as I
from routed_experts_b200 import moe as M

# Output tolerances: bf16 |g - o| <= 2e-2 + 1e-2 |o| elementwise and a
# normwise relative error <= 1e-2; fp32 |g - o| <= 1e-4 + 1e-4 |o| and
# normwise <= 1e-5. Gating weights (fp32 on both sides, fp32 exp on the GPU,
# fp64 in the oracle) within 1e-6.
TOL = {C.BF16: (2e-2, 1e-2, 1e-2), C.FP32: (1e-4, 1e-4, 1e-5)}
W_ATOL = 1e-6


def assert_close(got: np.ndarray, ref: np.ndarray, dtype: int, what: str):
    atol, rtol, nrm = TOL[dtype]
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    err = np.abs(got - ref)
    bad = err > atol + rtol * np.abs(ref)
    assert not bad.any(), f"{what}: {int(bad.sum())} elements out of tolerance, max err {err.max():.3e}"
    den = np.linalg.norm(ref)
    if den > 0:
        rel = np.linalg.norm(got - ref) / den
        assert rel <= nrm, f"{what}: normwise error {rel:.3e} > {nrm}"


def to_f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


# Bit patterns written into h and yp before a call: rows no entry maps to
# (padding) must come back either untouched or zero, never anything else.
SENTINEL = {C.BF16: 0x7FAB, C.FP32: 0x7FC0ABCD}


def sentinel_like(shape, cfg, device) -> torch.Tensor:
    if cfg.dtype == C.BF16:
        return torch.full(shape, SENTINEL[C.BF16], dtype=torch.int16, device=device).view(torch.bfloat16)
    return torch.full(shape, SENTINEL[C.FP32], dtype=torch.int32, device=device).view(torch.float32)


PATHS = ("staged", "fused", "fused_gather", "fc1_gather", "fc2_combine", "layer")


def run_path(cfg, inp: dict, path: str = "staged") -> dict:
    """moe_plan, then the FFN through one of the library's paths, then
    moe_combine, on device inputs:
      staged        moe_dispatch, moe_expert_ffn (FC1 launch, FC2 launch)
      fused         moe_dispatch, moe_expert_ffn_fused (FC1 and FC2 in one launch)
      fused_gather  moe_expert_ffn_fused_gather (dispatch, FC1 and FC2 in one launch)
      fc1_gather    moe_expert_fc1_gather (dispatch and FC1 in one launch), moe_expert_fc2
      fc2_combine   moe_dispatch, moe_expert_fc1, moe_expert_fc2_combine (FC2 and the combine
                    in one launch; no moe_combine), on a MOE_WS_LAYER workspace whose layer
                    part starts as 0xff bytes, so its arrival counters must be cleared
      layer         moe_layer_fwd alone (h and yp stay inside its workspace)."""
    dev = inp["x"].device
    T, K, E, d, F = cfg.T, cfg.K, cfg.E, cfg.d, cfg.F
    dt = M.act_dtype(cfg)
    cap = M.moe_rows_capacity(cfg)
    if path == "layer":
        layer = M.Layer(cfg, dev)
        out = layer.forward(inp["logits"], inp["x"], inp["w_gate_up"], inp["w_down"])
        status = layer.status()
        return {"out": out, "status": status, "plan": M.read_plan(cfg, layer.ws), "ws": layer.ws, "rows_cap": cap,
                "idx": None}
    idx = torch.empty(T, K, dtype=torch.int32, device=dev)
    w = torch.empty(T, K, dtype=torch.float32, device=dev)
    counts = torch.empty(E, dtype=torch.int32, device=dev)
    if path == "fc2_combine":
        ws = M.alloc_workspace(cfg, M.WS_LAYER, dev)
        ws[M.moe_workspace_size(cfg, M.WS_PLAN):].fill_(255)
    else:
        ws = M.alloc_workspace(cfg, M.WS_PLAN, dev)
    h = sentinel_like((cap, F), cfg, dev)
    yp = sentinel_like((cap, d), cfg, dev)
    out = torch.empty(T, d, dtype=dt, device=dev)
    M.moe_plan(cfg, inp["logits"], idx, w, counts, ws)
    xp = None
    if path in ("staged", "fused", "fc2_combine"):
        # dispatch leaves padding rows of xp alone: NaN there must not reach h, yp or out
        xp = torch.full((cap, d), float("nan"), dtype=dt, device=dev)
        M.moe_dispatch(cfg, inp["x"], xp, ws)
    if path == "staged":
        M.moe_expert_ffn(cfg, xp, inp["w_gate_up"], inp["w_down"], h, yp, ws)
    elif path == "fused":
        M.moe_expert_ffn_fused(cfg, xp, inp["w_gate_up"], inp["w_down"], h, yp, ws)
    elif path == "fused_gather":
        M.moe_expert_ffn_fused_gather(cfg, inp["x"], inp["w_gate_up"], inp["w_down"], h, yp, ws)
    elif path == "fc1_gather":
        M.moe_expert_fc1_gather(cfg, inp["x"], inp["w_gate_up"], h, ws)
        M.moe_expert_fc2(cfg, h, inp["w_down"], yp, ws)
    elif path == "fc2_combine":
        M.moe_expert_fc1(cfg, xp, inp["w_gate_up"], h, ws)
        M.moe_expert_fc2_combine(cfg, h, inp["w_down"], w, yp, out, ws)
    else:
        raise ValueError(path)
    if path != "fc2_combine":
        M.moe_combine(cfg, yp, w, out, ws)
    status = M.moe_read_status(ws)
    plan = M.read_plan(cfg, ws)
    return {"idx": idx, "w": w, "counts": counts, "xp": xp, "h": h, "yp": yp, "out": out,
            "status": status, "plan": plan, "ws": ws, "rows_cap": cap}


def run_stages(cfg, inp: dict) -> dict:
    """moe_plan, moe_dispatch, moe_expert_ffn, moe_combine on device inputs."""
    return run_path(cfg, inp, "staged")


def check_padding_rows(t: torch.Tensor, valid: np.ndarray, cfg, what: str):
    """Rows no entry maps to hold either the sentinel written before the call
    or zero in every element."""
    pad = torch.as_tensor(np.nonzero(~valid)[0], device=t.device)
    if not len(pad):
        return
    bits = t[pad].view(torch.int16 if cfg.dtype == C.BF16 else torch.int32)
    sent = SENTINEL[cfg.dtype]
    if cfg.dtype == C.BF16:
        sent = sent - (1 << 16) if sent >= (1 << 15) else sent
    ok = (bits == sent).all(dim=1) | (bits == 0).all(dim=1)
    assert bool(ok.all()), f"{what}: {int((~ok).sum())} padding rows written with values"


# ---------------------------------------------------------------- the oracle on many cores

ORACLE_THREADS = max(1, min(64, len(os.sched_getaffinity(0))))


def _threaded(fn, n: int, *arrays):
    """fn over ORACLE_THREADS contiguous shards of range(n), run on that many
    threads (each call is one single-threaded oracle call; ctypes releases
    the interpreter lock around it). Returns the shards' results in order."""
    shards = [s_ for s_ in np.array_split(np.arange(n), ORACLE_THREADS) if len(s_)]
    with concurrent.futures.ThreadPoolExecutor(max_workers=len(shards)) as ex:
        return list(ex.map(fn, shards))


def par_entry_ffn(tokens, experts, x, wgu, wdn, dtype, rm):
    """O.entry_ffn over shards of the entries, on several threads."""
    tokens = np.asarray(tokens, np.int64)
    experts = np.asarray(experts, np.int32)
    parts = _threaded(lambda sh: O.entry_ffn(tokens[sh], experts[sh], x, wgu, wdn, dtype, rm), len(tokens))
    return np.concatenate([p[0] for p in parts]), np.concatenate([p[1] for p in parts])


def par_token_out(tokens, x, idx, w, wgu, wdn, dtype, rm):
    """O.token_out over shards of the tokens, on several threads."""
    tokens = np.asarray(tokens, np.int64)
    return np.concatenate(_threaded(lambda sh: O.token_out(tokens[sh], x, idx, w, wgu, wdn, dtype, rm),
                                    len(tokens)))


# ---------------------------------------------------------------- a test-side reference at full size

class CloseOnGpu:
    """The bf16 output bound of assert_close, accumulated over many slices on
    the GPU: elementwise |g - o| <= atol + rtol |o| and the normwise error."""

    def __init__(self, dtype: int, what: str):
        self.atol, self.rtol, self.nrm = TOL[dtype]
        self.what = what
        self.bad = 0
        self.n = 0
        self.err2 = 0.0
        self.ref2 = 0.0
        self.max_err = 0.0

    def add(self, got: torch.Tensor, ref: torch.Tensor):
        g, o = got.double(), ref.double()
        err = (g - o).abs()
        self.bad += int((err > self.atol + self.rtol * o.abs()).sum())
        self.n += err.numel()
        self.err2 += float((err * err).sum())
        self.ref2 += float((o * o).sum())
        if err.numel():
            self.max_err = max(self.max_err, float(err.max()))

    def check(self):
        assert self.bad == 0, f"{self.what}: {self.bad} of {self.n} elements out of tolerance, max err {self.max_err:.3e}"
        if self.ref2 > 0:
            rel = (self.err2 / self.ref2) ** 0.5
            assert rel <= self.nrm, f"{self.what}: normwise error {rel:.3e} > {self.nrm}"


def check_every_row_fp64(cfg, inp: dict, ref: dict, g: dict):
    """Every valid row of h and yp, and every token of out, against a
    test-side fp64 evaluation of the same formula on the GPU (torch matmuls
    per expert, bf16 rounding where the layer stores: h = bf16(silu(a) g),
    y = bf16(h W2^T), out = bf16(sum_k w_k y_k) in fp64). It reaches every
    work item of a full-size layer, which the oracle's one-by-one rows
    cannot; the oracle pins it through the sampled rows beside it."""
    dev = inp["x"].device
    F = cfg.F
    blocks = ref["plan"]["blocks"]
    total = ref["plan"]["total_rows"]
    src = torch.as_tensor(ref["src_of"][:total], device=dev, dtype=torch.int64)
    y_ref = torch.zeros(total, cfg.d, dtype=torch.float32, device=dev)
    ch, cy = CloseOnGpu(cfg.dtype, "h (every valid row)"), CloseOnGpu(cfg.dtype, "yp (every valid row)")
    rdt = torch.bfloat16 if cfg.dtype == C.BF16 else torch.float32
    for e in np.unique(blocks[:, 0]):
        eb = blocks[blocks[:, 0] == e]
        rows = torch.as_tensor(np.concatenate([np.arange(b[1], b[1] + b[2]) for b in eb]), device=dev)
        xe = inp["x"][src[rows]].double()
        w1 = inp["w_gate_up"][int(e)].double()
        a = xe @ w1[:F].T
        gg = xe @ w1[F:].T
        h = (a / (1.0 + torch.exp(-a)) * gg).to(rdt)
        y = (h.double() @ inp["w_down"][int(e)].double().T).to(rdt)
        if g.get("h") is not None:
            ch.add(g["h"][rows], h)
            cy.add(g["yp"][rows], y)
        y_ref[rows] = y.float()
        del xe, w1, a, gg, h, y
    if g.get("h") is not None:
        ch.check()
        cy.check()
    row_of = torch.as_tensor(ref["row_of"], device=dev, dtype=torch.int64).view(cfg.T, cfg.K)
    wk = torch.as_tensor(ref["w"], device=dev).double()
    co = CloseOnGpu(cfg.dtype, "out (every token)")
    step = max(1, (1 << 28) // (cfg.K * cfg.d * 8))
    for t0 in range(0, cfg.T, step):
        t1 = min(cfg.T, t0 + step)
        acc = torch.zeros(t1 - t0, cfg.d, dtype=torch.float64, device=dev)
        for k in range(cfg.K):
            acc += wk[t0:t1, k:k + 1] * y_ref[row_of[t0:t1, k]].double()
        co.add(g["out"][t0:t1], acc.to(rdt))
    co.check()


def host_inputs(inp: dict, with_weights: bool = True) -> dict:
    keys = ("logits", "x", "w_gate_up", "w_down") if with_weights else ("logits", "x")
    return {k: I.to_numpy_bits(inp[k]) for k in keys}


def check_routing_and_plan(cfg, g: dict, ref: dict):
    """Bit-exact checks of top-k, counts, plan and row maps; weights within 1e-6."""
    if g.get("idx") is not None:
        assert np.array_equal(g["idx"].cpu().numpy(), ref["idx"]), "top-k indices differ"
        np.testing.assert_allclose(g["w"].cpu().numpy(), ref["w"], rtol=0, atol=W_ATOL)
        assert np.array_equal(g["counts"].cpu().numpy(), ref["counts"]), "counts differ"
    gp, rp = g["plan"], ref["plan"]
    assert gp["moves"] == rp["moves"]
    assert (gp["status"] & O.PLAN_INEXACT) == rp["status"]
    assert gp["total_rows"] == rp["total_rows"]
    assert np.array_equal(gp["pieces"].numpy(), rp["pieces"]), "pieces differ"
    assert np.array_equal(gp["blocks"].numpy(), rp["blocks"]), "blocks differ"
    assert np.array_equal(gp["rank_load"].numpy(), rp["rank_load"])
    assert np.array_equal(gp["rank_replicas"].numpy(), rp["rank_replicas"])
    assert np.array_equal(gp["rank_row0"].numpy(), rp["rank_row0"])
    assert gp["replicas"] == int(rp["rank_replicas"].sum())
    if getattr(cfg, "plan_mode", 0) == O.PLAN_BLOCKS:
        assert gp["tau"] == rp["info"][0] and gp["candidate"] == rp["info"][1]
    assert np.array_equal(gp["row_of"].numpy(), ref["row_of"]), "row_of differs"
    total = rp["total_rows"]
    assert np.array_equal(gp["src_of"].numpy(), ref["src_of"][:total]), "src_of differs"


def oracle_routing(cfg, hin: dict) -> dict:
    idx, w = O.topk_gate(hin["logits"], cfg.K, cfg.gating)
    counts = O.histogram(idx, cfg.E)
    pl = O.plan(cfg.T, cfg.E, cfg.K, cfg.R, cfg.tile, cfg.budget, counts, getattr(cfg, "plan_mode", 0))
    cap = O.rows_capacity(cfg.N, cfg.E, cfg.R, cfg.budget, cfg.tile)
    row_of, src_of = O.row_maps(idx, cfg.E, pl["pieces"], cap)
    return {"idx": idx, "w": w, "counts": counts, "plan": pl, "row_of": row_of, "src_of": src_of,
            "rows_cap": cap}


def f64_to_bits(v: np.ndarray, dtype: int) -> np.ndarray:
    """Values that are exactly representable in the layer's type, as its bits."""
    f = np.asarray(v, np.float64).astype(np.float32)
    return (f.view(np.uint32) >> 16).astype(np.uint16) if dtype == C.BF16 else f


def row_experts(blocks: np.ndarray, total: int) -> np.ndarray:
    """The expert of every padded row (-1 outside blocks)."""
    e = np.full(total, -1, np.int32)
    for b in blocks:
        e[b[1]:b[1] + b[2]] = b[0]
    return e


def check_full_small(cfg, seed: int, device="cuda", path: str = "staged", threads: bool = False):
    """Every stage against the oracle, every element (sizes the oracle runs in
    seconds). With threads=True the oracle's FFN runs as one entry_ffn per
    valid row, sharded over host threads, and its combine on those rows
    (the same arithmetic as the oracle's layer, for layers too large for one
    thread)."""
    inp = I.make_inputs(cfg, seed, device)
    g = run_path(cfg, inp, path)
    hin = host_inputs(inp)
    rm = O.default_round_mode(cfg.dtype)
    if not threads:
        ref = O.layer(hin["logits"], hin["x"], hin["w_gate_up"], hin["w_down"], K=cfg.K, R=cfg.R,
                      tile=cfg.tile, budget=cfg.budget, gating=cfg.gating, dtype=cfg.dtype,
                      plan_mode=getattr(cfg, "plan_mode", 0))
    else:
        ref = oracle_routing(cfg, hin)
    assert g["rows_cap"] == ref["rows_cap"]
    check_routing_and_plan(cfg, g, ref)
    assert (g["status"] & ~O.PLAN_INEXACT) == 0, f"device status {g['status']}"
    total = ref["plan"]["total_rows"]
    src = ref["src_of"][:total]
    valid = src >= 0
    if threads:
        vrows = np.nonzero(valid)[0]
        rh, ry = par_entry_ffn(src[vrows], row_experts(ref["plan"]["blocks"], total)[vrows], hin["x"],
                               hin["w_gate_up"], hin["w_down"], cfg.dtype, rm)
        yp_bits = np.zeros((ref["rows_cap"], cfg.d), np.uint16 if cfg.dtype == C.BF16 else np.float32)
        yp_bits[vrows] = f64_to_bits(ry, cfg.dtype)
        ref["out"] = O.combine(yp_bits, ref["row_of"], ref["w"], cfg.dtype, rm)
        ref_h = np.zeros((total, cfg.F)); ref_h[vrows] = rh
        ref_y = np.zeros((total, cfg.d)); ref_y[vrows] = ry
    else:
        ref_h = O.to_f64(ref["h"][:total], cfg.dtype)
        ref_y = O.to_f64(ref["yp"][:total], cfg.dtype)
    if g.get("xp") is not None:
        assert np.array_equal(I.to_numpy_bits(g["xp"][:total])[valid], hin["x"][src[valid]]), "xp differs"
    if g.get("h") is not None:
        assert_close(to_f64(g["h"][:total])[valid], ref_h[valid], cfg.dtype, "h")
        assert_close(to_f64(g["yp"][:total])[valid], ref_y[valid], cfg.dtype, "yp")
        check_padding_rows(g["h"][:total], valid, cfg, "h")
        check_padding_rows(g["yp"][:total], valid, cfg, "yp")
    assert_close(to_f64(g["out"]), O.to_f64(ref["out"], cfg.dtype), cfg.dtype, "out")
    return g, ref, inp


def check_routing_full_size(cfg, seed: int, device="cuda"):
    """Routing, gating, counts, plan and row maps of a full-size layer, bit-exact (weights within 1e-6)."""
    inp = I.make_inputs(cfg, seed, device, weights=False)
    dev = inp["x"].device
    idx = torch.empty(cfg.T, cfg.K, dtype=torch.int32, device=dev)
    w = torch.empty(cfg.T, cfg.K, dtype=torch.float32, device=dev)
    counts = torch.empty(cfg.E, dtype=torch.int32, device=dev)
    ws = M.alloc_workspace(cfg, M.WS_PLAN, dev)
    M.moe_plan(cfg, inp["logits"], idx, w, counts, ws)
    status = M.moe_read_status(ws)
    assert (status & ~O.PLAN_INEXACT) == 0, f"device status {status}"
    g = {"idx": idx, "w": w, "counts": counts, "plan": M.read_plan(cfg, ws)}
    ref = oracle_routing(cfg, host_inputs(inp, with_weights=False))
    check_routing_and_plan(cfg, g, ref)
    return ref


def check_full_size(cfg, seed: int, path: str = "staged", n_tokens: int = 64, device="cuda"):
    """A full-size layer through one of the library's paths:
      * routing, plan and row maps bit-exact, and the dispatched rows;
      * every valid row of h and yp, and every token of out, against the
        test-side fp64 evaluation (check_every_row_fp64);
      * one row of h and yp in every planned block, with the row inside the
        block drawn at random, and n_tokens tokens of out spread over the
        token range, against the oracle (one by one, sharded over threads);
      * rows no entry maps to untouched or zero."""
    inp = I.make_inputs(cfg, seed, device)
    g = run_path(cfg, inp, path)
    hin = host_inputs(inp, with_weights=False)
    ref = oracle_routing(cfg, hin)
    check_routing_and_plan(cfg, g, ref)
    assert (g["status"] & ~O.PLAN_INEXACT) == 0, f"device status {g['status']}"
    total = ref["plan"]["total_rows"]
    src = ref["src_of"][:total]
    x = hin["x"]
    valid = src >= 0
    if g.get("xp") is not None:
        xp = I.to_numpy_bits(g["xp"][:total])
        assert np.array_equal(xp[valid], x[src[valid]]), "xp rows differ from their token rows"
        del xp
    if g.get("h") is not None:
        check_padding_rows(g["h"][:total], valid, cfg, "h")
        check_padding_rows(g["yp"][:total], valid, cfg, "yp")
    check_every_row_fp64(cfg, inp, ref, g)
    wgu, wdn = I.to_numpy_bits(inp["w_gate_up"]), I.to_numpy_bits(inp["w_down"])
    rm = O.default_round_mode(cfg.dtype)
    rng = np.random.default_rng(seed + 17)
    blocks = ref["plan"]["blocks"]
    if g.get("h") is not None:
        rows = np.array([b[1] + rng.integers(b[2]) for b in blocks], np.int64)
        rh, ry = par_entry_ffn(src[rows], blocks[:, 0], x, wgu, wdn, cfg.dtype, rm)
        sel = torch.as_tensor(rows, device=device)
        assert_close(to_f64(g["h"][sel]), rh, cfg.dtype, "h, one row per block")
        assert_close(to_f64(g["yp"][sel]), ry, cfg.dtype, "yp, one row per block")
    toks = np.unique(np.clip(np.linspace(0, cfg.T - 1, n_tokens).astype(np.int64) +
                             rng.integers(0, max(1, cfg.T // n_tokens), n_tokens), 0, cfg.T - 1))
    o = par_token_out(toks, x, ref["idx"], ref["w"], wgu, wdn, cfg.dtype, rm)
    assert_close(to_f64(g["out"][torch.as_tensor(toks, device=device)]), o, cfg.dtype, "out, spread tokens")
    return g, ref, inp


def assert_grad_close(got: np.ndarray, ref: np.ndarray, what: str, rel: float = 1e-2):
    """The bf16 output bound (2e-2 absolute + 1e-2 relative) with its absolute
    part taken at the gradient's scale: |g - o| <= 2 rel rms(o) + rel |o|
    elementwise, and ||g - o|| <= rel ||o||. Each weight-gradient element is
    a sum of products of bf16 values that the GPU and the oracle round from
    fp32 and fp64 sums, so single terms may differ by one bf16 ulp."""
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    scale = np.sqrt(np.mean(ref ** 2)) if ref.size else 0.0
    err = np.abs(got - ref)
    bad = err > rel * (2 * scale + np.abs(ref))
    assert not bad.any(), f"{what}: {int(bad.sum())} of {bad.size} out of tolerance, max err {err.max():.3e}"
    den = np.linalg.norm(ref)
    if den > 0:
        assert np.linalg.norm(got - ref) / den <= rel, f"{what}: normwise {np.linalg.norm(got - ref) / den:.3e}"


def run_bwd(cfg, seed, device="cuda"):
    """The training forward then the backward of one seeded layer through the C ABI."""
    inp = I.make_inputs(cfg, seed, device)
    d_out = I.make_grad_out(cfg, seed, device)
    layer = M.Layer(cfg, device, train=True)
    layer.forward(inp["logits"], inp["x"], inp["w_gate_up"], inp["w_down"])
    dx, dwgu, dwdn, dl = layer.backward(inp["logits"], inp["w_gate_up"], inp["w_down"], d_out)
    assert layer.status() & ~M.DEV_PLAN_INEXACT == 0
    return inp, d_out, layer, (dx, dwgu, dwdn, dl)


def check_bwd_small(cfg, seed, device="cuda"):
    """The backward against the oracle's, every element (sizes the oracle runs in seconds)."""
    inp, d_out, _, (dx, dwgu, dwdn, dl) = run_bwd(cfg, seed, device)
    hin = {k: I.to_numpy_bits(v) for k, v in inp.items()}
    idx, w = O.topk_gate(hin["logits"], cfg.K, cfg.gating)
    ref = O.layer_bwd(hin["logits"], idx, w, hin["x"], hin["w_gate_up"], hin["w_down"], I.to_numpy_bits(d_out),
                      gating=cfg.gating, dtype=cfg.dtype, round_mode=O.ROUND_BF16)
    assert_close(to_f64(dx), O.to_f64(ref["dx"], cfg.dtype), cfg.dtype, "dx")
    assert_grad_close(dwgu.cpu().numpy(), ref["dw_gate_up"], "dw_gate_up")
    assert_grad_close(dwdn.cpu().numpy(), ref["dw_down"], "dw_down")
    assert_grad_close(dl.cpu().numpy(), ref["dlogits"], "dlogits")
    # experts no token chose have exactly zero gradients; so do unchosen logits
    counts = np.bincount(idx.ravel(), minlength=cfg.E)
    for e in np.nonzero(counts == 0)[0]:
        assert not dwgu[e].any() and not dwdn[e].any()
    chosen = np.zeros((cfg.T, cfg.E), bool)
    np.put_along_axis(chosen, idx, True, axis=1)
    assert not dl.cpu().numpy()[~chosen].any()


# ---------------------------------------------------------------- MXFP8 forward

def mx_scale_index(rows: int, K: int) -> np.ndarray:
    """For each (row, 32-block) of a [rows, K] MXFP8 matrix, the byte of its
    scale in the chunked layout include/moe.h documents (512-byte chunks per
    128 rows and 128 columns; row r, block b at 16 (r % 32) + 4 ((r % 128) / 32) + b % 4)."""
    r = np.arange(rows, dtype=np.int64)[:, None]
    b = np.arange(K // 32, dtype=np.int64)[None, :]
    return ((r // 128) * (K // 128) + b // 4) * 512 + (r % 32) * 16 + ((r % 128) // 32) * 4 + b % 4


def mx_unchunk(sc: torch.Tensor | np.ndarray, rows: int, K: int) -> np.ndarray:
    sc = sc.cpu().numpy() if isinstance(sc, torch.Tensor) else sc
    return sc[mx_scale_index(rows, K)]


def mx_chunk(logical: np.ndarray, K: int, nbytes: int) -> np.ndarray:
    rows = logical.shape[0]
    out = np.zeros(nbytes, np.uint8)
    out[mx_scale_index(rows, K)] = logical
    return out


def w1_tile_rows(E: int, F: int) -> np.ndarray:
    """Row order of the MX W1: row e*2F + 128 t + i is gate row 64 t + i (i < 64)
    or up row F + 64 t + (i - 64) of expert e."""
    i = np.arange(2 * F)
    t, r = i // 128, i % 128
    local = np.where(r < 64, 64 * t + r, F + 64 * t + (r - 64))
    return (np.arange(E)[:, None] * 2 * F + local[None, :]).ravel()


def mx_weights_on_device(cfg, inp: dict, wfmt: int = M.MX_W_E4M3):
    return M.MxWeights(cfg, inp["w_gate_up"], inp["w_down"], wfmt=wfmt)


def mx_oracle_weights(cfg, inp: dict, experts=None, wfmt: int = M.MX_W_E4M3):
    """Oracle MX codes (one per byte) and scales of W1 / W2 (logical order) for the given experts (all by
    default), in weight format wfmt."""
    es = range(cfg.E) if experts is None else experts
    wgu = np.stack([I.to_numpy_bits(inp["w_gate_up"][e]) for e in es])
    wdn = np.stack([I.to_numpy_bits(inp["w_down"][e]) for e in es])
    return O.mx_weights(wgu, wdn, O.BF16, wfmt)


def mx_weight_codes(q: torch.Tensor, rows: int, K: int, wfmt: int) -> np.ndarray:
    """Weight codes from the device, one per byte: E2M1 codes are packed two per
    byte, element 2i in the low nibble of byte i."""
    a = q.cpu().numpy()
    if wfmt == M.MX_W_E4M3:
        return a.reshape(rows, K)
    a = a.reshape(rows, K // 2)
    out = np.empty((rows, K), np.uint8)
    out[:, 0::2] = a & 0xF
    out[:, 1::2] = a >> 4
    return out


def run_mx_stages(cfg, inp: dict, wfmt: int = M.MX_W_E4M3) -> dict:
    """moe_plan, moe_dispatch_mx, moe_expert_fc1_mx, moe_expert_fc2_mx, moe_combine."""
    dev = inp["x"].device
    T, K, E, d, F = cfg.T, cfg.K, cfg.E, cfg.d, cfg.F
    idx = torch.empty(T, K, dtype=torch.int32, device=dev)
    w = torch.empty(T, K, dtype=torch.float32, device=dev)
    counts = torch.empty(E, dtype=torch.int32, device=dev)
    ws = M.alloc_workspace(cfg, M.WS_PLAN, dev)
    cap = M.moe_rows_capacity(cfg)
    # padding rows of xq / xs are not written: fill them with NaN codes (0x7F) and scale 255
    xq = torch.full((M.moe_mx_buffer_bytes(cfg, M.MX_XQ),), 0x7F, dtype=torch.uint8, device=dev)
    xs = torch.full((M.moe_mx_buffer_bytes(cfg, M.MX_XS),), 0xFF, dtype=torch.uint8, device=dev)
    hq = M.mx_buffer(cfg, M.MX_HQ, dev)
    hs = M.mx_buffer(cfg, M.MX_HS, dev)
    yp = torch.empty(cap, d, dtype=torch.bfloat16, device=dev)
    out = torch.empty(T, d, dtype=torch.bfloat16, device=dev)
    mxw = mx_weights_on_device(cfg, inp, wfmt)
    M.moe_plan(cfg, inp["logits"], idx, w, counts, ws)
    M.moe_dispatch_mx(cfg, inp["x"], xq, xs, ws)
    M.moe_expert_fc1_mx(cfg, xq, xs, mxw.w1q, mxw.w1s, hq, hs, ws, wfmt=wfmt)
    M.moe_expert_fc2_mx(cfg, hq, hs, mxw.w2q, mxw.w2s, yp, ws, wfmt=wfmt)
    M.moe_combine(cfg, yp, w, out, ws)
    status = M.moe_read_status(ws)
    return {"idx": idx, "w": w, "counts": counts, "xq": xq.view(cap, d), "xs": xs, "hq": hq.view(cap, F),
            "hs": hs, "yp": yp, "out": out, "status": status, "plan": M.read_plan(cfg, ws), "ws": ws,
            "rows_cap": cap, "mxw": mxw}


def assert_mx_h_close(g_hq: np.ndarray, g_hs: np.ndarray, r_h: np.ndarray, r_hq: np.ndarray, r_hs: np.ndarray,
                      what: str, max_code_frac: float = 2e-3):
    """h after FC1 and MXFP8 quantization. The GPU forms h in fp32 and the
    oracle in fp64, so where the bf16-rounded h lands on either side of a
    rounding boundary the codes (or a block's scale) may differ; such
    elements differ by at most one E4M3 step of the block and must stay
    rare. Elementwise: |g - o| <= one step of E4M3 at o's magnitude (2^-3
    relative) + 2^-9 of the block's scale; normwise <= 1e-2."""
    gd = O.mx_dequantize(g_hq, g_hs)
    rd = O.mx_dequantize(r_hq, r_hs)
    code_diff = (g_hq != r_hq)
    frac = code_diff.mean() if code_diff.size else 0.0
    assert frac <= max_code_frac, f"{what}: {frac:.2e} of the codes differ"
    scale = 2.0 ** (np.repeat(r_hs.astype(np.int64), 32, axis=1) - 127)
    err = np.abs(gd - rd)
    bad = err > 2.0 ** -3 * np.abs(rd) + 2.0 ** -9 * scale * 2
    assert not bad.any(), f"{what}: {int(bad.sum())} elements beyond one E4M3 step, max err {err.max():.3e}"
    den = np.linalg.norm(rd)
    if den > 0:
        assert np.linalg.norm(gd - rd) / den <= 1e-2, f"{what}: normwise error"


def mx_h_error_bound(exps, g_hq, g_hs, r_hq, r_hs, w2q, w2s, d: int, wfmt: int) -> np.ndarray:
    """|dequant(GPU h) - dequant(oracle h)| @ |W2_e|^T per row: how far FC2
    outputs computed from the two h's can drift apart before rounding. The
    GPU forms h in fp32 and the oracle in fp64, so a few of h's MXFP8 codes
    may sit one step apart (assert_mx_h_close bounds them); FC2 carries
    each such step into yp, weighted by the expert's W2 row."""
    dh = np.abs(O.mx_dequantize(g_hq, g_hs) - O.mx_dequantize(r_hq, r_hs))
    bound = np.zeros((len(exps), d))
    for e in np.unique(exps):
        rows = np.nonzero((exps == e) & dh.any(axis=1))[0]
        if len(rows):
            w = np.abs(O.mx_dequantize_fmt(w2q[e * d:(e + 1) * d], w2s[e * d:(e + 1) * d], wfmt))
            bound[rows] = dh[rows] @ w.T
    return bound


def assert_close_mx(got: np.ndarray, ref: np.ndarray, bound: np.ndarray, what: str):
    """The bf16 output tolerance plus the drift an h of one E4M3 step can cause."""
    atol, rtol, nrm = TOL[C.BF16]
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    err = np.abs(got - ref)
    bad = err > atol + rtol * np.abs(ref) + bound
    assert not bad.any(), f"{what}: {int(bad.sum())} elements out of tolerance, max err {err.max():.3e}"
    den = np.linalg.norm(ref)
    if den > 0:
        rel = np.linalg.norm(got - ref) / den
        assert rel <= nrm + np.linalg.norm(bound) / den, f"{what}: normwise error {rel:.3e}"


def mx_out_error_bound(cfg, toks, ref, g, xq_ref, xs_ref, w1q, w1s, w2q, w2s, wfmt) -> np.ndarray:
    """sum_k |w_k| times the FC2 drift bound of entry (t, k): the GPU's h row
    of the entry against the oracle's h of the same entry."""
    K, d, F = cfg.K, cfg.d, cfg.F
    ent_tok = np.repeat(np.asarray(toks, np.int64), K)
    ent_k = np.tile(np.arange(K), len(toks))
    exps = ref["idx"][ent_tok, ent_k].astype(np.int32)
    rows = ref["row_of"][ent_tok * K + ent_k].astype(np.int64)
    _, r_hq, r_hs = O.mx_fc1_rows(np.arange(len(rows)), exps, xq_ref[ent_tok], xs_ref[ent_tok], w1q, w1s, F, wfmt)
    g_hq = g["hq"][torch.as_tensor(rows, device=g["hq"].device)].cpu().numpy()
    g_hs = mx_unchunk(g["hs"], int(rows.max()) + 1, F)[rows]
    b = mx_h_error_bound(exps, g_hq, g_hs, r_hq, r_hs, w2q, w2s, d, wfmt)
    wk = np.abs(ref["w"][ent_tok, ent_k].astype(np.float64))[:, None]
    return (wk * b).reshape(len(toks), K, d).sum(axis=1)


def check_mx_small(cfg, seed: int, device="cuda", max_rows: int = 768, max_tokens: int = 192,
                   wfmt: int = M.MX_W_E4M3):
    """The MX layer stage by stage against the oracle: weights and dispatched
    rows on every element; h and yp on every valid row up to max_rows (a
    seeded sample beyond), out on every token up to max_tokens (likewise)."""
    inp = I.make_inputs(cfg, seed, device)
    g = run_mx_stages(cfg, inp, wfmt)
    hin = host_inputs(inp)
    ref = oracle_routing(cfg, hin)
    assert g["rows_cap"] == ref["rows_cap"]
    check_routing_and_plan(cfg, g, ref)
    assert (g["status"] & ~O.PLAN_INEXACT) == 0, f"device status {g['status']}"
    d, F, E, K = cfg.d, cfg.F, cfg.E, cfg.K
    total = ref["plan"]["total_rows"]
    src = ref["src_of"][:total]
    valid = src >= 0
    # weights: bit-exact codes and scales
    w1q, w1s, w2q, w2s = mx_oracle_weights(cfg, inp, wfmt=wfmt)
    perm = w1_tile_rows(E, F)
    gw1q = mx_weight_codes(g["mxw"].w1q, E * 2 * F, d, wfmt)
    assert np.array_equal(gw1q, w1q[perm]), "W1 codes differ"
    assert np.array_equal(mx_unchunk(g["mxw"].w1s, E * 2 * F, d), w1s[perm]), "W1 scales differ"
    assert np.array_equal(mx_weight_codes(g["mxw"].w2q, E * d, F, wfmt), w2q), "W2 codes differ"
    assert np.array_equal(mx_unchunk(g["mxw"].w2s, E * d, F), w2s), "W2 scales differ"
    # dispatch: every valid row holds its token's codes and scales, bit for bit
    xq_ref, xs_ref = O.mx_quantize(hin["x"], O.BF16)
    gxq = g["xq"][:total].cpu().numpy()
    gxs = mx_unchunk(g["xs"], total, d)
    assert np.array_equal(gxq[valid], xq_ref[src[valid]]), "dispatched codes differ"
    assert np.array_equal(gxs[valid], xs_ref[src[valid]]), "dispatched scales differ"
    # FC1 on the oracle's own operands: every valid row of small layers, a
    # seeded sample of at most max_rows rows (all blocks' row positions) otherwise
    blocks = ref["plan"]["blocks"]
    row_exp = np.zeros(total, np.int32)
    for b in blocks:
        row_exp[b[1]:b[1] + 128] = b[0]
    rng = np.random.default_rng(seed + 5)
    vrows = np.nonzero(valid)[0]
    if len(vrows) > max_rows:
        vrows = np.sort(rng.choice(vrows, size=max_rows, replace=False))
    rh, rhq, rhs = O.mx_fc1_rows(np.arange(len(vrows)), row_exp[vrows], xq_ref[src[vrows]], xs_ref[src[vrows]],
                                 w1q, w1s, F, wfmt)
    ghq = g["hq"][:total].cpu().numpy()
    ghs = mx_unchunk(g["hs"], total, F)
    assert_mx_h_close(ghq[vrows], ghs[vrows], rh, rhq, rhs, "h (MXFP8)")
    assert not ghq[~valid].any() and not ghs[~valid].any(), "padding rows of h must be zero codes and scales"
    # FC2 on the oracle's h, with the drift of h's codes that differ
    ry = O.mx_fc2_rows(row_exp[vrows], rhq, rhs, w2q, w2s, d, wfmt)
    gy = to_f64(g["yp"][:total])
    yb = mx_h_error_bound(row_exp[vrows], ghq[vrows], ghs[vrows], rhq, rhs, w2q, w2s, d, wfmt)
    assert_close_mx(gy[vrows], ry, yb, "yp")
    assert not gy[~valid].any(), "padding rows of yp must be zero"
    # the whole layer, on all tokens or a seeded sample
    toks = np.arange(cfg.T) if cfg.T <= max_tokens else np.sort(rng.choice(cfg.T, size=max_tokens, replace=False))
    rout = O.mx_token_out(toks, xq_ref, xs_ref, ref["idx"], ref["w"], w1q, w1s, w2q, w2s, F, wfmt)
    ob = mx_out_error_bound(cfg, toks, ref, g, xq_ref, xs_ref, w1q, w1s, w2q, w2s, wfmt)
    assert_close_mx(to_f64(g["out"])[toks], rout, ob, "out")
    return g, ref, inp


def par_mx_oracle_weights(cfg, inp: dict, wfmt: int):
    """Oracle MX codes and scales of every expert's W1 and W2 (logical order),
    one oracle call per expert, sharded over host threads."""
    E = cfg.E

    def one(sh):
        res = []
        for e in sh:
            res.append(O.mx_weights(I.to_numpy_bits(inp["w_gate_up"][int(e)])[None],
                                    I.to_numpy_bits(inp["w_down"][int(e)])[None], O.BF16, wfmt))
        return res

    parts = [r for chunk in _threaded(one, E) for r in chunk]
    return tuple(np.concatenate([p[i] for p in parts]) for i in range(4))


def check_mx_full_size(cfg, seed: int, n_tokens: int = 32, device="cuda", wfmt: int = M.MX_W_E4M3):
    """Full-size MX layer through the staged MX calls: bit-exact routing, plan
    and dispatched codes and scales; one row of h (codes and scales) and of
    yp in every planned block, and n_tokens tokens of out spread over the
    token range, against the oracle; the layer entry gives the same bits."""
    inp = I.make_inputs(cfg, seed, device)
    g = run_mx_stages(cfg, inp, wfmt)
    hin = host_inputs(inp, with_weights=False)
    ref = oracle_routing(cfg, hin)
    check_routing_and_plan(cfg, g, ref)
    assert (g["status"] & ~O.PLAN_INEXACT) == 0, f"device status {g['status']}"
    d, F = cfg.d, cfg.F
    total = ref["plan"]["total_rows"]
    src = ref["src_of"][:total]
    valid = src >= 0
    xq_ref, xs_ref = O.mx_quantize(hin["x"], O.BF16)
    gxq = g["xq"][:total].cpu().numpy()
    gxs = mx_unchunk(g["xs"], total, d)
    assert np.array_equal(gxq[valid], xq_ref[src[valid]]), "dispatched codes differ"
    assert np.array_equal(gxs[valid], xs_ref[src[valid]]), "dispatched scales differ"
    del gxq, gxs
    w1q, w1s, w2q, w2s = par_mx_oracle_weights(cfg, inp, wfmt)
    rng = np.random.default_rng(seed + 29)
    blocks = ref["plan"]["blocks"]
    rows = np.array([b[1] + rng.integers(b[2]) for b in blocks], np.int64)
    exps = blocks[:, 0].astype(np.int32)
    parts = _threaded(lambda sh: O.mx_fc1_rows(np.arange(len(sh)), exps[sh], xq_ref[src[rows[sh]]],
                                               xs_ref[src[rows[sh]]], w1q, w1s, F, wfmt), len(rows))
    rh, rhq, rhs = (np.concatenate([p[i] for p in parts]) for i in range(3))
    ghq = g["hq"][torch.as_tensor(rows, device=device)].cpu().numpy()
    ghs_all = mx_unchunk(g["hs"], total, F)
    assert_mx_h_close(ghq, ghs_all[rows], rh, rhq, rhs, "h (MXFP8), one row per block")
    ry = np.concatenate(_threaded(lambda sh: O.mx_fc2_rows(exps[sh], rhq[sh], rhs[sh], w2q, w2s, d, wfmt),
                                  len(rows)))
    yb = mx_h_error_bound(exps, ghq, ghs_all[rows], rhq, rhs, w2q, w2s, d, wfmt)
    assert_close_mx(to_f64(g["yp"][torch.as_tensor(rows, device=device)]), ry, yb, "yp, one row per block")
    toks = np.unique(np.linspace(0, cfg.T - 1, n_tokens).astype(np.int64))
    rout = np.concatenate(_threaded(lambda sh: O.mx_token_out(toks[sh], xq_ref, xs_ref, ref["idx"], ref["w"], w1q,
                                                               w1s, w2q, w2s, F, wfmt), len(toks)))
    ob = mx_out_error_bound(cfg, toks, ref, g, xq_ref, xs_ref, w1q, w1s, w2q, w2s, wfmt)
    assert_close_mx(to_f64(g["out"][torch.as_tensor(toks, device=device)]), rout, ob, "out, spread tokens")
    layer = M.Layer(cfg, device)
    out = layer.forward_mx(inp["logits"], inp["x"], g["mxw"])
    assert (layer.status() & ~O.PLAN_INEXACT) == 0
    assert torch.equal(out, g["out"]), "moe_layer_fwd_mx differs from the staged MX calls"
    return g
