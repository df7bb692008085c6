"""Helpers for the GPU parity tests: run the layer through the C ABI stage by
stage, and compare every stage with the CPU oracle on the same inputs."""
from __future__ import annotations

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


def run_stages(cfg, inp: dict) -> dict:
    """moe_plan, moe_dispatch, moe_expert_ffn, moe_combine on device inputs."""
    dev = inp["x"].device
    T, K, E, d, F = cfg.T, cfg.K, cfg.E, cfg.d, cfg.F
    dt = M.act_dtype(cfg)
    idx = torch.empty(T, K, dtype=torch.int32, device=dev)
    w = torch.empty(T, K, dtype=torch.float32, device=dev)
    counts = torch.empty(E, dtype=torch.int32, device=dev)
    ws = M.alloc_workspace(cfg, M.WS_PLAN, dev)
    cap = M.moe_rows_capacity(cfg)
    # dispatch leaves padding rows of xp alone: NaN there must not reach h, yp or out
    xp = torch.full((cap, d), float("nan"), dtype=dt, device=dev)
    h = torch.empty(cap, F, dtype=dt, device=dev)
    yp = torch.empty(cap, d, dtype=dt, device=dev)
    out = torch.empty(T, d, dtype=dt, device=dev)
    M.moe_plan(cfg, inp["logits"], idx, w, counts, ws)
    M.moe_dispatch(cfg, inp["x"], xp, ws)
    M.moe_expert_ffn(cfg, xp, inp["w_gate_up"], inp["w_down"], h, yp, ws)
    M.moe_combine(cfg, yp, w, out, ws)
    status = M.moe_read_status(ws)
    plan = M.read_plan(cfg, ws)
    return {"idx": idx, "w": w, "counts": counts, "xp": xp, "h": h, "yp": yp, "out": out,
            "status": status, "plan": plan, "ws": ws, "rows_cap": cap}


def host_inputs(inp: dict, with_weights: bool = True) -> dict:
    keys = ("logits", "x", "w_gate_up", "w_down") if with_weights else ("logits", "x")
    return {k: I.to_numpy_bits(inp[k]) for k in keys}


def check_routing_and_plan(cfg, g: dict, ref: dict):
    """Bit-exact checks of top-k, counts, plan and row maps; weights within 1e-6."""
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


def check_full_small(cfg, seed: int, device="cuda"):
    """Every stage against the oracle, every element (sizes the oracle runs in seconds)."""
    inp = I.make_inputs(cfg, seed, device)
    g = run_stages(cfg, inp)
    hin = host_inputs(inp)
    ref = O.layer(hin["logits"], hin["x"], hin["w_gate_up"], hin["w_down"], K=cfg.K, R=cfg.R,
                  tile=cfg.tile, budget=cfg.budget, gating=cfg.gating, dtype=cfg.dtype,
                  plan_mode=getattr(cfg, "plan_mode", 0))
    assert g["rows_cap"] == ref["rows_cap"]
    check_routing_and_plan(cfg, g, ref)
    assert (g["status"] & ~O.PLAN_INEXACT) == 0, f"device status {g['status']}"
    total = ref["plan"]["total_rows"]
    valid = ref["src_of"][:total] >= 0
    assert np.array_equal(I.to_numpy_bits(g["xp"][:total])[valid], ref["xp"][:total][valid]), "xp differs"
    gh, gy = to_f64(g["h"][:total]), to_f64(g["yp"][:total])
    rh, ry = O.to_f64(ref["h"][:total], cfg.dtype), O.to_f64(ref["yp"][:total], cfg.dtype)
    assert_close(gh[valid], rh[valid], cfg.dtype, "h")
    assert_close(gy[valid], ry[valid], cfg.dtype, "yp")
    assert not gh[~valid].any() and not gy[~valid].any(), "padding rows must be zero"
    assert_close(to_f64(g["out"]), O.to_f64(ref["out"], cfg.dtype), cfg.dtype, "out")
    return g, ref, inp


class ExpertWeights:
    """Host copies of single experts' weights, fetched on demand."""

    def __init__(self, inp: dict):
        self.wgu, self.wdn = inp["w_gate_up"], inp["w_down"]
        self.cache = {}

    def stack(self, experts):
        es = list(experts)
        for e in es:
            if e not in self.cache:
                self.cache[e] = (I.to_numpy_bits(self.wgu[e]), I.to_numpy_bits(self.wdn[e]))
        return (np.stack([self.cache[e][0] for e in es]), np.stack([self.cache[e][1] for e in es]))


def check_full_size(cfg, seed: int, n_tokens: int = 8, n_rows: int = 32, device="cuda"):
    """Full-size layer: bit-exact routing, plan, row maps and dispatch; sampled
    rows of h and yp and sampled tokens of out against the oracle."""
    inp = I.make_inputs(cfg, seed, device)
    g = run_stages(cfg, inp)
    hin = host_inputs(inp, with_weights=False)
    ref = oracle_routing(cfg, hin)
    check_routing_and_plan(cfg, g, ref)
    assert (g["status"] & ~O.PLAN_INEXACT) == 0, f"device status {g['status']}"
    total = ref["plan"]["total_rows"]
    src = ref["src_of"][:total]
    # dispatch: every row is the token row it names (or zero), bit for bit
    xp = I.to_numpy_bits(g["xp"][:total])
    x = hin["x"]
    valid = src >= 0
    assert np.array_equal(xp[valid], x[src[valid]]), "xp rows differ from their token rows"
    del xp
    # padding rows of h and yp are zero (xp holds NaN there)
    pad = torch.as_tensor(np.nonzero(~valid)[0], device=device)
    if len(pad):
        assert not g["h"][pad].any() and not g["yp"][pad].any(), "padding rows of h and yp must be zero"
    rng = np.random.default_rng(seed + 17)
    ew = ExpertWeights(inp)
    # sampled rows of h and yp, from a few experts
    blocks = ref["plan"]["blocks"]
    experts = rng.choice(np.unique(blocks[:, 0]), size=min(4, len(np.unique(blocks[:, 0]))), replace=False)
    rows, exps = [], []
    for k, e in enumerate(experts):
        eb = blocks[blocks[:, 0] == e]
        cand = np.concatenate([np.arange(b[1], b[1] + b[2]) for b in eb])
        pick = rng.choice(cand, size=min(n_rows // len(experts), len(cand)), replace=False)
        rows += pick.tolist()
        exps += [k] * len(pick)
    rows = np.array(rows)
    wgu, wdn = ew.stack(experts)
    rh, ry = O.entry_ffn(src[rows], np.array(exps), x, wgu, wdn, cfg.dtype, O.default_round_mode(cfg.dtype))
    assert_close(to_f64(g["h"][torch.as_tensor(rows, device=device)]), rh, cfg.dtype, "sampled h rows")
    assert_close(to_f64(g["yp"][torch.as_tensor(rows, device=device)]), ry, cfg.dtype, "sampled yp rows")
    # sampled tokens of the output
    toks = rng.choice(cfg.T, size=n_tokens, replace=False)
    gout = to_f64(g["out"][torch.as_tensor(toks, device=device)])
    for i, t in enumerate(toks):
        es = ref["idx"][t]
        wgu, wdn = ew.stack(es)
        o = O.token_out(np.array([0]), x[t:t + 1], np.arange(cfg.K, dtype=np.int32)[None, :],
                        ref["w"][t:t + 1], wgu, wdn, cfg.dtype, O.default_round_mode(cfg.dtype))
        assert_close(gout[i:i + 1], o, cfg.dtype, f"out[{t}]")
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
    # FC2 on the oracle's h
    ry = O.mx_fc2_rows(row_exp[vrows], rhq, rhs, w2q, w2s, d, wfmt)
    gy = to_f64(g["yp"][:total])
    assert_close(gy[vrows], ry, C.BF16, "yp")
    assert not gy[~valid].any(), "padding rows of yp must be zero"
    # the whole layer, on all tokens or a seeded sample
    toks = np.arange(cfg.T) if cfg.T <= max_tokens else np.sort(rng.choice(cfg.T, size=max_tokens, replace=False))
    rout = O.mx_token_out(toks, xq_ref, xs_ref, ref["idx"], ref["w"], w1q, w1s, w2q, w2s, F, wfmt)
    assert_close(to_f64(g["out"])[toks], rout, C.BF16, "out")
    return g, ref, inp


def check_mx_full_size(cfg, seed: int, n_tokens: int = 3, device="cuda", wfmt: int = M.MX_W_E4M3):
    """Full-size MX layer through moe_layer_fwd_mx: bit-exact routing and plan
    (moe_plan), and sampled tokens of out against the oracle."""
    inp = I.make_inputs(cfg, seed, device)
    hin = host_inputs(inp, with_weights=False)
    ref = oracle_routing(cfg, hin)
    layer = M.Layer(cfg, device)
    mxw = mx_weights_on_device(cfg, inp, wfmt)
    out = layer.forward_mx(inp["logits"], inp["x"], mxw)
    assert (layer.status() & ~O.PLAN_INEXACT) == 0
    plan = M.read_plan(cfg, layer.ws)
    assert np.array_equal(plan["row_of"].numpy(), ref["row_of"]), "row_of differs"
    rng = np.random.default_rng(seed + 29)
    toks = rng.choice(cfg.T, size=n_tokens, replace=False)
    gout = to_f64(out[torch.as_tensor(toks, device=device)])
    for i, t in enumerate(toks):
        es = ref["idx"][t]
        w1q, w1s, w2q, w2s = mx_oracle_weights(cfg, inp, es, wfmt)
        xq, xs = O.mx_quantize(hin["x"][t:t + 1], O.BF16)
        o = O.mx_token_out(np.array([0]), xq, xs, np.arange(cfg.K, dtype=np.int32)[None, :], ref["w"][t:t + 1],
                           w1q, w1s, w2q, w2s, cfg.F, wfmt)
        assert_close(gout[i:i + 1], o, C.BF16, f"out[{t}]")
    return out
