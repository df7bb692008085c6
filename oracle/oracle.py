"""Python face of the CPU oracle (``oracle.c``), over numpy arrays.

TEST INFRASTRUCTURE. Only the test suite, the package smoke check and the
benchmark's CPU-baseline leg import this module. The product path (the CUDA
library and its binding) never imports it, and it imports nothing from the
product package.

bf16 tensors travel as uint16 arrays of bf16 bit patterns, fp32 tensors as
float32 arrays. ``dtype`` is 0 for bf16 and 1 for fp32.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import time

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "oracle.c")
LIB = os.path.join(HERE, "liboracle.so")

BF16, FP32 = 0, 1
ROUND_NONE, ROUND_F32, ROUND_BF16 = 0, 1, 2
PLAN_INEXACT = 1

_PIECE_FIELDS = ("expert", "rank", "start", "len", "row0")
_BLOCK_FIELDS = ("expert", "row0", "valid", "rank")

_lib = None


def build(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so with gcc (plain -O2, no fast-math, no FMA contraction)."""
    if force or not os.path.exists(LIB) or os.path.getmtime(LIB) < os.path.getmtime(SRC):
        tmp = f"{LIB}.{os.getpid()}.tmp"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fno-fast-math",
                               "-ffp-contract=off", "-Wall", "-o", tmp, SRC, "-lm"])
        os.replace(tmp, LIB)
    return LIB


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(LIB)
        P = ctypes.c_void_p
        i32, i64 = ctypes.c_int32, ctypes.c_int64
        L.orc_topk_gate.argtypes = [i64, i32, i32, i32, P, P, P]
        L.orc_histogram.argtypes = [i64, i32, P, P]
        L.orc_plan.argtypes = [i64, i32, i32, i32, i32, i32, P, P, P, P, P, P, P, P, P, P]
        L.orc_plan_blocks.argtypes = [i64, i32, i32, i32, i32, i32, P, P, P, P, P, P, P, P, P, P, P]
        L.orc_row_maps.argtypes = [i64, i32, i32, P, P, i32, i64, P, P]
        L.orc_dispatch.argtypes = [i64, i32, i32, P, P, P]
        L.orc_expert_ffn.argtypes = [i32, i32, i32, i32, i32, P, i32, P, P, P, P, P]
        L.orc_combine.argtypes = [i64, i32, i32, i32, i32, P, P, P, P]
        L.orc_token_out.argtypes = [i32, i32, i32, i32, i32, i64, P, P, P, P, P, P, P]
        L.orc_dense_layer.argtypes = [i64, i32, i32, i32, i32, i32, P, P, P, P, P]
        L.orc_entry_ffn.argtypes = [i32, i32, i32, i32, i64, P, P, P, P, P, P, P]
        L.orc_double_to_bf16.argtypes = [ctypes.c_double]
        L.orc_layer_bwd.argtypes = [i64, i32, i32, i32, i32, i32, i32, i32, P, P, P, P, P, P, P, P, P, P, P, P]
        L.orc_bwd_tokens.argtypes = [i32, i32, i32, i32, i32, i32, i32, i64, P, P, P, P, P, P, P, P, P, P, P]
        L.orc_bwd_wgrad_elems.argtypes = [i64, i32, i32, i32, i32, i32, P, P, P, P, P, P, i32, i64, P, P, P, P]
        L.orc_double_to_bf16.restype = ctypes.c_uint16
        L.orc_mx_quantize.argtypes = [i64, i32, i32, P, P, P]
        L.orc_mx_dequantize.argtypes = [i64, i32, P, P, P]
        L.orc_e4m3_encode.argtypes = [ctypes.c_double]
        L.orc_e4m3_encode.restype = ctypes.c_uint8
        L.orc_e4m3_value.argtypes = [ctypes.c_uint8]
        L.orc_e4m3_value.restype = ctypes.c_double
        L.orc_mx_scale_code.argtypes = [ctypes.c_double]
        L.orc_mx_scale_code.restype = ctypes.c_uint8
        L.orc_mx_entry_ffn.argtypes = [i32, i32, i64, P, P, P, P, P, P, P, P, i32, P, P, P, P]
        L.orc_mx_token_out.argtypes = [i32, i32, i32, i64, P, P, P, P, P, P, P, P, P, i32, P]
        L.orc_mx_quantize_fmt.argtypes = [i64, i32, i32, i32, P, P, P]
        L.orc_mx_dequantize_fmt.argtypes = [i64, i32, i32, P, P, P]
        L.orc_e2m1_encode.argtypes = [ctypes.c_double]
        L.orc_e2m1_encode.restype = ctypes.c_uint8
        L.orc_e2m1_value.argtypes = [ctypes.c_uint8]
        L.orc_e2m1_value.restype = ctypes.c_double
        L.orc_mx_scale_code_fmt.argtypes = [ctypes.c_double, i32]
        L.orc_mx_scale_code_fmt.restype = ctypes.c_uint8
        L.orc_mx_fc1_rows.argtypes = [i32, i32, i64, P, P, P, P, P, P, i32, P, P, P]
        L.orc_mx_fc2_rows.argtypes = [i32, i32, i64, P, P, P, P, P, i32, P]
        for f in ("orc_mx_quantize", "orc_mx_dequantize", "orc_mx_entry_ffn", "orc_mx_token_out",
                  "orc_mx_fc1_rows", "orc_mx_fc2_rows", "orc_mx_quantize_fmt", "orc_mx_dequantize_fmt"):
            getattr(L, f).restype = ctypes.c_int
        for f in ("orc_topk_gate", "orc_histogram", "orc_plan", "orc_plan_blocks", "orc_row_maps", "orc_dispatch",
                  "orc_expert_ffn", "orc_combine", "orc_token_out", "orc_dense_layer", "orc_entry_ffn"):
            getattr(L, f).restype = ctypes.c_int
        _lib = L
    return _lib


def _p(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return a.ctypes.data_as(ctypes.c_void_p)


def _check(rc: int, what: str):
    if rc != 0:
        raise RuntimeError(f"oracle {what} failed with code {rc}")


def _elem_dtype(dtype: int):
    return np.uint16 if dtype == BF16 else np.float32


# ---------------------------------------------------------------- layout sizes

def rows_capacity(N: int, E: int, R: int, budget: int, tile: int) -> int:
    """Rows the padded expert-major buffer can need: every piece wastes < tile rows."""
    return N + (E + R * budget) * tile


def max_pieces(E: int, R: int, budget: int) -> int:
    return E + R * budget


def max_blocks(N: int, E: int, R: int, budget: int, tile: int) -> int:
    return -(-N // tile) + max_pieces(E, R, budget)


# ---------------------------------------------------------------- steps

def topk_gate(logits: np.ndarray, K: int, gating: int):
    logits = np.ascontiguousarray(logits, dtype=np.float32)
    T, E = logits.shape
    idx = np.empty((T, K), np.int32)
    w = np.empty((T, K), np.float32)
    _check(lib().orc_topk_gate(T, E, K, gating, _p(logits), _p(idx), _p(w)), "topk_gate")
    return idx, w


def histogram(idx: np.ndarray, E: int) -> np.ndarray:
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    counts = np.empty(E, np.int32)
    _check(lib().orc_histogram(idx.size, E, _p(idx), _p(counts)), "histogram")
    return counts


PLAN_EXACT, PLAN_BLOCKS = 0, 1


def plan(T: int, E: int, K: int, R: int, tile: int, budget: int, counts: np.ndarray,
         mode: int = PLAN_EXACT) -> dict:
    """The replication plan. mode PLAN_EXACT: the MoonEP-style greedy to exactly
    S*K entries per rank; PLAN_BLOCKS: MegaFlux's block-granular four-candidate
    search, pruning and refinement."""
    counts = np.ascontiguousarray(counts, dtype=np.int32)
    N = T * K
    pieces = np.zeros((max_pieces(E, R, budget), 5), np.int32)
    blocks = np.zeros((max_blocks(N, E, R, budget, tile), 4), np.int32)
    npc = np.zeros(1, np.int32)
    nbl = np.zeros(1, np.int32)
    rank_load = np.zeros(R, np.int64)
    rank_rep = np.zeros(R, np.int32)
    rank_row0 = np.zeros(R + 1, np.int64)
    moves = np.zeros(1, np.int32)
    status = np.zeros(1, np.uint32)
    info = np.zeros(4, np.int32)
    if mode == PLAN_EXACT:
        _check(lib().orc_plan(T, E, K, R, tile, budget, _p(counts), _p(pieces), _p(npc), _p(blocks),
                              _p(nbl), _p(rank_load), _p(rank_rep), _p(rank_row0), _p(moves),
                              _p(status)), "plan")
    else:
        _check(lib().orc_plan_blocks(T, E, K, R, tile, budget, _p(counts), _p(pieces), _p(npc), _p(blocks),
                                     _p(nbl), _p(rank_load), _p(rank_rep), _p(rank_row0), _p(moves),
                                     _p(status), _p(info)), "plan_blocks")
    return {"pieces": pieces[:npc[0]].copy(), "blocks": blocks[:nbl[0]].copy(),
            "rank_load": rank_load, "rank_replicas": rank_rep, "rank_row0": rank_row0,
            "moves": int(moves[0]), "status": int(status[0]),
            "total_rows": int(rank_row0[R]), "info": info}


def row_maps(idx: np.ndarray, E: int, pieces: np.ndarray, rows_cap: int):
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    T, K = idx.shape
    pieces = np.ascontiguousarray(pieces, dtype=np.int32)
    row_of = np.empty(T * K, np.int32)
    src_of = np.empty(rows_cap, np.int32)
    _check(lib().orc_row_maps(T, K, E, _p(idx), _p(pieces), pieces.shape[0], rows_cap,
                              _p(row_of), _p(src_of)), "row_maps")
    return row_of, src_of


def dispatch(x: np.ndarray, src_of: np.ndarray, dtype: int, rows: int | None = None) -> np.ndarray:
    x = np.ascontiguousarray(x)
    src_of = np.ascontiguousarray(src_of, dtype=np.int32)
    rows = src_of.shape[0] if rows is None else rows
    d = x.shape[1]
    xp = np.empty((rows, d), _elem_dtype(dtype))
    _check(lib().orc_dispatch(rows, d, dtype, _p(x), _p(src_of), _p(xp)), "dispatch")
    return xp


def expert_ffn(xp, w_gu, w_down, blocks, tile: int, dtype: int, round_mode: int, rows: int):
    xp = np.ascontiguousarray(xp)
    w_gu = np.ascontiguousarray(w_gu)
    w_down = np.ascontiguousarray(w_down)
    blocks = np.ascontiguousarray(blocks, dtype=np.int32)
    d = xp.shape[1]
    F = w_down.shape[2]
    h = np.zeros((rows, F), _elem_dtype(dtype))
    yp = np.zeros((rows, d), _elem_dtype(dtype))
    _check(lib().orc_expert_ffn(d, F, dtype, round_mode, tile, _p(blocks), blocks.shape[0],
                                _p(xp), _p(w_gu), _p(w_down), _p(h), _p(yp)), "expert_ffn")
    return h, yp


def combine(yp, row_of, w, dtype: int, round_mode: int):
    yp = np.ascontiguousarray(yp)
    row_of = np.ascontiguousarray(row_of, dtype=np.int32)
    w = np.ascontiguousarray(w, dtype=np.float32)
    T, K = w.shape
    d = yp.shape[1]
    out = np.empty((T, d), _elem_dtype(dtype))
    _check(lib().orc_combine(T, K, d, dtype, round_mode, _p(yp), _p(row_of), _p(w), _p(out)),
           "combine")
    return out


def token_out(tokens, x, idx, w, w_gu, w_down, dtype: int, round_mode: int) -> np.ndarray:
    tokens = np.ascontiguousarray(tokens, dtype=np.int64)
    x = np.ascontiguousarray(x)
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    w = np.ascontiguousarray(w, dtype=np.float32)
    w_gu = np.ascontiguousarray(w_gu)
    w_down = np.ascontiguousarray(w_down)
    K = idx.shape[1]
    d = x.shape[1]
    F = w_down.shape[2]
    out = np.empty((tokens.shape[0], d), np.float64)
    _check(lib().orc_token_out(d, F, K, dtype, round_mode, tokens.shape[0], _p(tokens), _p(x),
                               _p(idx), _p(w), _p(w_gu), _p(w_down), _p(out)), "token_out")
    return out


def entry_ffn(tokens, experts, x, w_gu, w_down, dtype: int, round_mode: int):
    """h [n,F] and y [n,d] (fp64 arrays holding the rounded values) of entries (tokens[i], experts[i])."""
    tokens = np.ascontiguousarray(tokens, dtype=np.int64)
    experts = np.ascontiguousarray(experts, dtype=np.int32)
    x = np.ascontiguousarray(x)
    w_gu = np.ascontiguousarray(w_gu)
    w_down = np.ascontiguousarray(w_down)
    d = x.shape[1]
    F = w_down.shape[2]
    n = tokens.shape[0]
    h = np.empty((n, F), np.float64)
    y = np.empty((n, d), np.float64)
    _check(lib().orc_entry_ffn(d, F, dtype, round_mode, n, _p(tokens), _p(experts), _p(x), _p(w_gu),
                               _p(w_down), _p(h), _p(y)), "entry_ffn")
    return h, y


def dense_layer(logits, x, w_gu, w_down, K: int, gating: int) -> np.ndarray:
    logits = np.ascontiguousarray(logits, dtype=np.float64)
    x = np.ascontiguousarray(x, dtype=np.float64)
    w_gu = np.ascontiguousarray(w_gu, dtype=np.float64)
    w_down = np.ascontiguousarray(w_down, dtype=np.float64)
    T, E = logits.shape
    d = x.shape[1]
    F = w_down.shape[2]
    out = np.empty((T, d), np.float64)
    _check(lib().orc_dense_layer(T, d, E, K, F, gating, _p(logits), _p(x), _p(w_gu),
                                 _p(w_down), _p(out)), "dense_layer")
    return out


def layer_bwd(logits, idx, w, x, w_gu, w_down, d_out, *, gating: int, dtype: int, round_mode: int) -> dict:
    """The backward of the routed layer for every token ([MegaFlux] §3.2
    "Backward"): dx (dtype), weight gradients, routing-weight and logit
    gradients (fp64)."""
    logits = np.ascontiguousarray(logits, dtype=np.float32)
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    w = np.ascontiguousarray(w, dtype=np.float32)
    x, w_gu, w_down, d_out = (np.ascontiguousarray(a) for a in (x, w_gu, w_down, d_out))
    T, E = logits.shape
    K = idx.shape[1]
    d = x.shape[1]
    F = w_down.shape[2]
    dx = np.empty((T, d), _elem_dtype(dtype))
    dw_gu = np.empty((E, 2 * F, d), np.float64)
    dw_down = np.empty((E, d, F), np.float64)
    dw = np.empty((T, K), np.float64)
    dl = np.empty((T, E), np.float64)
    _check(lib().orc_layer_bwd(T, d, E, K, F, gating, dtype, round_mode, _p(logits), _p(idx), _p(w), _p(x),
                               _p(w_gu), _p(w_down), _p(d_out), _p(dx), _p(dw_gu), _p(dw_down), _p(dw),
                               _p(dl)), "layer_bwd")
    return {"dx": dx, "dw_gate_up": dw_gu, "dw_down": dw_down, "dw": dw, "dlogits": dl}


def bwd_tokens(tokens, logits, idx, w, x, w_gu, w_down, d_out, *, gating: int, dtype: int, round_mode: int):
    """dx rows (rounded values, fp64 array), dw and logit-gradient rows of selected tokens."""
    tokens = np.ascontiguousarray(tokens, dtype=np.int64)
    logits = np.ascontiguousarray(logits, dtype=np.float32)
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    w = np.ascontiguousarray(w, dtype=np.float32)
    x, w_gu, w_down, d_out = (np.ascontiguousarray(a) for a in (x, w_gu, w_down, d_out))
    E = logits.shape[1]
    K = idx.shape[1]
    d = x.shape[1]
    F = w_down.shape[2]
    n = tokens.shape[0]
    dx = np.empty((n, d), np.float64)
    dw = np.empty((n, K), np.float64)
    dl = np.empty((n, E), np.float64)
    _check(lib().orc_bwd_tokens(d, E, K, F, gating, dtype, round_mode, n, _p(tokens), _p(logits), _p(idx),
                                _p(w), _p(x), _p(w_gu), _p(w_down), _p(d_out), _p(dx), _p(dw), _p(dl)),
           "bwd_tokens")
    return dx, dw, dl


def bwd_wgrad_elems(e: int, which, r, c, idx, w, x, w_gu, w_down, d_out, *, dtype: int, round_mode: int):
    """Single weight-gradient elements of expert e (which: 0 gate [f][i], 1 up [f][i], 2 down [i][f])."""
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    w = np.ascontiguousarray(w, dtype=np.float32)
    x, w_gu, w_down, d_out = (np.ascontiguousarray(a) for a in (x, w_gu, w_down, d_out))
    which = np.ascontiguousarray(which, dtype=np.int32)
    r = np.ascontiguousarray(r, dtype=np.int32)
    c = np.ascontiguousarray(c, dtype=np.int32)
    T, K = idx.shape
    d = x.shape[1]
    F = w_down.shape[2]
    out = np.empty(which.shape[0], np.float64)
    _check(lib().orc_bwd_wgrad_elems(T, d, K, F, dtype, round_mode, _p(idx), _p(w), _p(x), _p(w_gu),
                                     _p(w_down), _p(d_out), e, which.shape[0], _p(which), _p(r), _p(c),
                                     _p(out)), "bwd_wgrad_elems")
    return out


def double_to_bf16(v: float) -> int:
    return int(lib().orc_double_to_bf16(float(v)))


# ---------------------------------------------------------------- conversions

def bf16_bits_to_f64(a: np.ndarray) -> np.ndarray:
    return (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def to_f64(a: np.ndarray, dtype: int) -> np.ndarray:
    return bf16_bits_to_f64(a) if dtype == BF16 else a.astype(np.float64)


# ---------------------------------------------------------------- the whole layer

def default_round_mode(dtype: int) -> int:
    return ROUND_BF16 if dtype == BF16 else ROUND_F32


def layer(logits, x, w_gu, w_down, *, K, R, tile, budget, gating, dtype, round_mode=None,
          ffn=True, plan_mode: int = PLAN_EXACT) -> dict:
    """Every step of the layer on numpy inputs; returns each intermediate."""
    rm = default_round_mode(dtype) if round_mode is None else round_mode
    T, E = logits.shape
    idx, w = topk_gate(logits, K, gating)
    counts = histogram(idx, E)
    pl = plan(T, E, K, R, tile, budget, counts, plan_mode)
    cap = rows_capacity(T * K, E, R, budget, tile)
    row_of, src_of = row_maps(idx, E, pl["pieces"], cap)
    res = {"idx": idx, "w": w, "counts": counts, "plan": pl, "row_of": row_of,
           "src_of": src_of, "rows_cap": cap}
    if ffn:
        xp = dispatch(x, src_of, dtype, rows=cap)
        h, yp = expert_ffn(xp, w_gu, w_down, pl["blocks"], tile, dtype, rm, cap)
        out = combine(yp, row_of, w, dtype, rm)
        res.update(xp=xp, h=h, yp=yp, out=out)
    return res


def timed_sample(logits, x, w_gu, w_down, *, K, R, tile, budget, gating, dtype,
                 n_tokens: int, seed: int = 0) -> dict:
    """Time the oracle on a bounded sample of a layer.

    Routing, planning and row maps run over all tokens; the FFN and combine
    run on ``n_tokens`` evenly spaced tokens (their cost is per token), and
    the whole-layer time is that routing time plus the per-token FFN time
    times T. Single-threaded.
    """
    T = logits.shape[0]
    t0 = time.perf_counter()
    r = layer(logits, x, w_gu, w_down, K=K, R=R, tile=tile, budget=budget, gating=gating,
              dtype=dtype, ffn=False)
    t1 = time.perf_counter()
    toks = np.linspace(0, T - 1, num=min(n_tokens, T)).astype(np.int64)
    token_out(toks, x, r["idx"], r["w"], w_gu, w_down, dtype, default_round_mode(dtype))
    t2 = time.perf_counter()
    per_tok = (t2 - t1) / len(toks)
    est = (t1 - t0) + per_tok * T
    return {"routing_s": t1 - t0, "ffn_s_per_token": per_tok, "layer_s_est": est,
            "sample_tokens": int(len(toks)), "measured_s": t2 - t0}


# ---------------------------------------------------------------- MX (block-scaled) forward

MX_E4M3, MX_E2M1 = 0, 1   # element formats: MXFP8 (E4M3), MXFP4 (E2M1, one code per byte here)


def e2m1_encode(v: float) -> int:
    """A value rounded to an E2M1 code (nearest, ties to even, saturating at 6)."""
    return int(lib().orc_e2m1_encode(float(v)))


def e2m1_value(code: int) -> float:
    return float(lib().orc_e2m1_value(int(code)))


def mx_scale_code_fmt(amax: float, fmt: int) -> int:
    return int(lib().orc_mx_scale_code_fmt(float(amax), int(fmt)))


def mx_quantize_fmt(x: np.ndarray, dtype: int, fmt: int):
    """MX quantization of the rows of a [rows, K] matrix in element format fmt: (codes uint8 [rows, K],
    one code per byte, scale exponents uint8 [rows, K/32])."""
    x = np.ascontiguousarray(x)
    rows, K = x.shape
    codes = np.empty((rows, K), np.uint8)
    scales = np.empty((rows, K // 32), np.uint8)
    _check(lib().orc_mx_quantize_fmt(rows, K, dtype, fmt, _p(x), _p(codes), _p(scales)), "mx_quantize_fmt")
    return codes, scales


def mx_dequantize_fmt(codes: np.ndarray, scales: np.ndarray, fmt: int) -> np.ndarray:
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    scales = np.ascontiguousarray(scales, dtype=np.uint8)
    rows, K = codes.shape
    out = np.empty((rows, K), np.float64)
    _check(lib().orc_mx_dequantize_fmt(rows, K, fmt, _p(codes), _p(scales), _p(out)), "mx_dequantize_fmt")
    return out

def e4m3_encode(v: float) -> int:
    """A value rounded to an E4M3 code (nearest, ties to even, saturating at 448)."""
    return int(lib().orc_e4m3_encode(float(v)))


def e4m3_value(code: int) -> float:
    return float(lib().orc_e4m3_value(int(code)))


def mx_scale_code(amax: float) -> int:
    """The E8M0 scale exponent of an MXFP8 block whose largest magnitude is amax."""
    return int(lib().orc_mx_scale_code(float(amax)))


def mx_quantize(x: np.ndarray, dtype: int):
    """MXFP8 quantization of the rows of a [rows, K] matrix (bf16 bits or fp32), 32-element
    blocks along K: (codes uint8 [rows, K], scale exponents uint8 [rows, K/32])."""
    x = np.ascontiguousarray(x)
    rows, K = x.shape
    codes = np.empty((rows, K), np.uint8)
    scales = np.empty((rows, K // 32), np.uint8)
    _check(lib().orc_mx_quantize(rows, K, dtype, _p(x), _p(codes), _p(scales)), "mx_quantize")
    return codes, scales


def mx_dequantize(codes: np.ndarray, scales: np.ndarray) -> np.ndarray:
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    scales = np.ascontiguousarray(scales, dtype=np.uint8)
    rows, K = codes.shape
    out = np.empty((rows, K), np.float64)
    _check(lib().orc_mx_dequantize(rows, K, _p(codes), _p(scales), _p(out)), "mx_dequantize")
    return out


def mx_weights(w_gu: np.ndarray, w_down: np.ndarray, dtype: int, fmt: int = MX_E4M3):
    """MX expert weights (fmt: MXFP8 or MXFP4): W1 = w_gate_up [E, 2F, d] along d, W2 = w_down
    [E, d, F] along F."""
    E, F2, d = w_gu.shape
    F = F2 // 2
    w1q, w1s = mx_quantize_fmt(np.ascontiguousarray(w_gu).reshape(E * F2, d), dtype, fmt)
    w2q, w2s = mx_quantize_fmt(np.ascontiguousarray(w_down).reshape(E * d, F), dtype, fmt)
    return w1q, w1s, w2q, w2s


def mx_entry_ffn(tokens, experts, xq, xs, w1q, w1s, w2q, w2s, F: int, wfmt: int = MX_E4M3):
    """Routed entries of the MX expert FFN: h (bf16 values, fp64 array), h's MXFP8 codes and
    scales, and y (bf16 values, fp64 array)."""
    tokens = np.ascontiguousarray(tokens, dtype=np.int64)
    experts = np.ascontiguousarray(experts, dtype=np.int32)
    xq, xs, w1q, w1s, w2q, w2s = (np.ascontiguousarray(a, dtype=np.uint8) for a in (xq, xs, w1q, w1s, w2q, w2s))
    d = xq.shape[1]
    n = tokens.shape[0]
    h = np.empty((n, F), np.float64)
    hq = np.empty((n, F), np.uint8)
    hs = np.empty((n, F // 32), np.uint8)
    y = np.empty((n, d), np.float64)
    _check(lib().orc_mx_entry_ffn(d, F, n, _p(tokens), _p(experts), _p(xq), _p(xs), _p(w1q), _p(w1s), _p(w2q),
                                  _p(w2s), wfmt, _p(h), _p(hq), _p(hs), _p(y)), "mx_entry_ffn")
    return h, hq, hs, y


def mx_token_out(tokens, xq, xs, idx, w, w1q, w1s, w2q, w2s, F: int, wfmt: int = MX_E4M3) -> np.ndarray:
    """Layer output rows (bf16 values, fp64 array) of selected tokens of the MX layer."""
    tokens = np.ascontiguousarray(tokens, dtype=np.int64)
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    w = np.ascontiguousarray(w, dtype=np.float32)
    xq, xs, w1q, w1s, w2q, w2s = (np.ascontiguousarray(a, dtype=np.uint8) for a in (xq, xs, w1q, w1s, w2q, w2s))
    d = xq.shape[1]
    K = idx.shape[1]
    out = np.empty((tokens.shape[0], d), np.float64)
    _check(lib().orc_mx_token_out(d, F, K, tokens.shape[0], _p(tokens), _p(xq), _p(xs), _p(idx), _p(w), _p(w1q),
                                  _p(w1s), _p(w2q), _p(w2s), wfmt, _p(out)), "mx_token_out")
    return out


def mx_fc1_rows(rows, experts, xq, xs, w1q, w1s, F: int, wfmt: int = MX_E4M3):
    """FC1 of the MX FFN alone for rows of an MXFP8 activation matrix: h (bf16 values, fp64
    array) and its MXFP8 codes and scales."""
    rows = np.ascontiguousarray(rows, dtype=np.int64)
    experts = np.ascontiguousarray(experts, dtype=np.int32)
    xq, xs, w1q, w1s = (np.ascontiguousarray(a, dtype=np.uint8) for a in (xq, xs, w1q, w1s))
    d = xq.shape[1]
    n = rows.shape[0]
    h = np.empty((n, F), np.float64)
    hq = np.empty((n, F), np.uint8)
    hs = np.empty((n, F // 32), np.uint8)
    _check(lib().orc_mx_fc1_rows(d, F, n, _p(rows), _p(experts), _p(xq), _p(xs), _p(w1q), _p(w1s), wfmt, _p(h),
                                 _p(hq), _p(hs)), "mx_fc1_rows")
    return h, hq, hs


def mx_fc2_rows(experts, hq, hs, w2q, w2s, d: int, wfmt: int = MX_E4M3) -> np.ndarray:
    """FC2 of the MX FFN alone: MXFP8 rows of h through their experts' W2 (bf16 values, fp64 array)."""
    experts = np.ascontiguousarray(experts, dtype=np.int32)
    hq, hs, w2q, w2s = (np.ascontiguousarray(a, dtype=np.uint8) for a in (hq, hs, w2q, w2s))
    n, F = hq.shape
    y = np.empty((n, d), np.float64)
    _check(lib().orc_mx_fc2_rows(d, F, n, _p(experts), _p(hq), _p(hs), _p(w2q), _p(w2s), wfmt, _p(y)),
           "mx_fc2_rows")
    return y
