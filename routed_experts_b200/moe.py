"""ctypes binding of libmoe.so (include/moe.h), over torch CUDA tensors.

Argument marshalling only: every step of the layer runs in the library's
CUDA kernels. There is no CPU fallback; if the library is missing or a call
fails, this module raises.
"""
from __future__ import annotations

import ctypes
import os

import torch

from . import configs as _cfgs

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libmoe.so")

MOE_OK, MOE_ERR_INVALID_ARG, MOE_ERR_UNSUPPORTED, MOE_ERR_WORKSPACE, MOE_ERR_CUDA = range(5)
DEV_PLAN_INEXACT, DEV_TIMEOUT, DEV_BAD_INDEX = 1, 2, 4
WS_PLAN, WS_LAYER, WS_LAYER_HOST, WS_LAYER_TRAIN = 0, 1, 2, 3
MX_XQ, MX_XS, MX_HQ, MX_HS, MX_W1Q, MX_W1S, MX_W2Q, MX_W2S = range(8)
MX_W_E4M3, MX_W_E2M1 = 0, 1   # weight element formats: MXFP8, MXFP4
PATH_DISPATCH, PATH_GATHER_FC1 = 0, 1   # moe_layer_fwd's FC1 input path


class MoeError(RuntimeError):
    def __init__(self, what: str, code: int):
        super().__init__(f"{what} failed: {status_string(code)}")
        self.code = code


class MoeConfig(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in ("T", "d", "E", "K", "F", "R", "tile", "budget", "dtype",
                                              "gating", "plan_mode")]


class PlanLayout(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int64) for n in ("header", "pieces", "blocks", "rank_load", "rank_replicas",
                                              "rank_row0", "row_of", "src_of", "max_pieces", "max_blocks",
                                              "rows_cap")]


_lib = None


def lib() -> ctypes.CDLL:
    """The loaded library; raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m routed_experts_b200.build` (needs nvcc)")
        L = ctypes.CDLL(LIB_PATH)
        P, S = ctypes.c_void_p, ctypes.c_size_t
        C = ctypes.POINTER(MoeConfig)
        L.moe_workspace_size.argtypes = [C, ctypes.c_int32, ctypes.POINTER(ctypes.c_size_t)]
        L.moe_rows_capacity.argtypes = [C, ctypes.POINTER(ctypes.c_int64)]
        L.moe_plan_view.argtypes = [C, ctypes.POINTER(PlanLayout)]
        L.moe_plan.argtypes = [C, P, P, P, P, P, S, P]
        L.moe_dispatch.argtypes = [C, P, P, P, S, P]
        L.moe_expert_ffn.argtypes = [C, P, P, P, P, P, P, S, P]
        L.moe_expert_fc1.argtypes = [C, P, P, P, P, S, P]
        L.moe_expert_ffn_fused.argtypes = [C, P, P, P, P, P, P, S, P]
        L.moe_expert_ffn_fused_gather.argtypes = [C, P, P, P, P, P, P, S, P]
        L.moe_expert_fc2.argtypes = [C, P, P, P, P, S, P]
        L.moe_expert_fc1_gather.argtypes = [C, P, P, P, P, S, P]
        L.moe_combine.argtypes = [C, P, P, P, P, S, P]
        L.moe_expert_fc2_combine.argtypes = [C, P, P, P, P, P, P, S, P]
        L.moe_layer_fwd.argtypes = [C, P, P, P, P, P, P, S, P]
        L.moe_layer_path.argtypes = [C, ctypes.POINTER(ctypes.c_int32)]
        L.moe_layer_fwd_host.argtypes = [C, P, P, P, P, P, P, S, P]
        L.moe_layer_bwd.argtypes = [C, P, P, P, P, P, P, P, P, P, S, P]
        L.moe_layer_fwd_train.argtypes = [C, P, P, P, P, P, P, S, P]
        L.moe_read_status.argtypes = [P, P, ctypes.POINTER(ctypes.c_uint32)]
        L.moe_plan_noalloc.argtypes = [C, P, P, P, P, P, P, P]
        L.moe_probe_bounded_wait.argtypes = [P, ctypes.c_int64, P]
        L.moe_probe_expert_ffn_timeout.argtypes = [C, P, P, P, P, P, P, S, ctypes.c_int64, P]
        L.moe_probe_fc1_gather_timeout.argtypes = [C, P, P, P, P, S, ctypes.c_int64, P]
        L.moe_status_string.argtypes = [ctypes.c_int]
        I32 = ctypes.c_int32
        L.moe_mx_buffer_bytes.argtypes = [C, I32, I32, ctypes.POINTER(ctypes.c_size_t)]
        L.moe_mx_quantize_weights.argtypes = [C, P, P, I32, P, P, P, P, P]
        L.moe_dispatch_mx.argtypes = [C, P, P, P, P, S, P]
        L.moe_expert_fc1_mx.argtypes = [C, P, P, P, P, I32, P, P, P, S, P]
        L.moe_expert_fc2_mx.argtypes = [C, P, P, P, P, I32, P, P, S, P]
        L.moe_layer_fwd_mx.argtypes = [C, P, P, P, P, P, P, I32, P, P, S, P]
        L.moe_status_string.restype = ctypes.c_char_p
        for f in ("moe_workspace_size", "moe_rows_capacity", "moe_plan_view", "moe_plan", "moe_dispatch",
                  "moe_expert_ffn", "moe_expert_ffn_fused", "moe_expert_ffn_fused_gather", "moe_expert_fc1", "moe_expert_fc2", "moe_expert_fc1_gather", "moe_combine",
                  "moe_expert_fc2_combine",
                  "moe_layer_fwd", "moe_layer_path", "moe_layer_bwd", "moe_layer_fwd_train",
                  "moe_layer_fwd_host", "moe_read_status", "moe_plan_noalloc", "moe_probe_bounded_wait",
                  "moe_probe_expert_ffn_timeout", "moe_probe_fc1_gather_timeout",
                  "moe_mx_buffer_bytes", "moe_mx_quantize_weights", "moe_dispatch_mx", "moe_expert_fc1_mx",
                  "moe_expert_fc2_mx", "moe_layer_fwd_mx"):
            getattr(L, f).restype = ctypes.c_int
        _lib = L
    return _lib


def status_string(code: int) -> str:
    try:
        return lib().moe_status_string(code).decode()
    except Exception:  # pragma: no cover
        return f"status {code}"


def _check(code: int, what: str):
    if code != MOE_OK:
        raise MoeError(what, code)


def config(c: "_cfgs.LayerConfig") -> MoeConfig:
    return MoeConfig(c.T, c.d, c.E, c.K, c.F, c.R, c.tile, c.budget, c.dtype, c.gating,
                     getattr(c, "plan_mode", 0))


def _ptr(t: torch.Tensor | None):
    if t is None:
        return None
    if not t.is_contiguous():
        raise ValueError("tensors passed to libmoe must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _ws(ws: torch.Tensor):
    return _ptr(ws), ctypes.c_size_t(ws.numel() * ws.element_size())


# ---------------------------------------------------------------- the C calls

def moe_layer_path(c) -> int:
    """PATH_GATHER_FC1 when moe_layer_fwd reads FC1's rows straight from x, else PATH_DISPATCH."""
    p = ctypes.c_int32(-1)
    _check(lib().moe_layer_path(ctypes.byref(config(c)), ctypes.byref(p)), "moe_layer_path")
    return p.value


def moe_workspace_size(c, kind: int = WS_PLAN) -> int:
    n = ctypes.c_size_t(0)
    _check(lib().moe_workspace_size(ctypes.byref(config(c)), kind, ctypes.byref(n)), "moe_workspace_size")
    return n.value


def moe_rows_capacity(c) -> int:
    n = ctypes.c_int64(0)
    _check(lib().moe_rows_capacity(ctypes.byref(config(c)), ctypes.byref(n)), "moe_rows_capacity")
    return n.value


def moe_plan_view(c) -> dict:
    v = PlanLayout()
    _check(lib().moe_plan_view(ctypes.byref(config(c)), ctypes.byref(v)), "moe_plan_view")
    return {f: getattr(v, f) for f, _ in PlanLayout._fields_}


def moe_plan(c, logits, topk_idx, topk_w, counts, ws, stream=None):
    p, n = _ws(ws)
    _check(lib().moe_plan(ctypes.byref(config(c)), _ptr(logits), _ptr(topk_idx), _ptr(topk_w), _ptr(counts),
                          p, n, _stream(stream)), "moe_plan")


def moe_dispatch(c, x, xp, ws, stream=None):
    p, n = _ws(ws)
    _check(lib().moe_dispatch(ctypes.byref(config(c)), _ptr(x), _ptr(xp), p, n, _stream(stream)), "moe_dispatch")


def moe_expert_ffn(c, xp, w_gate_up, w_down, h, yp, ws, stream=None):
    p, n = _ws(ws)
    _check(lib().moe_expert_ffn(ctypes.byref(config(c)), _ptr(xp), _ptr(w_gate_up), _ptr(w_down), _ptr(h),
                                _ptr(yp), p, n, _stream(stream)), "moe_expert_ffn")


def moe_expert_ffn_fused(c, xp, w_gate_up, w_down, h, yp, ws, stream=None):
    """FC1 and FC2 in one persistent launch (FC2 tiles wait on per-pair readiness counts)."""
    p, n = _ws(ws)
    _check(lib().moe_expert_ffn_fused(ctypes.byref(config(c)), _ptr(xp), _ptr(w_gate_up), _ptr(w_down), _ptr(h),
                                      _ptr(yp), p, n, _stream(stream)), "moe_expert_ffn_fused")


def moe_expert_ffn_fused_gather(c, x, w_gate_up, w_down, h, yp, ws, stream=None):
    """Dispatch, FC1 and FC2 in one launch: FC1 reads x through the plan's row map."""
    p, n = _ws(ws)
    _check(lib().moe_expert_ffn_fused_gather(ctypes.byref(config(c)), _ptr(x), _ptr(w_gate_up), _ptr(w_down),
                                             _ptr(h), _ptr(yp), p, n, _stream(stream)), "moe_expert_ffn_fused_gather")


def moe_expert_fc1(c, xp, w_gate_up, h, ws, stream=None):
    p, n = _ws(ws)
    _check(lib().moe_expert_fc1(ctypes.byref(config(c)), _ptr(xp), _ptr(w_gate_up), _ptr(h), p, n, _stream(stream)),
           "moe_expert_fc1")


def moe_expert_fc1_gather(c, x, w_gate_up, h, ws, stream=None):
    p, n = _ws(ws)
    _check(lib().moe_expert_fc1_gather(ctypes.byref(config(c)), _ptr(x), _ptr(w_gate_up), _ptr(h), p, n,
                                       _stream(stream)), "moe_expert_fc1_gather")


def moe_expert_fc2(c, h, w_down, yp, ws, stream=None):
    p, n = _ws(ws)
    _check(lib().moe_expert_fc2(ctypes.byref(config(c)), _ptr(h), _ptr(w_down), _ptr(yp), p, n, _stream(stream)),
           "moe_expert_fc2")


def moe_expert_fc2_combine(c, h, w_down, topk_w, yp, out, ws, stream=None):
    """FC2 with the weighted top-k sum folded in: yp as moe_expert_fc2, out as moe_combine."""
    p, n = _ws(ws)
    _check(lib().moe_expert_fc2_combine(ctypes.byref(config(c)), _ptr(h), _ptr(w_down), _ptr(topk_w), _ptr(yp),
                                        _ptr(out), p, n, _stream(stream)), "moe_expert_fc2_combine")


def moe_combine(c, yp, topk_w, out, ws, stream=None):
    p, n = _ws(ws)
    _check(lib().moe_combine(ctypes.byref(config(c)), _ptr(yp), _ptr(topk_w), _ptr(out), p, n, _stream(stream)),
           "moe_combine")


def moe_layer_fwd(c, logits, x, w_gate_up, w_down, out, ws, stream=None):
    p, n = _ws(ws)
    _check(lib().moe_layer_fwd(ctypes.byref(config(c)), _ptr(logits), _ptr(x), _ptr(w_gate_up), _ptr(w_down),
                               _ptr(out), p, n, _stream(stream)), "moe_layer_fwd")


def moe_layer_fwd_host(c, logits_host, x_host, w_gate_up, w_down, out_host, ws, stream=None):
    p, n = _ws(ws)
    _check(lib().moe_layer_fwd_host(ctypes.byref(config(c)), _ptr(logits_host), _ptr(x_host), _ptr(w_gate_up),
                                    _ptr(w_down), _ptr(out_host), p, n, _stream(stream)), "moe_layer_fwd_host")


def moe_layer_fwd_train(c, logits, x, w_gate_up, w_down, out, ws, stream=None):
    """moe_layer_fwd that also keeps FC1's pre-activations for moe_layer_bwd (MOE_WS_LAYER_TRAIN)."""
    p, n = _ws(ws)
    _check(lib().moe_layer_fwd_train(ctypes.byref(config(c)), _ptr(logits), _ptr(x), _ptr(w_gate_up),
                                     _ptr(w_down), _ptr(out), p, n, _stream(stream)), "moe_layer_fwd_train")


def moe_layer_bwd(c, logits, w_gate_up, w_down, d_out, dx, dw_gate_up, dw_down, dlogits, ws, stream=None):
    """The layer's backward on a MOE_WS_LAYER_TRAIN workspace that moe_layer_fwd_train last ran on."""
    p, n = _ws(ws)
    _check(lib().moe_layer_bwd(ctypes.byref(config(c)), _ptr(logits), _ptr(w_gate_up), _ptr(w_down), _ptr(d_out),
                               _ptr(dx), _ptr(dw_gate_up), _ptr(dw_down), _ptr(dlogits), p, n, _stream(stream)),
           "moe_layer_bwd")


def moe_plan_noalloc(c, logits, topk_idx, topk_w, counts, row_of, header, stream=None):
    """moe_plan with its scratch in the library's static device array (no workspace)."""
    _check(lib().moe_plan_noalloc(ctypes.byref(config(c)), _ptr(logits), _ptr(topk_idx), _ptr(topk_w),
                                  _ptr(counts), _ptr(row_of), _ptr(header), _stream(stream)), "moe_plan_noalloc")


def moe_probe_bounded_wait(status_word, budget_cycles: int, stream=None):
    """Runs the device timeout check: a wait on an mbarrier nothing arrives on."""
    _check(lib().moe_probe_bounded_wait(_ptr(status_word), int(budget_cycles), _stream(stream)),
           "moe_probe_bounded_wait")


def moe_probe_expert_ffn_timeout(c, xp, w_gate_up, w_down, h, yp, ws, budget_cycles: int, stream=None):
    """moe_expert_ffn with every device-side wait limited to budget_cycles (a failure-handling check)."""
    p, n = _ws(ws)
    _check(lib().moe_probe_expert_ffn_timeout(ctypes.byref(config(c)), _ptr(xp), _ptr(w_gate_up), _ptr(w_down),
                                              _ptr(h), _ptr(yp), p, n, ctypes.c_int64(int(budget_cycles)),
                                              _stream(stream)), "moe_probe_expert_ffn_timeout")


def moe_probe_fc1_gather_timeout(c, x, w_gate_up, h, ws, budget_cycles: int, stream=None):
    """moe_expert_fc1_gather with every device-side wait limited to budget_cycles (a failure-handling check)."""
    p, n = _ws(ws)
    _check(lib().moe_probe_fc1_gather_timeout(ctypes.byref(config(c)), _ptr(x), _ptr(w_gate_up), _ptr(h), p, n,
                                              ctypes.c_int64(int(budget_cycles)), _stream(stream)),
           "moe_probe_fc1_gather_timeout")


def moe_read_status(ws, stream=None) -> int:
    v = ctypes.c_uint32(0)
    _check(lib().moe_read_status(_ptr(ws), _stream(stream), ctypes.byref(v)), "moe_read_status")
    return v.value


# ---------------------------------------------------------------- MXFP8 forward

def moe_mx_buffer_bytes(c, which: int, wfmt: int = MX_W_E4M3) -> int:
    v = ctypes.c_size_t(0)
    _check(lib().moe_mx_buffer_bytes(ctypes.byref(config(c)), int(which), int(wfmt), ctypes.byref(v)),
           "moe_mx_buffer_bytes")
    return v.value


def moe_mx_quantize_weights(c, w_gate_up, w_down, w1q, w1s, w2q, w2s, stream=None, wfmt: int = MX_W_E4M3):
    _check(lib().moe_mx_quantize_weights(ctypes.byref(config(c)), _ptr(w_gate_up), _ptr(w_down), int(wfmt),
                                         _ptr(w1q), _ptr(w1s), _ptr(w2q), _ptr(w2s), _stream(stream)),
           "moe_mx_quantize_weights")


def moe_dispatch_mx(c, x, xq, xs, ws, stream=None):
    p, n = _ws(ws)
    _check(lib().moe_dispatch_mx(ctypes.byref(config(c)), _ptr(x), _ptr(xq), _ptr(xs), p, n, _stream(stream)),
           "moe_dispatch_mx")


def moe_expert_fc1_mx(c, xq, xs, w1q, w1s, hq, hs, ws, stream=None, wfmt: int = MX_W_E4M3):
    p, n = _ws(ws)
    _check(lib().moe_expert_fc1_mx(ctypes.byref(config(c)), _ptr(xq), _ptr(xs), _ptr(w1q), _ptr(w1s), int(wfmt),
                                   _ptr(hq), _ptr(hs), p, n, _stream(stream)), "moe_expert_fc1_mx")


def moe_expert_fc2_mx(c, hq, hs, w2q, w2s, yp, ws, stream=None, wfmt: int = MX_W_E4M3):
    p, n = _ws(ws)
    _check(lib().moe_expert_fc2_mx(ctypes.byref(config(c)), _ptr(hq), _ptr(hs), _ptr(w2q), _ptr(w2s), int(wfmt),
                                   _ptr(yp), p, n, _stream(stream)), "moe_expert_fc2_mx")


def moe_layer_fwd_mx(c, logits, x, w1q, w1s, w2q, w2s, out, ws, stream=None, wfmt: int = MX_W_E4M3):
    p, n = _ws(ws)
    _check(lib().moe_layer_fwd_mx(ctypes.byref(config(c)), _ptr(logits), _ptr(x), _ptr(w1q), _ptr(w1s), _ptr(w2q),
                                  _ptr(w2s), int(wfmt), _ptr(out), p, n, _stream(stream)), "moe_layer_fwd_mx")


def mx_buffer(c, which: int, device="cuda", wfmt: int = MX_W_E4M3) -> torch.Tensor:
    return torch.empty(moe_mx_buffer_bytes(c, which, wfmt), dtype=torch.uint8, device=device)


class MxWeights:
    """A layer's expert weights in MXFP8 (wfmt MX_W_E4M3) or MXFP4 (MX_W_E2M1), quantized on the
    device from bf16."""

    def __init__(self, c, w_gate_up, w_down, stream=None, wfmt: int = MX_W_E4M3):
        dev = w_gate_up.device
        self.wfmt = wfmt
        self.w1q, self.w1s, self.w2q, self.w2s = (mx_buffer(c, k, dev, wfmt)
                                                  for k in (MX_W1Q, MX_W1S, MX_W2Q, MX_W2S))
        moe_mx_quantize_weights(c, w_gate_up, w_down, self.w1q, self.w1s, self.w2q, self.w2s, stream, wfmt)


# ---------------------------------------------------------------- conveniences

def act_dtype(c) -> torch.dtype:
    return torch.bfloat16 if c.dtype == _cfgs.BF16 else torch.float32


def alloc_workspace(c, kind: int = WS_PLAN, device="cuda") -> torch.Tensor:
    return torch.empty(moe_workspace_size(c, kind), dtype=torch.uint8, device=device)


def read_plan(c, ws: torch.Tensor) -> dict:
    """Copies the plan out of a workspace (after moe_plan) into host tensors."""
    v = moe_plan_view(c)
    raw = ws.cpu()

    def arr(off, n, dt=torch.int32):
        return raw[off: off + n * 4].view(dt).clone()

    hdr = arr(v["header"], 8)
    npc, nbl = int(hdr[1]), int(hdr[2])
    total = int(hdr[3])
    return {
        "status": int(hdr[0]), "n_pieces": npc, "n_blocks": nbl, "total_rows": total, "moves": int(hdr[4]),
        "replicas": int(hdr[5]), "tau": int(hdr[6]), "candidate": int(hdr[7]),
        "pieces": arr(v["pieces"], 5 * npc).view(npc, 5),
        "blocks": arr(v["blocks"], 4 * nbl).view(nbl, 4),
        "rank_load": arr(v["rank_load"], c.R),
        "rank_replicas": arr(v["rank_replicas"], c.R),
        "rank_row0": arr(v["rank_row0"], c.R + 1),
        "row_of": arr(v["row_of"], c.T * c.K),
        "src_of": arr(v["src_of"], total),
    }


class Layer:
    """Owns a workspace for one layer shape and runs the whole layer on it."""

    def __init__(self, c, device="cuda", host_io: bool = False, train: bool = False):
        self.cfg = c
        self.kind = WS_LAYER_TRAIN if train else (WS_LAYER_HOST if host_io else WS_LAYER)
        self.ws = alloc_workspace(c, self.kind, device)
        self.out = torch.empty(c.T, c.d, dtype=act_dtype(c), device=device)

    def forward(self, logits, x, w_gate_up, w_down, out=None, stream=None):
        """The layer; a `train=True` layer also keeps what backward() needs."""
        out = self.out if out is None else out
        fwd = moe_layer_fwd_train if self.kind == WS_LAYER_TRAIN else moe_layer_fwd
        fwd(self.cfg, logits, x, w_gate_up, w_down, out, self.ws, stream)
        return out

    def forward_host(self, logits_host, x_host, w_gate_up, w_down, out_host, stream=None):
        moe_layer_fwd_host(self.cfg, logits_host, x_host, w_gate_up, w_down, out_host, self.ws, stream)
        return out_host

    def backward(self, logits, w_gate_up, w_down, d_out, stream=None, dlogits: bool = True):
        """Gradients after forward() on the same inputs (a `train=True` layer):
        dx, dw_gate_up, dw_down (fp32) and the logits' gradient (or None)."""
        c, dev = self.cfg, d_out.device
        dx = torch.empty(c.T, c.d, dtype=act_dtype(c), device=dev)
        dwgu = torch.empty(c.E, 2 * c.F, c.d, dtype=torch.float32, device=dev)
        dwdn = torch.empty(c.E, c.d, c.F, dtype=torch.float32, device=dev)
        dl = torch.empty(c.T, c.E, dtype=torch.float32, device=dev) if dlogits else None
        moe_layer_bwd(c, logits, w_gate_up, w_down, d_out, dx, dwgu, dwdn, dl, self.ws, stream)
        return dx, dwgu, dwdn, dl

    def forward_mx(self, logits, x, mxw: "MxWeights", out=None, stream=None):
        """The layer on MXFP8 expert operands (weights from MxWeights)."""
        out = self.out if out is None else out
        moe_layer_fwd_mx(self.cfg, logits, x, mxw.w1q, mxw.w1s, mxw.w2q, mxw.w2s, out, self.ws, stream, mxw.wfmt)
        return out

    def status(self, stream=None) -> int:
        return moe_read_status(self.ws, stream)
