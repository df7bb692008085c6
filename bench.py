"""Benchmark of the routed-expert MoE layer on B200: tokens/s of one layer pass.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config olmoe] [--impl mine|reference]

One step = one pass of the whole layer (top-k and gating, histogram, planner,
row maps, dispatch, FC1 + SwiGLU, FC2, combine; FC1 reads x itself in place
of the dispatch when moe_layer_path says so) over one batch of seeded
synthetic inputs already resident in HBM: one moe_layer_fwd call through the
C ABI. The stages are timed in a second pass, one ABI call per stage, and
FC2 with the combine folded in (moe_expert_fc2_combine) and the other FC1
input path in further passes. Under torchrun
every rank runs its own independent layer (its own tokens, replicated
weights, no collective on the data path: weak scaling); the timed region is
bracketed by a barrier and a device synchronisation, and the time is the
maximum over ranks. Rank 0 prints one JSON line.

--impl reference times the CPU oracle (oracle/, plain fp64 C, one core) on a
bounded sample of the same workload: routing, planning and row maps over
every token, the expert FFN and combine over a few tokens, scaled to the
whole layer.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from routed_experts_b200 import configs as C  # noqa: E402
from routed_experts_b200 import inputs as I  # noqa: E402

METRIC = "routed MoE layer tokens/s at 1 B200; % of bf16 tensor / HBM roofline"
LAUNCHES_PER_STEP = 7   # moe_layer_fwd: topk_hist, plan, row_maps, dispatch, fc1, fc2, combine (6 when FC1 reads x)
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=20)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--config", default="dsv3", choices=sorted(C.NAMED))
    p.add_argument("--seed", type=int, default=0)
    p.add_argument("--impl", default="mine", choices=["mine", "reference"])
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--cpu-tokens", type=int, default=None,
                   help="tokens of the oracle's FFN sample (default: sized to a few seconds per leg)")
    p.add_argument("--no-backward", action="store_true", help="skip timing the layer's backward")
    p.add_argument("--no-mx", action="store_true", help="skip timing the layer on MXFP8 operands")
    return p.parse_args()


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return dict(PEAKS_FALLBACK), "fallback"


class ClockSampler:
    """SM clock, its maximum and the active clock-event (throttle) reasons of
    one GPU, polled through NVML every 2 ms while the timed region runs (the
    region can be only tens of milliseconds long). Reads settings only."""

    def __init__(self, device: torch.device):
        self.device = device
        self.samples = []
        self.sm_max = None
        self.handle = None
        self.stop = threading.Event()

    def _handle(self):
        import pynvml as N
        N.nvmlInit()
        p = torch.cuda.get_device_properties(self.device)
        try:
            bus = f"{p.pci_domain_id:08x}:{p.pci_bus_id:02x}:{p.pci_device_id:02x}.0"
            return N.nvmlDeviceGetHandleByPciBusId(bus.encode())
        except Exception:
            vis = os.environ.get("CUDA_VISIBLE_DEVICES", "")
            ids = [v for v in vis.split(",") if v.strip()]
            idx = self.device.index or 0
            return N.nvmlDeviceGetHandleByIndex(int(ids[idx]) if idx < len(ids) and ids[idx].isdigit() else idx)

    def __enter__(self):
        try:
            import pynvml as N
            self.N = N
            self.handle = self._handle()
            self.sm_max = N.nvmlDeviceGetMaxClockInfo(self.handle, N.NVML_CLOCK_SM)
            self.t = threading.Thread(target=self._poll, daemon=True)
            self.t.start()
        except Exception:
            self.handle = None
        return self

    def _poll(self):
        N = self.N
        while not self.stop.is_set():
            try:
                sm = N.nvmlDeviceGetClockInfo(self.handle, N.NVML_CLOCK_SM)
                rs = N.nvmlDeviceGetCurrentClocksEventReasons(self.handle)
                self.samples.append((sm, rs))
            except Exception:
                pass
            time.sleep(0.002)

    def __exit__(self, *a):
        self.stop.set()
        if self.handle is not None:
            self.t.join(timeout=2)

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.sm_max, "reasons": [], "samples": 0}
        N = self.N
        names = {"hw_slowdown": N.nvmlClocksEventReasonHwSlowdown,
                 "hw_thermal_slowdown": N.nvmlClocksEventReasonHwThermalSlowdown,
                 "sw_thermal_slowdown": N.nvmlClocksEventReasonSwThermalSlowdown,
                 "sw_power_cap": N.nvmlClocksEventReasonSwPowerCap,
                 "hw_power_brake": N.nvmlClocksEventReasonHwPowerBrakeSlowdown}
        reasons = sorted(n for n, bit in names.items() if any(r & bit for _, r in self.samples))
        return {"sm_mhz": statistics.median(s for s, _ in self.samples), "sm_max_mhz": self.sm_max,
                "reasons": reasons, "samples": len(self.samples), "source": "NVML, 2 ms polling"}


def source_sha(*rel):
    h = hashlib.sha256()
    for r in rel:
        with open(os.path.join(ROOT, r), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


GEMM_SOURCES = ("routed_experts_b200/csrc/ffn_tn.cu", "routed_experts_b200/csrc/ptx.cuh",
                "routed_experts_b200/csrc/common.cuh", "routed_experts_b200/csrc/tc_common.cuh")


def ncu_traffic(kernel_key: str):
    """DRAM bytes per launch of a kernel from a committed ncu capture, or None
    when the capture is missing or the kernel's sources changed since."""
    path = os.path.join(ROOT, "profiles", "ncu_counters.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        d = json.load(f)
    e = d.get(kernel_key)
    if not e or e.get("source_sha") != source_sha(*GEMM_SOURCES):
        return None
    return e.get("dram_bytes_per_launch")


def max_over_ranks(values, device=None):
    """Element-wise maximum of per-rank floats over all ranks (a no-op without a
    process group). The tensor lives on `device` (the rank's GPU under NCCL,
    the CPU under gloo)."""
    if not (torch.distributed.is_available() and torch.distributed.is_initialized()):
        return [float(v) for v in values]
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return [float(v) for v in t.cpu()]


def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


# ------------------------------------------------------------------ the CPU oracle, timed

# Rough fp64 rate of the oracle's plain loops on one core (FLOP/s), used only
# to size the token samples so that each leg takes seconds, not hours.
ORACLE_FLOPS_GUESS = 1.8e9


def host_facts() -> dict:
    model = None
    try:
        with open("/proc/cpuinfo") as f:
            for ln in f:
                if ln.startswith("model name"):
                    model = ln.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    return {"cpu_model": model, "logical_cpus": os.cpu_count(), "usable_cpus": len(os.sched_getaffinity(0))}


def oracle_tokens_for(cfg, seconds: float, lo: int, hi: int) -> int:
    """Tokens of the oracle's FFN sample that take about `seconds` on one core."""
    per_token = 6.0 * cfg.d * cfg.F * cfg.K / ORACLE_FLOPS_GUESS
    return int(max(lo, min(hi, cfg.T, round(seconds / per_token))))


def oracle_leg(cfg, logits, x, expert_weights, n_tokens: int, workers: int) -> dict:
    """One timed pass of the CPU oracle on a bounded sample of the layer.

    Routing, gating, histogram, planning and row maps run over every token
    on one thread (the planner is sequential). The expert FFN and combine
    run for `n_tokens` evenly spaced tokens, split into `workers` shards that
    run on that many threads at once (each shard is one single-threaded
    oracle call; ctypes releases the interpreter lock around it). The
    whole-layer time is the routing time plus the sample's wall time per
    token times T. `expert_weights(experts)` returns host bit arrays of those
    experts' weights (fetched outside the timed parts)."""
    import concurrent.futures
    from oracle import oracle as O
    T, E, K = cfg.T, cfg.E, cfg.K
    t0 = time.perf_counter()
    idx, w = O.topk_gate(logits, K, cfg.gating)
    counts = O.histogram(idx, E)
    pl = O.plan(T, E, K, cfg.R, cfg.tile, cfg.budget, counts, getattr(cfg, "plan_mode", 0))
    O.row_maps(idx, E, pl["pieces"], O.rows_capacity(T * K, E, cfg.R, cfg.budget, cfg.tile))
    routing_s = time.perf_counter() - t0
    toks = np.unique(np.linspace(0, T - 1, num=min(n_tokens, T)).astype(np.int64))
    experts, sub = np.unique(idx[toks], return_inverse=True)
    wgu, wdn = expert_weights(experts)
    sub_idx = np.ascontiguousarray(sub.reshape(len(toks), K).astype(np.int32))
    xs = np.ascontiguousarray(x[toks])
    ws_ = np.ascontiguousarray(w[toks])
    shards = [s_ for s_ in np.array_split(np.arange(len(toks), dtype=np.int64), workers) if len(s_)]
    rm = O.default_round_mode(cfg.dtype)
    t1 = time.perf_counter()
    with concurrent.futures.ThreadPoolExecutor(max_workers=len(shards)) as ex:
        list(ex.map(lambda sh: O.token_out(sh, xs, sub_idx, ws_, wgu, wdn, cfg.dtype, rm), shards))
    ffn_s = time.perf_counter() - t1
    per_tok = ffn_s / len(toks)
    return {"routing_s": routing_s, "ffn_wall_s": ffn_s, "sample_tokens": int(len(toks)),
            "threads": len(shards), "layer_s_est": routing_s + per_tok * T,
            "step_s": routing_s + ffn_s}


def oracle_sample_text(cfg, leg: dict) -> str:
    return (f"top-k, gating, histogram, plan and row maps over all {cfg.T} tokens on one thread "
            f"({leg['routing_s']:.2f} s); expert FFN and combine over {leg['sample_tokens']} evenly spaced tokens on "
            f"{leg['threads']} thread(s) ({leg['ffn_wall_s']:.2f} s wall), scaled to {cfg.T} tokens; fp64 C oracle, "
            f"each call single-threaded")


def bench_config(cfg, seed: int, world: int) -> dict:
    """The `config` object of the JSON line (identical in both arms)."""
    eb = cfg.elem_bytes
    w_bytes = 3 * cfg.E * cfg.F * cfg.d * eb
    buf_bytes = (cfg.N + (cfg.E + cfg.R * cfg.budget) * cfg.tile) * (2 * cfg.d + cfg.F) * eb
    big = w_bytes + buf_bytes > 126e6
    l2 = (f"no flush: inputs larger than L2 (expert weights {w_bytes / 1e9:.2f} GB, padded xp/h/yp "
          f"{buf_bytes / 1e9:.2f} GB, against a 126 MB L2)" if big else
          f"no flush; the working set ({(w_bytes + buf_bytes) / 1e6:.1f} MB) fits in L2 (a parity-sized shape)")
    return {"workload": cfg.name, **C.describe(cfg), "seed": seed, "l2": l2,
            "parallelism": f"replicas x{world} (independent layers, no collective)"}


# ------------------------------------------------------------------ reference arm

def run_reference(args, world, rank):
    """The CPU oracle as the reference arm, rank 0 only: each step is one
    oracle_leg on all usable host cores over a bounded token sample."""
    if rank != 0:
        return
    cfg = C.NAMED[args.config]
    dev = "cuda" if torch.cuda.is_available() else "cpu"   # input generation only
    inp = I.make_inputs(cfg, args.seed, dev, weights=False)
    logits, x = I.to_numpy_bits(inp["logits"]), I.to_numpy_bits(inp["x"])
    workers = max(1, len(os.sched_getaffinity(0)))
    n_tok = workers * oracle_tokens_for(cfg, 2.0, 1, 64) if args.cpu_tokens is None else args.cpu_tokens

    cache = {}

    def weights(experts):
        missing = [int(e) for e in experts if int(e) not in cache]
        if missing:
            wgu, wdn = I.expert_weights(cfg, args.seed, missing, dev)
            for i, e in enumerate(missing):
                cache[e] = (I.to_numpy_bits(wgu[i]), I.to_numpy_bits(wdn[i]))
        return (np.stack([cache[int(e)][0] for e in experts]), np.stack([cache[int(e)][1] for e in experts]))

    oracle_leg(cfg, logits, x, weights, n_tok, workers)   # fetches the sample's weights once
    for _ in range(args.warmup):
        oracle_leg(cfg, logits, x, weights, n_tok, workers)
    legs = [oracle_leg(cfg, logits, x, weights, n_tok, workers) for _ in range(args.steps)]
    est = sum(l_["layer_s_est"] for l_ in legs)
    value = cfg.T * len(legs) / est
    measured = sum(l_["step_s"] for l_ in legs)
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * measured / len(legs),
            "layer_ms_est": 1e3 * est / len(legs),
            "timing": "ms_per_step is the measured wall time of one sampled step; value is the whole layer's "
                      "tokens/s extrapolated from it (layer_ms_est per layer)",
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded SplitMix64 + Box-Muller inputs, the recipe in routed_experts_b200/inputs.py)",
            "config": bench_config(cfg, args.seed, world),
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": legs[0]["threads"], "kind": "oracle",
                             "sample": oracle_sample_text(cfg, legs[0]), "host": host_facts()},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ the CUDA path

def plan_comparison(cfg, inp, dev, reps=20):
    """The planners side by side on the step's routing: exact S*K (the layer's
    planner), MegaFlux's block-granular search, and fixed placement (no
    replica budget). Per mode: moe_plan time (top-k, histogram, planner, row
    maps; CUDA events), the whole layer's time with that plan (moe_layer_fwd),
    the busiest rank's tiles against the mean (the straggler an
    expert-parallel layer would wait for), valid entries on the busiest rank,
    padded rows, replicas, moves."""
    lg = inp["logits"]
    from routed_experts_b200 import moe as M
    out = {}
    T, K, E = cfg.T, cfg.K, cfg.E
    for name, c in (("exact_SK", cfg), ("blocks", cfg.replace(plan_mode=C.PLAN_BLOCKS)),
                    ("fixed_placement", cfg.replace(budget=0))):
        idx = torch.empty(T, K, dtype=torch.int32, device=dev)
        w = torch.empty(T, K, dtype=torch.float32, device=dev)
        counts = torch.empty(E, dtype=torch.int32, device=dev)
        ws = M.alloc_workspace(c, M.WS_PLAN, dev)
        for _ in range(3):
            M.moe_plan(c, lg, idx, w, counts, ws)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(reps):
            M.moe_plan(c, lg, idx, w, counts, ws)
        e1.record()
        torch.cuda.synchronize(dev)
        pl = M.read_plan(c, ws)
        tiles = np.diff(pl["rank_row0"].numpy()) // c.tile
        del ws
        layer = M.Layer(c, dev)
        for _ in range(3):
            layer.forward(lg, inp["x"], inp["w_gate_up"], inp["w_down"])
        l0, l1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        l0.record()
        for _ in range(reps // 2):
            layer.forward(lg, inp["x"], inp["w_gate_up"], inp["w_down"])
        l1.record()
        torch.cuda.synchronize(dev)
        del layer
        torch.cuda.empty_cache()
        out[name] = {"moe_plan_us": 1e3 * e0.elapsed_time(e1) / reps,
                     "layer_ms": l0.elapsed_time(l1) / (reps // 2),
                     "max_tiles_per_rank": int(tiles.max()), "mean_tiles_per_rank": float(tiles.mean()),
                     "max_entries_per_rank": int(pl["rank_load"].max()), "entries_per_rank_mean": T * K / c.R,
                     "padded_rows": pl["total_rows"] - T * K, "replicas": pl["replicas"], "moves": pl["moves"],
                     "inexact": bool(pl["status"] & 1)}
    return out


def cpu_baseline(cfg, inp, n_tokens):
    """The oracle on the host cores beside the GPU run: one leg on a single
    thread and one on every usable core, each on a bounded token sample."""
    logits, x = I.to_numpy_bits(inp["logits"]), I.to_numpy_bits(inp["x"])

    def weights(experts):
        sel = torch.as_tensor(np.asarray(experts, dtype=np.int64), device=inp["w_gate_up"].device)
        return I.to_numpy_bits(inp["w_gate_up"][sel]), I.to_numpy_bits(inp["w_down"][sel])

    workers = max(1, len(os.sched_getaffinity(0)))
    one = oracle_leg(cfg, logits, x, weights, n_tokens or oracle_tokens_for(cfg, 12.0, 8, 320), 1)
    allc = oracle_leg(cfg, logits, x, weights, workers * oracle_tokens_for(cfg, 8.0, 1, 256), workers)
    return {"value": cfg.T / allc["layer_s_est"], "unit": "tokens/s", "cores": allc["threads"], "kind": "oracle",
            "sample": oracle_sample_text(cfg, allc), "host": host_facts(),
            "single_core": {"value": cfg.T / one["layer_s_est"], "unit": "tokens/s", "cores": 1,
                            "sample": oracle_sample_text(cfg, one)}}


def skew_descriptors(cfg, counts: np.ndarray, plan: dict) -> dict:
    """Routing skew of the step's input and the balance the plan reached:
    kappa = max/mean entries per expert ([MegaFlux] §4.1, the workloads'
    skew measure), MaxVio = how far the busiest expert sits above the mean,
    as a ratio minus one ([MoonEP] "Per-expert breakdown"), and the virtual
    ranks' loads (entries, and 128-row tiles after padding) over their mean
    before planning (home experts only) and after."""
    c = np.asarray(counts, dtype=np.float64)
    mean_e = cfg.N / cfg.E
    home = c.reshape(cfg.R, cfg.E // cfg.R).sum(axis=1)
    C_ = cfg.N / cfg.R
    loads = plan["rank_load"].numpy().astype(np.float64)
    tiles = np.diff(plan["rank_row0"].numpy()) / cfg.tile
    return {"kappa": float(c.max() / mean_e), "maxvio": float(c.max() / mean_e - 1.0),
            "experts_chosen": int((c > 0).sum()),
            "rank_load_max_over_mean_before": float(home.max() / C_),
            "rank_load_min_over_mean_before": float(home.min() / C_),
            "rank_load_max_over_mean_after": float(loads.max() / C_),
            "rank_tiles_max_over_mean_after": float(tiles.max() / tiles.mean())}


def time_backward(cfg, inp, args, world, dev, stream, pg):
    """The training forward (moe_layer_fwd_train) and the backward
    (moe_layer_bwd) on a training workspace, each W untimed and K timed
    passes (CUDA events on the launching stream), max over ranks. The
    forward state does not change between backward passes."""
    from routed_experts_b200 import moe as M
    lg, x, wgu, wdn = inp["logits"], inp["x"], inp["w_gate_up"], inp["w_down"]
    layer = M.Layer(cfg, dev, train=True)
    layer.forward(lg, x, wgu, wdn, stream=stream)
    d_out = I.make_grad_out(cfg, args.seed, dev)
    T, d, E, F = cfg.T, cfg.d, cfg.E, cfg.F
    dx = torch.empty(T, d, dtype=M.act_dtype(cfg), device=dev)
    dwgu = torch.empty(E, 2 * F, d, dtype=torch.float32, device=dev)
    dwdn = torch.empty(E, d, F, dtype=torch.float32, device=dev)
    dl = torch.empty(T, E, dtype=torch.float32, device=dev)

    def bwd():
        M.moe_layer_bwd(cfg, lg, wgu, wdn, d_out, dx, dwgu, dwdn, dl, layer.ws, stream)

    def timed(fn):
        for _ in range(args.warmup):
            fn()
        if pg is not None:
            torch.distributed.barrier()
        torch.cuda.synchronize(dev)
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.steps):
            fn()
        e1.record(stream)
        torch.cuda.synchronize(dev)
        ms = e0.elapsed_time(e1)
        if pg is not None:
            ms = max_over_ranks([ms], dev)[0]
        return ms / args.steps

    fwd_ms = timed(lambda: layer.forward(lg, x, wgu, wdn, stream=stream))
    ms = timed(bwd)
    st = M.moe_read_status(layer.ws, stream)
    if st & (M.DEV_TIMEOUT | M.DEV_BAD_INDEX):
        raise RuntimeError(f"device status {st} after the backward passes")
    N = cfg.N
    alg = 12.0 * N * d * F        # DGrad W2 2NdF + WGrad W2 2NdF + DGrad W1 4NdF + WGrad W1 4NdF
    pk, _ = peaks()
    del layer, dwgu, dwdn
    torch.cuda.empty_cache()
    return {"ms_per_step": ms, "tokens_per_s": world * T / (ms * 1e-3), "forward_train_ms": fwd_ms,
            "train_step_tokens_per_s": world * T / ((ms + fwd_ms) * 1e-3),
            "tflops": alg / (ms * 1e-3) / 1e12, "frac": alg / (ms * 1e-3) / 1e12 / pk["bf16_tflops"],
            "flop_algorithmic": alg,
            "note": "moe_layer_bwd: dY and dw, zeroed padding rows, DGrad W2 with the SwiGLU derivative "
                    "(pre-activations kept by moe_layer_fwd_train), WGrad W2, DGrad W1, WGrad W1, dx, logits' "
                    "gradient (8 launches); frac of the measured bf16 peak counts algorithmic FLOP"}


def time_mx(cfg, inp, args, world, dev, stream, pg, wfmt=0):
    """The layer on MX expert operands (moe_layer_fwd_mx; wfmt 0: MXFP8 weights,
    1: MXFP4 weights; activations MXFP8), W untimed and K timed passes, plus its
    stages (plan, quantizing dispatch, FC1, FC2, combine) timed by events
    between the calls; max over ranks. Weights are quantized once, outside the
    timed region (an offline step)."""
    from routed_experts_b200 import moe as M
    lg, x, wgu, wdn = inp["logits"], inp["x"], inp["w_gate_up"], inp["w_down"]
    T, d, E, F, K = cfg.T, cfg.d, cfg.E, cfg.F, cfg.K
    q0, q1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    q0.record(stream)
    mxw = M.MxWeights(cfg, wgu, wdn, stream, wfmt=wfmt)
    q1.record(stream)
    layer = M.Layer(cfg, dev)
    ref = layer.forward(lg, x, wgu, wdn, stream=stream).float().clone()

    def timed(fn):
        for _ in range(args.warmup):
            fn()
        if pg is not None:
            torch.distributed.barrier()
        torch.cuda.synchronize(dev)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.steps):
            fn()
        e1.record(stream)
        torch.cuda.synchronize(dev)
        ms = e0.elapsed_time(e1)
        if pg is not None:
            ms = max_over_ranks([ms], dev)[0]
        return ms / args.steps

    with ClockSampler(dev) as clk:
        ms = timed(lambda: layer.forward_mx(lg, x, mxw, stream=stream))
    out = layer.forward_mx(lg, x, mxw, stream=stream).float()
    torch.cuda.synchronize(dev)
    rel_to_bf16 = (torch.linalg.norm(out - ref) / torch.linalg.norm(ref)).item()
    st = M.moe_read_status(layer.ws, stream)
    if st & (M.DEV_TIMEOUT | M.DEV_BAD_INDEX):
        raise RuntimeError(f"device status {st} after the MX layer passes")
    del layer
    # the stages, events between the calls
    idx = torch.empty(T, K, dtype=torch.int32, device=dev)
    w = torch.empty(T, K, dtype=torch.float32, device=dev)
    counts = torch.empty(E, dtype=torch.int32, device=dev)
    ws = M.alloc_workspace(cfg, M.WS_PLAN, dev)
    xq, xs, hq, hs = (M.mx_buffer(cfg, k, dev) for k in (M.MX_XQ, M.MX_XS, M.MX_HQ, M.MX_HS))
    cap = M.moe_rows_capacity(cfg)
    yp = torch.empty(cap, d, dtype=torch.bfloat16, device=dev)
    o = torch.empty(T, d, dtype=torch.bfloat16, device=dev)
    calls = (lambda: M.moe_plan(cfg, lg, idx, w, counts, ws, stream),
             lambda: M.moe_dispatch_mx(cfg, x, xq, xs, ws, stream),
             lambda: M.moe_expert_fc1_mx(cfg, xq, xs, mxw.w1q, mxw.w1s, hq, hs, ws, stream, wfmt),
             lambda: M.moe_expert_fc2_mx(cfg, hq, hs, mxw.w2q, mxw.w2s, yp, ws, stream, wfmt),
             lambda: M.moe_combine(cfg, yp, w, o, ws, stream))
    for _ in range(args.warmup):
        for f in calls:
            f()
    torch.cuda.synchronize(dev)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(len(calls) + 1)] for _ in range(args.steps)]
    for k in range(args.steps):
        evs[k][0].record(stream)
        for i, f in enumerate(calls):
            f()
            evs[k][i + 1].record(stream)
    torch.cuda.synchronize(dev)
    stage = np.array([[evs[k][i].elapsed_time(evs[k][i + 1]) for i in range(len(calls))] for k in range(args.steps)])
    mean = stage.mean(axis=0)
    if pg is not None:
        mean = np.array(max_over_ranks(list(mean), dev))
    pk, pk_kind = peaks()
    fp8_peak = 2.0 * pk["bf16_tflops"]   # E4M3 dense rate = 2 x bf16 (4.5 vs 2.25 PFLOP/s nominal)
    N = cfg.N
    fc1_flop, fc2_flop = 2.0 * N * d * (2 * F), 2.0 * N * F * d
    plan = M.read_plan(cfg, ws)
    active = int((np.bincount(plan["blocks"][:, 0].numpy(), minlength=E) > 0).sum()) if plan["n_blocks"] else 0
    w_bytes = active * 3 * F * d * ((0.5 if wfmt else 1.0) + 1 / 32)
    alg_bytes = 4 * T * E + T * d * 2 + w_bytes + T * d * 2
    t_roof = max((fc1_flop + fc2_flop) / (fp8_peak * 1e12), alg_bytes / (pk["hbm_gbs"] * 1e9))
    disp_bytes = T * d * 2 + N * d * (1 + 1 / 32) + 4 * N
    del mxw, xq, xs, hq, hs, yp
    torch.cuda.empty_cache()
    return {"ms_per_step": ms, "tokens_per_s": world * T / (ms * 1e-3),
            "stages_ms": {"plan": mean[0], "dispatch_mx": mean[1], "fc1_mx": mean[2], "fc2_mx": mean[3],
                          "combine": mean[4]},
            "fc1_tflops": fc1_flop / (mean[2] * 1e-3) / 1e12, "fc2_tflops": fc2_flop / (mean[3] * 1e-3) / 1e12,
            "fc1_frac": fc1_flop / (mean[2] * 1e-3) / 1e12 / fp8_peak,
            "fc2_frac": fc2_flop / (mean[3] * 1e-3) / 1e12 / fp8_peak,
            "fp8_peak_tflops": fp8_peak, "peak_kind": f"{pk_kind} bf16 burst x 2 (E4M3 / bf16 nominal ratio)",
            "dispatch_mx_gbs": disp_bytes / (mean[1] * 1e-3) / 1e9,
            "layer_roofline_frac": (t_roof * 1e3) / ms, "layer_roofline_ms": t_roof * 1e3,
            "weight_quantize_ms": q0.elapsed_time(q1),
            "rel_diff_to_bf16_layer": rel_to_bf16,
            "clocks": clk.summary(),
            "weights": "MXFP4 (E2M1)" if wfmt else "MXFP8 (E4M3)",
            "note": "moe_layer_fwd_mx: plan, dispatch with MXFP8 quantization of x, FC1 + SwiGLU with h "
                    "quantized to MXFP8 in the epilogue, FC2, combine; E8M0 scale per 32 elements; "
                    "weights quantized once outside the timed region"}


def run_mine(args, world, rank, local):
    from routed_experts_b200 import moe as M
    cfg = C.NAMED[args.config]
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    pg = None
    if world > 1:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=dev)
        pg = torch.distributed.group.WORLD
    inp = I.make_inputs(cfg, args.seed + rank, dev)
    stream = torch.cuda.current_stream(dev)
    T, K, E, d, F = cfg.T, cfg.K, cfg.E, cfg.d, cfg.F
    dt = M.act_dtype(cfg)
    idx = torch.empty(T, K, dtype=torch.int32, device=dev)
    w = torch.empty(T, K, dtype=torch.float32, device=dev)
    counts = torch.empty(E, dtype=torch.int32, device=dev)
    ws = M.alloc_workspace(cfg, M.WS_LAYER, dev)
    cap = M.moe_rows_capacity(cfg)
    xp = torch.empty(cap, d, dtype=dt, device=dev)
    h = torch.empty(cap, F, dtype=dt, device=dev)
    yp = torch.empty(cap, d, dtype=dt, device=dev)
    out = torch.empty(T, d, dtype=dt, device=dev)
    lg, x, wgu, wdn = inp["logits"], inp["x"], inp["w_gate_up"], inp["w_down"]
    fold = cfg.dtype == C.BF16

    # the timed step: the whole layer, one moe_layer_fwd call
    layer = M.Layer(cfg, dev)
    for _ in range(args.warmup):
        layer.forward(lg, x, wgu, wdn, stream=stream)
    st = layer.status(stream)
    if st & (M.DEV_TIMEOUT | M.DEV_BAD_INDEX):
        raise RuntimeError(f"device status {st} after warm-up")
    step_evs = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps + 1)]
    if pg is not None:
        torch.distributed.barrier()
    torch.cuda.synchronize(dev)
    with ClockSampler(dev) as clk:
        for k in range(args.steps):
            step_evs[k].record(stream)
            layer.forward(lg, x, wgu, wdn, stream=stream)
        step_evs[args.steps].record(stream)
        torch.cuda.synchronize(dev)
    if pg is not None:
        torch.distributed.barrier()
    elapsed_ms = step_evs[0].elapsed_time(step_evs[args.steps])
    step_ms = np.array([step_evs[k].elapsed_time(step_evs[k + 1]) for k in range(args.steps)])
    st = layer.status(stream)
    if st & (M.DEV_TIMEOUT | M.DEV_BAD_INDEX):
        raise RuntimeError(f"device status {st} after the timed steps")
    del layer

    # the same kernels, one ABI call per stage, so that each stage can be timed;
    # the FC1 input path is the one moe_layer_fwd takes for this shape (no
    # dispatch stage when FC1 reads x itself), or with dispatch=True the other
    gather = M.moe_layer_path(cfg) == M.PATH_GATHER_FC1
    def stages(evs, fold_fc2=False, dispatch=False):
        evs[0].record(stream)
        M.moe_plan(cfg, lg, idx, w, counts, ws, stream)
        evs[1].record(stream)
        if gather and not dispatch:
            evs[2].record(stream)
            M.moe_expert_fc1_gather(cfg, x, wgu, h, ws, stream)
        else:
            M.moe_dispatch(cfg, x, xp, ws, stream)
            evs[2].record(stream)
            M.moe_expert_fc1(cfg, xp, wgu, h, ws, stream)
        evs[3].record(stream)
        if fold_fc2:
            M.moe_expert_fc2_combine(cfg, h, wdn, w, yp, out, ws, stream)
            evs[4].record(stream)
            return
        M.moe_expert_fc2(cfg, h, wdn, yp, ws, stream)
        evs[4].record(stream)
        M.moe_combine(cfg, yp, w, out, ws, stream)
        evs[5].record(stream)

    def time_stages(fold_fc2, dispatch=False):
        n = 5 if fold_fc2 else 6
        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(6)] for _ in range(args.steps + args.warmup)]
        torch.cuda.synchronize(dev)
        for e in evs:
            stages(e, fold_fc2, dispatch)
        torch.cuda.synchronize(dev)
        st_ = M.moe_read_status(ws, stream)
        if st_ & (M.DEV_TIMEOUT | M.DEV_BAD_INDEX):
            raise RuntimeError(f"device status {st_} after the stage pass")
        return np.array([[e[i].elapsed_time(e[i + 1]) for i in range(n - 1)] for e in evs[args.warmup:]])

    fold_ms = time_stages(True) if fold else None
    disp_ms = time_stages(False, dispatch=True) if gather else None
    stage_ms = time_stages(False)
    plan = M.read_plan(cfg, ws)

    # the fused FFN (FC1 and FC2 in one launch) on the same plan and xp, K passes; then the
    # same with FC1 gathering x through the row map (dispatch, FC1 and FC2 in one launch)
    fused_ms = gather_ms = None
    if cfg.dtype == C.BF16:
        def timed_passes(fn):
            for _ in range(args.warmup):
                fn()
            if pg is not None:
                torch.distributed.barrier()
            torch.cuda.synchronize(dev)
            f0 = torch.cuda.Event(enable_timing=True)
            f1 = torch.cuda.Event(enable_timing=True)
            f0.record(stream)
            for _ in range(args.steps):
                fn()
            f1.record(stream)
            torch.cuda.synchronize(dev)
            t = f0.elapsed_time(f1)
            if pg is not None:
                t = max_over_ranks([t], dev)[0]
            return t / args.steps

        fused_ms = timed_passes(lambda: M.moe_expert_ffn_fused(cfg, xp, wgu, wdn, h, yp, ws, stream))
        gather_ms = timed_passes(lambda: M.moe_expert_ffn_fused_gather(cfg, x, wgu, wdn, h, yp, ws, stream))

    # end to end through the public API with host buffers: H2D of logits and x
    # from pinned memory, the layer, D2H of the output, every step
    layer_h = M.Layer(cfg, dev, host_io=True)
    lg_h = lg.cpu().pin_memory()
    x_h = x.cpu().pin_memory()
    out_h = torch.empty(T, d, dtype=dt).pin_memory()
    for _ in range(args.warmup):
        layer_h.forward_host(lg_h, x_h, wgu, wdn, out_h, stream)
    if pg is not None:
        torch.distributed.barrier()
    torch.cuda.synchronize(dev)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        layer_h.forward_host(lg_h, x_h, wgu, wdn, out_h, stream)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_serial_ms = e0.elapsed_time(e1)

    # the same calls as a serving loop issues them: three workspaces on three
    # streams, steps in turn, so a step's input copy, another's kernels and a
    # third's output copy run at once (with two, a stream's next input copy
    # waits for its previous output copy)
    NS = 3
    layers = [layer_h] + [M.Layer(cfg, dev, host_io=True) for _ in range(NS - 1)]
    streams = [torch.cuda.Stream(dev) for _ in range(NS)]
    outs = [out_h] + [torch.empty(T, d, dtype=dt).pin_memory() for _ in range(NS - 1)]
    for k in range(args.warmup):
        layers[k % NS].forward_host(lg_h, x_h, wgu, wdn, outs[k % NS], streams[k % NS])
    if pg is not None:
        torch.distributed.barrier()
    torch.cuda.synchronize(dev)
    e0.record(stream)
    for s_ in streams:
        s_.wait_event(e0)
    for k in range(args.steps):
        layers[k % NS].forward_host(lg_h, x_h, wgu, wdn, outs[k % NS], streams[k % NS])
    for s_ in streams:
        done = torch.cuda.Event()
        done.record(s_)
        stream.wait_event(done)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = e0.elapsed_time(e1)
    for L_ in layers:
        if L_.status() & (M.DEV_TIMEOUT | M.DEV_BAD_INDEX):
            raise RuntimeError("device status after the end-to-end steps")
    if pg is not None:
        torch.distributed.barrier()
        elapsed_ms, e2e_ms, e2e_serial_ms = max_over_ranks([elapsed_ms, e2e_ms, e2e_serial_ms], dev)

    del layer_h, layers
    torch.cuda.empty_cache()
    mx = mx4 = None
    if not args.no_mx and cfg.dtype == C.BF16:
        mx = time_mx(cfg, inp, args, world, dev, stream, pg, 0)
        torch.cuda.empty_cache()
        mx4 = time_mx(cfg, inp, args, world, dev, stream, pg, 1)

    bwd = None
    if not args.no_backward and cfg.dtype == C.BF16 and cfg.F % 256 == 0:
        torch.cuda.empty_cache()
        bwd = time_backward(cfg, inp, args, world, dev, stream, pg)

    plans = plan_comparison(cfg, inp, dev) if rank == 0 else None
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(cfg, inp, args.cpu_tokens)

    if pg is not None:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()
    if rank != 0:
        return

    pk, pk_kind = peaks()
    med = np.median(stage_ms, axis=0)
    mean = stage_ms.mean(axis=0)
    N = cfg.N
    # algorithmic work, valid entries only (padding rows are not counted)
    fc1_flop = 2.0 * N * d * (2 * F)
    fc2_flop = 2.0 * N * F * d
    fc1_s = mean[2] * 1e-3
    fc2_s = mean[3] * 1e-3
    tensor_peak = pk["bf16_tflops"]
    eb = cfg.elem_bytes
    active = int((np.bincount(plan["blocks"][:, 0].numpy(), minlength=E) > 0).sum()) if plan["n_blocks"] else 0
    weight_bytes = active * 3 * F * d * eb
    alg_bytes = 4 * T * E + T * d * eb + weight_bytes + T * d * eb
    layer_flop = fc1_flop + fc2_flop
    t_roof = max(layer_flop / (tensor_peak * 1e12), alg_bytes / (pk["hbm_gbs"] * 1e9))
    ms_per_step = elapsed_ms / args.steps
    value = world * T / (ms_per_step * 1e-3)
    # dispatch: x read once, N valid rows written, the row map read (padding rows are not written)
    gather_bytes = T * d * eb + N * d * eb + 4 * N
    combine_bytes = N * d * eb + 8 * N + T * d * eb
    line = {
        "metric": METRIC,
        "value": value,
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": ms_per_step,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16" if cfg.dtype == C.BF16 else "fp32",
        "data": "synthetic (seeded SplitMix64 + Box-Muller inputs, the recipe in routed_experts_b200/inputs.py)",
        "config": bench_config(cfg, args.seed, world),
        "roofline": {"bound": "tensor",
                     "kernel": "ffn_tn_kernel<3> (FC1 + SwiGLU reading x)" if gather else "ffn_tn_kernel<0> (FC1 + SwiGLU)",
                     "achieved": fc1_flop / fc1_s / 1e12, "peak": tensor_peak, "unit": "TFLOP/s",
                     "frac": fc1_flop / fc1_s / 1e12 / tensor_peak,
                     "traffic": ncu_traffic(f"{'fc1_gather' if gather else 'fc1'}@{cfg.name}"),
                     "peak_kind": f"{pk_kind} bf16 burst",
                     "flop_per_launch": fc1_flop, "launch_ms": mean[2]},
        "layer_roofline": {"frac": (t_roof * 1e3) / ms_per_step, "roofline_ms": t_roof * 1e3,
                           "flop": layer_flop, "alg_bytes": alg_bytes,
                           "peaks": {"bf16_tflops": tensor_peak, "hbm_gbs": pk["hbm_gbs"], "kind": pk_kind}},
        "stages_ms": ({"plan(topk+hist+plan+rowmaps)": med[0], "fc1 (reading x, no dispatch)": med[2],
                       "fc2": med[3], "combine": med[4]} if gather else
                      {"plan(topk+hist+plan+rowmaps)": med[0], "dispatch": med[1], "fc1": med[2], "fc2": med[3],
                       "combine": med[4]}),
        "fc1_input_paths_ms": None if disp_ms is None else {
            "fc1_reading_x": float(med[2]), "dispatch": float(np.median(disp_ms[:, 1])),
            "fc1_after_dispatch": float(np.median(disp_ms[:, 2])),
            "note": "moe_expert_fc1_gather (the layer's path for this shape) against moe_dispatch + moe_expert_fc1"},
        "fc2_combine_fold_ms": None if fold_ms is None else {
            "median": float(np.median(fold_ms[:, 3])), "separate_fc2_plus_combine": float(med[3] + med[4]),
            "note": "moe_expert_fc2_combine (FC2 with the top-k sum in its epilogue, bit-identical; its call "
                    "clears the arrival counters first) against moe_expert_fc2 + moe_combine"},
        "step_ms": {"median": float(np.median(step_ms)), "min": float(step_ms.min()),
                    "max": float(step_ms.max())},
        "stage_rates": {"fc1_tflops": fc1_flop / fc1_s / 1e12, "fc2_tflops": fc2_flop / fc2_s / 1e12,
                        "dispatch_gbs": (gather_bytes / (float(disp_ms[:, 1].mean()) * 1e-3) / 1e9 if gather else
                                         gather_bytes / (mean[1] * 1e-3) / 1e9),
                        "combine_gbs": combine_bytes / (mean[4] * 1e-3) / 1e9},
        "plan": {"moves": plan["moves"], "replicas": plan["replicas"], "status": plan["status"],
                 "padded_rows": plan["total_rows"] - N, "blocks": plan["n_blocks"]},
        "skew": skew_descriptors(cfg, counts.cpu().numpy(), plan),
        "planners": plans,
        "e2e": {"value": world * T / (e2e_ms / args.steps * 1e-3), "unit": "tokens/s",
                "h2d_bytes_per_step": 4 * T * E + T * d * eb, "d2h_bytes_per_step": T * d * eb,
                "ms_per_step": e2e_ms / args.steps,
                "path": "moe_layer_fwd_host per step (H2D of logits and x from pinned memory, the layer, D2H of "
                        "out), three workspaces on three streams with steps in turn",
                "one_stream_value": world * T / (e2e_serial_ms / args.steps * 1e-3),
                "one_stream_ms_per_step": e2e_serial_ms / args.steps},
        "gpu_launches": (LAUNCHES_PER_STEP - (1 if gather else 0)) * args.steps,
        "layer_path": ("moe_layer_fwd: top-k + histogram, plan, row maps, FC1 + SwiGLU reading x through the row "
                       "map, FC2, combine" if gather else
                       "moe_layer_fwd: top-k + histogram, plan, row maps, dispatch, FC1 + SwiGLU, FC2, combine"),
        "backward": bwd,
        "mx": mx,
        "mx_fp4_weights": mx4,
        "fused_ffn": None if fused_ms is None else {
            "ms": fused_ms, "gather_ms": gather_ms, "staged_fc1_fc2_ms": float(med[2] + med[3]),
            "staged_dispatch_fc1_fc2_ms": float(med[1] + med[2] + med[3]),
            "note": "moe_expert_ffn_fused: FC1 and FC2 in one launch, FC2 tiles released per block pair; "
                    "moe_expert_ffn_fused_gather: the same with FC1 gathering x through the row map "
                    "(the staged launches are what the layer runs)"},
        "clocks": clk.summary(),
    }
    if cpu is not None:
        line["cpu_baseline"] = cpu
    print(json.dumps(line), flush=True)


def main():
    args = parse()
    world, rank, local = dist_setup(args)
    if args.impl == "reference":
        run_reference(args, world, rank)
    else:
        run_mine(args, world, rank, local)


if __name__ == "__main__":
    main()
