#!/usr/bin/env python
"""Sparse-FFN decode benchmark: tokens/s per layer stack and achieved HBM GB/s
over the bytes the path touches, on seeded synthetic power-law-sparse inputs.

Default workload: the largest single-GPU configuration, the OPT-66B-shaped
stack (64 layers, d=9216, n=36864, predictor H=2048, fp16 weights, ~87 GB,
batch 32 on the union-mask tensor-core path, mean activation rate 1%,
alpha=1.0); ``--config 1`` is the OPT-6.7B-shaped stack at batch 1.  Weights
are generated in HBM, hot-first reordered offline (untimed), then K decode steps
are timed with CUDA events.  One step = spffn_decode over all layers: predictor
(two GEMVs + threshold + compaction), sparse FC1/FC2 with the deterministic
split reduction, and the chaining into the next layer.
With --lookahead the step is spffn_decode_lookahead instead (layer l+1's set
predicted from layer l's input, DejaVu's asynchronous predictor), reported
under its own workload name.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config 4] [--lookahead] [--impl ours|reference]
    python bench.py --config 3 --rate 0.05 --true-mask     # sparse FFN on the true set, no predictor
    python bench.py --dense                                # comparison: dense FFN with cuBLAS, same weights

Under torchrun each rank runs its own replica on its own decode stream
(independent requests: weak scaling, no data-path collective); the reported time
is the max over ranks.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import workload as wl  # noqa: E402

METRIC = "sparse-FFN decode tokens/s per layer-stack"
UNIT = "tokens/s"
PROFILE_TOKENS = 256
PREDICTION = {False: "each layer's set predicted from its own input",
              True: "look-ahead: layer l+1's set predicted from layer l's input"}


def workload_name(cfg, args) -> str:
    hot = "-l2hot%d" % args.l2_hot_rows if getattr(args, "l2_hot_rows", 0) else ""
    per = {0: "-perlayer", 1: "-wholestack"}.get(getattr(args, "union_stack", 2), "")
    return cfg.name + ("-lookahead" if args.lookahead else "") + hot + per


def config_dict(cfg, args, world: int) -> dict:
    """The workload as both arms print it (same keys and values in each), so a
    line of this implementation and a line of the reference arm name one config."""
    rate = args.rate or cfg.rate
    return {"workload": workload_name(cfg, args), "layers": cfg.layers, "d": cfg.d, "n": cfg.n, "H": cfg.H,
            "batch": cfg.batch, "dtype": cfg.dtype, "prediction": PREDICTION[args.lookahead],
            "activation_rate": rate, "alpha": cfg.alpha, "global_batch": cfg.batch * world,
            "parallelism": "replicas%d" % world,
            "placement": "hot-first dealt over the SM count of CTA ranges (offline profile of %d tokens)"
                         % PROFILE_TOKENS,
            "l2": l2_statement(cfg, args),
            "l2_hot_rows_per_range": getattr(args, "l2_hot_rows", 0)}


L2_BYTES = 126 * 2 ** 20


def l2_statement(cfg, args) -> str:
    weights = cfg.layers * (predictor_bytes(cfg) + dense_bytes_per_layer(cfg))
    if weights > 2 * L2_BYTES:
        return "inputs larger than L2: every layer's weights (%.1f GB in all) stream from HBM each step" % (weights / 1e9)
    if getattr(args, "flush_l2", False):
        return "weights (%.1f MB) fit in L2; L2 flushed (%d MB written) before every timed step" % (
            weights / 1e6, FLUSH_BYTES // 2 ** 20)
    return "weights (%.1f MB) fit in L2 and stay resident between steps (no flush)" % (weights / 1e6)


FLUSH_BYTES = 512 * 2 ** 20


# ---------------------------------------------------------------------------
# distributed plumbing (host-side only: barrier and max-over-ranks timing)
def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def dist_init(world, backend):
    import torch.distributed as dist
    if world > 1 and not dist.is_initialized():
        import datetime
        dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=120))
    return world > 1


def max_over_ranks(value: float, world: int, device=None) -> float:
    if world <= 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world: int, device=None):
    if world > 1:
        import torch.distributed as dist
        if device is not None and device.type == "cuda":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


def rank_seed(rank: int) -> int:
    """Each replica decodes its own request stream."""
    return 1 + rank


# ---------------------------------------------------------------------------
# bytes the path touches (algorithmic; x, y and L2-resident partials excluded)
def predictor_bytes(cfg) -> int:
    return 2 * (cfg.H * cfg.d + cfg.n * cfg.H) + 2 * cfg.n + 2 * cfg.H


def ffn_bytes_per_neuron(cfg) -> int:
    return 4 * cfg.d + 2 + 4          # W1 row + W2T row + b1 + table entry


def step_bytes(cfg, counts_sum: int, layers: int) -> int:
    return layers * predictor_bytes(cfg) + counts_sum * ffn_bytes_per_neuron(cfg)


def dense_bytes_per_layer(cfg) -> int:
    return 4 * cfg.n * cfg.d + 2 * cfg.n     # every W1 and W2T row + b1


# DRAM traffic (ncu dram__bytes_read.sum + dram__bytes_write.sum) of the
# persistent decode kernel per layer, from one capture of a 4-layer stack of the
# OPT-6.7B-shaped workload at batch 1 (traffic grows with layers, so a launch
# over L layers is L times this).  It holds only for the kernel sources it was
# captured on: any change to them and the bench reports null.
DECODE_SOURCES = ("spffn_fused.cu", "spffn_fused.cuh", "spffn_internal.cuh")
DECODE_TRAFFIC = {
    "sha256": "0c61c2bd06d4ce768ff9b8b7c12e6c676bbcb2829f49c481448ec202ddb0ee79",
    "workload": "opt6.7b-d4096-n16384-L32", "batch": 1, "rate": 0.05,
    "bytes_per_layer": (222.220544e6 + 4.9152e6) / 4,
}


# DRAM traffic of the union path's per-layer launches (predictor modes, FC1, FC2, chaining),
# from one capture of a 2-layer stack of the OPT-66B-shaped workload at batch 32: per layer
# a fixed part (predictor weights, chaining) plus a part per table neuron (its W1 and W2T
# rows), so a run's traffic is scaled by the neurons its layers actually selected.  It holds
# only for the kernel sources it was captured on: any change to them and the bench reports null.
UNION_SOURCES = ("spffn_union.cu", "spffn_umma.cuh", "spffn_internal.cuh", "spffn_kernels.cu")
UNION_TRAFFIC = {
    "sha256": "a33d7a16b83a54096f631f2d9ccafedbeb675db8b306cc3998d69452248e8a43",
    "workload": "opt66b-d9216-n36864-L64", "batch": 32, "rate": 0.01,
    "fixed_per_layer": 38.435e6 + 152.19e6 + 1.78e6,
    "per_neuron": (105.245e6 + 105.32e6) / 5639.17,
}


def decode_sources_sha256(files=DECODE_SOURCES) -> str:
    import hashlib
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "activation_sparse_ffn_predictor_b200", "csrc")
    for f in files:
        with open(os.path.join(csrc, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()


def union_traffic(cfg, batch: int, rate, lookahead: bool, per_layer_counts):
    """DRAM bytes per step of the union path for this run (mean over the timed steps), or None."""
    t = UNION_TRAFFIC
    if lookahead or cfg.name != t["workload"] or batch != t["batch"] or (rate or cfg.rate) != t["rate"]:
        return None
    if decode_sources_sha256(UNION_SOURCES) != t["sha256"]:
        return None
    steps = [t["fixed_per_layer"] * len(row) + t["per_neuron"] * float(sum(row)) for row in per_layer_counts]
    return sum(steps) / len(steps)


def decode_traffic(cfg, layers: int, batch: int, rate, lookahead: bool):
    """Measured DRAM bytes per launch of the decode kernel for this run, or None."""
    t = DECODE_TRAFFIC
    if lookahead or cfg.name != t["workload"] or batch != t["batch"] or (rate or cfg.rate) != t["rate"]:
        return None
    if decode_sources_sha256() != t["sha256"]:
        return None
    return t["bytes_per_layer"] * layers


# ---------------------------------------------------------------------------
class Clocks:
    """Samples SM clocks and throttle reasons (NVML, read-only) during the timed region."""

    def __init__(self, index: int, period_s: float = 0.01):
        self.index = index
        self.period = period_s
        self.rows = []
        self._stop = threading.Event()
        self._t = None

    def _sample(self):
        nv = self._nv
        sm = nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM)
        rs = nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
        self.rows.append((sm, self._mx, rs))

    def _run(self):
        try:
            while not self._stop.wait(self.period):
                self._sample()
        except Exception as e:
            self.error = repr(e)

    def __enter__(self):
        # NVML is opened and sampled once before the timed work starts, so a timed region
        # shorter than the sampling period still has a record (plus one at its end)
        try:
            import pynvml as nv
            nv.nvmlInit()
            self._nv = nv
            self._h = nv.nvmlDeviceGetHandleByIndex(self.index)
            self._mx = nv.nvmlDeviceGetMaxClockInfo(self._h, nv.NVML_CLOCK_SM)
            self._sample()
        except Exception as e:  # NVML missing: leave the record empty and say why
            self.error = repr(e)
            return self
        self._t = threading.Thread(target=self._run, daemon=True)
        self._t.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self._t:
            self._t.join(timeout=10)
            try:
                self._sample()
            except Exception as e:
                self.error = repr(e)

    def summary(self):
        if not self.rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0,
                    "error": getattr(self, "error", "no samples")}
        bits = {"hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40,
                "sw_power_cap": 0x4, "hw_power_brake_slowdown": 0x80}
        reasons = sorted({k for _, _, r in self.rows for k, b in bits.items() if r & b})
        return {"sm_mhz": statistics.median(r[0] for r in self.rows), "sm_max_mhz": max(r[1] for r in self.rows),
                "reasons": reasons, "samples": len(self.rows)}


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


# ---------------------------------------------------------------------------
def build_stack(cfg, layers, device, rate=None, reorder=True, log=print):
    """All layers in HBM; hot-first reordered from an offline profile (untimed)."""
    import torch
    import activation_sparse_ffn_predictor_b200 as sp
    out = []
    for l in range(layers):
        dl = wl.device_layer(cfg, l, device=device, rate=rate)
        L = sp.Layer.from_device_layer(dl, max_batch=cfg.batch)
        if reorder:
            Xp = wl.to_torch(wl.tokens(cfg, PROFILE_TOKENS, aux=l, tensor=wl.T_XPROF), cfg, device)
            counts = torch.zeros(cfg.n, dtype=torch.int32, device=device)
            L.profile_counts(Xp, counts)
            # hot-first order dealt over the decode kernel's per-CTA row ranges
            perm = sp.reorder_dealt(counts.cpu().numpy().astype(np.uint32), L.num_partials)
            pt = torch.from_numpy(perm).to(device)
            for name in ("W1", "W2T", "Wp2"):
                src = getattr(dl, name)
                dst = torch.empty_like(src)
                sp.permute_rows(src, dst, pt)
                setattr(dl, name, dst)
                del src
            for name in ("b1", "bp2"):
                src = getattr(dl, name)
                dst = torch.empty_like(src)
                sp.permute_vector(src, dst, pt)
                setattr(dl, name, dst)
            L.close()
            L = sp.Layer.from_device_layer(dl, max_batch=cfg.batch)
        out.append((dl, L))
    torch.cuda.synchronize()
    return out


def run_ours(args, cfg, world, rank, local):
    import torch
    import activation_sparse_ffn_predictor_b200 as sp
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    dist_init(world, "nccl")
    L = cfg.layers
    stack = build_stack(cfg, L, device, rate=args.rate)
    layers = [s[1] for s in stack]
    B, K, W = cfg.batch, args.steps, args.warmup
    seed = rank_seed(rank)
    dt = torch.bfloat16 if cfg.bf16 else torch.float16
    xs = torch.stack([wl.to_torch(wl.tokens(cfg, B, aux=s, seed=seed), cfg, device) for s in range(K + W)])
    x_in = torch.empty(B, cfg.d, dtype=dt, device=device)
    x_out = torch.empty(B, cfg.d, dtype=dt, device=device)
    y = torch.empty(B, cfg.d, dtype=torch.float32, device=device)
    counts = torch.zeros(L, dtype=torch.int32, device=device)
    hist = torch.zeros(K + W, L, dtype=torch.int32, device=device)
    stream = torch.cuda.Stream(device)

    sp.set_l2_hot_rows(args.l2_hot_rows)
    sp.set_union_stack(args.union_stack)

    def one_step():
        sp.decode(layers, x_in, x_out, y, counts, stream=stream, lookahead=args.lookahead)

    # CUDA graph of one decode step (removes host launch cost from the timed region)
    with torch.cuda.stream(stream):
        one_step()
    stream.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        one_step()
    launches_per_step = sp.decode_kernel_launches(layers, B)

    with torch.cuda.stream(stream):
        for s in range(W):
            x_in.copy_(xs[s])
            g.replay()
            hist[s].copy_(counts)
    stream.synchronize()
    barrier(world, device)
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    flush = torch.empty(FLUSH_BYTES // 4, dtype=torch.float32, device=device) if args.flush_l2 else None
    with Clocks(local) as clk:
        with torch.cuda.stream(stream):
            e0.record(stream)
            for s in range(K):
                x_in.copy_(xs[W + s])
                if flush is not None:
                    flush.fill_(float(s))           # evicts the weights from L2 (outside the step's events)
                ev[s][0].record(stream)
                g.replay()
                ev[s][1].record(stream)
                hist[W + s].copy_(counts)
            e1.record(stream)
        stream.synchronize()
    torch.cuda.synchronize()
    barrier(world, device)
    total_ms = e0.elapsed_time(e1)
    kernel_ms = [a.elapsed_time(b) for a, b in ev]
    # with a flush between steps the time is the steps' own (the flushes are not decode work)
    t_max = max_over_ranks(sum(kernel_ms) if flush is not None else total_ms, world, device)
    del flush
    ks = hist[W:].cpu().numpy()
    bytes_per_step = [step_bytes(cfg, int(ks[s].sum()), L) for s in range(K)]
    peak, peak_kind = measured_peaks()
    mean_launch_ms = sum(kernel_ms) / K
    achieved = (sum(bytes_per_step) / K) / (mean_launch_ms * 1e-3) / 1e9

    # end to end through the public API: each step copies x in from pinned host memory,
    # calls spffn_decode through the binding (argument checks, parameter staging and
    # every launch included) and copies y back to pinned host memory
    xh = torch.empty(K, B, cfg.d, dtype=dt).pin_memory()
    xh.copy_(xs[W:].cpu())
    yh = torch.empty(K, B, cfg.d, dtype=torch.float32).pin_memory()
    del g
    barrier(world, device)
    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        f0.record(stream)
        for s in range(K):
            x_in.copy_(xh[s], non_blocking=True)
            one_step()
            yh[s].copy_(y, non_blocking=True)
        f1.record(stream)
    stream.synchronize()
    e2e_ms = max_over_ranks(f0.elapsed_time(f1), world, device)
    if args.trace and launches_per_step == 1 and B <= 2 and rank == 0:
        # one more eager step with per-CTA, per-layer phase stamps (outside every timed region)
        G = layers[0].num_partials
        M = sp.trace_marks()
        buf = torch.zeros(G * L * M, dtype=torch.int64, device=device)
        sp.set_trace(buf)
        with torch.cuda.stream(stream):
            one_step()
        stream.synchronize()
        sp.set_trace(None)
        print(fused_phase_table(buf.cpu().numpy(), G, L, M), file=sys.stderr, flush=True)
    if args.trace and launches_per_step > 1 and B >= 16 and B <= 128 and rank == 0:
        # one more eager step with per-CTA phase stamps (outside every timed region)
        nl = 4 * L
        G = layers[0].num_partials
        buf = torch.zeros(nl * G * 8, dtype=torch.int64, device=device)
        sp.set_trace(buf)
        with torch.cuda.stream(stream):
            one_step()
        stream.synchronize()
        sp.set_trace(None)
        print(union_phase_table(buf.cpu().numpy(), nl, G), file=sys.stderr, flush=True)

    value = world * B * K / (t_max * 1e-3)
    res = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K, "warmup": W,
        "ms_per_step": t_max / K, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": cfg.dtype, "data": "synthetic",
        "config": config_dict(cfg, args, world),
        "workload_stats": {"mean_active_neurons": float(ks.mean()),
                           "touched_gb_per_step": sum(bytes_per_step) / K / 1e9,
                           "placement_ranges": layers[0].num_partials},
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak,
                     "traffic": (decode_traffic(cfg, L, B, args.rate, args.lookahead) if launches_per_step == 1
                                 else union_traffic(cfg, B, args.rate, args.lookahead, ks.tolist())),
                     "kernel": "spffn decode step (one graph replay per step, %d launch%s)"
                               % (launches_per_step, "" if launches_per_step == 1 else "es"),
                     "peak_kind": peak_kind},
        "e2e": {"value": world * B * K / (e2e_ms * 1e-3), "unit": UNIT,
                "h2d_bytes_per_step": B * cfg.d * 2, "d2h_bytes_per_step": B * cfg.d * 4,
                "path": "spffn_decode through the Python binding each step, pinned host copies in the timed region"},
        "gpu_launches": launches_per_step * K,
        "clocks": clk.summary(),
    }
    return res, (rank == 0)


def union_phase_table(stamps, launches: int, ctas: int) -> str:
    """Phase summary of one traced step of the union path's per-layer launches (four
    tensor-core launches per layer): per mode, the median over layers of the wait for the
    previous kernel, the streaming span (first stage consumed to last MMA issued) and the
    tail (last accumulator read to the last CTA's epilogue end), in microseconds."""
    t = stamps.reshape(launches, ctas, 8).astype(np.float64)
    rows = {m: [] for m in range(4)}
    for i in range(launches):
        m0 = t[i][:, 0]
        if not (m0 > 0).any():
            continue
        start = m0[m0 > 0].min()

        def med(k):
            v = t[i][:, k]
            v = v[v > 0]
            return float(np.median(v)) if v.size else float("nan")

        last5 = t[i][:, 5]
        tail_end = last5[last5 > 0].max() if (last5 > 0).any() else float("nan")
        rows[i % 4].append(((med(1) - start) / 1e3, (med(3) - med(2)) / 1e3, (tail_end - med(4)) / 1e3))
    names = ["mode 0 (predictor hidden)", "mode 1 (logits, compaction)", "mode 2 (FC1)", "mode 3 (FC2)"]
    out = ["%-30s %12s %12s %12s" % ("launch", "wait us", "stream us", "tail us")]
    for m in range(4):
        if rows[m]:
            a = np.median(np.array(rows[m]), axis=0)
            out.append("%-30s %12.1f %12.1f %12.1f" % (names[m], a[0], a[1], a[2]))
    return "\n".join(out)


FUSED_MARKS = {0: "input formed", 1: "first predictor-1 chunk ready", 2: "hidden layer done",
               3: "after barrier 1", 4: "h loaded", 5: "first predictor-2 chunk ready",
               6: "own neuron list final", 7: "first FFN rows ready", 8: "FFN partial written",
               9: "after barrier 2", 10: "reduction and table written", 11: "after barrier 3",
               12: "4th predictor-2 chunk ready", 13: "4th chunk computed", 14: "last predictor-2 chunk ready",
               15: "last chunk computed"}


def fused_phase_table(stamps, ctas: int, layers: int, marks: int) -> str:
    """Phase summary of one traced step of the small-batch whole-stack kernel: per mark,
    the median over layers of the median (and max) over CTAs of the time since the
    layer's earliest "input formed" stamp, and the median layer period, in microseconds."""
    t = stamps.reshape(ctas, layers, marks).astype(np.float64)
    t0 = np.array([t[:, l, 0][t[:, l, 0] > 0].min() if (t[:, l, 0] > 0).any() else np.nan for l in range(layers)])
    out = ["%-32s %10s %10s" % ("mark", "median us", "max us")]
    for m, name in FUSED_MARKS.items():
        med, mx = [], []
        for l in range(1, layers):                      # layer 0 includes the launch
            v = t[:, l, m]
            v = v[v > 0] - t0[l]
            if v.size:
                med.append(np.median(v) / 1e3)
                mx.append(v.max() / 1e3)
        if med:
            out.append("%-32s %10.1f %10.1f" % (name, np.median(med), np.median(mx)))
    per = np.diff(t0[1:]) / 1e3
    if per.size:
        out.append("%-32s %10.1f" % ("layer period", float(np.median(per))))
    return "\n".join(out)


def run_true_mask(args, cfg, world, rank, local):
    """The sparse FFN alone on each token's true activation set (z > 0), no predictor:
    one spffn_decode_tables per step (per layer the FFN over the true table, then
    the chaining).  The tables come
    from an untimed pass of the same deterministic steps (the library's profile
    kernel on one step's layer input gives that input's z > 0 set); the timed
    replays then see exactly the inputs the tables were taken from."""
    import torch
    import activation_sparse_ffn_predictor_b200 as sp
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    dist_init(world, "nccl")
    L = cfg.layers
    B, K, W = cfg.batch, args.steps, args.warmup
    if B >= 16:
        raise SystemExit("--true-mask measures the per-phase FFN kernels: batch < 16")
    stack = build_stack(cfg, L, device, rate=args.rate)
    layers = [s_[1] for s_ in stack]
    seed = rank_seed(rank)
    dt = torch.bfloat16 if cfg.bf16 else torch.float16
    xs = torch.stack([wl.to_torch(wl.tokens(cfg, B, aux=s_, seed=seed), cfg, device) for s_ in range(K + W)])
    xl = torch.empty(L + 1, B, cfg.d, dtype=dt, device=device)
    y = torch.empty(B, cfg.d, dtype=torch.float32, device=device)
    idx = torch.zeros(K + W, L, cfg.n, dtype=torch.int32, device=device)
    cnt = torch.zeros(K + W, L, 1, dtype=torch.int32, device=device)
    prof = torch.zeros(cfg.n, dtype=torch.int32, device=device)
    stream = torch.cuda.Stream(device)

    tabs = [[idx[s_, l] for l in range(L)] for s_ in range(K + W)]
    tcnt = cnt[:, :, 0].contiguous()
    sp.set_l2_hot_rows(args.l2_hot_rows)

    def ffn_step(s_):
        sp.decode_tables(layers, xl[0], tabs[s_], tcnt[s_], xl[L], y, stream=stream)

    graphs = []
    with torch.cuda.stream(stream):
        for s_ in range(K + W):
            xl[0].copy_(xs[s_])
            for l, Ly in enumerate(layers):
                prof.zero_()
                Ly.profile_counts(xl[l], prof, stream=stream)
                sel = torch.nonzero(prof > 0).flatten().to(torch.int32)
                idx[s_, l, :sel.numel()] = sel
                cnt[s_, l, 0] = sel.numel()
                Ly.forward(xl[l], idx[s_, l], cnt[s_, l], y, stream=stream)
                Ly.chain(xl[l], y, xl[l + 1], stream=stream)
    stream.synchronize()
    tcnt = cnt[:, :, 0].contiguous()
    for s_ in range(K + W):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            ffn_step(s_)
        graphs.append(g)
    with torch.cuda.stream(stream):
        for s_ in range(W):
            xl[0].copy_(xs[s_])
            graphs[s_].replay()
    stream.synchronize()
    barrier(world, device)
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with Clocks(local) as clk:
        with torch.cuda.stream(stream):
            e0.record(stream)
            for k in range(K):
                xl[0].copy_(xs[W + k])
                ev[k][0].record(stream)
                graphs[W + k].replay()
                ev[k][1].record(stream)
            e1.record(stream)
        stream.synchronize()
    torch.cuda.synchronize()
    barrier(world, device)
    t_max = max_over_ranks(e0.elapsed_time(e1), world, device)
    ks = cnt[W:, :, 0].cpu().numpy()
    bytes_per_step = [int(ks[k].sum()) * ffn_bytes_per_neuron(cfg) for k in range(K)]
    mean_launch_ms = sum(a.elapsed_time(b) for a, b in ev) / K
    achieved = (sum(bytes_per_step) / K) / (mean_launch_ms * 1e-3) / 1e9
    peak, peak_kind = measured_peaks()
    # end to end: pinned host x in, the last layer's y out, every step
    xh = torch.empty(K, B, cfg.d, dtype=dt).pin_memory()
    xh.copy_(xs[W:].cpu())
    yh = torch.empty(K, B, cfg.d, dtype=torch.float32).pin_memory()
    barrier(world, device)
    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        f0.record(stream)
        for k in range(K):
            xl[0].copy_(xh[k], non_blocking=True)
            graphs[W + k].replay()
            yh[k].copy_(y, non_blocking=True)
        f1.record(stream)
    stream.synchronize()
    e2e_ms = max_over_ranks(f0.elapsed_time(f1), world, device)
    del graphs
    rate = args.rate or cfg.rate
    res = {
        "metric": METRIC, "value": world * B * K / (t_max * 1e-3), "unit": UNIT, "n_gpus": world, "steps": K,
        "warmup": W, "ms_per_step": t_max / K, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": cfg.dtype, "data": "synthetic",
        "config": {"workload": "%s-truemask-r%g" % (cfg.name, rate), "layers": L, "d": cfg.d, "n": cfg.n,
                   "batch": B, "activation_rate": rate, "alpha": cfg.alpha, "global_batch": B * world,
                   "mean_active_neurons": float(ks.mean()), "parallelism": "replicas%d" % world,
                   "prediction": "none: each token's true activation set (z > 0), taken before timing",
                   "l2": "%.2f GB touched per step" % (sum(bytes_per_step) / K / 1e9)},
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                     "traffic": None, "kernel": "spffn_decode_tables (one graph per step)", "peak_kind": peak_kind},
        "e2e": {"value": world * B * K / (e2e_ms * 1e-3), "unit": UNIT, "h2d_bytes_per_step": B * cfg.d * 2,
                "d2h_bytes_per_step": B * cfg.d * 4},
        # the persistent kernel at B <= 2 (d <= 10240): one launch per step; else FFN + reduction + chaining per layer
        "gpu_launches": (1 if B <= 2 and cfg.d <= 10240 else 3 * L) * K,
        "clocks": clk.summary(),
    }
    return res, (rank == 0)


def dense_layer(dl, x):
    """One layer's dense FFN with cuBLAS: y = W2T^T ReLU(W1 x + b1) (fp16 GEMM
    outputs, fp32 accumulation inside cuBLAS), returned in fp32."""
    import torch
    a = torch.relu(torch.addmm(dl.b1, x, dl.W1.t()))
    return torch.mm(a, dl.W2T).float()


def dense_stack(dls, x, dt):
    """x through every layer's dense FFN and the chaining x' = (x + y) / rms(x + y)."""
    import torch
    for dl in dls:
        u = x.float() + dense_layer(dl, x)
        x = (u * torch.rsqrt(u.square().mean(dim=-1, keepdim=True) + 1e-6)).to(dt)
    return x


def run_dense(args, cfg, world, rank, local):
    """Comparison arm, not the product path: the dense FFN of every layer on the
    same weights with cuBLAS GEMMs (dense_layer), ReLU and the same chaining in
    plain torch ops, one CUDA graph per step.  It
    shows what the predictor and the sparse FFN save over computing every
    neuron."""
    import torch
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    dist_init(world, "nccl")
    L = cfg.layers
    B, K, W = cfg.batch, args.steps, args.warmup
    stack = build_stack(cfg, L, device, rate=args.rate, reorder=False)
    dls = [s_[0] for s_ in stack]
    dt = torch.bfloat16 if cfg.bf16 else torch.float16
    seed = rank_seed(rank)
    xs = torch.stack([wl.to_torch(wl.tokens(cfg, B, aux=s_, seed=seed), cfg, device) for s_ in range(K + W)])
    x_in = torch.empty(B, cfg.d, dtype=dt, device=device)
    out = {}
    stream = torch.cuda.Stream(device)

    def one_step():
        out["x"] = dense_stack(dls, x_in, dt)

    with torch.cuda.stream(stream):
        x_in.copy_(xs[0])
        one_step()
    stream.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        one_step()
    with torch.cuda.stream(stream):
        for s_ in range(W):
            x_in.copy_(xs[s_])
            g.replay()
    stream.synchronize()
    barrier(world, device)
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with Clocks(local) as clk:
        with torch.cuda.stream(stream):
            e0.record(stream)
            for k in range(K):
                x_in.copy_(xs[W + k])
                ev[k][0].record(stream)
                g.replay()
                ev[k][1].record(stream)
            e1.record(stream)
        stream.synchronize()
    torch.cuda.synchronize()
    barrier(world, device)
    t_max = max_over_ranks(e0.elapsed_time(e1), world, device)
    del g
    mean_ms = sum(a_.elapsed_time(b_) for a_, b_ in ev) / K
    achieved = L * dense_bytes_per_layer(cfg) / (mean_ms * 1e-3) / 1e9
    peak, peak_kind = measured_peaks()
    res = {
        "metric": METRIC, "value": world * B * K / (t_max * 1e-3), "unit": UNIT, "n_gpus": world, "steps": K,
        "warmup": W, "ms_per_step": t_max / K, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": cfg.dtype, "data": "synthetic", "impl": "dense-cublas",
        "config": {"workload": cfg.name + "-dense", "layers": L, "d": cfg.d, "n": cfg.n, "batch": B,
                   "global_batch": B * world, "parallelism": "replicas%d" % world,
                   "prediction": "none: every neuron computed (dense FFN, torch/cuBLAS)",
                   "l2": "inputs larger than L2 (%.2f GB of FFN weights per step)" % (L * dense_bytes_per_layer(cfg) / 1e9)},
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                     "traffic": None, "kernel": "cuBLAS GEMMs + torch elementwise (one graph per step)",
                     "peak_kind": peak_kind},
        "gpu_launches": 0,
        "clocks": clk.summary(),
    }
    return res, (rank == 0)


# ---------------------------------------------------------------------------
# head-sparse attention with the attention-head predictor (DejaVu's SP_A)
ATTN_METRIC = "head-sparse attention decode tokens/s per layer-stack"


def attn_step_bytes(acfg, count: int, t: int) -> int:
    """Bytes one layer's step touches: the head predictor, the selected heads'
    Wq/Wk/Wv/Wo rows, their cached K/V rows at positions 0..t, and the stored token."""
    pred = 2 * (acfg.Ha * acfg.d + acfg.nh * acfg.Ha) + 2 * acfg.nh
    per_head = 4 * acfg.dh * acfg.d * 2 + 2 * (t + 1) * acfg.dh * 2
    return pred + count * per_head + acfg.d * 2


def run_attn(args, world, rank, local):
    """Each step runs every layer's head-sparse attention on the step's token (the
    layers are independent here: the FFN between them is the other benchmark).
    Every layer's cache is first filled with ``context`` tokens by the same kernels
    (untimed), so the timed steps see the lazily filled caches decode reaches."""
    import torch
    import activation_sparse_ffn_predictor_b200 as sp
    acfg = wl.ATTN_CONFIGS[args.attn_config]
    if args.layers:
        acfg = acfg.with_(layers=args.layers)
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    dist_init(world, "nccl")
    L, K, W = acfg.layers, args.steps, args.warmup
    dt = torch.bfloat16 if acfg.bf16 else torch.float16
    assert acfg.context + 1 + W + 2 * K <= acfg.tmax, "cache too small for the run"
    layers = []
    for l in range(L):
        da = wl.device_attn(acfg, l, device=device)
        layers.append((da, sp.AttnLayer(da.Wq, da.Wk, da.Wv, da.WoT, da.Wa1, da.Wa2, nh=acfg.nh, tmax=acfg.tmax,
                                        ba2=da.ba2)))
    steps_total = acfg.context + 1 + W + 2 * K
    toks = torch.empty(steps_total, acfg.d, dtype=dt, device=device)
    wl.device_fill(toks, wl.stream_id(wl.T_XA, 0, 1000 + rank), 1.0, acfg.bf16)
    y_in = torch.empty(acfg.d, dtype=dt, device=device)
    heads = torch.zeros(L, acfg.nh, dtype=torch.int32, device=device)
    count = torch.zeros(L, 1, dtype=torch.int32, device=device)
    out = torch.empty(L, acfg.d, dtype=torch.float32, device=device)
    stream = torch.cuda.Stream(device)

    def one_step():
        for l, (_, A) in enumerate(layers):
            A.step(y_in, heads[l], count[l], out[l], stream=stream)

    pos = 0
    with torch.cuda.stream(stream):
        y_in.copy_(toks[pos]); pos += 1
        one_step()
    stream.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        one_step()
    with torch.cuda.stream(stream):
        for _ in range(acfg.context - 1 + W):           # fill the caches, then warm up
            y_in.copy_(toks[pos]); pos += 1
            g.replay()
    stream.synchronize()
    barrier(world, device)
    torch.cuda.synchronize()
    t0 = pos
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    hist = torch.zeros(K, L, dtype=torch.int32, device=device)
    with Clocks(local) as clk:
        with torch.cuda.stream(stream):
            e0 = torch.cuda.Event(enable_timing=True); e1 = torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            for k in range(K):
                y_in.copy_(toks[pos]); pos += 1
                ev[k][0].record(stream)
                g.replay()
                ev[k][1].record(stream)
                hist[k].copy_(count[:, 0])
            e1.record(stream)
        stream.synchronize()
    torch.cuda.synchronize()
    barrier(world, device)
    t_max = max_over_ranks(e0.elapsed_time(e1), world, device)
    kernel_ms = sum(a.elapsed_time(b) for a, b in ev) / K
    cnt = hist.cpu().numpy()
    bytes_per_step = [sum(attn_step_bytes(acfg, int(cnt[k, l]), t0 + k) for l in range(L)) for k in range(K)]
    achieved = (sum(bytes_per_step) / K) / (kernel_ms * 1e-3) / 1e9
    peak, peak_kind = measured_peaks()
    dense = L * (2 * (4 * acfg.nh * acfg.dh * acfg.d) + 2 * 2 * (t0 + K) * acfg.nh * acfg.dh)
    # end to end: token in from pinned host memory, every layer through the binding, out back
    del g
    yh = torch.empty(K, acfg.d, dtype=dt).pin_memory()
    yh.copy_(toks[pos:pos + K].cpu())
    oh = torch.empty(K, acfg.d, dtype=torch.float32).pin_memory()
    barrier(world, device)
    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        f0.record(stream)
        for k in range(K):
            y_in.copy_(yh[k], non_blocking=True)
            one_step()
            oh[k].copy_(out[L - 1], non_blocking=True)
        f1.record(stream)
    stream.synchronize()
    e2e_ms = max_over_ranks(f0.elapsed_time(f1), world, device)
    res = {
        "metric": ATTN_METRIC, "value": world * K / (t_max * 1e-3), "unit": UNIT, "n_gpus": world, "steps": K,
        "warmup": W, "ms_per_step": t_max / K, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": acfg.dtype, "data": "synthetic", "impl": "head-sparse-attention",
        "config": {"workload": acfg.name, "layers": L, "d": acfg.d, "heads": acfg.nh, "head_dim": acfg.dh,
                   "predictor_hidden": acfg.Ha, "head_rate": acfg.rate, "context_tokens": t0,
                   "batch": 1, "parallelism": "replicas%d" % world,
                   "l2": "inputs larger than L2 (%.2f GB touched per step)" % (sum(bytes_per_step) / K / 1e9)},
        "workload_stats": {"mean_selected_heads": float(cnt.mean()),
                           "dense_attention_gb_per_step": dense / 1e9},
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                     "traffic": None, "kernel": "spffn_attn_step x %d layers (one graph replay per step, %d launches)"
                     % (L, L * sp.attn_step_kernel_launches()), "peak_kind": peak_kind},
        "e2e": {"value": world * K / (e2e_ms * 1e-3), "unit": UNIT, "h2d_bytes_per_step": acfg.d * 2,
                "d2h_bytes_per_step": acfg.d * 4,
                "path": "spffn_attn_step through the binding for every layer, pinned host copies in the timed region"},
        "gpu_launches": L * sp.attn_step_kernel_launches() * K,
        "clocks": clk.summary(),
    }
    return res, (rank == 0)


# ---------------------------------------------------------------------------
def cpu_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return len(os.sched_getaffinity(0))


class OracleSampler:
    """Times the CPU oracle on (layer, step) samples of the workload: the first
    two layers' predictors are generated once and kept, then each sample draws a
    fresh batch of tokens, regenerates the FFN rows its table names (untimed) and
    times the oracle's predict + sparse FFN.  The rate is extrapolated to the
    whole stack (tokens/s per layer stack)."""

    def __init__(self, cfg, rate=None, seed=1):
        self.cfg, self.seed, self.s = cfg, seed, 0
        bf = cfg.bf16
        self.prepared = []
        for l in range(min(2, cfg.layers)):
            p, Wp1, bp1, Wp2, bp2 = wl.host_predictor(cfg, l, rate=rate)
            self.prepared.append((l, wl.widen(Wp1, bf), wl.widen(bp1, bf), wl.widen(Wp2, bf), wl.widen(bp2, bf),
                                  wl.widen(wl.fc1_bias(p, bf), bf)))

    def run(self, budget_s: float, threads=None):
        """Samples until `budget_s` of oracle compute is spent (at least one);
        `threads` caps the BLAS thread pool (None: all it has)."""
        import contextlib
        import oracle as O
        cfg = self.cfg
        ctx = contextlib.nullcontext()
        if threads is not None:
            from threadpoolctl import threadpool_limits
            ctx = threadpool_limits(limits=threads, user_api="blas")
        spent, samples = 0.0, 0
        with ctx:
            while (spent < budget_s or samples == 0) and samples < 10000:
                l, Wp1, bp1, Wp2, bp2, b1 = self.prepared[self.s % len(self.prepared)]
                x64 = wl.widen(wl.tokens(cfg, cfg.batch, aux=self.s, seed=self.seed), cfg.bf16)
                idx, k, _ = O.predict(Wp1, Wp2, bp2, x64, bp1)
                sc = 1.0 / math.sqrt(cfg.d)
                W1 = wl.widen(wl.fill_rows(wl.stream_id(wl.T_W1, l), cfg.d, idx, sc, cfg.bf16), cfg.bf16)
                W2T = wl.widen(wl.fill_rows(wl.stream_id(wl.T_W2T, l), cfg.d, idx, sc, cfg.bf16), cfg.bf16)
                t0 = time.perf_counter()
                idx, k, _ = O.predict(Wp1, Wp2, bp2, x64, bp1)
                O.sparse_ffn(W1, b1, W2T, None, x64, idx, row_ids=idx)
                spent += time.perf_counter() - t0
                samples += 1
                self.s += 1
        tok_s = cfg.batch / (spent / samples * cfg.layers)
        return tok_s, samples, spent


def cpu_baseline(cfg, budget_s: float, rate=None):
    """The oracle timed on all host cores (BLAS threads) and on one thread, on
    bounded samples of the workload; returns the JSON object."""
    sampler = OracleSampler(cfg, rate=rate)
    v_all, n_all, t_all = sampler.run(budget_s)
    v_one, n_one, t_one = sampler.run(budget_s, threads=1)
    return {"value": v_all, "unit": UNIT, "cores": cpu_threads(), "kind": "oracle",
            "sample": "%d (layer, step) samples of the first 2 layers, %.1f s of oracle compute, extrapolated "
                      "to %d layers" % (n_all, t_all, cfg.layers),
            "single_thread": {"value": v_one, "unit": UNIT, "cores": 1,
                              "sample": "%d samples, %.1f s of oracle compute" % (n_one, t_one)}}


def run_reference(args, cfg, world, rank, local):
    """The oracle as it stands on the host cores, same workload, bounded samples per step."""
    if rank != 0:
        return None, False
    K, W = args.steps, args.warmup
    per_step_budget = max(0.5, min(10.0, args.ref_budget / max(1, K + W)))
    sampler = OracleSampler(cfg, rate=args.rate)
    for _ in range(W):
        sampler.run(per_step_budget * 0.2)
    vals, spent, samples = [], 0.0, 0
    for _ in range(K):
        v, n_s, sp_ = sampler.run(per_step_budget)
        vals.append(v)
        spent += sp_
        samples += n_s
    value = statistics.mean(vals)
    v_one, n_one, t_one = sampler.run(per_step_budget, threads=1)
    cores = cpu_threads()
    ms = cfg.batch / value * 1e3
    res = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K, "warmup": W,
        "ms_per_step": ms, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f64", "data": "synthetic", "impl": "reference",
        "config": config_dict(cfg, args, world),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": "%d (layer, step) samples of the first 2 layers, %.1f s of oracle compute, "
                                   "extrapolated to %d layers" % (samples, spent, cfg.layers),
                         "single_thread": {"value": v_one, "unit": UNIT, "cores": 1,
                                           "sample": "%d samples, %.1f s of oracle compute" % (n_one, t_one)}},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    return res, True


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--config", type=int, default=4)
    ap.add_argument("--rate", type=float, default=None)
    ap.add_argument("--batch", type=int, default=None)
    ap.add_argument("--layers", type=int, default=None)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--cpu-budget", type=float, default=10.0,
                    help="seconds of oracle compute for each cpu_baseline leg (all cores, one thread)")
    ap.add_argument("--ref-budget", type=float, default=60.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--l2-hot-rows", type=int, default=0,
                    help="keep this many of the hottest slots of every dealt range in L2 (B <= 2 decode)")
    ap.add_argument("--union-stack", type=int, choices=[0, 1, 2], default=2,
                    help="decode 3 <= B <= 128: 0 per-layer launches, 1 one whole-stack launch, 2 (default) "
                         "the faster on the measured shapes (per-layer)")
    ap.add_argument("--flush-l2", action="store_true",
                    help="write a buffer larger than L2 before every timed step (for workloads that fit in L2)")
    ap.add_argument("--lookahead", action="store_true",
                    help="predict layer l+1's neuron set from layer l's input (DejaVu look-ahead)")
    ap.add_argument("--true-mask", action="store_true",
                    help="time the sparse FFN alone on each token's true activation set (no predictor)")
    ap.add_argument("--attn", action="store_true",
                    help="head-sparse attention decode with the attention-head predictor (its own metric)")
    ap.add_argument("--attn-config", type=int, default=1)
    ap.add_argument("--trace", action="store_true",
                    help="after the timed runs, print a phase table of one traced step to stderr (the "
                         "small-batch whole-stack kernel, or the union path's per-layer launches)")
    ap.add_argument("--dense", action="store_true",
                    help="comparison arm: the dense FFN of every layer with cuBLAS on the same weights")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    cfg = wl.CONFIGS[args.config]
    if args.batch:
        cfg = cfg.with_(batch=args.batch)
    if args.layers:
        cfg = cfg.with_(layers=args.layers)
    world, rank, local = dist_env()
    if args.impl == "reference":
        res, show = run_reference(args, cfg, world, rank, local)
    elif args.attn:
        res, show = run_attn(args, world, rank, local)
    elif args.true_mask:
        res, show = run_true_mask(args, cfg, world, rank, local)
    elif args.dense:
        res, show = run_dense(args, cfg, world, rank, local)
    else:
        res, show = run_ours(args, cfg, world, rank, local)
        if show and world == 1 and not args.no_cpu_baseline:
            res["cpu_baseline"] = cpu_baseline(cfg, args.cpu_budget, rate=args.rate)
    if show and res is not None:
        print(json.dumps(res), flush=True)
    if world > 1:
        import torch.distributed as dist
        if dist.is_initialized():
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
