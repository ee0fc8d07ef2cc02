#!/usr/bin/env python
"""Decode benchmark of the CSA/HCA attention operator on B200.

A step is one decode token through one CSA layer (m=4, top-k 1024) and one HCA
layer (m'=128) at 1,048,576 tokens of context, batch 1, 128 query heads, KV
dim 512 stored as BF16 rotary dims + FP8 remainder, indexer 32 x 128 FP8: the
whole hot path (append + compress, indexer scores, top-k, sparse attention;
append + compress, dense attention) through the C ABI's fused decode calls.

Timing: W untimed warm-up steps, then exactly K steps bracketed by a barrier
and a device synchronisation, timed with CUDA events on the launching stream,
max over ranks.  Each step runs on the next of R independent layer instances
(caches at distinct addresses), so a step never finds its keys in L2 (R=8:
>= 280 MB streamed between two uses of one instance vs 126 MB of L2).
Steps are CUDA-graph replays of the public API calls; the only event nodes in
the timed graphs bracket one indexer launch per cycle (the roofline sample).

`value` = tokens x attention layers processed by all ranks / time (tok/s per
attention layer).  `e2e` repeats the measurement with each step's inputs
copied host->device from pinned memory and its outputs copied back.
`--impl reference` times the CPU oracle on the same workload instead.
"""

import argparse
import hashlib
import json
import os
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "decode tok/s per attention layer at 1M ctx (CSA top-k 1024 + HCA m'=128, interleaved)"
UNIT = "tok/s"


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=200)
    p.add_argument("--warmup", type=int, default=10)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--workload", default="csa_hca_decode_1m",
                   choices=["csa_hca_decode_1m", "csa_decode_128k", "hca_decode_128k", "csa_prefill_8k"])
    p.add_argument("--replicas", type=int, default=8)
    p.add_argument("--cpu-seconds", type=float, default=10.0, help="CPU-baseline sample budget")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-extra-configs", action="store_true", help="skip the 128K configurations' lines")
    p.add_argument("--prefill-queries", type=int, default=None,
                   help="chunk size of --workload csa_prefill_8k (default: the workload's 8,192)")
    p.add_argument("--burn-seconds", type=float, default=0.5, help="untimed replays before timing (clocks settle)")
    return p.parse_args()


def workload_config(wl, replicas):
    layers = []
    for L in wl.layers:
        if L.kind == "csa":
            layers.append(f"csa m={L.m} overlap={L.ov} top-k={L.top_k} indexer {L.H_I}x{L.d_I} {L.idx_format}")
        else:
            layers.append(f"hca m'={L.m}")
    return {"workload": wl.name, "batch": wl.B, "context": wl.n, "layers": layers, "heads": wl.layers[0].H,
            "kv_dim": wl.layers[0].D, "kv_format": wl.layers[0].kv_format, "window": wl.layers[0].window,
            "l2": f"rotating {replicas} layer instances (inputs larger than L2)"}


# ----------------------------------------------------------------------------- algorithmic bytes

def index_kernel_bytes(layer, n_vis, B):
    """Algorithmic bytes of one indexer-score launch: keys + key scales read, scores written, queries
    (FP4 keys: d_I / 2 bytes of codes and a 4-byte scale word)."""
    per_entry = (layer.d_I // 2 if layer.idx_format == "e2m1" else layer.d_I) + 4 + 4
    per_query = layer.H_I * layer.d_I + 2 * 4 * layer.H_I
    return B * (n_vis * per_entry + per_query)


def step_bytes(layer, n, B):
    """Algorithmic HBM bytes of one decode step of a layer (per sequence x B)."""
    rb = {"f32": 4 * layer.D, "bf16": 2 * layer.D, "mixed": layer.D + 68}[layer.kv_format]
    ab = 4 if layer.act_format == "f32" else 2
    nv = n // layer.m
    w = min(layer.window, n)
    qo = 2 * layer.H * layer.D * ab
    if layer.kind == "csa":
        kb = layer.d_I // 2 if layer.idx_format == "e2m1" else layer.d_I
        idx = nv * (kb + 4 + 4) + layer.H_I * layer.d_I
        att = (min(layer.top_k, nv) + w) * rb
        return B * (idx + att + qo)
    return B * ((nv + w) * rb + qo)


# ----------------------------------------------------------------------------- clocks

class ClockSampler:
    """Polls NVML SM clock and clock-event reasons on a thread."""

    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
               0x10: "sync_boost", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
               0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting"}

    def __init__(self, index):
        self.samples = []
        self.ok = False
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # noqa: BLE001
            self.err = str(e)
        self._stop = threading.Event()

    def sample(self):
        if not self.ok:
            return
        nv = self.nv
        try:
            mhz = nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM)
            try:
                r = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
            except Exception:  # noqa: BLE001
                r = nv.nvmlDeviceGetCurrentClocksThrottleReasons(self.h)
            self.samples.append((time.perf_counter(), mhz, r))
        except Exception:  # noqa: BLE001
            pass

    def _run(self):
        while not self._stop.is_set():
            self.sample()
            time.sleep(0.005)

    def start(self):
        self.t = threading.Thread(target=self._run, daemon=True)
        self.t.start()

    def stop(self):
        self._stop.set()
        if hasattr(self, "t"):
            self.t.join()

    def summary(self, t0, t1):
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "note": getattr(self, "err", "no samples")}
        inside = [s for s in self.samples if t0 <= s[0] <= t1]
        if not inside:   # timed region shorter than one poll: nearest samples around it
            inside = sorted(self.samples, key=lambda s: min(abs(s[0] - t0), abs(s[0] - t1)))[:4]
        mhz = [s[1] for s in inside]
        bits = 0
        for s in inside:
            bits |= s[2]
        reasons = [name for b, name in self.REASONS.items() if bits & b and name != "gpu_idle"]
        return {"sm_mhz": float(np.median(mhz)), "sm_max_mhz": float(self.max_mhz), "reasons": reasons,
                "samples": len(inside)}


# ----------------------------------------------------------------------------- CPU oracle

def oracle_step(oracle_layers, datas):
    from oracle import csa as O
    outs = []
    for L, d in zip(oracle_layers, datas):
        for b in range(len(d["t"])):
            outs.append(O.decode_step(L, d, b)["o"])
    return outs


def cpu_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info()]
        return int(max(n)) if n else 1
    except Exception:  # noqa: BLE001
        return os.cpu_count() or 1


def run_cpu_oracle(wl, datas, budget_s, min_steps=1, max_steps=None):
    from oracle import csa as O
    Ls = [O.LayerSpec.of(L) for L in wl.layers]
    times = []
    t_all = time.perf_counter()
    while True:
        t0 = time.perf_counter()
        oracle_step(Ls, datas)
        times.append(time.perf_counter() - t0)
        if max_steps is not None and len(times) >= max_steps:
            break
        if len(times) >= min_steps and time.perf_counter() - t_all >= budget_s:
            break
    return times


def cpu_baseline(wl, datas, budget_s):
    """The oracle timed on the host cores on whole decode steps of the workload: with every BLAS
    thread (`value`, `cores`) and single-threaded (`single_thread`), each for about half the budget."""
    units = wl.B * len(wl.layers)
    times = run_cpu_oracle(wl, datas, budget_s / 2)
    line = {"value": units / float(np.mean(times)), "unit": UNIT, "cores": cpu_threads(), "kind": "oracle",
            "sample": f"{len(times)} full decode steps of the workload ({budget_s / 2:.0f} s budget per mode)"}
    try:
        from threadpoolctl import threadpool_limits
        with threadpool_limits(limits=1):
            t1 = run_cpu_oracle(wl, datas, budget_s / 2)
        line["single_thread"] = {"value": units / float(np.mean(t1)), "cores": 1, "steps": len(t1)}
    except Exception as e:  # noqa: BLE001
        line["single_thread"] = {"value": None, "note": f"thread limit unavailable: {e}"}
    return line


# ----------------------------------------------------------------------------- reference arm

def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    from csa_synth import decode_inputs, get_workload
    wl = get_workload(args.workload)
    datas = [decode_inputs(wl, li) for li in range(len(wl.layers))]
    from oracle import csa as O
    Ls = [O.LayerSpec.of(L) for L in wl.layers]
    for _ in range(args.warmup):
        oracle_step(Ls, datas)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle_step(Ls, datas)
    T = time.perf_counter() - t0
    units = wl.B * len(wl.layers) * args.steps
    value = units / T
    cores = cpu_threads()
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * T / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": workload_config(wl, 1),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                             "sample": f"{args.steps} full decode steps (every layer, every sequence) of the workload"},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------------- multi-rank plumbing

def max_over_ranks(x, world, dist=None, device=None):
    """Maximum of a per-rank float over all ranks (the slowest rank's time); identity at world 1."""
    if world == 1:
        return x
    import torch
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_value(units_per_rank, world, T_ms):
    """Whole-job throughput under weak scaling: every rank processes units_per_rank units (its own
    replicas, no data-path exchange), so the job's units over the slowest rank's time."""
    return units_per_rank * world / (T_ms / 1e3)


# ----------------------------------------------------------------------------- our arm

def _code_only(text):
    """Source text without comments or blank lines, so a comment edit does not change the hash."""
    import re
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    lines = [re.sub(r"//.*$", "", ln).rstrip() for ln in text.splitlines()]
    return "\n".join(ln for ln in lines if ln)


def sha_of(paths):
    """Hash of the kernel sources' code (comments excluded)."""
    h = hashlib.sha256()
    for p in paths:
        with open(os.path.join(ROOT, p), encoding="utf-8") as f:
            h.update(_code_only(f.read()).encode())
    return h.hexdigest()[:16]


INDEX_KERNEL_SOURCES = ["long_context_sparse_csa_b200/csrc/index_score.cu", "long_context_sparse_csa_b200/csrc/sm100.cuh",
                        "long_context_sparse_csa_b200/csrc/common.cuh", "long_context_sparse_csa_b200/csrc/kernels.h",
                        "long_context_sparse_csa_b200/csrc/api.cu"]


def recorded_traffic(workload):
    """DRAM bytes per launch of the indexer kernel from the committed ncu summary, if it is current."""
    p = os.path.join(ROOT, "profiles", "index_score_tc_traffic.json")
    try:
        with open(p) as f:
            rec = json.load(f)
    except OSError:
        return None
    if rec.get("kernel_sha") != sha_of(INDEX_KERNEL_SOURCES):
        return None
    return rec.get("per_launch_bytes", {}).get(workload)


class DecodeRig:
    """Device state of one decode workload: R independent instances of every layer's caches (at
    distinct addresses, so consecutive steps stream different bytes), the step inputs, one
    workspace per layer, and CUDA graphs of whole steps through the C ABI's fused decode calls."""

    def __init__(self, wl, R, dev, indexed=False):
        import torch
        from csa_synth import decode_inputs
        from long_context_sparse_csa_b200 import binding as C
        from long_context_sparse_csa_b200.state import LayerState, to_device
        self.wl, self.R, self.dev, self.indexed = wl, R, dev, indexed
        self.datas, self.layers = [], []
        for li, spec in enumerate(wl.layers):
            d = decode_inputs(wl, li, indexed=indexed and spec.kind == "csa")
            self.datas.append(d)
            base = LayerState.from_arrays(spec, wl.B, d, device=dev)
            insts = [base]
            for _ in range(R - 1):
                insts.append(LayerState(spec, wl.B, 0, entries=base.entries.clone(), window=base.window.clone(),
                                        raw=base.raw.clone(), gate=base.gate.clone(),
                                        idx_keys=None if base.idx_keys is None else base.idx_keys.clone(),
                                        idx_key_scale=None if base.idx_key_scale is None else base.idx_key_scale.clone(),
                                        pos_bias=base.pos_bias, gamma_kv=base.gamma_kv, gamma_q=base.gamma_q,
                                        sinks=base.sinks))
            cap = d["entries"].shape[1]
            io = {k: to_device(d[k], dev) for k in ["q", "x_new", "g_new", "t"]}
            if spec.kind == "csa":
                for k in ["idx_q", "idx_q_scale", "head_w"]:
                    io[k] = to_device(d[k], dev)
                io["topk"] = torch.zeros((wl.B, spec.top_k), dtype=torch.int32, device=dev)
            io["out"] = torch.zeros((wl.B, spec.H, spec.D),
                                    dtype=torch.int16 if spec.act_format == "bf16" else torch.float32, device=dev)
            ix = indexed and spec.kind == "csa"
            ws = base.workspace("decode_step_indexed" if ix else "decode_step", 1, cap)
            lay = {"spec": spec, "insts": insts, "io": io, "ws": ws, "indexed": ix,
                   "caches": [s.cache() for s in insts], "params": base.params(), "L": base.L}
            if ix:
                # the index side made in the step: index-key stream rings per instance, latent and weights
                for k in ["c_q", "W_iq", "idx_x_new", "idx_g_new"]:
                    io[k] = to_device(d[k], dev)
                bias = to_device(np.asarray(d["idx_pos_bias"], np.float32), dev)
                lay["rings"] = [(to_device(d["idx_raw_ring"], dev), to_device(d["idx_gate_ring"], dev), bias)
                                for _ in range(R)]
                lay["streams"] = [C.make_index_stream(*rg) for rg in lay["rings"]]
            self.layers.append(lay)
        self.stream = torch.cuda.Stream(device=dev)

    def call(self, li, r):
        """The public decode call of layer li on instance r (eager or under capture)."""
        from long_context_sparse_csa_b200 import binding as C
        lay = self.layers[li]
        io, spec = lay["io"], lay["spec"]
        if spec.kind == "csa" and lay["indexed"]:
            C.csa_decode_step_indexed(lay["L"], lay["caches"][r], lay["params"], lay["streams"][r], io["q"],
                                      io["c_q"], io["W_iq"], spec.idx_rank, io["head_w"], io["x_new"], io["g_new"],
                                      io["idx_x_new"], io["idx_g_new"], io["t"], io["out"], io["topk"], lay["ws"])
        elif spec.kind == "csa":
            C.csa_decode_step(lay["L"], lay["caches"][r], lay["params"], io["q"], io["idx_q"], io["idx_q_scale"],
                              io["head_w"], io["x_new"], io["g_new"], io["t"], io["out"], io["topk"], lay["ws"])
        else:
            C.hca_decode_step(lay["L"], lay["caches"][r], lay["params"], io["q"], io["x_new"], io["g_new"],
                              io["t"], io["out"], lay["ws"])

    def warm(self):
        """Eager steps of every instance (module load, attributes, the second stream), then a check
        of every layer's device error word."""
        import torch
        from long_context_sparse_csa_b200 import binding as C
        for r in range(self.R):
            for li in range(len(self.layers)):
                self.call(li, r)
        torch.cuda.synchronize()
        for lay in self.layers:
            assert C.csa_device_error(lay["ws"]) == 0

    def capture(self, rs, lis, idx_events=False):
        """One CUDA graph running steps of instances rs (layers lis of each, in order).  With
        idx_events, a pair of events brackets the indexer-score launch of the first step (the only
        event nodes: each one breaks the chain of kernel nodes and costs a few microseconds)."""
        import torch
        from long_context_sparse_csa_b200 import binding as C
        pair = None
        if idx_events:
            pair = (_ext_event(), _ext_event())
            for x in pair:
                x.record()
            torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        n0 = C.csa_launch_count()
        with torch.cuda.graph(g, stream=self.stream):
            for j, r in enumerate(rs):
                for li in lis:
                    csa = self.layers[li]["spec"].kind == "csa"
                    if idx_events and j == 0 and csa:
                        C.csa_profile_events(*pair)
                    self.call(li, r)
                    C.csa_profile_events(None, None)
        return g, pair, C.csa_launch_count() - n0

    def graphs(self, lis, steps, idx_events=False):
        """(cycle graphs, single-step graphs, launches per step) for layers lis: n_cyc copies of the
        cycle over the R instances, replayed round-robin (the last replay of each copy lies in the
        timed region, so its event pair samples one indexer launch of the timed steps)."""
        n_cyc = max(1, min(8, steps // self.R))
        cycles = [self.capture(list(range(self.R)), lis, idx_events) for _ in range(n_cyc)]
        singles = [self.capture([r], lis)[0] for r in range(self.R)]
        return cycles, singles, cycles[0][2] // self.R


def _ext_event():
    import torch
    return torch.cuda.Event(enable_timing=True, external=True)


def run_steps(cycles, singles, R, k):
    """Exactly k decode steps: whole cycles of the R instances, then single steps."""
    for c in range(k // R):
        cycles[c % len(cycles)][0].replay()
    for r in range(k % R):
        singles[r].replay()


def timed(fn, world, dist, dev):
    """Device time (ms) of fn() on the current stream, bracketed by a barrier and a device
    synchronisation on both sides, max over ranks."""
    import torch
    cur = torch.cuda.current_stream()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(cur)
    fn()
    e1.record(cur)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    return max_over_ranks(e0.elapsed_time(e1), world, dist, dev)


# Replicas of the 128K configurations: enough instances that one cycle streams more than the 126 MB
# of L2 (config B: 4.7 MB of rows per instance; config C: 190 MB).
EXTRA_CONFIGS = {"hca_decode_128k": 32, "csa_decode_128k": 2}


def hbm_summary(wl, ms_per_step, peak):
    """tok/s, algorithmic bytes and HBM fraction of one decode step of every layer of wl."""
    b = sum(step_bytes(L, wl.n, wl.B) for L in wl.layers)
    gbs = b / (ms_per_step / 1e3) / 1e9
    return {"tok_s": wl.B * len(wl.layers) / (ms_per_step / 1e3), "us_per_step": 1e3 * ms_per_step,
            "algorithmic_bytes": b, "achieved_gbs": gbs, "hbm_frac": gbs / peak}


def run_ours(args):
    import torch
    import torch.distributed as dist

    from csa_synth import get_workload
    from long_context_sparse_csa_b200 import binding as C

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300), device_id=torch.device("cuda", local))
    C.lib()
    wl = get_workload(args.workload)
    R = max(1, args.replicas)
    dev = torch.device("cuda", local)
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            peak, peak_note = float(json.load(f)["hbm_gbs"]), "of measured"
    except (OSError, KeyError, ValueError):
        peak, peak_note = 6650.0, "of fallback"

    rig = DecodeRig(wl, R, dev)
    layers, datas = rig.layers, rig.datas
    rig.warm()
    all_li = list(range(len(layers)))
    has_csa = any(l["spec"].kind == "csa" for l in layers)
    cycles, singles, launches_per_step = rig.graphs(all_li, args.steps, idx_events=has_csa)
    torch.cuda.synchronize()

    clocks = ClockSampler(local)
    clocks.start()
    # warm-up: W steps, plus a short burn so clocks settle at load before the timed region
    run_steps(cycles, singles, R, args.warmup)
    t_burn = time.perf_counter()
    while time.perf_counter() - t_burn < args.burn_seconds:
        cycles[0][0].replay()
        torch.cuda.synchronize()
    clocks.sample()
    w0 = time.perf_counter()
    T_ms = timed(lambda: run_steps(cycles, singles, R, args.steps), world, dist, dev)
    w1 = time.perf_counter()
    clocks.sample()
    clk = clocks.summary(w0, w1)
    # indexer launch durations sampled inside the timed region (one per cycle-graph copy)
    idx_ms = [c[1][0].elapsed_time(c[1][1]) for c in cycles] if has_csa else []

    # ------------------------------------------------------------------ each layer on its own (timed the same way)
    per_layer = {}
    if len(layers) > 1:
        for li, lay in enumerate(layers):
            cy, si, _ = rig.graphs([li], args.steps)
            run_steps(cy, si, R, args.warmup)
            ms = timed(lambda: run_steps(cy, si, R, args.steps), world, dist, dev) / args.steps
            spec = lay["spec"]
            b = step_bytes(spec, wl.n, wl.B)
            per_layer[f"{spec.kind}{li}"] = {"us_per_step": 1e3 * ms, "tok_s": wl.B / (ms / 1e3),
                                             "algorithmic_bytes": b, "achieved_gbs": b / (ms / 1e3) / 1e9,
                                             "hbm_frac": b / (ms / 1e3) / 1e9 / peak}
            del cy, si

    # ------------------------------------------------------------------ per-kernel timeline (diagnostic, untimed)
    # launch order of the sequential (diagnostic) step: the second stream is off while it is timed
    labels = {"csa": ["append+compress", "indexer scores", "top-k", "q preparation", "attention", "combine"],
              "hca": ["append+compress", "q preparation", "attention", "combine"]}
    tl_events = []
    g_tl = torch.cuda.CUDAGraph()
    for lay in layers:
        evs = [_ext_event() for _ in range(17)]
        for x in evs:
            x.record()
        tl_events.append(evs)
    torch.cuda.synchronize()
    with torch.cuda.graph(g_tl, stream=rig.stream):
        for li, lay in enumerate(layers):
            evs = tl_events[li]
            C.csa_profile_timeline(evs[:16])
            rig.call(li, 0)
            lay["tl_n"] = C.csa_profile_timeline_count()
            C.csa_profile_timeline(None)
            evs[lay["tl_n"]].record()
    timeline = {}
    reps = []
    for rep in range(5):
        for r in range(1, R):          # touch the other instances so instance 0 is cold in L2
            singles[r].replay()
        g_tl.replay()
        torch.cuda.synchronize()
        reps.append([[tl_events[li][i].elapsed_time(tl_events[li][i + 1]) * 1e3 for i in range(lay["tl_n"])]
                     for li, lay in enumerate(layers)])
    for li, lay in enumerate(layers):
        med = np.median(np.array([r[li] for r in reps]), axis=0)
        names = labels[lay["spec"].kind] if len(labels[lay["spec"].kind]) == lay["tl_n"] else \
            [f"launch{i}" for i in range(lay["tl_n"])]
        timeline[f"{lay['spec'].kind}{li}"] = {n: round(float(v), 2) for n, v in zip(names, med)}
    del g_tl

    # ------------------------------------------------------------------ end to end through host memory
    h2d, d2h = [], []
    for lay in layers:
        for k in ["q", "idx_q", "idx_q_scale", "head_w", "x_new", "g_new", "t"]:
            if k in lay["io"]:
                t = lay["io"][k]
                h2d.append((torch.empty(t.shape, dtype=t.dtype, pin_memory=True).copy_(t), t))
        o = lay["io"]["out"]
        d2h.append((o, torch.empty(o.shape, dtype=o.dtype, pin_memory=True)))
    h2d_bytes = sum(h.numel() * h.element_size() for h, _ in h2d)
    d2h_bytes = sum(h.numel() * h.element_size() for _, h in d2h)

    def e2e_steps(k):
        for s in range(k):
            for h, dv in h2d:
                dv.copy_(h, non_blocking=True)
            singles[s % R].replay()
            for dv, h in d2h:
                h.copy_(dv, non_blocking=True)

    e2e_steps(args.warmup)
    E_ms = timed(lambda: e2e_steps(args.steps), world, dist, dev)
    clocks.stop()

    for lay in layers:
        assert C.csa_device_error(lay["ws"]) == 0

    units = wl.B * len(layers) * args.steps
    value = job_value(units, world, T_ms)
    e2e_value = job_value(units, world, E_ms)

    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": T_ms / args.steps, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "e4m3+bf16 (fp32 accumulate)", "data": "synthetic",
            "config": workload_config(wl, R)}
    if has_csa:
        csa_li = [i for i, l in enumerate(layers) if l["spec"].kind == "csa"][0]
        spec = layers[csa_li]["spec"]
        nv = wl.n // spec.m
        bytes_idx = index_kernel_bytes(spec, nv, wl.B)
        t_idx = float(np.mean(idx_ms)) / 1e3
        achieved = bytes_idx / t_idx / 1e9
        line["roofline"] = {"bound": "hbm", "kernel": "index_score_tc_kernel", "achieved": achieved, "peak": peak,
                            "unit": "GB/s", "frac": achieved / peak, "peak_source": peak_note,
                            "traffic": recorded_traffic(wl.name), "algorithmic_bytes": bytes_idx,
                            "launch_us": 1e6 * t_idx, "launches_sampled": len(idx_ms)}
    else:
        spec = layers[0]["spec"]
        b = step_bytes(spec, wl.n, wl.B)
        t = T_ms / args.steps / 1e3
        line["roofline"] = {"bound": "hbm", "kernel": "hca layer step", "achieved": b / t / 1e9, "peak": peak,
                            "unit": "GB/s", "frac": b / t / 1e9 / peak, "peak_source": peak_note, "traffic": None,
                            "algorithmic_bytes": b}
    step_alg = sum(step_bytes(l["spec"], wl.n, wl.B) for l in layers)
    line["step_hbm"] = {"algorithmic_bytes": step_alg, "achieved_gbs": step_alg / (T_ms / args.steps / 1e3) / 1e9,
                        "frac": step_alg / (T_ms / args.steps / 1e3) / 1e9 / peak}
    if per_layer:
        line["layers"] = per_layer
    line["e2e"] = {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d_bytes, "d2h_bytes_per_step": d2h_bytes,
                   "ms_per_step": E_ms / args.steps}
    line["gpu_launches"] = int(launches_per_step) * args.steps
    line["timeline_us"] = timeline
    line["clocks"] = clk
    del cycles, singles

    # ------------------------------------------------------------------ the 128K configurations
    if args.workload == "csa_hca_decode_1m" and not args.no_extra_configs:
        extra = {}
        for name, r_extra in EXTRA_CONFIGS.items():
            wl2 = get_workload(name)
            rig2 = DecodeRig(wl2, r_extra, dev)
            rig2.warm()
            cy, si, _ = rig2.graphs(list(range(len(rig2.layers))), args.steps)
            run_steps(cy, si, r_extra, args.warmup)
            ms = timed(lambda: run_steps(cy, si, r_extra, args.steps), world, dist, dev) / args.steps
            for lay in rig2.layers:
                assert C.csa_device_error(lay["ws"]) == 0
            extra[name] = dict(hbm_summary(wl2, ms, peak), batch=wl2.B, context=wl2.n,
                               l2=f"rotating {r_extra} instances (inputs larger than L2)")
            del cy, si, rig2
            torch.cuda.empty_cache()
        line["configs"] = extra

    # ------------------------------------------------------------------ variants of the 1M CSA layer
    if args.workload == "csa_hca_decode_1m" and not args.no_extra_configs:
        from csa_synth.configs import CSA_PRO, scaled_layer
        variants = {}
        for name, layer, indexed in [("csa_1m_fp4_keys", scaled_layer(CSA_PRO, idx_format="e2m1"), False),
                                     ("csa_1m_index_side_in_step", CSA_PRO, True)]:
            wl2 = get_workload("csa_hca_decode_1m", layers=(layer,))
            rig2 = DecodeRig(wl2, R, dev, indexed=indexed)
            rig2.warm()
            cy, si, _ = rig2.graphs([0], args.steps, idx_events=True)
            run_steps(cy, si, R, args.warmup)
            ms = timed(lambda: run_steps(cy, si, R, args.steps), world, dist, dev) / args.steps
            idx = [c[1][0].elapsed_time(c[1][1]) for c in cy]
            for lay in rig2.layers:
                assert C.csa_device_error(lay["ws"]) == 0
            key_bytes = layer.d_I // 2 + 4 if layer.idx_format == "e2m1" else layer.d_I + 4
            b = step_bytes(layer, wl2.n, wl2.B)
            if indexed:
                b += layer.H_I * layer.d_I * layer.idx_rank * 2 + (1 + layer.ov) * layer.m * layer.d_I * 2 * 2
            variants[name] = {"us_per_step": 1e3 * ms, "tok_s": wl2.B / (ms / 1e3), "algorithmic_bytes": b,
                              "hbm_frac": b / (ms / 1e3) / 1e9 / peak, "index_key_bytes_per_entry": key_bytes,
                              "indexer_launch_us": 1e3 * float(np.mean(idx)),
                              "indexer_gbs": index_kernel_bytes(layer, wl2.n // layer.m, wl2.B) /
                              (float(np.mean(idx)) / 1e3) / 1e9}
            del cy, si, rig2
            torch.cuda.empty_cache()
        line["variants"] = variants

    # ------------------------------------------------------------------ the chunked prefill (config E)
    if args.workload == "csa_hca_decode_1m" and not args.no_extra_configs and world == 1:
        res, _, _ = prefill_measure("csa_prefill_8k", args.steps, args.warmup)
        res.pop("clocks", None)
        line["prefill"] = res
        torch.cuda.empty_cache()

    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(wl, datas, args.cpu_seconds)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


# ----------------------------------------------------------------------------- chunked prefill (diagnostic mode)

def prefill_work(layer, t, n_max, B=1):
    """Work of one chunked-prefill call for queries at positions t (pos0 = 0): FP8 indexer FLOPs (every
    visible entry of every query, all index heads), BF16 attention FLOPs (QK^T and PV over each
    query's top-k entries and window rows, all heads) and the rows the attention gathers (bytes)."""
    t = np.asarray(t, dtype=np.int64)
    n_vis = np.minimum((t + 1) // layer.m, n_max).astype(np.float64)
    idx_flops = 2.0 * layer.H_I * layer.d_I * float(n_vis.sum()) * B
    rows = np.minimum(n_vis, layer.top_k) + np.minimum(t + 1, layer.window)
    att_flops = 4.0 * layer.H * layer.D * float(rows.sum()) * B
    row_bytes = layer.D * 2 if layer.kv_format == "bf16" else layer.D * 4
    return idx_flops, att_flops, float(rows.sum()) * B * row_bytes


def prefill_measure(workload, steps, warmup, queries=None):
    """Times csa_prefill on the 8,192-query chunk (one GPU): the whole call (CUDA events around
    back-to-back calls), and the launch list of one call (an event before each launch, one after the
    call: the last interval is the attention kernel's own).  The work of a call (FP8 indexer FLOPs,
    BF16 attention FLOPs, gathered bytes) is set against the measured dense BF16 peak (FP8 = 2x, the
    nominal ratio).  The workload's inputs (512 MiB of queries alone) exceed L2, so calls run back to
    back."""
    import torch
    from csa_synth import get_workload, prefill_inputs
    from long_context_sparse_csa_b200 import binding as C
    from long_context_sparse_csa_b200.state import LayerState, to_device
    wl = get_workload(workload)
    layer = wl.layers[0]
    pf = prefill_inputs(wl, Tq=queries)
    st = LayerState.from_arrays(layer, wl.B, pf, raw_key="raw", gate_key="gate", raw_base=pf["raw_first_row"])
    Tq, n_max = pf["Tq"], pf["n"] // layer.m
    out = torch.zeros((wl.B, Tq, layer.H, layer.D), dtype=torch.int16, device="cuda")
    topk = torch.zeros((wl.B, Tq, layer.top_k), dtype=torch.int32, device="cuda")
    ws = st.workspace("prefill", Tq, n_max)
    io = {k: to_device(pf[k]) for k in ("q", "idx_q", "idx_q_scale", "head_w", "t")}

    def call():
        C.csa_prefill(st.L, st.cache(), st.params(), io["q"], io["idx_q"], io["idx_q_scale"], io["head_w"], io["t"],
                      Tq, n_max, out, topk, ws)

    for _ in range(max(3, warmup)):
        call()
    torch.cuda.synchronize()
    steps = max(1, min(steps, 10))
    clocks = ClockSampler(torch.cuda.current_device())
    clocks.start()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks.sample()
    w0 = time.perf_counter()
    e0.record()
    for _ in range(steps):
        call()
    e1.record()
    torch.cuda.synchronize()
    w1 = time.perf_counter()
    clocks.sample()
    clocks.stop()
    ms = e0.elapsed_time(e1) / steps
    # launch list of one call (the library records an event before each of its launches)
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(17)]
    for x in evs:                      # recorded once here, so torch accepts the library's records
        x.record()
    torch.cuda.synchronize()
    C.csa_profile_timeline(evs[:16])
    call()
    n = C.csa_profile_timeline_count()
    C.csa_profile_timeline(None)
    evs[n].record()
    torch.cuda.synchronize()
    assert C.csa_device_error(ws) == 0
    launches_ms = [evs[i].elapsed_time(evs[i + 1]) for i in range(n)]
    idx_flops, att_flops, gather_bytes = prefill_work(layer, pf["t"][0], n_max, wl.B)
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            bf16_peak, note = float(json.load(f)["bf16_tflops"]), "of measured"
    except (OSError, KeyError, ValueError):
        bf16_peak, note = 1590.0, "of fallback"
    res = {"workload": wl.name, "tok_s": wl.B * Tq / (ms / 1e3), "ms_per_call": ms, "queries": Tq,
           "prefix": pf["prefix"], "heads": layer.H, "kv_format": layer.kv_format, "launch_ms": launches_ms,
           "work": {"indexer_fp8_tflop": idx_flops / 1e12, "attention_bf16_tflop": att_flops / 1e12,
                    "attention_gather_gb": gather_bytes / 1e9},
           "bf16_peak_tflops": bf16_peak, "peak_source": note, "clocks": clocks.summary(w0, w1)}
    if n in (4, 5):     # append+compress, indexer scores, top-k, (q preparation,) attention, in order
        names = ["append_compress", "indexer", "topk"] + (["q_preparation"] if n == 5 else []) + ["attention"]
        res["kernels_ms"] = dict(zip(names, launches_ms))
        att_ms, idx_ms = launches_ms[n - 1], launches_ms[1]
        res["attention"] = {"kernel": "attend_prefill_tc_kernel" if layer.H == 64 and layer.kv_format == "bf16"
                            else "attend_mma_kernel", "ms": att_ms, "tflops": att_flops / (att_ms / 1e3) / 1e12,
                            "frac_of_bf16_peak": att_flops / (att_ms / 1e3) / 1e12 / bf16_peak}
        res["indexer"] = {"kernel": "index_score_tc_kernel", "ms": idx_ms, "tflops": idx_flops / (idx_ms / 1e3) / 1e12,
                          "frac_of_fp8_peak": idx_flops / (idx_ms / 1e3) / 1e12 / (2 * bf16_peak)}
    return res, steps, max(3, warmup)


def run_prefill(args):
    """The chunked-prefill line on its own (`--workload csa_prefill_8k`); the default decode line
    carries the same measurement under its "prefill" key."""
    res, steps, warmup = prefill_measure(args.workload, args.steps, args.warmup, args.prefill_queries)
    line = {"metric": f"prefill tok/s ({res['queries']:,}-query CSA chunk after a {res['prefix']:,}-token prefix)",
            "value": res["tok_s"], "unit": "tok/s", "n_gpus": 1, "steps": steps, "warmup": warmup,
            "ms_per_call": res["ms_per_call"], "higher_is_better": True, "dtype": "e4m3+bf16 (fp32 accumulate)",
            "data": "synthetic",
            "config": {"workload": res["workload"], "queries": res["queries"], "prefix": res["prefix"],
                       "heads": res["heads"], "kv_format": res["kv_format"],
                       "l2": "inputs larger than L2 (queries alone 512 MiB)"},
            "prefill": res, "clocks": res["clocks"]}
    print(json.dumps(line), flush=True)


def main():
    args = parse()
    if args.impl == "reference":
        run_reference(args)
    elif args.workload == "csa_prefill_8k":
        run_prefill(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
