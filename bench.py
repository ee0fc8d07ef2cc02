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
    """Algorithmic bytes of one indexer-score launch: keys + key scales read, scores written, queries."""
    per_entry = layer.d_I + 4 + 4
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
        idx = nv * (layer.d_I + 4 + 4) + layer.H_I * layer.d_I
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
                        "long_context_sparse_csa_b200/csrc/common.cuh"]


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


def run_ours(args):
    import torch
    import torch.distributed as dist

    from csa_synth import decode_inputs, get_workload
    from long_context_sparse_csa_b200 import binding as C
    from long_context_sparse_csa_b200.state import LayerState, to_device

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

    datas, layers = [], []
    for li, spec in enumerate(wl.layers):
        d = decode_inputs(wl, li)
        datas.append(d)
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
        io["out"] = torch.zeros((wl.B, spec.H, spec.D), dtype=torch.int16 if spec.act_format == "bf16" else torch.float32,
                                device=dev)
        ws = base.workspace("decode_step", 1, cap)
        layers.append({"spec": spec, "insts": insts, "io": io, "ws": ws,
                       "caches": [s.cache() for s in insts], "params": base.params(), "L": base.L})

    def run_step(r):
        for li, lay in enumerate(layers):
            io, spec = lay["io"], lay["spec"]
            if spec.kind == "csa":
                C.csa_decode_step(lay["L"], lay["caches"][r], lay["params"], io["q"], io["idx_q"], io["idx_q_scale"],
                                  io["head_w"], io["x_new"], io["g_new"], io["t"], io["out"], io["topk"], lay["ws"])
            else:
                C.hca_decode_step(lay["L"], lay["caches"][r], lay["params"], io["q"], io["x_new"], io["g_new"],
                                  io["t"], io["out"], lay["ws"])

    # eager warm-up of every instance (module load, attributes), then one graph per instance
    for r in range(R):
        run_step(r)
    torch.cuda.synchronize()
    for lay in layers:
        assert C.csa_device_error(lay["ws"]) == 0
    has_csa = any(l["spec"].kind == "csa" for l in layers)
    ev = lambda: torch.cuda.Event(enable_timing=True, external=True)  # noqa: E731
    stream = torch.cuda.Stream(device=dev)

    def capture(rs, idx_events):
        """One CUDA graph running the steps of instances rs in order.  With idx_events, a pair of
        events brackets the indexer-score launch of the first step (the only event nodes: each one
        breaks the chain of kernel nodes and costs a few microseconds)."""
        pair = None
        if idx_events:
            pair = (ev(), ev())
            for x in pair:
                x.record()
            torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        n0 = C.csa_launch_count()
        with torch.cuda.graph(g, stream=stream):
            for j, r in enumerate(rs):
                for li, lay in enumerate(layers):
                    io, spec = lay["io"], lay["spec"]
                    if spec.kind == "csa":
                        if idx_events and j == 0:
                            C.csa_profile_events(*pair)
                        C.csa_decode_step(lay["L"], lay["caches"][r], lay["params"], io["q"], io["idx_q"],
                                          io["idx_q_scale"], io["head_w"], io["x_new"], io["g_new"], io["t"],
                                          io["out"], io["topk"], lay["ws"])
                        C.csa_profile_events(None, None)
                    else:
                        C.hca_decode_step(lay["L"], lay["caches"][r], lay["params"], io["q"], io["x_new"],
                                          io["g_new"], io["t"], io["out"], lay["ws"])
        return g, pair, C.csa_launch_count() - n0

    # n_cyc copies of the cycle graph, replayed round-robin: the last replay of each copy lies in the
    # timed region, so its event pair samples one indexer launch of the timed steps
    n_cyc = max(1, min(8, args.steps // R))
    cycles = [capture(list(range(R)), has_csa) for _ in range(n_cyc)]
    launches_per_step = cycles[0][2] // R
    singles = [capture([r], False)[0] for r in range(R)]
    torch.cuda.synchronize()

    def run_steps(k):
        """Exactly k decode steps: whole cycles of the R instances, then single steps."""
        for c in range(k // R):
            cycles[c % n_cyc][0].replay()
        for r in range(k % R):
            singles[r].replay()

    def barrier():
        if world > 1:
            dist.barrier()

    cur = torch.cuda.current_stream()
    clocks = ClockSampler(local)
    clocks.start()
    # warm-up: W steps, plus a short burn so clocks settle at load before the timed region
    run_steps(args.warmup)
    t_burn = time.perf_counter()
    while time.perf_counter() - t_burn < args.burn_seconds:
        cycles[0][0].replay()
        torch.cuda.synchronize()
    torch.cuda.synchronize()
    barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks.sample()
    w0 = time.perf_counter()
    e0.record(cur)
    run_steps(args.steps)
    e1.record(cur)
    torch.cuda.synchronize()
    w1 = time.perf_counter()
    clocks.sample()
    barrier()
    T_ms = max_over_ranks(e0.elapsed_time(e1), world, dist, dev)
    clk = clocks.summary(w0, w1)
    # indexer launch durations sampled inside the timed region (one per cycle-graph copy)
    idx_ms = [c[1][0].elapsed_time(c[1][1]) for c in cycles] if has_csa else []

    # ------------------------------------------------------------------ per-kernel timeline (diagnostic, untimed)
    # launch order of the sequential (diagnostic) step: the second stream is off while it is timed
    labels = {"csa": ["append+compress", "indexer scores", "top-k", "q preparation", "attention", "combine"],
              "hca": ["append+compress", "q preparation", "attention", "combine"]}
    tl_events = []
    g_tl = torch.cuda.CUDAGraph()
    for lay in layers:
        evs = [ev() for _ in range(17)]
        for x in evs:
            x.record()
        tl_events.append(evs)
    torch.cuda.synchronize()
    with torch.cuda.graph(g_tl, stream=stream):
        for li, lay in enumerate(layers):
            io, spec = lay["io"], lay["spec"]
            evs = tl_events[li]
            C.csa_profile_timeline(evs[:16])
            if spec.kind == "csa":
                C.csa_decode_step(lay["L"], lay["caches"][0], lay["params"], io["q"], io["idx_q"], io["idx_q_scale"],
                                  io["head_w"], io["x_new"], io["g_new"], io["t"], io["out"], io["topk"], lay["ws"])
            else:
                C.hca_decode_step(lay["L"], lay["caches"][0], lay["params"], io["q"], io["x_new"], io["g_new"],
                                  io["t"], io["out"], lay["ws"])
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
    for s in range(args.warmup):
        for h, dv in h2d:
            dv.copy_(h, non_blocking=True)
        singles[s % R].replay()
        for dv, h in d2h:
            h.copy_(dv, non_blocking=True)
    torch.cuda.synchronize()
    barrier()
    torch.cuda.synchronize()
    f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    f0.record(cur)
    for s in range(args.steps):
        for h, dv in h2d:
            dv.copy_(h, non_blocking=True)
        singles[s % R].replay()
        for dv, h in d2h:
            h.copy_(dv, non_blocking=True)
    f1.record(cur)
    torch.cuda.synchronize()
    barrier()
    E_ms = max_over_ranks(f0.elapsed_time(f1), world, dist, dev)
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
    peaks = {}
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            peaks = json.load(f)
        peak, peak_note = float(peaks["hbm_gbs"]), "of measured"
    except (OSError, KeyError, ValueError):
        peak, peak_note = 6650.0, "of fallback"
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
    line["e2e"] = {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d_bytes, "d2h_bytes_per_step": d2h_bytes,
                   "ms_per_step": E_ms / args.steps}
    line["gpu_launches"] = int(launches_per_step) * args.steps
    line["timeline_us"] = timeline
    line["clocks"] = clk

    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        times = run_cpu_oracle(wl, datas, args.cpu_seconds)
        line["cpu_baseline"] = {"value": wl.B * len(layers) / float(np.mean(times)), "unit": UNIT,
                                "cores": cpu_threads(), "kind": "oracle",
                                "sample": f"{len(times)} full decode steps of the workload ({args.cpu_seconds:.0f} s budget)"}
    if rank == 0:
        print(json.dumps(line), flush=True)
    del cycles, singles
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


def run_prefill(args):
    """Times csa_prefill on the 8,192-query chunk (one GPU): tokens/s, the launch list of one call
    (CUDA events before each launch), and the indexer's FP8 and the attention's BF16 TFLOP/s against
    the measured dense BF16 peak (FP8 = 2x, the nominal ratio).  Not the headline line: the
    workload's inputs (512 MiB of queries alone) exceed L2, so calls run back to back."""
    import torch
    from csa_synth import get_workload, prefill_inputs
    from long_context_sparse_csa_b200 import binding as C
    from long_context_sparse_csa_b200.state import LayerState, to_device
    wl = get_workload(args.workload)
    layer = wl.layers[0]
    pf = prefill_inputs(wl)
    st = LayerState.from_arrays(layer, wl.B, pf, raw_key="raw", gate_key="gate", raw_base=pf["raw_first_row"])
    Tq, n_max = pf["Tq"], pf["n"] // layer.m
    out = torch.zeros((wl.B, Tq, layer.H, layer.D), dtype=torch.int16, device="cuda")
    topk = torch.zeros((wl.B, Tq, layer.top_k), dtype=torch.int32, device="cuda")
    ws = st.workspace("prefill", Tq, n_max)
    io = {k: to_device(pf[k]) for k in ("q", "idx_q", "idx_q_scale", "head_w", "t")}

    def call():
        C.csa_prefill(st.L, st.cache(), st.params(), io["q"], io["idx_q"], io["idx_q_scale"], io["head_w"], io["t"],
                      Tq, n_max, out, topk, ws)

    for _ in range(max(3, args.warmup)):
        call()
    torch.cuda.synchronize()
    steps = max(1, min(args.steps, 10))
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
    # launch list of one call
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
    launches_ms = [evs[i].elapsed_time(evs[i + 1]) for i in range(n)]
    idx_flops, att_flops, gather_bytes = prefill_work(layer, pf["t"][0], n_max, wl.B)
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            bf16_peak, note = float(json.load(f)["bf16_tflops"]), "of measured"
    except (OSError, KeyError, ValueError):
        bf16_peak, note = 1590.0, "of fallback"
    longest = sorted(range(n), key=lambda i: -launches_ms[i])
    line = {"metric": "prefill tok/s (8,192-query CSA chunk after a 65,536-token prefix)",
            "value": wl.B * Tq / (ms / 1e3), "unit": "tok/s", "n_gpus": 1, "steps": steps, "warmup": max(3, args.warmup),
            "ms_per_call": ms, "higher_is_better": True, "dtype": "e4m3+bf16 (fp32 accumulate)", "data": "synthetic",
            "config": {"workload": wl.name, "batch": wl.B, "queries": Tq, "prefix": pf["prefix"], "heads": layer.H,
                       "kv_dim": layer.D, "kv_format": layer.kv_format, "top_k": layer.top_k,
                       "l2": "inputs larger than L2 (queries alone 512 MiB)"},
            "launch_ms": [round(x, 3) for x in launches_ms],
            "work": {"indexer_fp8_tflop": idx_flops / 1e12, "attention_bf16_tflop": att_flops / 1e12,
                     "attention_gather_gb": gather_bytes / 1e9},
            "tensor": {"bf16_peak_tflops": bf16_peak, "fp8_peak_tflops": 2 * bf16_peak, "peak_source": note},
            "longest_launches": [{"launch": i, "ms": round(launches_ms[i], 3)} for i in longest[:3]],
            "clocks": clocks.summary(w0, w1)}
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
