"""Throughput bench for the GLA token mixer (libgla.so) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step = the whole hot path over one batch of the 640-px workload (40x40
patch grid, B=1, H=6, d_k=d_v=64, fp16): four gla_fwd launches, one per
scan direction (L->R, R->L, T->B, B->T), each on its own input set taken
from a rotating pool larger than the 126 MB L2, so every launch reads cold
inputs from HBM.  The K timed steps run as CUDA-graph replays; timing uses
CUDA events on the launching stream with a barrier and synchronize on both
sides, and the max over ranks.  With N > 1 (torchrun) every rank runs an
independent replica (the operator has no cross-GPU exchange) and `value` is
the total over ranks.

--impl reference times the fp64 CPU oracle (test infrastructure, the only
reference implementation that exists) on the machine's host cores on a bounded
sample of the same workload; under torchrun only rank 0 runs it.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "GLA fwd Mtokens/s (B·H·L) at 40×40 grid fp16; % of HBM/tensor roofline"
WORKLOAD = "gtr640"
DIRECTIONS = (0, 1, 2, 3)
L2_BYTES = 126 * 1024 * 1024
FALLBACK_HBM_GBS = 6650.0
PROFILE_TRAFFIC = os.path.join(ROOT, "profiles", "traffic.json")
GATE_KERNEL = "gate projection (tcgen05)"
GATE_RANK = 16
SSWIGLU_KERNEL = "spatial swiglu mix"
LINEAR_KERNEL = "dense projection (tcgen05)"
FALLBACK_TENSOR_TFLOPS = 1590.0
SSWIGLU_EXPANSION = 4


def gate_shape(wl, d_model: int):
    """(tokens, d_model, n_out) of the gate projection feeding the workload's operator."""
    return wl.B * wl.L, d_model, wl.H * wl.d_k


def linear_bytes(rows: int, k_dim: int, n_dim: int) -> int:
    """Algorithmic HBM bytes of one projection: x read, y written and W read once (fp16)."""
    return 2 * (rows * k_dim + rows * n_dim + k_dim * n_dim)


def measured_tensor_peak():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["bf16_tflops"]), "measured"
    except Exception:
        return FALLBACK_TENSOR_TFLOPS, "fallback"


def sswiglu_bytes(wl, d_model: int) -> int:
    """Algorithmic HBM bytes of one Spatial SwiGLU mixing step: value and gate read and h
    written once (fp16), the taps and bias (fp32) read once."""
    C = SSWIGLU_EXPANSION * d_model
    return 3 * 2 * wl.B * wl.L * C + 4 * 10 * C


def gate_bytes(wl, d_model: int) -> int:
    """Algorithmic HBM bytes of one projection: x read and a written once (fp16), the weights
    (fp16) and bias (fp32) read once."""
    T, d, n = gate_shape(wl, d_model)
    return 2 * T * d + 2 * T * n + 2 * GATE_RANK * (d + n) + 4 * n


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--e2e-steps", type=int, default=50)
    ap.add_argument("--cpu-seconds", type=float, default=10.0,
                    help="CPU-oracle sample budget for cpu_baseline / --impl reference")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--kernel", choices=["auto", "tc128", "tc64", "pipe64", "simt"], default="auto",
                    help="kernel to time (default: the one gla_fwd picks for the workload)")
    ap.add_argument("--workload", default=WORKLOAD,
                    help="synthetic workload to time (default: the 40x40 headline); the others "
                         "are reported with their own metric name")
    ap.add_argument("--op", choices=["gla", "gate", "sswiglu", "proj_in", "proj_out"], default="gla",
                    help="gla: the operator (default); gate: the retention gate's low-rank "
                         "projection a = x W1 W2 + b over the workload's tokens (B*L), its output "
                         "width H*d_k, model width --d-model; sswiglu: Spatial SwiGLU's "
                         "dwconv + gating step on the workload's grid, 4 x d_model channels; "
                         "proj_in / proj_out: the block's input projections (x -> q, k, v, W_r) "
                         "and output projection (heads -> d_model)")
    ap.add_argument("--d-model", type=int, default=384,
                    help="with --op gate / sswiglu: the model width d (GTR-L: 384)")
    ap.add_argument("--record-traffic", metavar="NCU_CSV",
                    help="no bench: read an ncu CSV (dram__bytes_read.sum / dram__bytes_write.sum "
                         "of the kernel --kernel / --workload select) and print the traffic entry "
                         "for profiles/traffic.json, stamped with this build's sources digest")
    ap.add_argument("--ncu-command", default="",
                    help="with --record-traffic: the ncu command line that wrote the CSV")
    return ap.parse_args()


def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def max_over_ranks(value_ms: float, device) -> float:
    """Max of a per-rank time over the job (the job ends when its slowest rank does)."""
    import torch
    import torch.distributed as dist
    t = torch.tensor([value_ms], dtype=torch.float64, device=device)
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(tokens_per_step: int, steps: int, world_size: int, max_ms: float) -> float:
    """Whole-job Mtokens/s: every rank's tokens over the slowest rank's time."""
    return tokens_per_step * world_size * steps / (max_ms / 1e3) / 1e6


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def profile_traffic(workload: str, kernel: str):
    """DRAM bytes per launch from the committed ncu entries (profiles/traffic.json), if one was
    taken on this workload, this kernel and this exact kernel build (sources digest); else None."""
    try:
        with open(PROFILE_TRAFFIC) as f:
            d = json.load(f)
        from recurrent_vision_backbone_only_b200 import build as _b
        digest = _b.sources_digest()
        for e in d.get("entries", []):
            if (e.get("workload") == workload and e.get("kernel") == kernel and
                    e.get("lib_sources_digest") == digest):
                return e.get("dram_bytes_per_launch")
        return None
    except Exception:
        return None


def read_ncu_csv(path: str):
    """Launches of an ncu --csv log (details layout: one row per metric; raw layout: one column
    per metric) as [(kernel name, {metric: value})], in capture order; the launch's grid size is
    kept as the pseudo-metric "grid"."""
    import csv
    with open(path, newline="") as f:
        lines = [ln for ln in f if ln.startswith('"')]
    rows = list(csv.reader(lines))
    if not rows or rows[0][:1] != ["ID"]:
        raise ValueError("%s: no ncu CSV header" % path)
    head = rows[0]
    launches = {}
    order = []
    if "Metric Name" in head:
        i_id, i_k = head.index("ID"), head.index("Kernel Name")
        i_g = head.index("Grid Size") if "Grid Size" in head else None
        i_n, i_v = head.index("Metric Name"), head.index("Metric Value")
        i_u = head.index("Metric Unit")
        scale = {"byte": 1, "Kbyte": 1e3, "Mbyte": 1e6, "Gbyte": 1e9}
        for r in rows[1:]:
            if len(r) <= i_v:
                continue
            key = r[i_id]
            if key not in launches:
                launches[key] = (r[i_k], {"grid": r[i_g] if i_g is not None else ""})
                order.append(key)
            v = float(r[i_v].replace(",", ""))
            launches[key][1][r[i_n]] = v * scale.get(r[i_u], 1)
    else:
        units = rows[1]
        i_id, i_k = head.index("ID"), head.index("Kernel Name")
        i_g = head.index("Grid Size") if "Grid Size" in head else None
        scale = {"byte": 1, "Kbyte": 1e3, "Mbyte": 1e6, "Gbyte": 1e9}
        for r in rows[2:]:
            vals = {"grid": r[i_g] if i_g is not None else ""}
            for j, name in enumerate(head):
                if name.startswith(("dram__", "gpu__time")) and j < len(r) and r[j]:
                    vals[name] = float(r[j].replace(",", "")) * scale.get(units[j], 1)
            launches[r[i_id]] = (r[i_k], vals)
            order.append(r[i_id])
    return [launches[k] for k in order]


def record_traffic(args):
    """Print the profiles/traffic.json entry for the launches of `args.record_traffic`."""
    import re
    from recurrent_vision_backbone_only_b200 import build as _b, gla, synth
    wl = synth.WORKLOADS[args.workload]
    op = getattr(args, "op", "gla")
    if op in ("gate", "sswiglu", "proj_in", "proj_out"):
        T, n = wl.B * wl.L, wl.H * wl.d_k
        symbol, kname, alg = {
            "gate": ("gla_gate_kernel", GATE_KERNEL, gate_bytes),
            "sswiglu": ("gla_sswiglu_kernel", SSWIGLU_KERNEL, sswiglu_bytes),
            "proj_in": ("gla_linear_kernel", LINEAR_KERNEL + ", input side", lambda w_, d: linear_bytes(T, d, 4 * n)),
            "proj_out": ("gla_linear_kernel", LINEAR_KERNEL + ", output side",
                         lambda w_, d: linear_bytes(T, w_.H * w_.d_v, d)),
        }[op]
        got = [v for k, v in read_ncu_csv(args.record_traffic) if re.search(symbol, k)]
        got = [v for v in got if "dram__bytes_read.sum" in v and "dram__bytes_write.sum" in v]
        if not got:
            raise SystemExit("no %s launch with dram bytes in %s" % (symbol, args.record_traffic))
        rd = statistics.mean(v["dram__bytes_read.sum"] for v in got)
        wr = statistics.mean(v["dram__bytes_write.sum"] for v in got)
        print(json.dumps({"workload": wl.name, "kernel": kname,
                          "lib_sources_digest": _b.sources_digest(), "launches": len(got),
                          "launch_shapes": sorted({v.get("grid", "") for v in got}),
                          "dram_read_bytes": rd, "dram_write_bytes": wr,
                          "dram_bytes_per_launch": rd + wr,
                          "algorithmic_bytes_per_launch": alg(wl, args.d_model),
                          "command": args.ncu_command}))
        return
    kid = {"auto": 0, "tc128": gla.KERNEL_TC128, "tc64": gla.KERNEL_TC64,
           "pipe64": gla.KERNEL_PIPE64, "simt": gla.KERNEL_SIMT}[args.kernel]
    symbol = {gla.KERNEL_TC128: "gla_tc_kernel", gla.KERNEL_TC64: "gla_chunk_kernel",
              gla.KERNEL_PIPE64: "gla_pipe_kernel", gla.KERNEL_SIMT: "gla_simt_kernel"}
    if not kid:
        raise SystemExit("--record-traffic needs an explicit --kernel")
    got = [v for k, v in read_ncu_csv(args.record_traffic) if re.search(symbol[kid], k)]
    got = [v for v in got if "dram__bytes_read.sum" in v and "dram__bytes_write.sum" in v]
    if not got:
        raise SystemExit("no %s launch with dram__bytes_read/write.sum in %s"
                         % (symbol[kid], args.record_traffic))
    # one gla_fwd call may issue two launches (a partial wave split off): per call, the mean
    # over launches of each grid shape, summed over the shapes
    shapes = sorted({v.get("grid", "") for v in got})
    rd = sum(statistics.mean(v["dram__bytes_read.sum"] for v in got if v.get("grid", "") == g)
             for g in shapes)
    wr = sum(statistics.mean(v["dram__bytes_write.sum"] for v in got if v.get("grid", "") == g)
             for g in shapes)
    print(json.dumps({"workload": wl.name, "kernel": gla.KERNEL_NAMES[kid],
                      "lib_sources_digest": _b.sources_digest(), "launches": len(got),
                      "launch_shapes": shapes,
                      "dram_read_bytes": rd, "dram_write_bytes": wr,
                      "dram_bytes_per_launch": rd + wr,
                      "algorithmic_bytes_per_launch": wl.tokens * wl.bytes_per_token,
                      "command": args.ncu_command}))


class ClockSampler:
    """nvidia-smi clock / throttle sampling during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "--query-gpu=" + self.FIELDS, "--format=csv,noheader,nounits",
                 "-lms", "50", "-i", str(self.gpu)],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            time.sleep(0.3)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *exc):
        self.out = ""
        if self.proc is not None:
            time.sleep(0.1)
            self.proc.terminate()
            try:
                self.out, _ = self.proc.communicate(timeout=5)
            except Exception:
                self.proc.kill()
                self.out = ""

    def summary(self):
        rows = []
        for line in (self.out or "").splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                rows.append(dict(sm=float(parts[1]), max=float(parts[2]), reasons=parts[5:9]))
            except ValueError:
                continue
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"], "samples": 0}
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        seen = sorted({names[i] for r in rows for i, v in enumerate(r["reasons"])
                       if v.lower() == "active"})
        return {"sm_mhz": statistics.median(r["sm"] for r in rows),
                "sm_max_mhz": max(r["max"] for r in rows), "reasons": seen,
                "samples": len(rows)}


def cpu_oracle_sample(wl, x, budget_s: float, directions=DIRECTIONS):
    """Time the fp64 oracle on whole (direction) passes of the workload until the budget."""
    import numpy as np
    import oracle
    xs = {n: np.asarray(x[n], dtype=np.float64) for n in ("q", "k", "v", "a", "g", "w")}
    threads = os.cpu_count() or 1
    oracle.gla_forward(xs["q"][:, :16], xs["k"][:, :16], xs["v"][:, :16], xs["a"][:, :16],
                       xs["g"][:, :16], xs["w"], 4, 4, 0, threads=threads)   # warm
    passes, tokens = 0, 0
    t0 = time.perf_counter()
    while True:
        d = directions[passes % len(directions)]
        oracle.gla_forward(xs["q"], xs["k"], xs["v"], xs["a"], xs["g"], xs["w"],
                           wl.grid_h, wl.grid_w, d, threads=threads)
        passes += 1
        tokens += wl.tokens
        el = time.perf_counter() - t0
        if el >= budget_s or passes >= 4000:
            break
    out = {"value": tokens / el / 1e6, "unit": "Mtokens/s", "cores": threads, "kind": "oracle",
           "sample": "%d full passes (directions cycling L2R,R2L,T2B,B2T) of the %s workload, "
                     "%.1f s, fp64, OpenMP over (b,h)" % (passes, wl.name, el)}
    # the same on one host thread (a bounded sample of (b,h) pairs: the oracle's cost is
    # linear in the pairs and independent across them)
    b1, h1 = 1, min(wl.H, 2)
    sl = {n: np.ascontiguousarray(xs[n][:b1, :, :h1]) for n in ("q", "k", "v", "a", "g")}
    passes1, tokens1 = 0, 0
    t0 = time.perf_counter()
    while True:
        d = directions[passes1 % len(directions)]
        oracle.gla_forward(sl["q"], sl["k"], sl["v"], sl["a"], sl["g"], xs["w"],
                           wl.grid_h, wl.grid_w, d, threads=1)
        passes1 += 1
        tokens1 += b1 * h1 * wl.L
        el1 = time.perf_counter() - t0
        if el1 >= min(3.0, budget_s / 3) or passes1 >= 4000:
            break
    out["single_thread"] = {"value": tokens1 / el1 / 1e6, "unit": "Mtokens/s", "cores": 1,
                            "sample": "%d passes over %d (b,h) pair(s), %.1f s" % (passes1, b1 * h1, el1)}
    return out


def run_reference(args, ws, rank):
    """The reference arm: the fp64 CPU oracle on this arm's workload and step definition.

    One step = the four scan directions over H' of the workload's heads, H'
    chosen (from a timed probe) so that K steps take about two minutes;
    H' = H is the full workload.  Tokens are counted as processed.
    """
    from recurrent_vision_backbone_only_b200 import synth
    if rank != 0:
        return
    import numpy as np
    import oracle
    wl = synth.WORKLOADS[WORKLOAD]
    x = synth.make_inputs(wl)
    xs = {n: np.asarray(x[n], dtype=np.float64) for n in ("q", "k", "v", "a", "g", "w")}
    threads = os.cpu_count() or 1
    K = max(1, args.steps)

    sliced = {}

    def one_step(heads):
        if heads not in sliced:
            sliced[heads] = [np.ascontiguousarray(xs[n][:, :, :heads])
                             for n in ("q", "k", "v", "a", "g")]
        for d in DIRECTIONS:
            oracle.gla_forward(*sliced[heads], xs["w"], wl.grid_h, wl.grid_w, d, threads=threads)

    t0 = time.perf_counter()
    one_step(wl.H)
    full_s = time.perf_counter() - t0
    heads = wl.H
    while heads > 1 and K * full_s * heads / wl.H > 120.0:
        heads -= 1
    for _ in range(args.warmup):
        one_step(heads)
    t0 = time.perf_counter()
    done = 0
    for _ in range(K):
        one_step(heads)
        done += 1
        if time.perf_counter() - t0 > 240.0:
            break
    el = time.perf_counter() - t0
    tokens_per_step = wl.B * heads * wl.L * len(DIRECTIONS)
    value = done * tokens_per_step / el / 1e6
    sample = ("%d steps x 4 directions over %d of %d heads of the %s workload, fp64, %d host "
              "threads" % (done, heads, wl.H, wl.name, threads))
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "Mtokens/s",
        "n_gpus": args.gpus, "steps": done, "warmup": args.warmup,
        "ms_per_step": el / done * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": "%s: %dx%d patch grid (L=%d), B=%d, H=%d, d_k=d_v=%d, fp16-rounded "
                               "inputs; one step = 4 directions" % (wl.name, wl.grid_h, wl.grid_w,
                                                                   wl.L, wl.B, wl.H, wl.d_k),
                   "sample_heads": heads},
        "cpu_baseline": {"value": value, "unit": "Mtokens/s", "cores": threads, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "Mtokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def launch_floor_us(gla, wl, stream, launches: int):
    """Per-launch time of the do-nothing kernel launched with gla_fwd's exact shape for this
    workload (cluster, block, shared memory, programmatic dependent launch), replayed from a
    CUDA graph like the timed steps: the floor no work inside the kernel can remove.  None
    when the workload does not use the tensor-core kernel."""
    import torch
    try:
        gla.empty_launch(wl.B, wl.H, wl.grid_h, wl.grid_w, stream=stream)
    except gla.GLAError:
        return None
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(stream):
        with torch.cuda.graph(g, stream=stream):
            for _ in range(launches):
                gla.empty_launch(wl.B, wl.H, wl.grid_h, wl.grid_w, stream=stream)
        g.replay()
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    reps = 5
    with torch.cuda.stream(stream):
        e0.record(stream)
        for _ in range(reps):
            g.replay()
        e1.record(stream)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) * 1e3 / (reps * launches)


def run_ours(args, ws, rank, local):
    import numpy as np
    import torch
    import torch.distributed as dist
    from recurrent_vision_backbone_only_b200 import build as _b, gla, synth

    _b.build()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    wl = synth.WORKLOADS[args.workload]
    x = synth.make_inputs(wl)
    gh, gw = wl.grid_h, wl.grid_w
    directions = wl.directions if args.workload != WORKLOAD else DIRECTIONS

    # rotating pool of input sets, total larger than L2
    set_bytes = wl.tokens * wl.bytes_per_token
    n_sets = max(2 if set_bytes > L2_BYTES else 8, math.ceil(2 * L2_BYTES / set_bytes))
    base = {n: torch.from_numpy(x[n]).to(dev) for n in ("q", "k", "v", "a", "g")}
    w = torch.from_numpy(x["w"]).to(dev)
    sets = []
    for _ in range(n_sets):
        s = {n: base[n].clone() for n in base}
        s["out"] = torch.empty_like(base["v"])
        sets.append(s)
    launches_per_step = len(directions)
    dt = torch.float16 if wl.dtype == "f16" else torch.float32

    kernel = {"auto": 0, "tc128": gla.KERNEL_TC128, "tc64": gla.KERNEL_TC64,
              "pipe64": gla.KERNEL_PIPE64, "simt": gla.KERNEL_SIMT}[args.kernel]
    kernel_name = (gla.KERNEL_NAMES[kernel] if kernel else
                   gla.plan(wl.B, wl.H, gh, gw, wl.d_k, wl.d_v, 0 if wl.dtype == "f16" else 1)["kernel"])
    # kernel launches per gla_fwd call: two when the library splits off a partial wave (its
    # plan then has more CTAs than pairs x segments); gla_fwd_ex with an explicit kernel and
    # automatic segments splits the same way
    _pl = gla.plan(wl.B, wl.H, gh, gw, wl.d_k, wl.d_v, 0 if wl.dtype == "f16" else 1)
    calls_split = (_pl["kernel"] == kernel_name and
                   _pl["ctas"] > wl.B * wl.H * _pl["segments"])

    def step(i):
        for j, d in enumerate(directions):
            s = sets[(i * launches_per_step + j) % n_sets]
            if kernel:
                gla.gla_fwd_ex(s["q"], s["k"], s["v"], s["a"], s["g"], w, s["out"], gh, gw, d,
                               kernel=kernel)
            else:
                gla.gla_fwd(s["q"], s["k"], s["v"], s["a"], s["g"], w, s["out"], gh, gw, d)

    stream = torch.cuda.Stream(device=dev)
    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        for i in range(args.warmup):
            step(i)
    torch.cuda.synchronize()
    if gla.get_status(stream) != 0:
        raise RuntimeError("device status set during warm-up")

    # capture the K timed steps as replays of a graph of G steps (+ a remainder graph)
    K = args.steps
    G = min(K, 100)
    graphs = []
    with torch.cuda.stream(stream):
        g_main = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g_main, stream=stream):
            for i in range(G):
                step(i)
        rem = K % G
        g_rem = None
        if rem:
            g_rem = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g_rem, stream=stream):
                for i in range(rem):
                    step(i)
    plan = [g_main] * (K // G) + ([g_rem] if g_rem is not None else [])
    with torch.cuda.stream(stream):
        g_main.replay()                     # untimed: graph upload
        if g_rem is not None:
            g_rem.replay()
    torch.cuda.synchronize()

    ev0 = torch.cuda.Event(enable_timing=True)
    ev1 = torch.cuda.Event(enable_timing=True)
    if ws > 1:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        with torch.cuda.stream(stream):
            ev0.record(stream)
            for gr in plan:
                gr.replay()
            ev1.record(stream)
        torch.cuda.synchronize()
    if ws > 1:
        dist.barrier()
    elapsed_ms = ev0.elapsed_time(ev1)
    if gla.get_status(stream) != 0:
        raise RuntimeError("device status set during the timed region")
    max_ms = max_over_ranks(elapsed_ms, dev)

    tokens_per_step = wl.tokens * launches_per_step
    value = job_throughput(tokens_per_step, K, ws, max_ms)
    launch_s = (elapsed_ms / 1e3) / (K * launches_per_step)
    bytes_per_launch = wl.tokens * wl.bytes_per_token
    peak, peak_kind = measured_peaks()
    achieved = bytes_per_launch / launch_s / 1e9

    # ---- e2e through the public host-buffer entry point (H2D + kernel + D2H) ----
    e2e_steps = max(1, min(args.e2e_steps, K))
    hx = {n: torch.from_numpy(np.ascontiguousarray(x[n])).pin_memory()
          for n in ("q", "k", "v", "a", "g", "w")}
    hout = torch.empty(tuple(x["v"].shape), dtype=dt).pin_memory()
    with torch.cuda.stream(stream):
        for d in directions:  # warm the staging buffers
            gla.gla_fwd_host(hx["q"], hx["k"], hx["v"], hx["a"], hx["g"], hx["w"], hout, gh, gw,
                             d, stream=stream)
        if ws > 1:
            dist.barrier()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for i in range(e2e_steps):
            for d in directions:
                gla.gla_fwd_host(hx["q"], hx["k"], hx["v"], hx["a"], hx["g"], hx["w"], hout, gh,
                                 gw, d, stream=stream)
        e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), dev)
    h2d = launches_per_step * sum(hx[n].numel() * hx[n].element_size()
                                  for n in ("q", "k", "v", "a", "g", "w"))
    d2h = launches_per_step * hout.numel() * hout.element_size()
    e2e = {"value": job_throughput(tokens_per_step, e2e_steps, ws, e2e_ms), "unit": "Mtokens/s",
           "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
           "steps": e2e_steps, "ms_per_step": e2e_ms / e2e_steps}

    tc_shape = wl.dtype == "f16" and wl.d_k == 64 and wl.d_v == 64
    floor_us = launch_floor_us(gla, wl, stream, G * launches_per_step) if tc_shape else None
    if gla.get_status(stream) != 0:
        raise RuntimeError("device status set by the launch-floor measurement")

    if rank != 0:
        return
    clocks = clk.summary()
    dnames = {0: "L2R", 1: "R2L", 2: "T2B", 3: "B2T", 4: "cycle b%4"}
    line = {
        "metric": METRIC if args.workload == WORKLOAD else
                  "GLA fwd Mtokens/s (B·H·L), %s workload" % wl.name, "value": value, "unit": "Mtokens/s", "n_gpus": ws, "steps": K,
        "warmup": args.warmup, "ms_per_step": max_ms / K, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": wl.dtype, "data": "synthetic",
        "config": {
            "workload": "%s: %dx%d patch grid (L=%d), B=%d, H=%d, d_k=d_v=%d, %s I/O, fp32 "
                        "accumulation; one step = %d launch(es) (%s)"
                        % (wl.name, gh, gw, wl.L, wl.B, wl.H, wl.d_k, wl.dtype, launches_per_step,
                           ", ".join(dnames[d] for d in directions)),
            "tokens_per_step": tokens_per_step,
            "l2": "rotating pool of %d input sets (%.0f MB > 126 MB L2); no flush kernel"
                  % (n_sets, n_sets * set_bytes / 1e6),
            "timing": "CUDA-graph replays (graphs of %d steps), CUDA events on the launch "
                      "stream; warm-up = %d eager steps + one untimed replay" % (G, args.warmup),
            "parallelism": "replicas" if ws > 1 else "single GPU",
            "schedule": gla.plan(wl.B, wl.H, gh, gw, wl.d_k, wl.d_v, 0 if wl.dtype == "f16" else 1)
                        if not kernel else {"kernel": gla.KERNEL_NAMES[kernel]},
        },
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak,
                     "traffic": profile_traffic(wl.name, kernel_name),
                     "peak_source": "%s (MEASURED_PEAKS.json hbm_gbs)" % peak_kind
                     if peak_kind == "measured" else "fallback 6.65 TB/s",
                     "bytes_per_launch": bytes_per_launch,
                     "launch_us": launch_s * 1e6,
                     "launch_floor_us": floor_us,
                     "launch_floor": "do-nothing kernel, same launch shape, same graph replay"},
        "e2e": e2e,
        "gpu_launches": K * launches_per_step * (2 if calls_split else 1),
        "clocks": clocks,
    }
    if ws == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_oracle_sample(wl, x, args.cpu_seconds, directions)
    print(json.dumps(line), flush=True)


class AuxOp:
    """One of the steps next to the operator, timed like it: `step(i)` launches on the current
    stream with device-resident input set i mod the pool, `e2e_step()` copies a host input
    set in, launches, and copies the result out."""

    def __init__(self, **kw):
        self.__dict__.update(kw)


def gate_op(args, wl, dev):
    """gla_gate_proj (the retention gate's low-rank projection) on the workload's tokens."""
    import torch
    from recurrent_vision_backbone_only_b200 import gla, synth
    T, d, n = gate_shape(wl, args.d_model)
    inp = synth.make_gate_inputs(T, d, n, seed=wl.seed)
    w1, w2, b = (torch.from_numpy(inp[k]).to(dev) for k in ("w1", "w2", "b"))
    set_bytes = 2 * T * (d + n)
    n_sets = max(2 if set_bytes > L2_BYTES else 8, math.ceil(2 * L2_BYTES / set_bytes))
    x0 = torch.from_numpy(inp["x"]).to(dev)
    sets = [(x0.clone(), torch.empty((T, n), dtype=torch.float16, device=dev)) for _ in range(n_sets)]
    hx = torch.from_numpy(inp["x"]).pin_memory()
    ha = torch.empty((T, n), dtype=torch.float16).pin_memory()

    def step(i):
        xs, a = sets[i % n_sets]
        gla.gate_proj(xs, w1, w2, b, a)

    def e2e_step():
        xs, a = sets[0]
        xs.copy_(hx, non_blocking=True)
        gla.gate_proj(xs, w1, w2, b, a)
        ha.copy_(a, non_blocking=True)

    return AuxOp(
        name="gate", kernel=GATE_KERNEL, tokens=T, bytes_per_launch=gate_bytes(wl, d), step=step,
        e2e_step=e2e_step, h2d=hx.numel() * 2, d2h=ha.numel() * 2, n_sets=n_sets, set_bytes=set_bytes,
        metric="gate projection Mtokens/s (B·L), %s workload" % wl.name,
        workload="%s tokens: a = x W1 W2 + b, tokens=%d (B=%d x %dx%d), d_model=%d, rank=%d, "
                 "n_out=H*d_k=%d, fp16 I/O, fp32 accumulation; one step = 1 launch"
                 % (wl.name, T, wl.B, wl.grid_h, wl.grid_w, d, GATE_RANK, n),
        cpu=lambda budget: cpu_gate_sample(inp, budget))


def sswiglu_op(args, wl, dev):
    """gla_sswiglu (Spatial SwiGLU's dwconv + gating step) on the workload's grid, with
    channels = expansion 4 x the model width."""
    import torch
    from recurrent_vision_backbone_only_b200 import gla, synth
    B, gh, gw, C = wl.B, wl.grid_h, wl.grid_w, SSWIGLU_EXPANSION * args.d_model
    inp = synth.make_sswiglu_inputs(B, gh, gw, C, seed=wl.seed)
    cw, cb = (torch.from_numpy(inp[k]).to(dev) for k in ("conv_w", "conv_b"))
    set_bytes = 3 * B * gh * gw * C * 2
    n_sets = max(2 if set_bytes > L2_BYTES else 8, math.ceil(2 * L2_BYTES / set_bytes))
    v0, g0 = (torch.from_numpy(inp[k]).to(dev) for k in ("value", "gate"))
    sets = [(v0.clone(), g0.clone(), torch.empty_like(v0)) for _ in range(n_sets)]
    hv, hg = (torch.from_numpy(inp[k]).pin_memory() for k in ("value", "gate"))
    hh = torch.empty(tuple(hv.shape), dtype=torch.float16).pin_memory()

    def step(i):
        v, g, h = sets[i % n_sets]
        gla.sswiglu(v, g, cw, cb, h, gh, gw)

    def e2e_step():
        v, g, h = sets[0]
        v.copy_(hv, non_blocking=True)
        g.copy_(hg, non_blocking=True)
        gla.sswiglu(v, g, cw, cb, h, gh, gw)
        hh.copy_(h, non_blocking=True)

    return AuxOp(
        name="sswiglu", kernel=SSWIGLU_KERNEL, tokens=B * gh * gw, bytes_per_launch=sswiglu_bytes(wl, args.d_model),
        step=step, e2e_step=e2e_step, h2d=2 * hv.numel() * 2, d2h=hh.numel() * 2, n_sets=n_sets,
        set_bytes=set_bytes,
        metric="Spatial SwiGLU mix Mtokens/s (B·L), %s workload" % wl.name,
        workload="%s grid: h = SiLU(gate) * (DWConv3x3(value) + b), B=%d, %dx%d, channels=%d "
                 "(expansion %d x d_model %d), fp16 I/O, fp32 arithmetic; one step = 1 launch"
                 % (wl.name, B, gh, gw, C, SSWIGLU_EXPANSION, args.d_model),
        cpu=lambda budget: cpu_sswiglu_sample(inp, gh, gw, budget))


def linear_op(args, wl, dev, side):
    """gla_linear as the block's input side (x -> q, k, v and the output gate's pre-activation,
    four [B][L][H][d] parts) or output side (the concatenated heads -> the model width)."""
    import torch
    from recurrent_vision_backbone_only_b200 import gla, synth
    T, d, n = wl.B * wl.L, args.d_model, wl.H * wl.d_k
    rows, K, N, n_part = (T, d, 4 * n, n) if side == "in" else (T, wl.H * wl.d_v, d, d)
    inp = synth.make_linear_inputs(rows, K, N, seed=wl.seed)
    w = torch.from_numpy(inp["w"]).to(dev)
    set_bytes = 2 * rows * (K + N)
    n_sets = max(2 if set_bytes > L2_BYTES else 8, math.ceil(2 * L2_BYTES / set_bytes))
    x0 = torch.from_numpy(inp["x"]).to(dev)
    sets = [(x0.clone(), torch.empty((N // n_part, rows, n_part), dtype=torch.float16, device=dev))
            for _ in range(n_sets)]
    hx = torch.from_numpy(inp["x"]).pin_memory()
    hy = torch.empty((N // n_part, rows, n_part), dtype=torch.float16).pin_memory()

    def step(i):
        xs, y = sets[i % n_sets]
        gla.linear(xs, w, y, n_part=n_part)

    def e2e_step():
        xs, y = sets[0]
        xs.copy_(hx, non_blocking=True)
        gla.linear(xs, w, y, n_part=n_part)
        hy.copy_(y, non_blocking=True)

    what = ("x -> q, k, v, W_r pre-activation (4 parts of H*d_k=%d)" % n if side == "in"
            else "concatenated heads (H*d_v=%d) -> d_model" % K)
    return AuxOp(
        name="proj_" + side, kernel="%s, %s side" % (LINEAR_KERNEL, "input" if side == "in" else "output"), tokens=rows, bytes_per_launch=linear_bytes(rows, K, N),
        flops_per_launch=2 * rows * K * N, step=step, e2e_step=e2e_step, h2d=hx.numel() * 2,
        d2h=hy.numel() * 2, n_sets=n_sets, set_bytes=set_bytes,
        metric="%s projection Mtokens/s (B·L), %s workload" % ("input" if side == "in" else "output", wl.name),
        workload="%s tokens: %s, rows=%d (B=%d x %dx%d), K=%d, N=%d, fp16 I/O, fp32 accumulation; "
                 "one step = 1 launch" % (wl.name, what, rows, wl.B, wl.grid_h, wl.grid_w, K, N),
        cpu=lambda budget: cpu_linear_sample(inp, budget))


def aux_roofline(bytes_per_launch: int, flops_per_launch: int, launch_s: float, hbm, tensor):
    """Roofline entry for one launch: HBM-bound unless its FLOPs need more time on the tensor
    roof than its bytes need on the HBM roof.  hbm = (GB/s, kind), tensor = (TFLOP/s, kind)."""
    peak, peak_kind = hbm
    achieved = bytes_per_launch / launch_s / 1e9
    roof = {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
            "peak_source": "%s (MEASURED_PEAKS.json hbm_gbs)" % peak_kind
            if peak_kind == "measured" else "fallback 6.65 TB/s"}
    if flops_per_launch:
        tpeak, tkind = tensor
        if flops_per_launch / (tpeak * 1e12) > bytes_per_launch / (peak * 1e9):
            ta = flops_per_launch / launch_s / 1e12
            roof = {"bound": "tensor", "achieved": ta, "peak": tpeak, "unit": "TFLOP/s", "frac": ta / tpeak,
                    "peak_source": "%s (MEASURED_PEAKS.json bf16_tflops; fp16 runs at the same nominal "
                                   "dense rate)" % tkind if tkind == "measured" else "fallback 1.59 PFLOP/s",
                    "hbm_achieved_gbs": achieved, "hbm_frac": achieved / peak}
        roof["flops_per_launch"] = flops_per_launch
    return roof


def run_aux(args, ws, rank, local):
    """Time one of the steps next to the operator (--op gate / sswiglu / proj_in / proj_out) like
    the operator."""
    import torch
    import torch.distributed as dist
    from recurrent_vision_backbone_only_b200 import build as _b, gla, synth

    _b.build()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    wl = synth.WORKLOADS[args.workload]
    op = {"gate": gate_op, "sswiglu": sswiglu_op,
          "proj_in": lambda a, w_, d_: linear_op(a, w_, d_, "in"),
          "proj_out": lambda a, w_, d_: linear_op(a, w_, d_, "out")}[args.op](args, wl, dev)

    stream = torch.cuda.Stream(device=dev)
    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        for i in range(args.warmup):
            op.step(i)
    if gla.get_status(stream) != 0:
        raise RuntimeError("device status set during warm-up")
    K = args.steps
    G = min(K, 100)
    with torch.cuda.stream(stream):
        g_main = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g_main, stream=stream):
            for i in range(G):
                op.step(i)
        g_rem = None
        if K % G:
            g_rem = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g_rem, stream=stream):
                for i in range(K % G):
                    op.step(i)
        g_main.replay()
        if g_rem is not None:
            g_rem.replay()
    torch.cuda.synchronize()
    plan = [g_main] * (K // G) + ([g_rem] if g_rem is not None else [])
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if ws > 1:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        with torch.cuda.stream(stream):
            ev0.record(stream)
            for gr in plan:
                gr.replay()
            ev1.record(stream)
        torch.cuda.synchronize()
    if ws > 1:
        dist.barrier()
    if gla.get_status(stream) != 0:
        raise RuntimeError("device status set during the timed region")
    max_ms = max_over_ranks(ev0.elapsed_time(ev1), dev)
    value = job_throughput(op.tokens, K, ws, max_ms)
    launch_s = max_ms / 1e3 / K
    roof = aux_roofline(op.bytes_per_launch, getattr(op, "flops_per_launch", 0), launch_s,
                        measured_peaks(), measured_tensor_peak())

    # e2e: inputs from pinned host memory, the launch, the result back to pinned host memory
    e2e_steps = max(1, min(args.e2e_steps, K))
    with torch.cuda.stream(stream):
        op.e2e_step()
        if ws > 1:
            dist.barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(e2e_steps):
            op.e2e_step()
        e1.record(stream)
    torch.cuda.synchronize()
    if gla.get_status(stream) != 0:
        raise RuntimeError("device status set during the e2e region")
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), dev)
    if rank != 0:
        return
    line = {
        "metric": op.metric, "value": value,
        "unit": "Mtokens/s", "n_gpus": ws, "steps": K, "warmup": args.warmup,
        "ms_per_step": max_ms / K, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f16", "data": "synthetic",
        "config": {
            "workload": op.workload,
            "tokens_per_step": op.tokens,
            "l2": "rotating pool of %d input/output sets (%.0f MB > 126 MB L2); no flush kernel"
                  % (op.n_sets, op.n_sets * op.set_bytes / 1e6),
            "timing": "CUDA-graph replays (graphs of %d steps), CUDA events on the launch stream"
                      % G,
            "parallelism": "replicas" if ws > 1 else "single GPU",
        },
        "roofline": dict(roof, traffic=profile_traffic(wl.name, op.kernel),
                         bytes_per_launch=op.bytes_per_launch, launch_us=launch_s * 1e6),
        "e2e": {"value": job_throughput(op.tokens, e2e_steps, ws, e2e_ms), "unit": "Mtokens/s",
                "h2d_bytes_per_step": op.h2d, "d2h_bytes_per_step": op.d2h,
                "steps": e2e_steps, "ms_per_step": e2e_ms / e2e_steps},
        "gpu_launches": K,
        "clocks": clk.summary(),
    }
    if ws == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = op.cpu(args.cpu_seconds)
    print(json.dumps(line), flush=True)


def cpu_gate_sample(inp, budget_s: float):
    """The oracle's gate projection (fp64) timed on the host over repeated whole-input calls
    until about a tenth of the budget has passed."""
    import oracle
    x, w1, w2, b = (inp[k].astype("float64") for k in ("x", "w1", "w2", "b"))
    t0 = time.perf_counter()
    calls = 0
    while True:
        oracle.gate_projection(x, w1, w2, b)
        calls += 1
        el = time.perf_counter() - t0
        if el >= budget_s / 10:
            break
    return {"value": calls * x.shape[0] / el / 1e6, "unit": "Mtokens/s",
            "cores": os.cpu_count(), "kind": "oracle",
            "sample": "%d whole-input calls of the fp64 oracle (numpy matmuls, %d tokens each)"
                      % (calls, x.shape[0])}


def cpu_linear_sample(inp, budget_s: float):
    """The oracle's dense projection (fp64 numpy matmul) over the whole input, repeated until
    about a tenth of the budget has passed."""
    import oracle
    x, w = inp["x"].astype("float64"), inp["w"].astype("float64")
    t0 = time.perf_counter()
    calls = 0
    while True:
        oracle.linear(x, w)
        calls += 1
        el = time.perf_counter() - t0
        if el >= budget_s / 10:
            break
    return {"value": calls * x.shape[0] / el / 1e6, "unit": "Mtokens/s", "cores": os.cpu_count(),
            "kind": "oracle", "sample": "%d whole-input calls of the fp64 oracle (numpy matmul, %d x %d x %d)"
                                        % (calls, x.shape[0], x.shape[1], w.shape[1])}


def cpu_sswiglu_sample(inp, gh: int, gw: int, budget_s: float):
    """The oracle's Spatial SwiGLU mixing step (fp64 numpy) on the first image, repeated until
    about a tenth of the budget has passed."""
    import oracle
    v, g, w, b = (inp[k][:1].astype("float64") if k in ("value", "gate") else inp[k].astype("float64")
                  for k in ("value", "gate", "conv_w", "conv_b"))
    t0 = time.perf_counter()
    calls = 0
    while True:
        oracle.spatial_swiglu_mix(v, g, w, b, gh, gw)
        calls += 1
        el = time.perf_counter() - t0
        if el >= budget_s / 10:
            break
    return {"value": calls * gh * gw / el / 1e6, "unit": "Mtokens/s", "cores": os.cpu_count(),
            "kind": "oracle",
            "sample": "%d calls of the fp64 oracle (numpy) on one %dx%d image of %d channels"
                      % (calls, gh, gw, v.shape[2])}


def main():
    args = parse()
    ws, rank, local = dist_env()
    if args.record_traffic:
        record_traffic(args)
        return
    if args.impl == "reference":
        run_reference(args, ws, rank)
        return
    if ws > 1:
        import datetime
        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    try:
        (run_ours if args.op == "gla" else run_aux)(args, ws, rank, local)
    finally:
        if ws > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
