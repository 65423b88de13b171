"""Benchmark of the QMoE forward on B200 (one JSON line on rank 0).

Default workload: Mixtral-like decode (T=8, H=4096, I=14336, E=8, k=2, int4
block_size 128, bf16 activations and scales, swiglu fused not interleaved,
renormalised routing), seeded synthetic inputs. One step = one whole forward
(routing, permutation, FC1 + SwiGLU, FC2, combine) over the batch, launched
as one CUDA graph replay; the JSON line also gives the step time with direct
launches, the per-kernel times of a separate event-bracketed pass, and the
end-to-end rate through the public call with host buffers.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
    python bench.py --impl reference ...   # the CPU oracle, timed on host cores

With N > 1 (torchrun) every rank runs an independent replica on its own
token batch (tokens are independent; no collective on the data path) and the
job throughput is all ranks' tokens over the slowest rank's time.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from weight_only_quantized_warp_b200 import inputs as gen  # noqa: E402

METRIC = "QMoE fwd tokens/s; HBM GB/s (decode) / TFLOP/s (prefill) vs roofline"
L2_BYTES = 126 * 2**20
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="mixtral_decode")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--path", type=int, default=None,
                    help="force the expert-FFN kernels: 1 mma.sync streaming, 2 tcgen05 GEMM, "
                         "3 tcgen05 streaming (default: by shape)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-sample-tokens", type=int, default=0,
                    help="tokens in the CPU-baseline sample (0: whole batch, capped by time)")
    return ap.parse_args()


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def config_of(cfg, name, world):
    return {"workload": name, "T": cfg.T, "H": cfg.H, "I": cfg.I, "E": cfg.E, "k": cfg.k,
            "bits": cfg.bits, "block_size": cfg.block_size, "swiglu_fusion": cfg.fusion,
            "act_dtype": "bf16" if cfg.act_dtype == gen.DT_BF16 else "f32",
            "compute": "int8 block tier" if cfg.compute_mode == gen.COMPUTE_INT8_BLOCK else "float",
            "tokens_per_step": cfg.T * world, "parallelism": f"replicas x{world}",
            "l2": "no flush: the expert weights a step streams exceed the 126 MB L2"}


def launch_names(path, launches, weights_on_input):
    """Names of the forward's launches in order, for a path and the launch
    count the library reports: routing and permutation (one launch or two),
    the row gather (tensor-core paths, or router weights on the input), the
    int8 tier's two rounding launches, FC1, FC2 and the combine."""
    from weight_only_quantized_warp_b200 import qmoe
    gather = path in (qmoe.PATH_TC, qmoe.PATH_TC_DECODE) or weights_on_input
    ffn = ["quantize_x", "fc1", "quantize_h", "fc2"] if path == qmoe.PATH_INT8 else ["fc1", "fc2"]
    routing = launches - int(gather) - len(ffn) - 1
    if routing not in (1, 2):
        raise ValueError(f"{launches} launches do not fit path {path}")
    return ((["route_permute"] if routing == 1 else ["route", "permute"]) + (["gather"] if gather else [])
            + ffn + ["combine"])


def algorithmic(cfg, offsets):
    """Algorithmic bytes / FLOPs of one forward, from the routing (experts
    with at least one routed row count once)."""
    counts = np.diff(offsets)
    touched = int((counts > 0).sum())
    ssz = {gen.DT_F32: 4, gen.DT_BF16: 2, gen.DT_E8M0: 1}[cfg.scale_dtype]
    asz = 2 if cfg.act_dtype == gen.DT_BF16 else 4
    n1 = cfg.n1 + (cfg.I if cfg.has_fc3 else 0)
    nsb1 = cfg.H // cfg.block_size if cfg.block_size else 1
    nsb2 = cfg.I // cfg.block_size if cfg.block_size else 1
    fc1 = n1 * cfg.H * cfg.bits // 8 + n1 * nsb1 * ssz + (n1 * asz if cfg.has_fc1_bias else 0)
    fc2 = cfg.H * cfg.I * cfg.bits // 8 + cfg.H * nsb2 * ssz + (cfg.H * asz if cfg.has_fc2_bias else 0)
    R = cfg.T * cfg.k
    act_fc1 = cfg.T * cfg.H * asz + R * cfg.I * asz                # x in, h out
    io = cfg.T * cfg.H * asz * (2 + int(cfg.has_shared)) + cfg.T * cfg.E * asz
    flops = 2 * R * 3 * cfg.H * cfg.I if (cfg.fusion or cfg.has_fc3) else 2 * R * 2 * cfg.H * cfg.I
    return dict(touched=touched, fc1_bytes=touched * fc1 + act_fc1, fc2_bytes=touched * fc2,
                total_bytes=touched * (fc1 + fc2) + io, flops=flops,
                fc1_per_expert=fc1, fc2_per_expert=fc2)


class ClockSampler:
    """nvidia-smi clocks and throttle reasons during the timed region."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        # raw samples: QMOE_CLOCKS_DIR if set, else the system temp directory
        folder = os.environ.get("QMOE_CLOCKS_DIR") or tempfile.gettempdir()
        self.path = os.path.join(folder, f"clocks_bench_{os.getpid()}.csv")

    def start(self):
        try:
            os.makedirs(os.path.dirname(self.path), exist_ok=True)
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.Q}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=self.f, stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.f.close()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        loaded = [s for s in sm if mx and s > 0.5 * max(mx)] or sm
        return {"sm_mhz": statistics.median(loaded) if loaded else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons, "samples": len(rows)}


def traffic_record(kernel_key):
    """Per-launch DRAM bytes of the dominant kernel from a committed ncu
    summary, valid only while the kernel's source is unchanged."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f).get(kernel_key)
    if not d:
        return None
    return d if source_digest(d["source"]) == d.get("sha256_16") else None


def source_digest(sources):
    """First 16 hex digits of the sha256 over the named csrc files, in order."""
    h = hashlib.sha256()
    for name in ([sources] if isinstance(sources, str) else sources):
        with open(os.path.join(ROOT, "weight_only_quantized_warp_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


# ---------------------------------------------------------------- reference arm

def cpu_oracle_timing(inp, tokens, budget_s=20.0):
    """Time the CPU oracle on a bounded sample of the workload's tokens:
    repeated calls on ``tokens`` until about ``budget_s`` / 2 has passed."""
    import oracle
    t0 = time.perf_counter()
    done = 0
    while True:
        oracle.forward(inp, tokens=tokens)
        done += len(tokens)
        if time.perf_counter() - t0 >= budget_s / 2:
            break
    el = time.perf_counter() - t0
    return done / el, el, done, oracle.num_threads()


def run_reference(args):
    ws, rank, _ = dist_env()
    if rank != 0:
        return 0
    import oracle
    cfg, seed, kw = gen.workload(args.workload)
    inp = gen.make_inputs(cfg, seed, **kw)
    ntok = args.cpu_sample_tokens or 1
    rng = np.random.default_rng(0)
    samples = [sorted(rng.choice(cfg.T, size=min(ntok, cfg.T), replace=False).tolist())
               for _ in range(args.warmup + args.steps)]
    for s in samples[:args.warmup]:
        oracle.forward(inp, tokens=s)
    times = []
    for s in samples[args.warmup:]:
        t0 = time.perf_counter()
        oracle.forward(inp, tokens=s)
        times.append(time.perf_counter() - t0)
    total = sum(times)
    tok = ntok * args.steps
    value = tok / total
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * total / args.steps, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded)",
            "config": config_of(cfg, args.workload, 1),
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": oracle.num_threads(),
                             "kind": "oracle",
                             "sample": f"{ntok} token(s) of the {cfg.T}-token batch per step"},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------------- our arm

def run_ours(args):
    import torch
    import torch.distributed as dist
    from weight_only_quantized_warp_b200 import qmoe, replicas

    world, rank, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)

    # every replica: the same weights, its own token batch
    inp = replicas.replica_inputs(args.workload, rank)
    cfg = inp.cfg

    m = qmoe.QMoE(cfg, dev, path=args.path)
    m.set_weights_from(inp)
    x = qmoe.to_device(inp.x, dev)
    lg = qmoe.to_device(inp.logits, dev)
    sh = qmoe.to_device(inp.shared, dev)
    y = torch.empty_like(x)
    T = cfg.T
    ws = m.workspace(T)
    nws = ws.numel()
    h = m.handle
    launches = qmoe.qmoe_launches_for(h, T)
    stream = torch.cuda.current_stream()

    def fwd():
        qmoe.qmoe_forward(h, T, x, lg, sh, y, ws, nws, stream)

    # warm-up
    for _ in range(max(args.warmup, 3)):
        fwd()
    torch.cuda.synchronize()

    # one step = one forward, replayed from a CUDA graph (the forward enqueues
    # only stream-ordered device work, so it captures as is)
    graph = torch.cuda.CUDAGraph()
    # captures on a side stream and replays on `stream`; thread-local capture
    # so that other threads' CUDA calls (a process group's watchdog) are not
    # treated as part of the capture
    with torch.cuda.graph(graph, capture_error_mode="thread_local"):
        qmoe.qmoe_forward(h, T, x, lg, sh, y, ws, nws, torch.cuda.current_stream())
    for _ in range(3):
        graph.replay()
    torch.cuda.synchronize()

    # routing of this batch (for the algorithmic byte count)
    off = torch.empty(cfg.E + 1, dtype=torch.int32, device=dev)
    qmoe.qmoe_debug_routing(h, T, ws, offsets=off)
    alg = algorithmic(cfg, off.cpu().numpy())

    # ---- timed region: K whole forwards, events per kernel on this stream
    K = args.steps
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(launches + 1)] for _ in range(K)]
    for row in evs:
        for e in row:
            e.record(stream)  # materialise the event handles
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(local)

    def keep_loaded(seconds):
        # the same forward, back to back, so clock samples bracket the timed
        # region under its own load (a short region ends between samples)
        t_end = time.perf_counter() + seconds
        while time.perf_counter() < t_end:
            for _ in range(20):
                graph.replay()
            torch.cuda.synchronize()

    clocks.start()
    keep_loaded(0.6)
    if world > 1:
        dist.barrier(device_ids=[local])
    torch.cuda.synchronize()
    start.record(stream)
    for i in range(K):
        graph.replay()
    stop.record(stream)
    torch.cuda.synchronize()
    keep_loaded(0.4)
    clk = clocks.stop()
    if clk is not None:
        clk["window"] = "timed region bracketed by 0.6 s / 0.4 s of the same forward"
    ms = replicas.max_over_ranks([start.elapsed_time(stop)], dev)[0]
    if world > 1:
        dist.barrier(device_ids=[local])

    # after the timed region: the same K steps as direct launches, and once
    # more with an event between kernels for the per-kernel times (the events
    # themselves add a few microseconds per launch)
    s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s0.record(stream)
    for i in range(K):
        fwd()
    s1.record(stream)
    for i in range(K):
        qmoe.qmoe_forward_profiled(h, T, x, lg, sh, y, ws, nws, evs[i], stream)
    torch.cuda.synchronize()
    stream_ms = replicas.max_over_ranks([s0.elapsed_time(s1)], dev)[0]
    del graph
    if world > 1:
        dist.barrier(device_ids=[local])
    per_kernel = np.array([[evs[i][j].elapsed_time(evs[i][j + 1]) for j in range(launches)]
                           for i in range(K)]).mean(axis=0)
    path = qmoe.qmoe_path_for(h, T)
    i8 = path == qmoe.PATH_INT8
    names = launch_names(path, launches, bool(cfg.apply_router_weight_on_input))

    # ---- end to end through the public call, host buffers, copies inside
    x_h = torch.empty(x.shape, dtype=x.dtype, pin_memory=True).copy_(x.cpu())
    lg_h = torch.empty(lg.shape, dtype=lg.dtype, pin_memory=True).copy_(lg.cpu())
    sh_h = None if sh is None else torch.empty(sh.shape, dtype=sh.dtype, pin_memory=True).copy_(sh.cpu())
    y_h = torch.empty(y.shape, dtype=y.dtype, pin_memory=True)
    x_d, lg_d = torch.empty_like(x), torch.empty_like(lg)
    sh_d = None if sh is None else torch.empty_like(sh)

    def e2e_step():
        x_d.copy_(x_h, non_blocking=True)
        lg_d.copy_(lg_h, non_blocking=True)
        if sh_d is not None:
            sh_d.copy_(sh_h, non_blocking=True)
        qmoe.qmoe_forward(h, T, x_d, lg_d, sh_d, y, ws, nws, stream)
        y_h.copy_(y, non_blocking=True)

    for _ in range(3):
        e2e_step()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier(device_ids=[local])
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(K):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = replicas.max_over_ranks([e0.elapsed_time(e1)], dev)[0]
    h2d = x_h.numel() * x_h.element_size() + lg_h.numel() * lg_h.element_size() + (
        0 if sh_h is None else sh_h.numel() * sh_h.element_size())
    d2h = y_h.numel() * y_h.element_size()

    # ---- CPU baseline (rank 0, N = 1 only)
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        ntok = args.cpu_sample_tokens or min(T, 8)
        rng = np.random.default_rng(1)
        toks = sorted(rng.choice(T, size=ntok, replace=False).tolist())
        v, el, done, cores = cpu_oracle_timing(inp, toks)
        cpu = {"value": v, "unit": "tokens/s", "cores": cores, "kind": "oracle",
               "sample": f"{done} tokens ({ntok} per call) of the {T}-token batch, {el:.1f} s"}

    if world > 1:
        dist.destroy_process_group()
    if rank != 0:
        return 0

    peaks, peaks_kind = load_peaks()
    kms = dict(zip(names, [float(v) for v in per_kernel]))
    fc1_ms = kms["fc1"]
    step_ms = ms / K
    value = replicas.job_tokens_per_s(T, world, K, ms)
    # dominant kernel by algorithmic work: FC1 (gate + up rows); its bound is
    # the slower of its bytes at HBM bandwidth and its FLOPs at bf16 peak
    hbm_peak = float(peaks["hbm_gbs"])
    tc_peak = float(peaks["bf16_tflops"])
    fc1_flops = 2.0 * cfg.T * cfg.k * (cfg.n1 + (cfg.I if cfg.has_fc3 else 0)) * cfg.H
    t_hbm = alg["fc1_bytes"] / (hbm_peak * 1e9)
    t_tc = fc1_flops / (tc_peak * 1e12)
    tile = qmoe.qmoe_token_tile_for(h, T)
    kbase = ("ffn_tc_wide_kernel" if tile > 128 else "ffn_tc_kernel") if path == qmoe.PATH_TC else \
        {qmoe.PATH_TC_DECODE: "ffn_tc_decode_kernel", qmoe.PATH_SIMT: "ffn_simt_kernel",
         qmoe.PATH_INT8: "ffn_i8_kernel"}.get(path, "ffn_decode_kernel")
    kname = kbase + " (FC1 + activation)"
    tr = traffic_record("fc1_" + kbase + "_" + args.workload)
    if t_hbm >= t_tc:
        achieved = alg["fc1_bytes"] / (fc1_ms / 1e3) / 1e9
        roofline = {"bound": "hbm", "achieved": achieved, "peak": hbm_peak, "unit": "GB/s",
                    "frac": achieved / hbm_peak, "algorithmic_bytes": alg["fc1_bytes"]}
    else:
        achieved = fc1_flops / (fc1_ms / 1e3) / 1e12
        roofline = {"bound": "tensor", "achieved": achieved, "peak": tc_peak, "unit": "TFLOP/s",
                    "frac": achieved / tc_peak, "algorithmic_flops": fc1_flops}
    roofline.update({"kernel": kname, "peak_kind": peaks_kind + (" (burst bf16)" if roofline["bound"] == "tensor" else ""),
                     "traffic": tr["bytes_per_launch"] if tr else None, "avg_launch_ms": fc1_ms,
                     "roofline_frac_of_step": max(alg["total_bytes"] / (hbm_peak * 1e9),
                                                  alg["flops"] / (tc_peak * 1e12)) / (ms / K / 1e3)})
    whole = alg["total_bytes"] / (step_ms / 1e3) / 1e9
    line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": K,
            "warmup": args.warmup, "ms_per_step": step_ms, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None,
            "dtype": "s8" if i8 else ("bf16" if cfg.act_dtype else "f32"),
            "data": "synthetic (seeded, shapes of the workload; no trained weights)",
            "config": config_of(cfg, args.workload, world),
            "roofline": roofline,
            "step": {"hbm_gbs": whole, "tflops": alg["flops"] / (step_ms / 1e3) / 1e12,
                     "hbm_frac": whole / hbm_peak, "experts_touched": alg["touched"],
                     "algorithmic_bytes": alg["total_bytes"],
                     "kernel_ms": kms, "path": path, "token_tile": tile,
                     "launch": "CUDA graph of one forward per step",
                     "ms_per_step_direct_launches": stream_ms / K,
                     "kernel_ms_note": "from a separate pass with an event between kernels"},
            "cpu_baseline": cpu,
            "e2e": {"value": replicas.job_tokens_per_s(T, world, K, e2e_ms), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h},
            "gpu_launches": launches * K,
            "clocks": clk}
    print(json.dumps(line), flush=True)
    return 0


def main():
    args = parse()
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
