"""Benchmark of the QMoE forward on B200 (one JSON line on rank 0).

Headline workload: the prefill sweep's largest shape (T=8192, H=4096,
I=14336, E=8, k=2, int4 block_size 64, bf16 activations and scales, swiglu
fused not interleaved, renormalised uniform-random routing), the largest
single-GPU configuration, bound by the tensor cores. The same line carries
the decode half of the metric as a nested record (Mixtral-like decode: T=8,
int4 block_size 128, bound by HBM bandwidth) with its own roofline, per-kernel
times and clocks, and the decode-to-compute crossover measured over T on the
headline's weights. Inputs are seeded synthetic draws of the shapes; no
trained weights.

One step = one whole forward (routing, permutation, row gather, FC1 + SwiGLU,
FC2, combine) over the batch, launched as one CUDA graph replay. The line
also gives the step time with direct launches, the per-kernel times of a
separate event-bracketed pass, and the end-to-end rate through the public
call with host buffers copied in and out inside the timed region.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
    python bench.py --impl reference ...   # the CPU oracle, timed on host cores

With N > 1 (torchrun) every rank runs an independent replica of the headline
workload on its own token batch (tokens are independent; no collective on the
data path) and the job throughput is all ranks' tokens over the slowest
rank's time; the nested decode record and the crossover run at N = 1 only.
"""
from __future__ import annotations

import argparse
import hashlib
import json
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
HEADLINE = "sweep_int4_T8192"
DECODE = "mixtral_decode"
CROSSOVER_T = (1, 16, 64, 128, 256, 512, 1024, 2048, 4096, 8192)
L2_BYTES = 126 * 2**20
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=HEADLINE)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--path", type=int, default=None,
                    help="force the expert-FFN kernels: 1 mma.sync streaming, 2 tcgen05 GEMM, "
                         "3 tcgen05 streaming (default: by shape)")
    ap.add_argument("--decode-workload", default=DECODE,
                    help="workload of the nested decode record ('none' to skip)")
    ap.add_argument("--no-crossover", action="store_true", help="skip the crossover sweep over T")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-sample-tokens", type=int, default=0,
                    help="tokens per oracle call in the CPU-baseline sample (0: 32, capped by the batch)")
    return ap.parse_args()


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def cpu_model():
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def l2_note(alg):
    if alg["weight_bytes"] > L2_BYTES:
        return "no flush: the expert weights a step streams exceed the 126 MB L2"
    return "weights fit L2 (not flushed between steps)"


def config_of(cfg, name, world, alg=None):
    d = {"workload": name, "T": cfg.T, "H": cfg.H, "I": cfg.I, "E": cfg.E, "k": cfg.k,
         "bits": cfg.bits, "block_size": cfg.block_size, "swiglu_fusion": cfg.fusion,
         "act_dtype": "bf16" if cfg.act_dtype == gen.DT_BF16 else "f32",
         "compute": "int8 block tier" if cfg.compute_mode == gen.COMPUTE_INT8_BLOCK else "float",
         "tokens_per_step": cfg.T * world, "parallelism": f"replicas x{world}"}
    if alg is not None:
        d["l2"] = l2_note(alg)
    return d


def launch_names(path, launches, weights_on_input):
    """Names of the forward's launches in order, for a path and the launch
    count the library reports: routing and permutation (one launch or two),
    the row gather (tensor-core paths, or router weights on the input), the
    int8 tier's two rounding launches, FC1, FC2 and the combine."""
    from weight_only_quantized_warp_b200 import qmoe
    gather = path in (qmoe.PATH_TC, qmoe.PATH_TC_DECODE, qmoe.PATH_INT8_TC) or weights_on_input
    int8_tier = path in (qmoe.PATH_INT8, qmoe.PATH_INT8_TC)
    ffn = ["quantize_x", "fc1", "quantize_h", "fc2"] if int8_tier else ["fc1", "fc2"]
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
    gated = cfg.fusion or cfg.has_fc3
    flops = 2 * R * 3 * cfg.H * cfg.I if gated else 2 * R * 2 * cfg.H * cfg.I
    fc1_flops = 2.0 * R * n1 * cfg.H
    return dict(touched=touched, fc1_bytes=touched * fc1 + act_fc1, fc2_bytes=touched * fc2,
                total_bytes=touched * (fc1 + fc2) + io, weight_bytes=touched * (fc1 + fc2), flops=flops,
                fc1_flops=fc1_flops, fc1_per_expert=fc1, fc2_per_expert=fc2)


def tc_peak_of(peaks):
    """The bf16 tensor peak a kernel timed here is held to: every timed
    region runs inside a seconds-long loop of the same forward (the clock
    sampler's bracketing load included), where the GPU settles at its power
    cap, so the sustained figure applies (the burst one when only that is
    known)."""
    if "bf16_tflops_sustained" in peaks:
        return float(peaks["bf16_tflops_sustained"]), "sustained bf16"
    return float(peaks["bf16_tflops"]), "burst bf16"


def roofline_of(cfg, alg, fc1_ms, peaks, peaks_kind, kname, traffic):
    """Roofline record of the FC1 launch: the slower of its algorithmic bytes
    at the measured HBM bandwidth and its FLOPs at the sustained bf16 peak
    binds."""
    hbm_peak = float(peaks["hbm_gbs"])
    tc_peak, tc_kind = tc_peak_of(peaks)
    if kname.startswith("ffn_tc_i8_kernel"):
        # integer MMAs: the bf16 figure times the nominal int8 / bf16 ratio (4.5 / 2.25)
        tc_peak, tc_kind = 2.0 * tc_peak, tc_kind + " x 2 for int8"
    t_hbm = alg["fc1_bytes"] / (hbm_peak * 1e9)
    t_tc = alg["fc1_flops"] / (tc_peak * 1e12)
    if t_hbm >= t_tc:
        achieved = alg["fc1_bytes"] / (fc1_ms / 1e3) / 1e9
        r = {"bound": "hbm", "achieved": achieved, "peak": hbm_peak, "unit": "GB/s",
             "frac": achieved / hbm_peak, "algorithmic_bytes": alg["fc1_bytes"]}
    else:
        achieved = alg["fc1_flops"] / (fc1_ms / 1e3) / 1e12
        r = {"bound": "tensor", "achieved": achieved, "peak": tc_peak, "unit": "TFLOP/s",
             "frac": achieved / tc_peak, "algorithmic_flops": alg["fc1_flops"]}
    r.update({"kernel": kname, "peak_kind": peaks_kind + (f" ({tc_kind})" if r["bound"] == "tensor" else ""),
              "traffic": traffic["bytes_per_launch"] if traffic else None, "avg_launch_ms": fc1_ms})
    return r


class ClockSampler:
    """nvidia-smi clocks and throttle reasons during the timed region."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index, tag="bench"):
        self.index = index
        self.proc = None
        # raw samples: QMOE_CLOCKS_DIR if set, else the system temp directory
        folder = os.environ.get("QMOE_CLOCKS_DIR") or tempfile.gettempdir()
        self.path = os.path.join(folder, f"clocks_{tag}_{os.getpid()}.csv")

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
        pw = [float(r[3]) for r in rows if r[3].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        loaded = [s for s in sm if mx and s > 0.5 * max(mx)] or sm
        return {"sm_mhz": statistics.median(loaded) if loaded else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons, "samples": len(rows),
                "power_w_median": statistics.median(pw) if pw else None}


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


def fc1_kernel_name(qmoe, path, tile):
    if path == qmoe.PATH_TC:
        return "ffn_tc_wide_kernel" if tile > 128 else "ffn_tc_kernel"
    return {qmoe.PATH_TC_DECODE: "ffn_tc_decode_kernel", qmoe.PATH_SIMT: "ffn_simt_kernel",
            qmoe.PATH_INT8: "ffn_i8_kernel", qmoe.PATH_INT8_TC: "ffn_tc_i8_kernel"}.get(path, "ffn_decode_kernel")


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
    tok = len(samples[0]) * args.steps
    value = tok / total
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * total / args.steps, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded)",
            "config": config_of(cfg, args.workload, 1),
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": oracle.num_threads(),
                             "cpu_model": cpu_model(), "kind": "oracle",
                             "sample": f"{len(samples[0])} token(s) of the {cfg.T}-token batch per step"},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------------- our arm

class Bound:
    """One operator instance with its device inputs, workspace and a graph of
    one forward."""

    def __init__(self, inp, dev, path=None, m=None):
        import torch
        from weight_only_quantized_warp_b200 import qmoe
        self.qmoe, self.torch = qmoe, torch
        self.inp, self.cfg, self.dev = inp, inp.cfg, dev
        if m is None:
            m = qmoe.QMoE(inp.cfg, dev, path=path)
            m.set_weights_from(inp)
        self.m = m
        self.h = m.handle
        self.x = qmoe.to_device(inp.x, dev)
        self.lg = qmoe.to_device(inp.logits, dev)
        self.sh = qmoe.to_device(inp.shared, dev)
        self.y = torch.empty_like(self.x)
        self.T = inp.cfg.T
        self.ws = m.workspace(self.T)
        self.nws = self.ws.numel()
        self.launches = qmoe.qmoe_launches_for(self.h, self.T)
        self.path = qmoe.qmoe_path_for(self.h, self.T)
        self.tile = qmoe.qmoe_token_tile_for(self.h, self.T)
        self.graph = None

    def fwd(self, stream):
        self.qmoe.qmoe_forward(self.h, self.T, self.x, self.lg, self.sh, self.y, self.ws, self.nws, stream)

    def capture(self):
        torch = self.torch
        self.graph = torch.cuda.CUDAGraph()
        # captures on a side stream and replays on the current one;
        # thread-local capture so that other threads' CUDA calls (a process
        # group's watchdog) are not treated as part of the capture
        with torch.cuda.graph(self.graph, capture_error_mode="thread_local"):
            self.fwd(torch.cuda.current_stream())

    def release(self):
        self.graph = None

    def offsets(self):
        torch = self.torch
        off = torch.empty(self.cfg.E + 1, dtype=torch.int32, device=self.dev)
        self.qmoe.qmoe_debug_routing(self.h, self.T, self.ws, offsets=off)
        return off.cpu().numpy()

    def per_kernel_ms(self, stream, n):
        torch = self.torch
        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(self.launches + 1)] for _ in range(n)]
        for row in evs:
            for e in row:
                e.record(stream)  # materialise the event handles
        torch.cuda.synchronize()
        for i in range(n):
            self.qmoe.qmoe_forward_profiled(self.h, self.T, self.x, self.lg, self.sh, self.y, self.ws, self.nws,
                                            evs[i], stream)
        torch.cuda.synchronize()
        per = np.array([[evs[i][j].elapsed_time(evs[i][j + 1]) for j in range(self.launches)]
                        for i in range(n)]).mean(axis=0)
        names = launch_names(self.path, self.launches, bool(self.cfg.apply_router_weight_on_input))
        return dict(zip(names, [float(v) for v in per]))


def timed_replays(b, stream, K, local, world, clocks_tag=None, dist=None):
    """K graph replays bracketed by events (and a barrier with N > 1); the
    clock sampler brackets the region with the same forward under load."""
    import torch
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(local, clocks_tag) if clocks_tag else None

    def keep_loaded(seconds):
        t_end = time.perf_counter() + seconds
        while time.perf_counter() < t_end:
            for _ in range(5):
                b.graph.replay()
            torch.cuda.synchronize()

    if clocks:
        clocks.start()
        keep_loaded(0.6)
    if world > 1:
        dist.barrier(device_ids=[local])
    torch.cuda.synchronize()
    start.record(stream)
    for _ in range(K):
        b.graph.replay()
    stop.record(stream)
    torch.cuda.synchronize()
    clk = None
    if clocks:
        keep_loaded(0.4)
        clk = clocks.stop()
        if clk is not None:
            clk["window"] = "timed region bracketed by 0.6 s / 0.4 s of the same forward"
    return start.elapsed_time(stop), clk


def measure_record(b, stream, K, warmup, local, peaks, peaks_kind, workload, clocks_tag):
    """Graph-timed step, per-kernel times and the FC1 roofline of one bound
    workload at N = 1 (the nested decode record and the crossover points)."""
    import torch
    for _ in range(max(warmup, 3)):
        b.fwd(stream)
    torch.cuda.synchronize()
    b.capture()
    for _ in range(3):
        b.graph.replay()
    torch.cuda.synchronize()
    alg = algorithmic(b.cfg, b.offsets())
    ms, clk = timed_replays(b, stream, K, local, 1, clocks_tag)
    kms = b.per_kernel_ms(stream, min(K, 10))
    b.release()
    step_ms = ms / K
    kbase = fc1_kernel_name(b.qmoe, b.path, b.tile)
    rl = roofline_of(b.cfg, alg, kms["fc1"], peaks, peaks_kind, kbase + " (FC1 + activation)",
                     traffic_record("fc1_" + kbase + "_" + workload))
    hbm_peak, tc_peak = float(peaks["hbm_gbs"]), tc_peak_of(peaks)[0]
    t_roof = max(alg["total_bytes"] / (hbm_peak * 1e9), alg["flops"] / (tc_peak * 1e12))
    return {"workload": workload, "T": b.T, "value": b.T / (step_ms / 1e3), "unit": "tokens/s",
            "ms_per_step": step_ms, "steps": K, "roofline": rl,
            "step": {"hbm_gbs": alg["total_bytes"] / (step_ms / 1e3) / 1e9,
                     "tflops": alg["flops"] / (step_ms / 1e3) / 1e12,
                     "roofline_frac_of_step": t_roof / (step_ms / 1e3),
                     "experts_touched": alg["touched"], "algorithmic_bytes": alg["total_bytes"],
                     "kernel_ms": kms, "path": b.path, "token_tile": b.tile,
                     "launch": "CUDA graph of one forward per step"},
            "gpu_launches": b.launches * K, "clocks": clk, "l2": l2_note(alg)}


def crossover(head_inp, m, dev, stream, peaks, peaks_kind, ts=CROSSOVER_T):
    """Step time over T on the headline's weights (token batches of each T
    from their own seeds): the flat part is bound by streaming the touched
    experts' weights, the rising part by the tensor cores. The measured
    crossover is where the compute line through the two largest T meets the
    streaming floor (the mean step time of the T <= 128 points)."""
    import torch
    cfg0 = head_inp.cfg
    pts = []
    for T in ts:
        cfg = gen.MoEConfig(**{**cfg0.__dict__, "T": T})
        x, lg, sh = gen.make_token_batch(cfg, 5000 + T, logits="uniform")
        inp = gen.MoEInputs(cfg, x, lg, head_inp.fc1_w, head_inp.fc1_s, head_inp.fc2_w, head_inp.fc2_s,
                            shared=sh)
        b = Bound(inp, dev, m=m)
        K = 20 if T <= 1024 else 8
        r = measure_record(b, stream, K, 3, 0, peaks, peaks_kind, f"crossover_T{T}", None)
        pts.append({"T": T, "ms_per_step": r["ms_per_step"], "tokens_per_s": r["value"],
                    "fc1_kernel": r["roofline"]["kernel"].split(" ")[0], "fc1_bound": r["roofline"]["bound"],
                    "fc1_frac": r["roofline"]["frac"], "path": r["step"]["path"], "token_tile": r["step"]["token_tile"],
                    "step_roofline_frac": r["step"]["roofline_frac_of_step"]})
        del b
        torch.cuda.synchronize()
    floor = float(np.mean([p["ms_per_step"] for p in pts if p["T"] <= 128]))
    big = sorted(pts, key=lambda p: p["T"])[-2:]
    slope = (big[1]["ms_per_step"] - big[0]["ms_per_step"]) / (big[1]["T"] - big[0]["T"])
    icept = big[1]["ms_per_step"] - slope * big[1]["T"]
    measured = (floor - icept) / slope if slope > 0 else None
    alg = algorithmic(gen.MoEConfig(**{**cfg0.__dict__, "T": 1}), np.arange(cfg0.E + 1))
    wbytes = cfg0.E * (alg["fc1_per_expert"] + alg["fc2_per_expert"])
    per_tok_flops = 2 * cfg0.k * 3 * cfg0.H * cfg0.I
    model = wbytes * tc_peak_of(peaks)[0] * 1e12 / (float(peaks["hbm_gbs"]) * 1e9 * per_tok_flops)
    return {"weights": HEADLINE + " (all T share them)", "points": pts,
            "streaming_floor_ms": floor, "compute_ms_per_token": slope,
            "measured_crossover_T": measured, "model_crossover_T": model,
            "model": "all experts' weight bytes at the HBM peak = T tokens' FLOPs at the sustained bf16 peak"}


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
    peaks, peaks_kind = load_peaks()

    # every replica: the same weights, its own token batch
    inp = replicas.replica_inputs(args.workload, rank)
    cfg = inp.cfg
    b = Bound(inp, dev, path=args.path)
    T, h = b.T, b.h
    stream = torch.cuda.current_stream()
    K = args.steps

    for _ in range(max(args.warmup, 3)):
        b.fwd(stream)
    torch.cuda.synchronize()
    b.capture()
    for _ in range(3):
        b.graph.replay()
    torch.cuda.synchronize()
    alg = algorithmic(cfg, b.offsets())

    # ---- timed region: K graph replays of the whole forward
    ms, clk = timed_replays(b, stream, K, local, world, "headline", dist)
    ms = replicas.max_over_ranks([ms], dev)[0]
    if world > 1:
        dist.barrier(device_ids=[local])

    # after the timed region: the same K steps as direct launches, and a
    # pass with an event between kernels for the per-kernel times (the events
    # themselves add a few microseconds per launch)
    s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s0.record(stream)
    for _ in range(K):
        b.fwd(stream)
    s1.record(stream)
    torch.cuda.synchronize()
    stream_ms = replicas.max_over_ranks([s0.elapsed_time(s1)], dev)[0]
    kms = b.per_kernel_ms(stream, min(K, 10))
    b.release()
    if world > 1:
        dist.barrier(device_ids=[local])

    # ---- end to end through the public call, host buffers, copies inside.
    # As a serving loop does, two buffer slots and two copy streams let the
    # copy engines bring step i+1's inputs in and take step i-1's result out
    # while step i computes; every step's own copies lie inside the timed
    # region, which runs from before the first input copy to after the last
    # result copy. The same K steps with copies and compute in one stream
    # give the serial figure reported beside it.
    x_h = torch.empty(b.x.shape, dtype=b.x.dtype, pin_memory=True).copy_(b.x.cpu())
    lg_h = torch.empty(b.lg.shape, dtype=b.lg.dtype, pin_memory=True).copy_(b.lg.cpu())
    sh_h = None if b.sh is None else torch.empty(b.sh.shape, dtype=b.sh.dtype, pin_memory=True).copy_(b.sh.cpu())
    y_h = [torch.empty(b.y.shape, dtype=b.y.dtype, pin_memory=True) for _ in range(2)]
    x_d = [torch.empty_like(b.x) for _ in range(2)]
    lg_d = [torch.empty_like(b.lg) for _ in range(2)]
    sh_d = [None if b.sh is None else torch.empty_like(b.sh) for _ in range(2)]
    y_d = [b.y, torch.empty_like(b.y)]
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_comp = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]
    used = [False, False]

    def e2e_step(i):
        k = i % 2
        with torch.cuda.stream(s_in):
            if used[k]:
                s_in.wait_event(ev_comp[k])  # the slot's previous forward has read its inputs
            x_d[k].copy_(x_h, non_blocking=True)
            lg_d[k].copy_(lg_h, non_blocking=True)
            if sh_d[k] is not None:
                sh_d[k].copy_(sh_h, non_blocking=True)
            ev_in[k].record(s_in)
        stream.wait_event(ev_in[k])
        if used[k]:
            stream.wait_event(ev_out[k])  # the slot's previous result has left the device
        qmoe.qmoe_forward(h, T, x_d[k], lg_d[k], sh_d[k], y_d[k], b.ws, b.nws, stream)
        ev_comp[k].record(stream)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev_comp[k])
            y_h[k].copy_(y_d[k], non_blocking=True)
            ev_out[k].record(s_out)
        used[k] = True

    def serial_step():
        with torch.cuda.stream(stream):
            x_d[0].copy_(x_h, non_blocking=True)
            lg_d[0].copy_(lg_h, non_blocking=True)
            if sh_d[0] is not None:
                sh_d[0].copy_(sh_h, non_blocking=True)
            qmoe.qmoe_forward(h, T, x_d[0], lg_d[0], sh_d[0], y_d[0], b.ws, b.nws, stream)
            y_h[0].copy_(y_d[0], non_blocking=True)

    for i in range(3):
        e2e_step(i)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier(device_ids=[local])
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s_in)
    for i in range(K):
        e2e_step(3 + i)
    e1.record(s_out)
    torch.cuda.synchronize()
    e2e_ms = replicas.max_over_ranks([e0.elapsed_time(e1)], dev)[0]
    for _ in range(3):
        serial_step()
    torch.cuda.synchronize()
    e0.record(stream)
    for _ in range(K):
        serial_step()
    e1.record(stream)
    torch.cuda.synchronize()
    serial_ms = replicas.max_over_ranks([e0.elapsed_time(e1)], dev)[0]
    h2d = x_h.numel() * x_h.element_size() + lg_h.numel() * lg_h.element_size() + (
        0 if sh_h is None else sh_h.numel() * sh_h.element_size())
    d2h = y_h[0].numel() * y_h[0].element_size()

    if world > 1:
        dist.destroy_process_group()
    if rank != 0:
        return 0

    # ---- N = 1 only: the nested decode record and the crossover over T
    decode = None
    if world == 1 and args.decode_workload != "none":
        dinp = replicas.replica_inputs(args.decode_workload, 0)
        db = Bound(dinp, dev)
        decode = measure_record(db, stream, max(K, 20), args.warmup, local, peaks, peaks_kind,
                                args.decode_workload, "decode")
        decode["config"] = config_of(dinp.cfg, args.decode_workload, 1)
        del db
        torch.cuda.synchronize()
    cross = None
    if world == 1 and not args.no_crossover and args.workload == HEADLINE:
        cross = crossover(inp, b.m, dev, stream, peaks, peaks_kind)

    # ---- CPU baseline (rank 0, N = 1 only): the oracle on a bounded sample
    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        ntok = min(T, args.cpu_sample_tokens or 32)
        rng = np.random.default_rng(1)
        toks = sorted(rng.choice(T, size=ntok, replace=False).tolist())
        v, el, done, cores = cpu_oracle_timing(inp, toks)
        cpu = {"value": v, "unit": "tokens/s", "cores": cores, "cpu_model": cpu_model(), "kind": "oracle",
               "sample": f"{done} tokens ({ntok} per call) of the {T}-token batch, {el:.1f} s"}

    step_ms = ms / K
    value = replicas.job_tokens_per_s(T, world, K, ms)
    kbase = fc1_kernel_name(qmoe, b.path, b.tile)
    roofline = roofline_of(cfg, alg, kms["fc1"], peaks, peaks_kind, kbase + " (FC1 + activation)",
                           traffic_record("fc1_" + kbase + "_" + args.workload))
    hbm_peak, tc_peak = float(peaks["hbm_gbs"]), tc_peak_of(peaks)[0]
    t_roof = max(alg["total_bytes"] / (hbm_peak * 1e9), alg["flops"] / (tc_peak * 1e12))
    roofline["roofline_frac_of_step"] = t_roof / (step_ms / 1e3)
    line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": K,
            "warmup": args.warmup, "ms_per_step": step_ms, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None,
            "dtype": "s8" if cfg.compute_mode == gen.COMPUTE_INT8_BLOCK else (
                "bf16" if cfg.act_dtype == gen.DT_BF16 else "f32"),
            "data": "synthetic (seeded, shapes of the workload; no trained weights)",
            "config": config_of(cfg, args.workload, world, alg),
            "roofline": roofline,
            "step": {"hbm_gbs": alg["total_bytes"] / (step_ms / 1e3) / 1e9,
                     "tflops": alg["flops"] / (step_ms / 1e3) / 1e12,
                     "experts_touched": alg["touched"], "algorithmic_bytes": alg["total_bytes"],
                     "algorithmic_flops": alg["flops"],
                     "kernel_ms": kms, "path": b.path, "token_tile": b.tile,
                     "launch": "CUDA graph of one forward per step",
                     "ms_per_step_direct_launches": stream_ms / K,
                     "kernel_ms_note": "from a separate pass with an event between kernels"},
            "decode": decode,
            "crossover": cross,
            "cpu_baseline": cpu,
            "e2e": {"value": replicas.job_tokens_per_s(T, world, K, e2e_ms), "unit": "tokens/s",
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "copies": "pinned host buffers; input and result copies of neighbouring steps "
                              "overlap the forward on separate copy streams (two buffer slots)",
                    "serial_value": replicas.job_tokens_per_s(T, world, K, serial_ms)},
            "gpu_launches": b.launches * K,
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
