"""Benchmark of the ternary-weight decoder projections on B200.

Default workload: the full decode sweep — 28 layers x 7 projections = 196
ternary matrices of a Qwen2.5-1.5B-shaped decoder (q/o 1536x1536, k/v
256x1536, gate/up 8960x1536, down 1536x8960; 1,310,195,712 weights,
327,548,928 bytes of 2-bit codes), one token (M = 1), seeded synthetic
weights N(0, 0.02^2) and activations N(0, 1) with 1% outlier channels x20.
A step is one pass of the whole hot path over every projection: activation
quantisation (one launch), then ternary product and rescale (one persistent
launch per token group, started early by programmatic dependent launch).
Prefill sizes (--m > 32) take int8 activations quantised beforehand and run
the tensor-core kernel (one persistent launch).

--chain times the decoder-layer chain instead: the layers' projections in
dependency order (q/k/v on one input, identity attention, o and a residual,
gate/up, SiLU * up, down and a residual), each step all layers from one
token state, under its own metric name.

Prints one JSON line (rank 0).  Multi-GPU (torchrun): every rank runs its own
replica of the sweep on its own token (data-parallel decode; no collective
on the data path), value = all ranks' tokens / max-over-ranks time.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "196-matrix ternary decode sweep tokens/s & weight GB/s (% of HBM roofline)"
UNIT = "tokens/s"
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20000)
    ap.add_argument("--warmup", type=int, default=200)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--m", type=int, default=1, help="tokens per step (decode: 1..32)")
    ap.add_argument("--layers", type=int, default=28)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--chain", action="store_true",
                    help="time the dependent decoder-layer chain instead of the sweep")
    return ap.parse_args()


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d.get("hbm_gbs", FALLBACK_HBM_GBS), "measured"
    return FALLBACK_HBM_GBS, "fallback"


def _strip_comments(text):
    """C/C++/CUDA source without comments, trailing blanks or empty lines."""
    import re
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    text = re.sub(r"//[^\n]*", "", text)
    return "\n".join(l.rstrip() for l in text.splitlines() if l.strip())


def code_digest(kernel_src, read=None):
    """sha256 over the code of one kernel source file and of the library's
    headers (comments and blank lines removed): an ncu capture stays valid
    across comment edits and stops applying on any change of code.
    `read(relpath)` returns a file's text (default: the working tree)."""
    import glob
    import hashlib
    if read is None:
        def read(rel):
            with open(os.path.join(ROOT, rel)) as f:
                return f.read()
    csrc = os.path.join("ternary_weight_decoder_b200", "csrc")
    rels = [os.path.join(csrc, kernel_src)]
    for pat in (os.path.join(csrc, "*.cuh"), os.path.join(csrc, "*.h"), os.path.join("include", "*.h")):
        rels += sorted(os.path.relpath(q, ROOT) for q in glob.glob(os.path.join(ROOT, pat)))
    h = hashlib.sha256()
    for rel in rels:
        h.update(rel.encode() + b"\0" + _strip_comments(read(rel)).encode() + b"\0")
    return h.hexdigest()


def profiled_traffic(kernel_src, M, layers):
    """DRAM bytes (read + write) per launch of the dominant kernel, from the
    ncu capture recorded in profiles/traffic.json, or None when there is no
    capture for this M or the kernel's code has changed since it was taken.
    A capture of fewer layers is scaled by the layer count (the traffic of a
    sweep grows in proportion to its projections at fixed M)."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    digest = code_digest(kernel_src)
    for e in json.load(open(p)).get("captures", []):
        if e["kernel_src"] == kernel_src and e["M"] == M and e["code_sha256"] == digest:
            return e["dram_bytes_per_launch"] * layers / e["layers"]
    return None


def sweep_bytes(shapes, M):
    codes = sum((-(-N // 16) * 16) * K // 4 for (_, _, _, N, K) in shapes)
    algo_codes = sum(N * K // 4 for (_, _, _, N, K) in shapes)
    xin = sum(M * K * 4 for (_, _, _, N, K) in shapes)
    yout = sum(M * N * 4 for (_, _, _, N, K) in shapes)
    return algo_codes + xin + yout, algo_codes, codes


class ClockSampler:
    """Polls SM clock, power and throttle reasons through NVML while running."""

    def __init__(self, index: int):
        self.samples, self.reasons, self.stop_ev = [], set(), threading.Event()
        self.max_mhz = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception as e:  # no NVML: report that instead of clocks
            self.nv, self.err = None, str(e)

    def _run(self):
        nv = self.nv
        names = {
            "hw_slowdown": getattr(nv, "nvmlClocksThrottleReasonHwSlowdown", 0x8),
            "hw_thermal_slowdown": getattr(nv, "nvmlClocksThrottleReasonHwThermalSlowdown", 0x40),
            "sw_thermal_slowdown": getattr(nv, "nvmlClocksThrottleReasonSwThermalSlowdown", 0x20),
            "sw_power_cap": getattr(nv, "nvmlClocksThrottleReasonSwPowerCap", 0x4),
        }
        while not self.stop_ev.is_set():
            try:
                mhz = nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM)
                r = nv.nvmlDeviceGetCurrentClocksThrottleReasons(self.h)
                self.samples.append(mhz)
                for k, bit in names.items():
                    if r & bit:
                        self.reasons.add(k)
            except Exception:
                pass
            time.sleep(0.002)

    def __enter__(self):
        if self.nv:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        if self.nv:
            self.stop_ev.set()
            self.t.join()

    def summary(self):
        if not self.nv:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "note": self.err}
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                "samples": len(self.samples)}


def rank_layer_seed(layer, rank):
    """Layer index the activations of `rank` are seeded with: every rank of a
    data-parallel run decodes its own token stream over the same weights."""
    return layer + 1000 * rank


def max_over_ranks(ms, dist, device):
    """The slowest rank's time (all ranks take the same collective step)."""
    if dist is None:
        return ms
    import torch
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_value(M, world, steps, max_ms):
    """Whole-job tokens/s: every rank's tokens over the slowest rank's time."""
    return M * world * steps / (max_ms / 1e3)


def build_workload(api, torch, dev, M, layers, rank):
    """Generate, upload and ternarise the sweep; return descriptors and buffers."""
    from ternary_weight_decoder_b200 import synth
    shapes = synth.sweep_shapes(layers)
    x_off, y_off, xo, yo = [], [], 0, 0
    for (_, _, _, N, K) in shapes:
        x_off.append(xo)
        y_off.append(yo)
        xo += M * K
        yo += M * N
    x_host = torch.empty(xo, dtype=torch.float32).pin_memory()
    xn = x_host.numpy()
    descs = []
    x_all = torch.empty(xo, dtype=torch.float32, device=dev)
    y_all = torch.empty(yo, dtype=torch.float32, device=dev)
    import concurrent.futures as cf
    pool = cf.ThreadPoolExecutor(max_workers=min(16, os.cpu_count() or 4))
    window = 16   # bounds host memory: at most this many fp32 matrices alive
    futs = {}
    for i, (l, p, name, N, K) in enumerate(shapes):
        for j in range(i, min(i + window, len(shapes))):
            if j not in futs:
                lj, pj, _, Nj, Kj = shapes[j]
                futs[j] = pool.submit(synth.weights, lj, pj, Nj, Kj)
        W = futs.pop(i).result()
        Wd = torch.from_numpy(W).to(dev)
        packed, mean_abs, wscale = api.ternarize_pack(Wd)
        del Wd, W
        # each rank decodes its own token stream
        xn[x_off[i]:x_off[i] + M * K] = synth.activations(rank_layer_seed(l, rank), p, M, K).ravel()
        descs.append(dict(x=x_all[x_off[i]:x_off[i] + M * K].view(M, K), packed=packed,
                          wscale=wscale, y=y_all[y_off[i]:y_off[i] + M * N].view(M, N),
                          N=N, K=K))
    api.check()
    pool.shutdown()
    x_all.copy_(x_host)
    torch.cuda.synchronize()
    return shapes, descs, x_host, x_all, y_all


CHAIN_METRIC = "decoder-layer chain tokens/s (28 dependent layers; % of HBM roofline)"
CHAIN_DIMS = (1536, 256, 128, 8960)   # hidden, kv_dim, head_dim, inter (Qwen2.5-1.5B)


def chain_bytes(shapes, M, dims=CHAIN_DIMS):
    """Algorithmic bytes of one chain step: the sweep's (codes, fp32 x read
    and y written per projection) plus the element-wise steps per layer
    (attention stand-in: v read, a written; two residual adds: two reads and
    a write each; SiLU * up: two reads and a write)."""
    hidden, kv, hd, inter = dims
    algo, codes, _ = sweep_bytes(shapes, M)
    layers = len(shapes) // 7
    ew = M * 4 * ((kv + hidden) + 2 * 3 * hidden + 3 * inter)
    return algo + layers * ew, codes


def run_chain(args, api, torch, dev, rank, world, dist, local):
    from ternary_weight_decoder_b200 import synth
    M = args.m
    if not 1 <= M <= 32:
        raise SystemExit("--chain runs decode token counts only (1..32)")
    shapes, descs, _, x_all, y_all = build_workload(api, torch, dev, M, args.layers, rank)
    layers = [dict() for _ in range(args.layers)]
    for (l, _, name, _, _), d in zip(shapes, descs):
        layers[l][name] = (d["packed"], d["wscale"])
    del descs, x_all, y_all
    hidden, kv, hd, inter = CHAIN_DIMS
    chain = api.DecoderChain(layers, M, hidden, kv, hd, inter, dev)
    h0_host = torch.from_numpy(synth.activations(rank_layer_seed(0, rank), 0, M, hidden)).pin_memory()
    h0 = h0_host.to(dev)
    stream = torch.cuda.current_stream()

    def step():
        chain.h.copy_(h0, non_blocking=True)   # every step starts from the same token state
        api.decoder_chain(chain)

    for _ in range(args.warmup):
        step()
    api.check()

    def barrier():
        if dist is not None:
            dist.barrier()
        torch.cuda.synchronize()

    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clk:
        barrier()
        e0.record(stream)
        for _ in range(args.steps):
            step()
        e1.record(stream)
        barrier()
    api.check()
    ms = max_over_ranks(e0.elapsed_time(e1), dist, dev)
    ms_per_step = ms / args.steps
    algo, codes = chain_bytes(shapes, M)
    hbm, src = peaks()
    achieved = algo / (ms_per_step / 1e3) / 1e9

    e2e = None
    if not args.no_e2e:
        out = torch.empty(M * hidden, dtype=torch.float32).pin_memory()
        k2 = max(3, min(args.steps, 500))
        barrier()
        f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        f0.record(stream)
        for _ in range(k2):
            chain.h.copy_(h0_host, non_blocking=True)
            api.decoder_chain(chain)
            out.copy_(chain.h.view(-1), non_blocking=True)
            stream.synchronize()
        f1.record(stream)
        barrier()
        ems = max_over_ranks(f0.elapsed_time(f1), dist, dev)
        e2e = {"value": job_value(M, world, k2, ems), "unit": UNIT,
               "h2d_bytes_per_step": M * hidden * 4, "d2h_bytes_per_step": M * hidden * 4,
               "steps": k2, "ms_per_step": ems / k2}
    if dist is not None:
        dist.destroy_process_group()
    if rank != 0:
        return
    print(json.dumps({
        "metric": CHAIN_METRIC, "value": job_value(M, world, args.steps, ms), "unit": UNIT,
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "int8xternary->int32, f32 in/out", "data": "synthetic",
        "config": {"workload": f"decoder_chain_{args.layers}L_M{M}", "M": M,
                   "layers": args.layers, "hidden": hidden, "kv_dim": kv, "head_dim": hd,
                   "inter": inter, "parallelism": f"dp{world} (independent replicas)",
                   "l2": f"codes {codes / 1e6:.0f} MB > 126 MB L2; no flush"},
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": hbm, "unit": "GB/s",
                     "frac": achieved / hbm, "traffic": None,
                     "peak_source": f"{src} (MEASURED_PEAKS.json hbm_gbs)" if src == "measured"
                     else "fallback 6650 GB/s",
                     "algorithmic_bytes_per_step": algo, "weight_bytes_per_step": codes,
                     "note": "step = all layers: per layer 4 sweeps + 4 element-wise launches"},
        "cpu_baseline": None, "e2e": e2e,
        "gpu_launches": chain.launches * args.steps, "clocks": clk.summary(),
    }))


def cpu_oracle_sample(M, budget_s=10.0, sample_layers=4, layers=28):
    """Time the reference oracle, as it stands, on one host core: repeated
    passes over the projections of the first `sample_layers` layers until
    about budget_s of timed work; tokens/s is scaled to the full sweep by
    weight count."""
    from oracle import oracle as orc
    from ternary_weight_decoder_b200 import synth
    shapes = synth.sweep_shapes(layers)
    total_w = sum(N * K for (_, _, _, N, K) in shapes)
    sample = []
    for (l, p, name, N, K) in synth.sweep_shapes(min(sample_layers, layers)):
        codes, mean = orc.ternarize(synth.weights(l, p, N, K))
        sample.append((synth.activations(l, p, M, K), codes, mean))
    sample_w = sum(c.size for _, c, _ in sample)
    timed, passes = 0.0, 0
    while timed < budget_s or passes == 0:
        t0 = time.perf_counter()
        for x, codes, mean in sample:
            orc.ternary_linear(x, codes, mean)
        timed += time.perf_counter() - t0
        passes += 1
    sweep_s = timed / passes * total_w / sample_w
    return {"value": M / sweep_s, "unit": UNIT, "cores": 1, "kind": "oracle",
            "sample": (f"{len(sample)} of {len(shapes)} projections (layers 0-"
                       f"{min(sample_layers, layers) - 1}, {sample_w / total_w:.3f} of the "
                       f"weights) at M={M}, {passes} passes, {timed:.1f} s timed, scaled to "
                       f"the full sweep by weight count")}


def run_reference(args):
    """The oracle as it stands, on host cores, on the same metric and config."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    from oracle import oracle as orc
    from ternary_weight_decoder_b200 import synth
    M = args.m
    shapes = synth.sweep_shapes(args.layers)
    total_w = sum(N * K for (_, _, _, N, K) in shapes)
    # per-step sample: leading rows of each projection of layer 0, sized so
    # that warm-up + steps take about 60 s in total (at most ~2 s a step)
    per_step_s = min(2.0, 60.0 / max(1, args.steps + args.warmup))
    calib = []
    for (l, p, name, N, K) in shapes[:7]:
        W = synth.weights(l, p, N, K)
        codes, mean = orc.ternarize(W)
        x = synth.activations(l, p, M, K)
        calib.append((codes, mean, x, N, K))
    t0 = time.perf_counter()
    for codes, mean, x, N, K in calib:
        orc.ternary_linear(x, codes[:16], mean)
    per_row_s = (time.perf_counter() - t0) / (16 * len(calib))
    rows = max(1, int(per_step_s / (per_row_s * len(calib))))
    sample = [(c[:min(rows, N)], m, x) for (c, m, x, N, K) in calib]
    sample_w = sum(c.size for c, _, _ in sample)
    for _ in range(args.warmup):
        for c, m, x in sample:
            orc.ternary_linear(x, c, m)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        for c, m, x in sample:
            orc.ternary_linear(x, c, m)
    el = time.perf_counter() - t0
    step_s = el / args.steps
    value = M / (step_s * total_w / sample_w)
    samp = (f"per step: first {rows} rows of each of layer 0's 7 projections "
            f"({sample_w} weights, M={M}), scaled to the {len(shapes)}-projection sweep by "
            f"weight count")
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": step_s * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "int8xternary->int32, f32 in/out", "data": "synthetic",
        "config": {"workload": f"decode_sweep_196x_M{M}", "M": M,
                   "projections": len(shapes)},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": 1, "kind": "oracle",
                         "sample": samp},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }))


def main():
    args = parse()
    if args.impl == "reference":
        return run_reference(args)
    import torch
    from ternary_weight_decoder_b200 import build
    build.build()
    from ternary_weight_decoder_b200 import api

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)

    if args.chain:
        return run_chain(args, api, torch, dev, rank, world, dist, local)
    M = args.m
    shapes, descs, x_host, x_all, y_all = build_workload(api, torch, dev, M, args.layers, rank)
    if M > 32:   # prefill sweeps consume int8 activations quantised beforehand
        for d in descs:
            d["xq"], d["amax"], d["qsum"] = api.quantize_act(d["x"])
    table = api.SweepTable(descs, M, device=dev)
    algo_bytes, algo_codes, _ = sweep_bytes(shapes, M)
    launches_per_step = table.launches

    stream = torch.cuda.current_stream()
    for _ in range(args.warmup):
        api.decoder_projection_sweep(table)
    api.check()

    def barrier():
        if dist is not None:
            dist.barrier()
        torch.cuda.synchronize()

    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clk:
        barrier()
        e0.record(stream)
        for _ in range(args.steps):
            api.decoder_projection_sweep(table)
        e1.record(stream)
        barrier()
    api.check()
    ms = max_over_ranks(e0.elapsed_time(e1), dist, dev)
    ms_per_step = ms / args.steps
    value = job_value(M, world, args.steps, ms)

    hbm, src = peaks()
    if M <= 32:
        # decode: HBM-bound; algorithmic bytes = 2-bit codes + fp32 x + fp32 y
        achieved = algo_bytes / (ms_per_step / 1e3) / 1e9
        roofline = {"bound": "hbm", "achieved": achieved, "peak": hbm, "unit": "GB/s",
                    "frac": achieved / hbm,
                    # sweeps of more than 16 tokens run the tensor-core decode kernel
                    "traffic": profiled_traffic("tw_decode_tc.cu" if M > 16 else "tw_decode.cu",
                                                M, args.layers),
                    "peak_source": f"{src} (MEASURED_PEAKS.json hbm_gbs)" if src == "measured"
                    else "fallback 6650 GB/s",
                    "algorithmic_bytes_per_step": algo_bytes,
                    "weight_bytes_per_step": algo_codes,
                    "weight_gbs": algo_codes / (ms_per_step / 1e3) / 1e9,
                    "note": "step = quantise launch + decode launch; time of the whole step"}
    else:
        # prefill: int8 tensor-core bound; 2*M*N*K ops per projection
        ops = sum(2 * M * N * K for (_, _, _, N, K) in shapes)
        tops = ops / (ms_per_step / 1e3) / 1e12
        pk = json.load(open(os.path.join(ROOT, "MEASURED_PEAKS.json"))).get("bf16_tflops") \
            if os.path.exists(os.path.join(ROOT, "MEASURED_PEAKS.json")) else FALLBACK_BF16_TFLOPS
        roofline = {"bound": "tensor", "achieved": tops, "peak": 2 * pk, "unit": "TOP/s",
                    "frac": tops / (2 * pk),
                    "traffic": profiled_traffic("tw_prefill.cu", M, args.layers),
                    "peak_source": "2 x measured bf16 burst (int8 dense = 2 x bf16 nominal)",
                    "ops_per_step": ops}

    e2e = None
    if not args.no_e2e and M <= 32:
        y_host = torch.empty(y_all.numel(), dtype=torch.float32).pin_memory()
        k2 = max(3, min(args.steps, 2000))
        for _ in range(3):
            x_all.copy_(x_host, non_blocking=True)
            api.decoder_projection_sweep(table)
            y_host.copy_(y_all, non_blocking=True)
            stream.synchronize()
        barrier()
        t0 = time.perf_counter()
        f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        f0.record(stream)
        for _ in range(k2):
            x_all.copy_(x_host, non_blocking=True)
            api.decoder_projection_sweep(table)
            y_host.copy_(y_all, non_blocking=True)
            stream.synchronize()   # the host reads every step's result
        f1.record(stream)
        barrier()
        wall = time.perf_counter() - t0
        ems = max_over_ranks(f0.elapsed_time(f1), dist, dev)
        e2e = {"value": job_value(M, world, k2, ems), "unit": UNIT,
               "h2d_bytes_per_step": x_all.numel() * 4, "d2h_bytes_per_step": y_all.numel() * 4,
               "steps": k2, "ms_per_step": ems / k2, "host_wall_ms_per_step": wall * 1e3 / k2}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu:
        cpu = cpu_oracle_sample(M, layers=args.layers)

    if dist is not None:
        dist.destroy_process_group()
    if rank != 0:
        return
    print(json.dumps({
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None,
        "dtype": "int8xternary->int32, f32 in/out", "data": "synthetic",
        "config": {"workload": f"decode_sweep_196x_M{M}" if args.layers == 28
                   else f"decode_sweep_{7 * args.layers}x_M{M}",
                   "M": M, "projections": len(shapes), "layers": args.layers,
                   "parallelism": f"dp{world} (independent replicas, no collective)",
                   "l2": f"inputs {algo_bytes / 1e6:.0f} MB > 126 MB L2; no flush"},
        "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e,
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clk.summary(),
    }))


if __name__ == "__main__":
    main()
