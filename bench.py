"""Benchmark of the ternary-weight decoder projections on B200.

Headline workload: the full decode sweep -- 28 layers x 7 projections = 196
ternary matrices of a Qwen2.5-1.5B-shaped decoder (q/o 1536x1536, k/v
256x1536, gate/up 8960x1536, down 1536x8960; 1,310,195,712 weights,
327,548,928 bytes of 2-bit codes), one token (M = 1), seeded synthetic
weights N(0, 0.02^2) and activations N(0, 1) with 1% outlier channels x20.
A step is one pass of the whole hot path over every projection: activation
quantisation, then ternary product and rescale (one persistent launch per
token group, started early by programmatic dependent launch).

The same JSON line carries a ``configs`` object with every workload of the
benchmark definition, measured in the same run on the same weights:

  1. one 1536x1536 GEMV at M = 1 (x without outliers), L2 flushed before
     every call: us per call, median and p10/p90; and back to back over a
     rotating pool of distinct matrices whose codes exceed twice the L2;
  2. one decoder layer's 7 projections at M = 1 as one sweep call, L2
     flushed before every call: us per matrix;
  3. the headline (196 projections, M = 1);
  4. the 196-projection sweep at M = 4, 8, 16, 32 (fraction of HBM);
  5. the 196-projection prefill sweep at M = 256, 1024, 4096 on int8
     activations quantised beforehand (fraction of the int8 tensor peak);
  and the 196-projection sweep at M = 64, 128, 192 (more than 32 tokens:
  the default weights-in-TMEM GEMM against the expanded-weights GEMM on the
  same descriptors), the I8_S int8 linear layer with bias and ReLU, and the
  decoder-layer chain (28 dependent layers at M = 1).
Each decode/prefill entry also carries the oracle timed on the host's cores
on a bounded sample (labelled, extrapolated by weight count and tokens).

--chain times only the decoder-layer chain, under its own metric name.

Prints one JSON line (rank 0).  Multi-GPU (torchrun): every rank runs its own
replica of the sweep on its own token (data-parallel decode; no collective
on the data path), value = all ranks' tokens / max-over-ranks time.
"""
from __future__ import annotations

import argparse
import json
import os
import re
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
DTYPE = "int8xternary->int32, f32 in/out"
DECODE_MS = (4, 8, 16, 32)
PREFILL_MS = (256, 1024, 4096)
MID_MS = (64, 128, 192)          # more than 32 tokens, below the expanded-weights crossover
L2_FLUSH_BYTES = 256 << 20   # > 2 x the 126 MB L2
PREFILL_DISTINCT_ROWS = 256  # distinct generated token rows per projection (tiled up to M)
# I8_S encoder layer shapes (tokens M, channels K -> N = 4K): activations
# outweigh weights 16 : 1 (M*K = 16 * N*K)
I8_SHAPES = ((16384, 256, 1024), (32768, 512, 2048))


def parse(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--m", type=int, default=1, help="tokens per step of the headline sweep")
    ap.add_argument("--layers", type=int, default=28)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--no-configs", action="store_true",
                    help="headline only (no configs object)")
    ap.add_argument("--configs", default="1,2,4,5,mid,i8,chain",
                    help="comma list of the extra workloads to measure")
    ap.add_argument("--chain", action="store_true",
                    help="time the dependent decoder-layer chain instead of the sweep")
    return ap.parse_args(argv)


def peaks():
    """(HBM GB/s, int8 dense TOP/s, source).  The int8 peak is 2 x the
    measured bf16 burst (the nominal int8 : bf16 dense ratio, 4.5 : 2.25)."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return (d.get("hbm_gbs", FALLBACK_HBM_GBS),
                2 * d.get("bf16_tflops", FALLBACK_BF16_TFLOPS), "measured")
    return FALLBACK_HBM_GBS, 2 * FALLBACK_BF16_TFLOPS, "fallback"


def peak_source(src):
    return ("measured (MEASURED_PEAKS.json hbm_gbs; int8 = 2 x bf16_tflops)"
            if src == "measured" else "fallback 6650 GB/s; int8 = 2 x 1590 TFLOP/s")


def _strip_comments(text):
    """C/C++/CUDA source without comments, trailing blanks or empty lines."""
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    text = re.sub(r"//[^\n]*", "", text)
    return "\n".join(l.rstrip() for l in text.splitlines() if l.strip())


# The public C header declares host entry points only; no kernel's device
# code depends on it, so an edit there keeps a capture valid.
_HOST_ONLY_HEADERS = (os.path.join("include", "ternary_decoder.h"),)


def kernel_sources(kernel_src, read=None):
    """The kernel's source file and every local header it includes,
    transitively (quoted includes), minus the host-only public header."""
    if read is None:
        def read(rel):
            with open(os.path.join(ROOT, rel)) as f:
                return f.read()
    csrc = os.path.join("ternary_weight_decoder_b200", "csrc")
    todo, seen = [os.path.join(csrc, kernel_src)], []
    while todo:
        rel = os.path.normpath(todo.pop(0))
        if rel in seen or rel in _HOST_ONLY_HEADERS:
            continue
        seen.append(rel)
        for inc in re.findall(r'^\s*#\s*include\s+"([^"]+)"', _strip_comments(read(rel)), re.M):
            todo.append(os.path.join(os.path.dirname(rel), inc))
    return seen


def code_digest(kernel_src, read=None):
    """sha256 over the code of one kernel source file and of the local
    headers it includes (comments and blank lines removed): an ncu capture
    stays valid across comment edits and stops applying on any change of
    the code the kernel is compiled from.  `read(relpath)` returns a file's
    text (default: the working tree)."""
    import hashlib
    if read is None:
        def read(rel):
            with open(os.path.join(ROOT, rel)) as f:
                return f.read()
    h = hashlib.sha256()
    for rel in kernel_sources(kernel_src, read):
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


def decode_kernel_src(M):
    """Source file of the dominant kernel of a sweep of M tokens."""
    if M > 192:
        return "tw_prefill.cu"
    if M > 32:
        return "tw_mid.cu"
    return "tw_decode_tc.cu" if M > 8 else "tw_decode.cu"


def sweep_bytes(shapes, M):
    codes = sum((-(-N // 16) * 16) * K // 4 for (_, _, _, N, K) in shapes)
    algo_codes = sum(N * K // 4 for (_, _, _, N, K) in shapes)
    xin = sum(M * K * 4 for (_, _, _, N, K) in shapes)
    yout = sum(M * N * 4 for (_, _, _, N, K) in shapes)
    return algo_codes + xin + yout, algo_codes, codes


def sweep_ops(shapes, M):
    return sum(2 * M * N * K for (_, _, _, N, K) in shapes)


def dist_summary(per_ms):
    """Median and 10th/90th percentiles (us) of per-step times in ms."""
    a = np.asarray(per_ms, np.float64) * 1e3
    return {"median_us": float(np.median(a)), "p10_us": float(np.percentile(a, 10)),
            "p90_us": float(np.percentile(a, 90)), "samples": int(a.size)}


def cpu_info():
    model = None
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    try:
        avail = len(os.sched_getaffinity(0))
    except AttributeError:
        avail = os.cpu_count()
    return {"cpu_model": model, "nproc": os.cpu_count(), "cpus_available": avail}


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

    def _sample(self):
        nv = self.nv
        names = {
            "hw_slowdown": getattr(nv, "nvmlClocksThrottleReasonHwSlowdown", 0x8),
            "hw_thermal_slowdown": getattr(nv, "nvmlClocksThrottleReasonHwThermalSlowdown", 0x40),
            "sw_thermal_slowdown": getattr(nv, "nvmlClocksThrottleReasonSwThermalSlowdown", 0x20),
            "sw_power_cap": getattr(nv, "nvmlClocksThrottleReasonSwPowerCap", 0x4),
        }
        try:
            mhz = nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM)
            r = nv.nvmlDeviceGetCurrentClocksThrottleReasons(self.h)
            self.samples.append(mhz)
            for k, bit in names.items():
                if r & bit:
                    self.reasons.add(k)
        except Exception:
            pass

    def _run(self):
        while not self.stop_ev.is_set():
            self._sample()
            time.sleep(0.002)

    def __enter__(self):
        if self.nv:
            self._sample()   # at least one sample inside the region
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        if self.nv:
            self.stop_ev.set()
            self.t.join()
            self._sample()

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


def _pool():
    import concurrent.futures as cf
    return cf.ThreadPoolExecutor(max_workers=min(16, os.cpu_count() or 4))


def build_weights(api, torch, dev, layers):
    """Generate and ternarise the 196 (7 x layers) projections on the GPU:
    [(layer, proj, name, N, K)] and [(packed, wscale)]."""
    from ternary_weight_decoder_b200 import synth
    shapes = synth.sweep_shapes(layers)
    pool = _pool()
    window = 16   # bounds host memory: at most this many fp32 matrices alive
    futs, weights = {}, []
    for i, (l, p, name, N, K) in enumerate(shapes):
        for j in range(i, min(i + window, len(shapes))):
            if j not in futs:
                lj, pj, _, Nj, Kj = shapes[j]
                futs[j] = pool.submit(synth.weights, lj, pj, Nj, Kj)
        W = futs.pop(i).result()
        Wd = torch.from_numpy(W).to(dev)
        packed, _, wscale = api.ternarize_pack(Wd)
        del Wd, W
        weights.append((packed, wscale))
    api.check()
    pool.shutdown()
    return shapes, weights


def decode_inputs(api, torch, dev, shapes, weights, M, rank, with_host=False):
    """Decode-sweep descriptors over M tokens: per projection its own seeded
    x (one contiguous device buffer) and y.  Returns (descs, x_host, x_all,
    y_all); x_host (pinned) only when with_host."""
    from ternary_weight_decoder_b200 import synth
    x_off, y_off, xo, yo = [], [], 0, 0
    for (_, _, _, N, K) in shapes:
        x_off.append(xo)
        y_off.append(yo)
        xo += M * K
        yo += M * N
    x_host = torch.empty(xo, dtype=torch.float32)
    if with_host:
        x_host = x_host.pin_memory()
    xn = x_host.numpy()
    pool = _pool()
    futs = [pool.submit(synth.activations, rank_layer_seed(l, rank), p, M, K)
            for (l, p, _, _, K) in shapes]
    for i, f in enumerate(futs):
        K = shapes[i][4]
        xn[x_off[i]:x_off[i] + M * K] = f.result().ravel()
    pool.shutdown()
    x_all = x_host.to(dev)
    y_all = torch.empty(yo, dtype=torch.float32, device=dev)
    descs = []
    for i, (_, _, _, N, K) in enumerate(shapes):
        packed, wscale = weights[i]
        descs.append(dict(x=x_all[x_off[i]:x_off[i] + M * K].view(M, K), packed=packed,
                          wscale=wscale, y=y_all[y_off[i]:y_off[i] + M * N].view(M, N),
                          N=N, K=K))
    torch.cuda.synchronize()
    return descs, (x_host if with_host else None), x_all, y_all


def prefill_inputs(api, torch, dev, shapes, weights, M, rank):
    """Prefill-sweep descriptors over M tokens: per projection
    PREFILL_DISTINCT_ROWS seeded token rows (with outliers) tiled up to M,
    quantised once by tw_quantize_act; y [M x N] per projection."""
    from ternary_weight_decoder_b200 import synth
    R = min(M, PREFILL_DISTINCT_ROWS)
    pool = _pool()
    futs = [pool.submit(synth.activations, rank_layer_seed(l, rank), p, R, K)
            for (l, p, _, _, K) in shapes]
    descs = []
    for i, (_, _, _, N, K) in enumerate(shapes):
        xr = torch.from_numpy(futs[i].result()).to(dev)
        x = xr.repeat((M + R - 1) // R, 1)[:M].contiguous()
        xq, amax, qsum = api.quantize_act(x)
        del x, xr
        packed, wscale = weights[i]
        descs.append(dict(xq=xq, amax=amax, qsum=qsum, packed=packed, wscale=wscale,
                          y=torch.empty((M, N), dtype=torch.float32, device=dev), N=N, K=K))
    pool.shutdown()
    api.check()
    return descs


def timed_steps(torch, stream, fn, steps, barrier):
    """Run fn `steps` times between a barrier + synchronize on each side;
    an event at every step boundary on `stream`.  Returns (total ms, per-step
    ms list)."""
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(steps + 1)]
    barrier()
    evs[0].record(stream)
    for i in range(steps):
        fn()
        evs[i + 1].record(stream)
    barrier()
    per = [evs[i].elapsed_time(evs[i + 1]) for i in range(steps)]
    return evs[0].elapsed_time(evs[steps]), per


def cold_calls(torch, stream, fn, n, flush, batch=32, sleep_cycles=40_000_000):
    """Device time of `n` calls of fn, each after an L2 flush (`flush()`
    writes more than the L2 holds; it is not timed).  A spin kernel at the
    head of every batch lets the host queue the whole batch, so the events
    bracket device work and not host launch gaps.  Returns per-call ms."""
    per = []
    for b0 in range(0, n, batch):
        nb = min(batch, n - b0)
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(nb)]
        torch.cuda._sleep(sleep_cycles)
        for a, b in evs:
            flush()
            a.record(stream)
            fn()
            b.record(stream)
        torch.cuda.synchronize()
        per += [a.elapsed_time(b) for a, b in evs]
    return per


def pool_calls(torch, stream, fns, batch=64, sleep_cycles=40_000_000):
    """Device time of each call in `fns`, run back to back in batches; a spin
    kernel at the head of every batch lets the host queue the whole batch,
    so an event after each call brackets device work only.  Returns
    per-call ms (the first call of each batch is not timed)."""
    per = []
    for b0 in range(0, len(fns), batch):
        chunk = fns[b0:b0 + batch]
        evs = [torch.cuda.Event(enable_timing=True) for _ in range(len(chunk))]
        torch.cuda._sleep(sleep_cycles)
        chunk[0]()
        evs[0].record(stream)
        for fn, ev in zip(chunk[1:], evs[1:]):
            fn()
            ev.record(stream)
        torch.cuda.synchronize()
        per += [evs[i - 1].elapsed_time(evs[i]) for i in range(1, len(chunk))]
    return per


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


def make_chain(api, torch, dev, shapes, weights, M, layers):
    per_layer = [dict() for _ in range(layers)]
    for (l, _, name, _, _), w in zip(shapes, weights):
        per_layer[l][name] = w
    hidden, kv, hd, inter = CHAIN_DIMS
    return api.DecoderChain(per_layer, M, hidden, kv, hd, inter, dev)


def run_chain(args, api, torch, dev, rank, world, dist, local):
    from ternary_weight_decoder_b200 import synth
    M = args.m
    if not 1 <= M <= 32:
        raise SystemExit("--chain runs decode token counts only (1..32)")
    shapes, weights = build_weights(api, torch, dev, args.layers)
    chain = make_chain(api, torch, dev, shapes, weights, M, args.layers)
    hidden = CHAIN_DIMS[0]
    h0_host = torch.from_numpy(synth.activations(rank_layer_seed(0, rank), 0, M, hidden)).pin_memory()
    h0 = h0_host.to(dev)
    stream = torch.cuda.current_stream()

    def step():
        chain.h.copy_(h0, non_blocking=True)   # every step starts from the same token state
        api.decoder_chain_fused(chain)

    for _ in range(args.warmup):
        step()
    api.check()

    def barrier():
        if dist is not None:
            dist.barrier()
        torch.cuda.synchronize()

    with ClockSampler(local) as clk:
        ms, per = timed_steps(torch, stream, step, args.steps, barrier)
    api.check()
    ms = max_over_ranks(ms, dist, dev)
    ms_per_step = ms / args.steps
    algo, codes = chain_bytes(shapes, M)
    hbm, _, src = peaks()
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
            api.decoder_chain_fused(chain)
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
    hidden, kv, hd, inter = CHAIN_DIMS
    print(json.dumps({
        "metric": CHAIN_METRIC, "value": job_value(M, world, args.steps, ms), "unit": UNIT,
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": DTYPE, "data": "synthetic",
        "config": {"workload": f"decoder_chain_{args.layers}L_M{M}", "M": M,
                   "layers": args.layers, "hidden": hidden, "kv_dim": kv, "head_dim": hd,
                   "inter": inter, "parallelism": f"dp{world} (independent replicas)",
                   "l2": f"codes {codes / 1e6:.0f} MB > 126 MB L2; no flush"},
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": hbm, "unit": "GB/s",
                     "frac": achieved / hbm, "traffic": None, "peak_source": peak_source(src),
                     "algorithmic_bytes_per_step": algo, "weight_bytes_per_step": codes,
                     "note": "the fused chain: one persistent launch per 8 tokens"},
        "step_times": dist_summary(per),
        "cpu_baseline": None, "e2e": e2e,
        "gpu_launches": chain.fused_launches * args.steps, "clocks": clk.summary(),
    }))


# ------------------------------------------------------------ oracle timing
_ORACLE_CODES = {}


def _oracle_sample(M, rows_cap, token_cap, budget_s, layers=28, sample_layers=1):
    """Time the oracle, as it stands, on one host core over the first
    `rows_cap` weight rows of each projection of the first `sample_layers`
    layers and min(M, token_cap) token rows, repeated for about budget_s;
    tokens/s of the full sweep extrapolated by weight count (and by tokens
    when fewer than M were run)."""
    from oracle import oracle as orc
    from ternary_weight_decoder_b200 import synth
    shapes = synth.sweep_shapes(layers)
    total_w = sum(N * K for (_, _, _, N, K) in shapes)
    toks = min(M, token_cap)
    sample = []
    for (l, p, name, N, K) in synth.sweep_shapes(min(sample_layers, layers)):
        r = min(rows_cap, N)
        if (l, p) not in _ORACLE_CODES:   # the oracle's ternarisation, done once per run
            _ORACLE_CODES[(l, p)] = orc.ternarize(synth.weights(l, p, N, K))
        codes, mean = _ORACLE_CODES[(l, p)]
        sample.append((synth.activations(l, p, toks, K), np.ascontiguousarray(codes[:r]), mean))
    sample_w = sum(c.size for _, c, _ in sample)
    timed, passes = 0.0, 0
    while timed < budget_s or passes == 0:
        t0 = time.perf_counter()
        for x, codes, mean in sample:
            orc.ternary_linear(x, codes, mean)
        timed += time.perf_counter() - t0
        passes += 1
    sweep_s = timed / passes * (total_w / sample_w) * (M / toks)
    desc = (f"{len(sample)} of {len(shapes)} projections, {'all rows' if rows_cap >= 8960 else f'first {rows_cap} rows each'} "
            f"({sample_w / total_w:.4f} of the weights), {toks} of {M} tokens, {passes} passes, "
            f"{timed:.1f} s timed; extrapolated to the full sweep by weight count"
            + (" and token count" if toks < M else ""))
    return {"value": M / sweep_s, "unit": UNIT, "cores": 1, "kind": "oracle",
            "sample": desc, **cpu_info()}


def _oracle_call_us(projs, M, budget_s):
    """Microseconds per call of the oracle on one host core, run back to back
    for about budget_s over the given (layer, projection) indices at M tokens
    (the whole matrices)."""
    from oracle import oracle as orc
    from ternary_weight_decoder_b200 import synth
    shapes = {(l, p): (N, K) for (l, p, _, N, K) in synth.sweep_shapes(1)}
    sample = []
    for lp in projs:
        N, K = shapes[lp]
        if lp not in _ORACLE_CODES:
            _ORACLE_CODES[lp] = orc.ternarize(synth.weights(lp[0], lp[1], N, K))
        codes, mean = _ORACLE_CODES[lp]
        sample.append((synth.activations(lp[0], lp[1], M, K), codes, mean))
    timed, passes = 0.0, 0
    while timed < budget_s or passes == 0:
        t0 = time.perf_counter()
        for x, codes, mean in sample:
            orc.ternary_linear(x, codes, mean)
        timed += time.perf_counter() - t0
        passes += 1
    return {"value": timed / passes * 1e6, "unit": "us per call", "cores": 1, "kind": "oracle",
            "sample": f"{len(sample)} whole projection(s) of layer 0 at {M} token(s), {passes} passes, "
                      f"{timed:.1f} s timed", **cpu_info()}


def _oracle_i8_us(W, bias, x, M, budget_s):
    """Microseconds per call of the oracle's I8_S layer over all M rows, from
    the rows of x (a sample of the rows) run back to back for about budget_s
    and extrapolated by row count."""
    from oracle import oracle as orc
    wq, amax_w = orc.i8_quantize_weights(W)
    timed, passes = 0.0, 0
    while timed < budget_s or passes == 0:
        t0 = time.perf_counter()
        orc.i8_linear(x, wq, amax_w, bias, relu=True)
        timed += time.perf_counter() - t0
        passes += 1
    return {"value": timed / passes * 1e6 * M / x.shape[0], "unit": "us per call", "cores": 1,
            "kind": "oracle", "sample": f"{x.shape[0]} of {M} token rows, {passes} passes, "
            f"{timed:.1f} s timed; extrapolated by row count", **cpu_info()}


def _oracle_chain_us(M, layers, budget_s):
    """Microseconds per token step of the oracle's decoder-layer chain: one
    layer (layer 0's projections) run back to back for about budget_s,
    times the layer count."""
    from oracle import oracle as orc
    from ternary_weight_decoder_b200 import synth
    layer = {}
    for (l, p, name, N, K) in synth.sweep_shapes(1):
        if (l, p) not in _ORACLE_CODES:
            _ORACLE_CODES[(l, p)] = orc.ternarize(synth.weights(l, p, N, K))
        layer[name] = _ORACLE_CODES[(l, p)]
    h = synth.activations(0, 0, M, CHAIN_DIMS[0])
    timed, passes = 0.0, 0
    while timed < budget_s or passes == 0:
        t0 = time.perf_counter()
        orc.decoder_layer(h, layer, head_dim=CHAIN_DIMS[2])
        timed += time.perf_counter() - t0
        passes += 1
    return {"value": timed / passes * 1e6 * layers, "unit": "us per step", "cores": 1,
            "kind": "oracle", "sample": f"1 of {layers} layers, {M} token(s), {passes} passes, "
            f"{timed:.1f} s timed; extrapolated by layer count", **cpu_info()}


def cpu_oracle_sample(M, budget_s=10.0, sample_layers=4, layers=28):
    """Headline CPU baseline: the oracle over all rows of the projections
    of the first `sample_layers` layers at M tokens."""
    return _oracle_sample(M, rows_cap=1 << 30, token_cap=M, budget_s=budget_s, layers=layers,
                          sample_layers=sample_layers)


def headline_config(M, layers, world):
    """The `config` of the headline line, the same for both arms."""
    shapes = [(N, K) for (_, _, _, N, K) in _sweep_shapes(layers)]
    algo = sum(N * K // 4 + M * K * 4 + M * N * 4 for (N, K) in shapes)
    if M <= 32:
        workload = (f"decode_sweep_196x_M{M}" if layers == 28
                    else f"decode_sweep_{7 * layers}x_M{M}")
    else:
        workload = f"prefill_sweep_{7 * layers}x_M{M}"
    return {"workload": workload, "M": M, "projections": len(shapes), "layers": layers,
            "parallelism": f"dp{world} (independent replicas, no collective)",
            "l2": f"inputs {algo / 1e6:.0f} MB > 126 MB L2; no flush"}


def _sweep_shapes(layers):
    from ternary_weight_decoder_b200 import synth
    return synth.sweep_shapes(layers)


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
        "vs_baseline": None, "dtype": DTYPE, "data": "synthetic",
        "config": headline_config(M, args.layers, args.gpus),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": 1, "kind": "oracle",
                         "sample": samp, **cpu_info()},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }))


# ------------------------------------------------------------ configs
def measure_configs(args, api, torch, dev, rank, shapes, weights, descs_m1, want, cpu_ok):
    """The benchmark definition's other workloads on the same weights."""
    from ternary_weight_decoder_b200 import synth
    hbm, int8_peak, src = peaks()
    stream = torch.cuda.current_stream()
    out = {}
    csteps = max(3, min(args.steps, 200))
    psteps = max(3, min(args.steps, 20))
    cwarm = max(3, min(args.warmup, 10))

    def barrier():
        torch.cuda.synchronize()

    flush_buf = None
    if "1" in want or "2" in want:
        flush_buf = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.int32, device=dev)
    flush_ctr = [0]

    def flush():
        flush_ctr[0] += 1
        flush_buf.fill_(flush_ctr[0])

    if "1" in want:
        # layer 0's q projection, x ~ N(0, 1) without outliers
        N = K = 1536
        assert shapes[0][3:] == (N, K)
        packed, wscale = weights[0]
        x = torch.from_numpy(synth.activations(rank_layer_seed(0, rank), 0, 1, K,
                                               outliers=False)).to(dev)
        y = torch.empty((1, N), dtype=torch.float32, device=dev)
        ws = torch.zeros(api.linear_workspace_bytes(1, N, K), dtype=torch.uint8, device=dev)

        def one():
            api.ternary_linear(x, packed, wscale, N, y=y, ws=ws)
        for _ in range(cwarm):
            one()
        api.check()
        per = cold_calls(torch, stream, one, max(32, min(args.steps, 512)), flush)
        api.check()
        s = dist_summary(per)
        nbytes = N * K // 4 + K * 4 + N * 4
        out["1_gemv_1536x1536_M1"] = {
            "us_per_call": s, "algorithmic_bytes": nbytes,
            "gbs_at_median": nbytes / (s["median_us"] * 1e-6) / 1e9,
            "frac_hbm_at_median": nbytes / (s["median_us"] * 1e-6) / 1e9 / hbm,
            "launches_per_call": 2, "l2": "flushed (256 MB written) before every call",
            "note": "launch-latency bound: the 0.6 MB of work is 0.09 us of HBM time"}
        # A rotating pool of distinct seeded 1536^2 matrices whose codes
        # exceed twice the L2, called back to back: each call's matrix was
        # last read a whole pool earlier, so it streams from HBM.
        pool_n = -(-L2_FLUSH_BYTES // (N * K // 4))
        gen = torch.Generator(device=dev)
        gen.manual_seed(20261202 + rank)
        pool = []
        for _ in range(pool_n):
            Wi = torch.randn((N, K), generator=gen, device=dev).mul_(0.02)
            pk, _, wsc = api.ternarize_pack(Wi)
            pool.append((pk, wsc))
            del Wi
        api.check()

        def call(i):
            return lambda: api.ternary_linear(x, pool[i][0], pool[i][1], N, y=y, ws=ws)
        fns = [call(i % pool_n) for i in range(2 * pool_n)]
        for f in fns[:pool_n]:
            f()
        api.check()
        per = pool_calls(torch, stream, fns)
        api.check()
        s = dist_summary(per)
        out["1_gemv_1536x1536_M1"]["rotating_pool"] = {
            "us_per_call": s, "matrices": pool_n, "pool_code_bytes": pool_n * (N * K // 4),
            "gbs_at_median": nbytes / (s["median_us"] * 1e-6) / 1e9,
            "frac_hbm_at_median": nbytes / (s["median_us"] * 1e-6) / 1e9 / hbm,
            "note": "calls back to back over distinct W ~ N(0, 0.02^2) (device-seeded), "
                    "codes of the pool > 2 x L2; one x and one y"}
        del pool, fns
        if cpu_ok:
            out["1_gemv_1536x1536_M1"]["oracle"] = _oracle_call_us([(0, 0)], 1, 2.0)

    if "2" in want:
        layer0 = descs_m1[:7]
        t1 = api.SweepTable(layer0, 1, device=dev)
        for _ in range(cwarm):
            api.decoder_projection_sweep(t1)
        api.check()
        per = cold_calls(torch, stream, lambda: api.decoder_projection_sweep(t1),
                         max(32, min(args.steps, 512)), flush)
        api.check()
        s = dist_summary(per)
        nbytes, _, _ = sweep_bytes(shapes[:7], 1)
        out["2_layer_7proj_M1"] = {
            "us_per_sweep": s, "us_per_matrix_median": s["median_us"] / 7,
            "algorithmic_bytes": nbytes,
            "frac_hbm_at_median": nbytes / (s["median_us"] * 1e-6) / 1e9 / hbm,
            "launches_per_call": t1.launches, "l2": "flushed (256 MB written) before every call"}
        if cpu_ok:
            out["2_layer_7proj_M1"]["oracle"] = _oracle_call_us([(0, p) for p in range(7)], 1, 3.0)
        del t1
    del flush_buf

    if "4" in want:
        for M in DECODE_MS:
            descs, _, x_all, y_all = decode_inputs(api, torch, dev, shapes, weights, M, rank)
            table = api.SweepTable(descs, M, device=dev)
            for _ in range(cwarm):
                api.decoder_projection_sweep(table)
            api.check()
            ms, per = timed_steps(torch, stream, lambda: api.decoder_projection_sweep(table),
                                  csteps, barrier)
            api.check()
            algo, codes, _ = sweep_bytes(shapes, M)
            step_s = ms / csteps / 1e3
            e = {"M": M, "tokens_per_s": M / step_s, "us_per_step": step_s * 1e6,
                 "step_times": dist_summary(per), "algorithmic_bytes": algo,
                 "achieved_gbs": algo / step_s / 1e9, "frac_hbm": algo / step_s / 1e9 / hbm,
                 "weight_gbs": codes / step_s / 1e9, "launches_per_step": table.launches,
                 "dominant_kernel_src": decode_kernel_src(M),
                 "traffic": profiled_traffic(decode_kernel_src(M), M, args.layers)}
            if cpu_ok:
                e["oracle"] = _oracle_sample(M, rows_cap=512, token_cap=M, budget_s=2.5,
                                             layers=args.layers)
            out[f"4_decode_sweep_196x_M{M}"] = e
            del table, descs, x_all, y_all
            torch.cuda.empty_cache()

    if "5" in want:
        for M in PREFILL_MS:
            descs = prefill_inputs(api, torch, dev, shapes, weights, M, rank)
            table = api.SweepTable(descs, M, device=dev)
            for _ in range(cwarm):
                api.decoder_projection_sweep(table)
            api.check()
            ms, per = timed_steps(torch, stream, lambda: api.decoder_projection_sweep(table),
                                  psteps, barrier)
            api.check()
            step_s = ms / psteps / 1e3
            ops = sweep_ops(shapes, M)
            e = {"M": M, "tokens_per_s": M / step_s, "us_per_step": step_s * 1e6,
                 "step_times": dist_summary(per), "int8_ops": ops,
                 "achieved_tops": ops / step_s / 1e12, "peak_tops": int8_peak,
                 "frac_int8": ops / step_s / 1e12 / int8_peak,
                 "launches_per_step": table.launches,
                 "inputs": f"{min(M, PREFILL_DISTINCT_ROWS)} distinct seeded token rows per "
                           f"projection tiled to {M}, quantised before the timed region",
                 "traffic": profiled_traffic("tw_prefill.cu", M, args.layers)}
            if cpu_ok:
                e["oracle"] = _oracle_sample(M, rows_cap=64, token_cap=256, budget_s=3.0,
                                             layers=args.layers)
            out[f"5_prefill_sweep_196x_M{M}"] = e
            del table, descs
            torch.cuda.empty_cache()

    if "mid" in want:
        # 33..192 tokens: the default (weights expanded into tensor memory)
        # against the expanded-weights GEMM on the same descriptors
        for M in MID_MS:
            descs = prefill_inputs(api, torch, dev, shapes, weights, M, rank)
            e = {"M": M, "inputs": f"{min(M, PREFILL_DISTINCT_ROWS)} distinct seeded token rows "
                                   f"per projection, quantised before the timed region"}
            ops = sweep_ops(shapes, M)
            _, codes, _ = sweep_bytes(shapes, M)
            nbytes = codes + sum(M * K + M * N * 4 for (_, _, _, N, K) in shapes)
            for gemm, name in (("auto", "tmem_weights"), ("expanded", "expanded_weights")):
                table = api.SweepTable(descs, M, device=dev, gemm=gemm)
                for _ in range(cwarm):
                    api.decoder_projection_sweep(table)
                api.check()
                ms, per = timed_steps(torch, stream, lambda: api.decoder_projection_sweep(table),
                                      psteps, barrier)
                api.check()
                step_s = ms / psteps / 1e3
                e[name] = {"tokens_per_s": M / step_s, "us_per_step": step_s * 1e6,
                           "step_times": dist_summary(per),
                           "achieved_tops": ops / step_s / 1e12,
                           "frac_int8": ops / step_s / 1e12 / int8_peak,
                           "achieved_gbs": nbytes / step_s / 1e9,
                           "frac_hbm": nbytes / step_s / 1e9 / hbm,
                           "launches_per_step": table.launches}
                del table
            e["default"] = "tmem_weights"
            e["speedup_vs_expanded"] = (e["expanded_weights"]["us_per_step"]
                                        / e["tmem_weights"]["us_per_step"])
            e["int8_ops"], e["algorithmic_bytes"] = ops, nbytes
            e["traffic"] = profiled_traffic("tw_mid.cu", M, args.layers)
            if cpu_ok:
                e["oracle"] = _oracle_sample(M, rows_cap=64, token_cap=M, budget_s=2.5,
                                             layers=args.layers)
            out[f"f2_mid_sweep_196x_M{M}"] = e
            del descs
            torch.cuda.empty_cache()

    if "i8" in want:
        for (M, K, N) in I8_SHAPES:
            W = synth.weights(7000 + K, 0, N, K, 0.05)
            wq, amax_w = api.i8_quantize_weights(torch.from_numpy(W).to(dev))
            bias = torch.from_numpy((np.random.default_rng(K).standard_normal(N) * 0.1)
                                    .astype(np.float32)).to(dev)
            xr = torch.from_numpy(synth.activations(7000 + K, 1, min(M, 1024), K)).to(dev)
            x = xr.repeat((M + xr.shape[0] - 1) // xr.shape[0], 1)[:M].contiguous()
            xq, amax_x, _ = api.quantize_act(x)
            y = torch.empty((M, N), dtype=torch.float32, device=dev)
            ws = torch.empty(api.tw_i8_workspace_bytes(M, K), dtype=torch.uint8, device=dev)
            api.check()

            def gemm():
                api.i8_linear_q(xq, amax_x, wq, amax_w, bias, relu=True, y=y)

            def layer():
                api.i8_linear(x, wq, amax_w, bias, relu=True, y=y, ws=ws)
            res = {}
            for name, fn in (("gemm", gemm), ("layer", layer)):
                for _ in range(cwarm):
                    fn()
                api.check()
                ms, per = timed_steps(torch, stream, fn, csteps, barrier)
                api.check()
                step_s = ms / csteps / 1e3
                ops = 2 * M * N * K
                nbytes = M * K + N * K + 4 * M * N + 4 * M + (4 * M * K + M * K if name == "layer" else 0)
                res[name] = {"us_per_call": step_s * 1e6, "step_times": dist_summary(per),
                             "algorithmic_bytes": nbytes, "achieved_gbs": nbytes / step_s / 1e9,
                             "frac_hbm": nbytes / step_s / 1e9 / hbm,
                             "achieved_tops": ops / step_s / 1e12,
                             "frac_int8": ops / step_s / 1e12 / int8_peak,
                             "bound": "hbm" if nbytes / hbm / 1e9 > ops / int8_peak / 1e12 else "tensor",
                             "launches_per_call": 1 if name == "gemm" else 2}
            out[f"i8_linear_bias_relu_M{M}_K{K}_N{N}"] = {
                **res, "inputs": f"{min(M, 1024)} distinct seeded token rows tiled to {M}; "
                                 "W ~ N(0, 0.05^2); bias ~ N(0, 0.1^2)",
                "note": "gemm: int8 activations quantised beforehand; layer: fp32 activations "
                        "quantised in the call (two launches)"}
            if cpu_ok:
                out[f"i8_linear_bias_relu_M{M}_K{K}_N{N}"]["oracle"] = _oracle_i8_us(
                    W, bias.cpu().numpy(), xr[:64].cpu().numpy(), M, 2.0)
            del W, wq, xq, x, xr, y, ws
            torch.cuda.empty_cache()

    if "chain" in want:
        M = 1
        chain = make_chain(api, torch, dev, shapes, weights, M, args.layers)
        h0 = torch.from_numpy(synth.activations(rank_layer_seed(0, rank), 0, M,
                                                CHAIN_DIMS[0])).to(dev)

        res = {}
        for name, run, launches in (("fused", api.decoder_chain_fused, chain.fused_launches),
                                    ("unfused", api.decoder_chain, chain.launches)):
            def cstep():
                chain.h.copy_(h0, non_blocking=True)
                run(chain)
            for _ in range(cwarm):
                cstep()
            api.check()
            ms, per = timed_steps(torch, stream, cstep, csteps, barrier)
            api.check()
            algo, codes = chain_bytes(shapes, M)
            step_s = ms / csteps / 1e3
            res[name] = {"tokens_per_s": M / step_s, "us_per_step": step_s * 1e6,
                         "step_times": dist_summary(per), "frac_hbm": algo / step_s / 1e9 / hbm,
                         "launches_per_step": launches + 1}
        out["chain_28L_M1"] = {
            "M": M, **res, "algorithmic_bytes": algo,
            "note": "28 dependent layers from one token state (the +1 launch copies it in); "
                    "fused: one persistent launch, 112 grid-wide barriers; unfused: per layer "
                    "4 sweeps and 4 element-wise launches"}
        if cpu_ok:
            out["chain_28L_M1"]["oracle"] = _oracle_chain_us(M, args.layers, 3.0)
        del chain
    return out


def measure_e2e(args, api, torch, dev, dist, world, M, descs, table, x_host, x_all, y_all,
                barrier):
    """The headline metric through the public API with host buffers: every
    step copies its x from pinned host memory, runs the sweep and copies its
    y back to pinned host memory, and the host reads every step's result.
    Two sets of device buffers (and sweep tables) let step k's copies run on
    their own streams (one per direction) while the sweep of step k - 1
    runs; the host waits for step k - 1's result after issuing step k."""
    x_b = [x_all, torch.empty_like(x_all)]
    y_b = [y_all, torch.empty_like(y_all)]
    descs2 = []
    for d in descs:
        xo = (d["x"].data_ptr() - x_all.data_ptr()) // 4
        yo = (d["y"].data_ptr() - y_all.data_ptr()) // 4
        descs2.append(dict(d, x=x_b[1][xo:xo + d["x"].numel()].view(d["x"].shape),
                           y=y_b[1][yo:yo + d["y"].numel()].view(d["y"].shape)))
    tables = [table, api.SweepTable(descs2, M, device=dev)]
    y_host = [torch.empty(y_all.numel(), dtype=torch.float32).pin_memory() for _ in range(2)]
    compute = torch.cuda.current_stream()
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_comp = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]

    def step(k):
        b = k & 1
        with torch.cuda.stream(s_in):
            if k >= 2:
                s_in.wait_event(ev_comp[b])      # the sweep of k - 2 has read x[b]
            x_b[b].copy_(x_host, non_blocking=True)
            ev_in[b].record(s_in)
        compute.wait_event(ev_in[b])
        if k >= 2:
            compute.wait_event(ev_out[b])        # y[b] of k - 2 is in host memory
        api.decoder_projection_sweep(tables[b], stream=compute)
        ev_comp[b].record(compute)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev_comp[b])
            y_host[b].copy_(y_b[b], non_blocking=True)
            ev_out[b].record(s_out)
        if k >= 1:
            ev_out[(k - 1) & 1].synchronize()   # the host reads step k - 1's result

    def run(n):
        for k in range(n):
            step(k)
        ev_out[(n - 1) & 1].synchronize()

    run(4)
    api.check()
    k2 = max(3, min(args.steps, 2000))
    barrier()
    t0 = time.perf_counter()
    f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    f0.record(s_in)
    for k in range(k2):
        step(k)
    f1.record(s_out)
    f1.synchronize()
    barrier()
    wall = time.perf_counter() - t0
    api.check()
    ems = max_over_ranks(f0.elapsed_time(f1), dist, dev)
    return {"value": job_value(M, world, k2, ems), "unit": UNIT,
            "h2d_bytes_per_step": x_all.numel() * 4, "d2h_bytes_per_step": y_all.numel() * 4,
            "steps": k2, "ms_per_step": ems / k2, "host_wall_ms_per_step": wall * 1e3 / k2,
            "pipeline": "two device buffer sets; each step's H2D and D2H copies on their own "
                        "streams overlap the neighbouring steps' sweeps; the host reads every "
                        "step's result, one step behind"}


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
    shapes, weights = build_weights(api, torch, dev, args.layers)
    if M > 32:
        descs = prefill_inputs(api, torch, dev, shapes, weights, M, rank)
        x_host = x_all = None
        y_all = None
    else:
        descs, x_host, x_all, y_all = decode_inputs(api, torch, dev, shapes, weights, M, rank,
                                                    with_host=True)
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

    with ClockSampler(local) as clk:
        ms, per = timed_steps(torch, stream, lambda: api.decoder_projection_sweep(table),
                              args.steps, barrier)
    api.check()
    ms = max_over_ranks(ms, dist, dev)
    ms_per_step = ms / args.steps
    value = job_value(M, world, args.steps, ms)

    hbm, int8_peak, src = peaks()
    if M <= 32:
        # decode: HBM-bound; algorithmic bytes = 2-bit codes + fp32 x + fp32 y
        achieved = algo_bytes / (ms_per_step / 1e3) / 1e9
        roofline = {"bound": "hbm", "achieved": achieved, "peak": hbm, "unit": "GB/s",
                    "frac": achieved / hbm,
                    "traffic": profiled_traffic(decode_kernel_src(M), M, args.layers),
                    "peak_source": peak_source(src),
                    "algorithmic_bytes_per_step": algo_bytes,
                    "weight_bytes_per_step": algo_codes,
                    "weight_gbs": algo_codes / (ms_per_step / 1e3) / 1e9,
                    "note": "step = quantise launch + decode launch; time of the whole step"}
    else:
        # prefill: int8 tensor-core bound; 2*M*N*K ops per projection
        ops = sweep_ops(shapes, M)
        tops = ops / (ms_per_step / 1e3) / 1e12
        roofline = {"bound": "tensor", "achieved": tops, "peak": int8_peak, "unit": "TOP/s",
                    "frac": tops / int8_peak,
                    "traffic": profiled_traffic("tw_prefill.cu", M, args.layers),
                    "peak_source": peak_source(src), "ops_per_step": ops}

    e2e = None
    if not args.no_e2e and M <= 32:
        e2e = measure_e2e(args, api, torch, dev, dist, world, M, descs, table, x_host, x_all,
                          y_all, barrier)

    cpu_ok = rank == 0 and world == 1 and not args.no_cpu
    cpu = cpu_oracle_sample(M, layers=args.layers) if cpu_ok and M <= 32 else None

    configs, cclk = None, None
    if not args.no_configs and M == 1 and args.layers == 28:
        want = set(w.strip() for w in args.configs.split(",") if w.strip())
        del table
        with ClockSampler(local) as cs:
            configs = measure_configs(args, api, torch, dev, rank, shapes, weights, descs,
                                      want, cpu_ok)
        cclk = cs.summary()

    if dist is not None:
        dist.destroy_process_group()
    if rank != 0:
        return
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": DTYPE, "data": "synthetic",
        "config": headline_config(M, args.layers, world),
        "roofline": roofline, "step_times": dist_summary(per), "cpu_baseline": cpu, "e2e": e2e,
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clk.summary(),
    }
    if configs is not None:
        line["configs"] = configs
        line["configs_clocks"] = cclk
    print(json.dumps(line))


if __name__ == "__main__":
    main()
