"""Benchmark of the packed variable-length attention forward on B200.

Metric: effective TFLOP/s over valid FLOPs, 4 * sum(L_i^2) * d * H per call
(block-diagonal work only; masked tail work and padding do not count), on the
mixed-resolution pack (512x512, 1024x1024 and 768x432 images at patch 16 ->
segments [1024, 4096, 1296], 24 heads, head_dim 128, bf16).  One step = one
call of the C-ABI entry point ``pa_varlen_attn_fwd`` (schedule kernel +
attention kernel) on inputs resident in HBM; L2 is flushed between timed steps.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--config NAME]

Beside the headline the line carries: ``steady_state`` (at least --steady-s seconds of
back-to-back calls, with the clock samples of that region and the roofline against the
sustained bf16 figure), ``per_config`` (the other workloads, each with its kernel's
roofline), ``short_segments`` (packs of small images, where the path is bound by HBM:
unique bytes / time against the measured copy bandwidth), and the backward, the
projections and the FP8 variant of the same pack.

With N > 1 (torchrun, one rank per GPU) every rank runs its own pack of the same
shape (independent replicas: the forward has no exchange step), the timed
region is bracketed by barriers, and the time is the max over ranks.
``--impl reference`` times the fp64 CPU oracle on bounded samples of the same
workload on the host cores.
"""
import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

import workloads  # noqa: E402

FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
L2_FLUSH_BYTES = 256 << 20


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def dist_setup(n_gpus):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if torch.cuda.is_available():
            torch.cuda.set_device(local)
        torch.distributed.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=120))
    return world, rank, local


def barrier(world):
    if world > 1:
        torch.distributed.barrier()


def allreduce_max(x, world, device):
    if world <= 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


class ClockSampler:
    """nvidia-smi samples of the SM clock, power and throttle reasons, each with its own
    timestamp, so that only the samples taken inside the timed region are reported."""
    FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    PERIOD_MS = 20

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.rows = []
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", str(self.PERIOD_MS)], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except (OSError, FileNotFoundError):
            self.proc = None

    def _read(self):
        import datetime
        for line in self.proc.stdout:
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 10:
                continue
            ts = None
            for fmt in ("%Y/%m/%d %H:%M:%S.%f", "%Y/%m/%d %H:%M:%S", "%a %b %d %H:%M:%S %Y"):
                try:
                    ts = datetime.datetime.strptime(parts[0], fmt).timestamp()
                    break
                except ValueError:
                    pass
            if ts is None:
                continue
            self.rows.append([ts] + parts[1:])

    def summary(self, t0, t1):
        """Summary of the samples taken in [t0, t1] (host wall-clock seconds); the sampler keeps running."""
        if self.proc is None:
            return None
        rows = [r for r in list(self.rows) if t0 <= r[0] <= t1]
        in_region = bool(rows)
        if not rows and self.rows:  # region shorter than the sampling period: nearest sample (within 1 s)
            near = min(self.rows, key=lambda r: abs(r[0] - t0))
            rows = [near] if abs(near[0] - t0) <= 1.0 else []
        if not rows:
            return None
        num = lambda x: x.replace(".", "", 1).isdigit()
        sm = [float(r[2]) for r in rows if num(r[2])]
        mx = [float(r[3]) for r in rows if num(r[3])]
        pw = [float(r[4]) for r in rows if num(r[4])]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[6 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows) if in_region else 0,
                "power_w_median": statistics.median(pw) if pw else None,
                "window": "samples taken inside the timed region" if in_region
                          else "timed region shorter than the sampling period: nearest sample"}

    def stop(self, t0=None, t1=None):
        """Stops sampling; returns the summary of [t0, t1] when a window is given."""
        if self.proc is None:
            return None
        time.sleep(2.5 * self.PERIOD_MS / 1e3)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        return self.summary(t0, t1) if t0 is not None else None


def workload_desc(cfg):
    segs = cfg["segments"]
    desc = {"workload": f"{cfg['name']} pack: {cfg.get('description', '')}",
            "segments": segs if len(segs) <= 32 else f"{len(segs)} segments",
            "total_tokens": int(sum(segs)), "heads": cfg["heads"], "head_dim": cfg["head_dim"],
            "valid_flops_per_step": workloads.valid_flops(segs, cfg["heads"], cfg["head_dim"])}
    return desc


def oracle_sample_rate(p, cfg, target_s, seed=0, max_rows=None):
    """Times the fp64 oracle on a bounded random sample of (token, head) rows; returns
    (TFLOP/s over the sample's valid FLOPs, rows, seconds, threads)."""
    import oracle
    segs = cfg["segments"]
    T, H, d = sum(segs), cfg["heads"], cfg["head_dim"]
    cu = np.concatenate([[0], np.cumsum(segs)])
    seg_len = np.repeat(np.array(segs), segs)  # length of the segment of every token
    rng = np.random.default_rng(seed)
    n = 8
    while True:
        tok = rng.integers(0, T, size=n)
        head = rng.integers(0, H, size=n).astype(np.int32)
        t0 = time.perf_counter()
        oracle.varlen_attention(p["q"], p["k"], p["v"], cu, p["scale"], rows=(tok, head))
        dt = time.perf_counter() - t0
        if dt >= target_s or (max_rows and n >= max_rows):
            flops = float(np.sum(4.0 * seg_len[tok] * d))
            return flops / dt / 1e12, n, dt, oracle.default_threads()
        n = int(n * min(8.0, max(2.0, 1.2 * target_s / max(dt, 1e-4))))
        if max_rows:
            n = min(n, max_rows)


def run_reference(args, world, rank):
    if rank != 0:
        return 0
    cfg = workloads.load_config(args.config)
    p = workloads.make_inputs(cfg)
    # size one step so that (warmup + steps) samples take about two minutes in all
    per_step = max(0.02, 120.0 / max(1, args.steps + args.warmup))
    rates = []
    rows = secs = threads = 0
    for i in range(args.warmup + args.steps):
        r, rows, secs, threads = oracle_sample_rate(p, cfg, per_step, seed=i)
        if i >= args.warmup:
            rates.append(r)
    value = statistics.median(rates)
    flops = workloads.valid_flops(cfg["segments"], cfg["heads"], cfg["head_dim"])
    line = {"impl": "reference", "metric": HEADLINE_METRIC, "value": value, "unit": "TFLOP/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": flops / (value * 1e12) * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": dict(workload_desc(cfg), parallelism="host cores"),
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
                             "sample": f"{rows} random (token, head) rows per step, about {secs:.1f} s each; "
                                       "rate extrapolated to the whole pack by valid FLOPs"},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line))
    return 0


HEADLINE_METRIC = "varlen attn fwd effective TFLOP/s (valid FLOPs) on 1 B200; % of BF16 peak"


def traffic_for_current_kernel(record="attn_fwd_traffic.json"):
    """DRAM bytes per launch from a committed ncu summary, if it matches the kernel source as built."""
    import hashlib
    path = os.path.join(ROOT, "profiles", record)
    if not os.path.exists(path):
        return None
    with open(path) as f:
        rec = json.load(f)
    h = hashlib.sha256()
    for name in rec.get("sources", []):
        with open(os.path.join(ROOT, name), "rb") as f:
            h.update(f.read())
    if h.hexdigest() != rec.get("sources_sha256"):
        return None
    return rec


def time_steps(call, flush, stream, warmup, steps, world, device, flush_each=True):
    """W untimed calls, then K calls each bracketed by CUDA events on the launching stream (L2
    flushed before every call when flush_each), barriers + synchronize around the region.
    Returns (per-call ms list, host t0, host t1) with the per-call times max-reduced over ranks."""
    for _ in range(warmup):
        if flush_each:
            flush.fill_(1.0)
        call()
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    barrier(world)
    torch.cuda.synchronize()
    t0 = time.time()
    for a, b in ev:
        if flush_each:
            flush.fill_(1.0)  # evict the operands from L2 (untimed)
        a.record(stream)
        call()
        b.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    t1 = time.time()
    ms = [a.elapsed_time(b) for a, b in ev]
    if world > 1:
        t = torch.tensor(ms, dtype=torch.float64, device=device)
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
        ms = t.tolist()
    return ms, t0, t1


def kernel_ms(pa, call, flush, steps, flush_each=True):
    """Average duration (ms) of the library's main kernel over `steps` calls, from the events
    the library records around it on its launch stream; also the host seconds the run took."""
    pa.pa_profile_read()  # clear
    pa.pa_profile_enable(True)
    t0 = time.time()
    for _ in range(steps):
        if flush_each:
            flush.fill_(1.0)
        call()
    torch.cuda.synchronize()
    dt = time.time() - t0
    pa.pa_profile_enable(False)
    tot, n = pa.pa_profile_read()
    return tot / max(1, n), dt


def paired_steps(pa, call, flush, stream, warmup, steps, world, device):
    """Per-call times and the main kernel's time from one region: `steps` pairs of calls, L2
    flushed before each; the first call of a pair is bracketed by CUDA events, the second runs
    with the library's kernel events on. Both numbers then come from the same clock and power
    state (two back-to-back loops can see different ones). Returns (per-call ms list, kernel
    ms average)."""
    for _ in range(warmup):
        flush.fill_(1.0)
        call()
    torch.cuda.synchronize()
    pa.pa_profile_read()  # clear
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    barrier(world)
    torch.cuda.synchronize()
    for a, b in ev:
        flush.fill_(1.0)
        a.record(stream)
        call()
        b.record(stream)
        flush.fill_(1.0)
        pa.pa_profile_enable(True)
        call()
        pa.pa_profile_enable(False)
    torch.cuda.synchronize()
    barrier(world)
    ms = [a.elapsed_time(b) for a, b in ev]
    if world > 1:
        t = torch.tensor(ms, dtype=torch.float64, device=device)
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
        ms = t.tolist()
    tot, n = pa.pa_profile_read()
    return ms, tot / max(1, n)


def fp8_compare(pa, pack, flush, stream, warmup, steps):
    """bf16 call against the FP8 path on one pack (d = 128), interleaved step by step so that
    all four see the same clocks: the bf16 call; the quantiser (maxima of this call) + FP8
    attention; the delayed-scaling quantiser (a previous step's maxima) + FP8 attention; the FP8
    attention alone. L2 flushed before each; returns the mean ms of each."""
    T, H, d = pack.T, pack.H, pack.d
    dev = pack.q.device
    B = pack.cu.numel() - 1
    q8, k8 = (torch.empty(T, H, d, dtype=torch.uint8, device=dev) for _ in range(2))
    v8t = torch.empty(H * d, pa.pa_fp8_vt_keys(B, T), dtype=torch.uint8, device=dev)
    sc8 = torch.empty(4 + H * d, dtype=torch.float32, device=dev)
    out8, lse8 = torch.empty_like(pack.out), torch.empty_like(pack.lse)
    am_in = torch.ones(4 + H * d, dtype=torch.float32, device=dev)
    am_out = torch.empty_like(am_in)

    def check(rc, what):
        if rc != pa.PA_OK:
            raise pa.PackAttnError(rc, what)

    check(pa.pa_fp8_quantize_qkv_delayed(pack.q, pack.k, pack.v, pack.cu, am_out, am_in, q8, k8, v8t, sc8, stream),
          "pa_fp8_quantize_qkv_delayed")  # am_in = this pack's maxima (a previous step's record)
    quant = lambda: check(pa.pa_fp8_quantize_qkv(pack.q, pack.k, pack.v, pack.cu, q8, k8, v8t, sc8, stream),
                          "pa_fp8_quantize_qkv")
    dquant = lambda: check(pa.pa_fp8_quantize_qkv_delayed(pack.q, pack.k, pack.v, pack.cu, am_in, am_out, q8, k8,
                                                          v8t, sc8, stream), "pa_fp8_quantize_qkv_delayed")
    attn = lambda: check(pa.pa_varlen_attn_fwd_fp8(q8, k8, v8t, sc8, pack.cu, pack.p["max_seqlen"],
                                                   pack.p["scale"], out8, lse8, stream), "pa_varlen_attn_fwd_fp8")
    arms = [pack, lambda: (quant(), attn()), lambda: (dquant(), attn()), attn]
    for _ in range(warmup):
        for fn in arms:
            flush.fill_(1.0)
            fn()
    torch.cuda.synchronize()
    ev = [[(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in arms]
          for _ in range(steps)]
    for row in ev:
        for fn, (a, b) in zip(arms, row):
            flush.fill_(1.0)
            a.record(stream)
            fn()
            b.record(stream)
    torch.cuda.synchronize()
    check(pa.pa_get_error(stream), "fp8 comparison")
    ms = [sum(row[i][0].elapsed_time(row[i][1]) for row in ev) / steps for i in range(len(arms))]
    return dict(bf16_ms=ms[0], quant_attn_ms=ms[1], delayed_attn_ms=ms[2], attn_ms=ms[3], steps=steps)


def unique_bytes(T, H, d):
    """Algorithmic HBM bytes of one forward call: q, k, v read and out written (bf16), lse written (fp32)."""
    return 4.0 * T * H * d * 2 + 4.0 * T * H


class Pack:
    """Device-resident inputs and outputs of one workload, and the C-ABI call on them."""

    def __init__(self, pa, cfg, device, stream, seed_offset=0):
        self.pa, self.cfg, self.stream = pa, cfg, stream
        p = workloads.make_inputs(dict(cfg, seed=int(cfg["seed"]) + seed_offset))
        self.p = p
        self.segs = [int(n) for n in cfg["segments"]]
        self.T, self.H, self.d = sum(self.segs), int(cfg["heads"]), int(cfg["head_dim"])
        self.flops = workloads.valid_flops(self.segs, self.H, self.d)
        self.bytes = unique_bytes(self.T, self.H, self.d)
        self.q, self.k, self.v = (p[n].to(device) for n in ("q", "k", "v"))
        self.cu = p["cu_seqlens"].to(device)
        self.out = torch.empty_like(self.q)
        self.lse = torch.empty(self.T, self.H, dtype=torch.float32, device=device)

    def __call__(self):
        pa = self.pa
        rc = pa.pa_varlen_attn_fwd(self.q, self.k, self.v, self.cu, self.p["max_seqlen"], self.p["scale"],
                                   self.out, self.lse, self.stream)
        if rc != pa.PA_OK:
            raise pa.PackAttnError(rc, "pa_varlen_attn_fwd")


def measure_pack(pa, pack, flush, stream, args, world, device, target_s=0.5, clocks=None):
    """Per-call time of one pack (L2 flushed before every call) and its kernel alone; the step
    count is the bench's, capped so that the region stays under about `target_s` seconds."""
    pack()
    torch.cuda.synchronize()
    t0 = time.time()
    pack()
    torch.cuda.synchronize()
    est = max(time.time() - t0, 1e-5)
    steps = max(5, min(args.steps, int(target_s / est)))
    t0 = time.time()
    ms, kms = paired_steps(pa, pack, flush, stream, args.warmup, steps, world, device)
    t1 = time.time()
    rc = pa.pa_get_error(stream)
    if rc != pa.PA_OK:
        raise pa.PackAttnError(rc, pack.cfg["name"])
    ledger = pa.pa_schedule_stats(stream)  # the tile ledger of the last call
    call_ms = sum(ms) / len(ms)
    return dict(steps=steps, ms_per_call=call_ms, kernel_ms=kms, ledger=ledger,
                clocks=clocks.summary(t0, t1) if clocks else None,
                tflops=pack.flops * world / (call_ms * 1e-3) / 1e12,
                kernel_tflops=pack.flops / (kms * 1e-3) / 1e12,
                gbs=pack.bytes * world / (call_ms * 1e-3) / 1e9,
                kernel_gbs=pack.bytes / (kms * 1e-3) / 1e9)


def head_kernel_name(d):
    return "attn_fwd_kernel<128>" if d == 128 else "attn_fwd_kernel<64>"


def run_ours(args, world, rank, local):
    import dit_resolution_packed_b200 as pa
    if not torch.cuda.is_available():
        raise RuntimeError("bench.py needs a CUDA device")
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    cfg = workloads.load_config(args.config)
    stream = torch.cuda.current_stream()
    head = Pack(pa, cfg, device, stream, seed_offset=7919 * rank)  # each replica its own data, same shapes
    p, segs, T, H, d, flops = head.p, head.segs, head.T, head.H, head.d, head.flops
    q, k, v, cu, out, lse = head.q, head.k, head.v, head.cu, head.out, head.lse
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=device)
    call = head

    # the clock sampler runs from here to the end; each record keeps the samples of its own region
    clocks = ClockSampler(local) if rank == 0 else None
    if clocks:
        clocks.start()
        time.sleep(0.3)  # nvidia-smi needs a moment to start

    # ---- headline: K calls after W warm-up calls, L2 flushed before each (a burst of K calls)
    step_ms, t_region0, t_region1 = time_steps(call, flush, stream, args.warmup, args.steps, world, device)
    rc = pa.pa_get_error(stream)
    if rc != pa.PA_OK:
        raise pa.PackAttnError(rc, "timed region")
    # attention kernel alone (for the roofline): the library brackets it with events on its
    # launch stream; the schedule kernel is outside the events
    kern_avg_ms, t_prof = kernel_ms(pa, call, flush, args.steps)
    head_ledger = pa.pa_schedule_stats(stream)
    clock_rec = clocks.summary(t_region0, t_region1) if clocks else None
    rc = pa.pa_get_error(stream)
    if rc != pa.PA_OK:
        raise pa.PackAttnError(rc, "timed region")
    q10, q50, q90 = (float(x) for x in np.percentile(step_ms, [10, 50, 90]))
    ms_per_step = sum(step_ms) / args.steps
    value = flops * world / (ms_per_step * 1e-3) / 1e12

    # ---- steady state under the board's power limit: back-to-back calls of the same pack for
    # at least `steady_s` seconds (no flush between calls: the 158 MB of operands exceed the
    # 126 MB L2), per-call events and the kernel's own events, clock samples inside the region
    n_ss = max(args.steps, int(args.steady_s / max(ms_per_step * 1e-3, 1e-6)) + 1)
    ss_ms, ss_t0, ss_t1 = time_steps(call, flush, stream, 0, n_ss, world, device, flush_each=False)
    ss_kern_ms, _ = kernel_ms(pa, call, flush, n_ss, flush_each=False)
    ss_clock = clocks.summary(ss_t0, ss_t1 + 0.02) if clocks else None
    rc = pa.pa_get_error(stream)
    if rc != pa.PA_OK:
        raise pa.PackAttnError(rc, "steady-state region")
    ss_call_ms = sum(ss_ms) / len(ss_ms)

    # ---- backward (the gradients of the same call): out and lse from the forward above, dout a
    # seeded N(0,1) tensor; same warm-up, step count and L2 flush as the forward
    dout = workloads.random_dout(q.shape, 7919 + rank).to(device)
    gq, gk, gv = (torch.empty_like(q) for _ in range(3))

    def bwd_call():
        rc = pa.pa_varlen_attn_bwd(q, k, v, out, lse, dout, cu, p["max_seqlen"], p["scale"], gq, gk, gv, stream)
        if rc != pa.PA_OK:
            raise pa.PackAttnError(rc, "pa_varlen_attn_bwd")

    bwd_step_ms, bkern_ms = paired_steps(pa, bwd_call, flush, stream, args.warmup, args.steps, world, device)
    t_bprof = 2e-3 * sum(bwd_step_ms)  # the paired region's length, about
    rc = pa.pa_get_error(stream)
    if rc != pa.PA_OK:
        raise pa.PackAttnError(rc, "backward region")
    bwd_flops = 2.5 * flops  # five GEMMs (S^T, dP^T, dV, dK, dQ) against the forward's two
    bwd_ms = allreduce_max(sum(bwd_step_ms), world, device) / args.steps
    bq10, bq50, bq90 = (float(x) for x in np.percentile(bwd_step_ms, [10, 50, 90]))

    # ---- the projections around the attention at this pack's shape (hidden = H*d): the fused
    # QKV projection with RoPE and the output projection, on synthetic x and weights
    C = H * d
    px = workloads.random_dout((T, C), 31 + rank).to(device)
    pw = (workloads.random_dout((3 * H * d, C), 32).float() * C ** -0.5).to(torch.bfloat16).to(device)
    pwo = (workloads.random_dout((C, H * d), 33).float() * (H * d) ** -0.5).to(torch.bfloat16).to(device)
    pq, pk, pv = (torch.empty(T, H, d, dtype=torch.bfloat16, device=device) for _ in range(3))
    py = torch.empty(T, C, dtype=torch.bfloat16, device=device)
    o2 = out.view(T, H * d)

    def proj_time(fn):
        for _ in range(args.warmup):
            flush.fill_(1.0)
            fn()
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
        barrier(world)
        torch.cuda.synchronize()
        for a, b in evs:
            flush.fill_(1.0)
            a.record(stream)
            fn()
            b.record(stream)
        torch.cuda.synchronize()
        barrier(world)
        return allreduce_max(sum(a.elapsed_time(b) for a, b in evs), world, device) / args.steps

    qkv_ms = proj_time(lambda: pa.pa_qkv_rope_fwd(px, pw, cu, p["max_seqlen"], 10000.0, pq, pk, pv, stream))
    out_ms = proj_time(lambda: pa.pa_linear_fwd(o2, pwo, py, stream))
    rc = pa.pa_get_error(stream)
    if rc != pa.PA_OK:
        raise pa.PackAttnError(rc, "projections")
    qkv_flops, out_flops = 2.0 * T * C * 3 * H * d, 2.0 * T * H * d * C

    # ---- FP8 variant on the same pack (head_dim 128): the quantiser, then the FP8 attention
    # on its output; same steps, warm-up and L2 flush
    fp8_rec = None
    if d == 128:
        B = cu.numel() - 1
        q8, k8 = torch.empty(T, H, d, dtype=torch.uint8, device=device), torch.empty(T, H, d, dtype=torch.uint8,
                                                                                    device=device)
        v8t = torch.empty(H * d, pa.pa_fp8_vt_keys(B, T), dtype=torch.uint8, device=device)
        sc8 = torch.empty(4 + H * d, dtype=torch.float32, device=device)
        out8, lse8 = torch.empty_like(out), torch.empty_like(lse)

        def quant_call():
            rc = pa.pa_fp8_quantize_qkv(q, k, v, cu, q8, k8, v8t, sc8, stream)
            if rc != pa.PA_OK:
                raise pa.PackAttnError(rc, "pa_fp8_quantize_qkv")

        def fp8_call():
            rc = pa.pa_varlen_attn_fwd_fp8(q8, k8, v8t, sc8, cu, p["max_seqlen"], p["scale"], out8, lse8, stream)
            if rc != pa.PA_OK:
                raise pa.PackAttnError(rc, "pa_varlen_attn_fwd_fp8")

        # delayed scaling: one pass with the maxima of a previous step (here the same tensors'
        # maxima, recorded by a first call), this call's maxima returned for the next step
        am_prev = torch.ones(4 + H * d, dtype=torch.float32, device=device)
        am_in, am_out = torch.empty_like(am_prev), torch.empty_like(am_prev)
        if pa.pa_fp8_quantize_qkv_delayed(q, k, v, cu, am_prev, am_in, q8, k8, v8t, sc8, stream) != pa.PA_OK:
            raise RuntimeError("pa_fp8_quantize_qkv_delayed")

        def dquant_call():
            rc = pa.pa_fp8_quantize_qkv_delayed(q, k, v, cu, am_in, am_out, q8, k8, v8t, sc8, stream)
            if rc != pa.PA_OK:
                raise pa.PackAttnError(rc, "pa_fp8_quantize_qkv_delayed")

        quant_ms = proj_time(quant_call)
        dquant_ms = proj_time(dquant_call)
        fp8_ms = proj_time(fp8_call)
        both_ms = proj_time(lambda: (quant_call(), fp8_call()))
        dboth_ms = proj_time(lambda: (dquant_call(), fp8_call()))
        bf16_ms = proj_time(call)  # the bf16 call again, in the same stretch of the run
        pa.pa_profile_read()  # clear
        pa.pa_profile_enable(True)
        t_fprof0 = time.time()
        for _ in range(args.steps):
            flush.fill_(1.0)
            fp8_call()
        torch.cuda.synchronize()
        t_fprof = time.time() - t_fprof0
        pa.pa_profile_enable(False)
        fkern_ms_total, fkern_n = pa.pa_profile_read()
        rc = pa.pa_get_error(stream)
        if rc != pa.PA_OK:
            raise pa.PackAttnError(rc, "fp8 region")
        fp8_rec = dict(quant_ms=quant_ms, fp8_ms=fp8_ms, both_ms=both_ms, t_prof=t_fprof,
                       dquant_ms=dquant_ms, dboth_ms=dboth_ms, bf16_ms=bf16_ms,
                       kern_s=fkern_ms_total / max(1, fkern_n) * 1e-3,
                       # algorithmic bytes: q, k, v read once (6 B per element) and the E4M3 codes
                       # written (3 B); the two-pass quantiser moves 15 B (the amax pass reads
                       # q, k, v once more)
                       quant_bytes=9.0 * T * H * d, quant_bytes_moved=15.0 * T * H * d)

    # ---- end to end through the public API with host buffers (pinned): every step copies its
    # q, k, v, cu_seqlens host -> device and its out, lse device -> host inside the timed region.
    # Steps are pipelined the way an input pipeline runs them: two device buffer sets and three
    # streams, so the copies of neighbouring steps overlap this step's kernels.
    hq, hk, hv = (p[n].pin_memory() for n in ("q", "k", "v"))
    hcu = p["cu_seqlens"].pin_memory()
    hout = [torch.empty(q.shape, dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    hlse = [torch.empty(T, H, dtype=torch.float32).pin_memory() for _ in range(2)]
    bufs = [(q, k, v, cu, out, lse), tuple(torch.empty_like(t) for t in (q, k, v, cu, out, lse))]
    s_in, s_comp, s_out = torch.cuda.Stream(device), torch.cuda.Stream(device), torch.cuda.Stream(device)

    def e2e_run(n_steps):
        comp_done, out_done = [None, None], [None, None]
        for i in range(n_steps):
            b = i & 1
            dq, dk, dv, dcu, dout, dlse = bufs[b]
            with torch.cuda.stream(s_in):
                if comp_done[b] is not None:  # the kernels of step i-2 have read this set
                    s_in.wait_event(comp_done[b])
                dq.copy_(hq, non_blocking=True)
                dk.copy_(hk, non_blocking=True)
                dv.copy_(hv, non_blocking=True)
                dcu.copy_(hcu, non_blocking=True)
                ready = torch.cuda.Event()
                ready.record(s_in)
            s_comp.wait_event(ready)
            if out_done[b] is not None:  # the outputs of step i-2 have left this set
                s_comp.wait_event(out_done[b])
            rc = pa.pa_varlen_attn_fwd(dq, dk, dv, dcu, p["max_seqlen"], p["scale"], dout, dlse, s_comp)
            if rc != pa.PA_OK:
                raise pa.PackAttnError(rc, "pa_varlen_attn_fwd")
            comp_done[b] = torch.cuda.Event()
            comp_done[b].record(s_comp)
            with torch.cuda.stream(s_out):
                s_out.wait_event(comp_done[b])
                hout[b].copy_(dout, non_blocking=True)
                hlse[b].copy_(dlse, non_blocking=True)
                out_done[b] = torch.cuda.Event()
                out_done[b].record(s_out)

    e2e_run(max(2, args.warmup))
    torch.cuda.synchronize()
    barrier(world)
    e2e_t0, e2e_t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e2e_t0.record(s_in)
    e2e_run(args.steps)
    s_out.wait_stream(s_comp)
    e2e_t1.record(s_out)
    torch.cuda.synchronize()
    barrier(world)
    rc = pa.pa_get_error(s_comp)
    if rc != pa.PA_OK:
        raise pa.PackAttnError(rc, "end-to-end region")
    e2e_ms = allreduce_max(e2e_t0.elapsed_time(e2e_t1), world, device) / args.steps
    h2d = sum(t.numel() * t.element_size() for t in (hq, hk, hv, hcu))
    d2h = hout[0].numel() * hout[0].element_size() + hlse[0].numel() * hlse[0].element_size()

    # ---- every other configuration of the workload list, and the short-segment regime: the same
    # call, L2 flushed before each call, step count capped per pack
    per_config = {}
    if not args.no_configs:
        del bufs, hq, hk, hv, hout, hlse
        for name in workloads.CONFIG_NAMES + workloads.SHORT_PACK_NAMES:
            if name == args.config:
                continue
            pk = Pack(pa, workloads.load_config(name), device, stream, seed_offset=7919 * rank)
            # each pack from the same state as the headline: a short idle gap (the board's power
            # average recovers), then its own warm-up and a burst region; its clocks are recorded
            torch.cuda.synchronize()
            time.sleep(1.0)
            rec = measure_pack(pa, pk, flush, stream, args, world, device, clocks=clocks)
            rec.update(tokens=pk.T, segments=len(pk.segs), heads=pk.H, head_dim=pk.d, valid_flops=pk.flops,
                       unique_bytes=pk.bytes)
            if pk.d == 128 and name in workloads.CONFIG_NAMES and name != "tiny":
                rec["fp8"] = fp8_compare(pa, pk, flush, stream, args.warmup, rec["steps"])
            if name in workloads.SHORT_PACK_NAMES or name == "tiny":
                # the same pack with short-segment packing off: every segment its own tiles
                pa.pa_set_short_packing(False)
                try:
                    torch.cuda.synchronize()
                    time.sleep(1.0)
                    rec["packing_off"] = measure_pack(pa, pk, flush, stream, args, world, device, clocks=clocks)
                finally:
                    pa.pa_set_short_packing(True)
            per_config[name] = rec
            del pk
            torch.cuda.empty_cache()
    if clocks:
        clocks.stop()

    if rank != 0:
        return 0
    peaks, peak_src = load_peaks()
    kern_avg_s = kern_avg_ms * 1e-3
    achieved = flops / kern_avg_s / 1e12
    peak_burst = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    peak_sust = float(peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"]))
    hbm = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    # The roofline's kernel is timed inside a run of back-to-back steps; once that run is
    # long enough to settle under the board's power limit (>= 0.25 s), its denominator is
    # the sustained cuBLAS figure, else the burst one.
    sustained = t_prof >= 0.25
    peak = peak_sust if sustained else peak_burst
    bpeak = peak_sust if t_bprof >= 0.25 else peak_burst
    bpeak_src = (f"bf16_tflops_sustained ({peak_src}; kernel timed inside {t_bprof:.2f} s of back-to-back steps)"
                 if t_bprof >= 0.25 else f"bf16_tflops ({peak_src}, burst)")
    trec = traffic_for_current_kernel()
    btrec = traffic_for_current_kernel("attn_bwd_traffic.json")
    ss_achieved = flops / (ss_kern_ms * 1e-3) / 1e12
    steady = {
        "what": (f"{n_ss} back-to-back calls of the same pack, no idle gap and no L2 flush between them "
                 f"(q, k, v, out: {head.bytes / 1e6:.0f} MB > 126 MB L2); per-call CUDA events"),
        "region_s": ss_t1 - ss_t0, "calls": n_ss, "ms_per_call": ss_call_ms,
        "value": flops * world / (ss_call_ms * 1e-3) / 1e12, "unit": "TFLOP/s",
        "pct_of_bf16_sustained": 100.0 * flops / (ss_call_ms * 1e-3) / 1e12 / peak_sust,
        "roofline": {"bound": "tensor", "kernel": head_kernel_name(d), "achieved": ss_achieved,
                     "peak": peak_sust, "unit": "TFLOP/s", "frac": ss_achieved / peak_sust,
                     "peak_source": f"bf16_tflops_sustained ({peak_src}; cuBLAS timed back to back under the "
                                    "power limit)",
                     "frac_of_burst": ss_achieved / peak_burst},
        "clocks": ss_clock,
    }
    if ss_clock and ss_clock.get("sm_mhz"):
        # clock-normalised rate: valid FLOPs per SM clock cycle of the whole GPU
        steady["flops_per_sm_cycle"] = flops / (ss_kern_ms * 1e-3) / (ss_clock["sm_mhz"] * 1e6)
    configs_rec, short_rec = {}, {}
    for name, rec in per_config.items():
        led = rec["ledger"]
        r = {"tokens": rec["tokens"], "segments": rec["segments"], "heads": rec["heads"],
             "head_dim": rec["head_dim"], "steps": rec["steps"], "ms_per_call": rec["ms_per_call"],
             "tile_ledger": {"score_tiles": led["score_tiles"], "useful_pairs": led["useful_pairs"],
                             "tile_utilisation": led["tile_utilisation"], "units": led["units"],
                             "groups": led["groups"], "grouped_segments": led["grouped_segments"]},
             "value": rec["tflops"], "unit": "TFLOP/s", "pct_of_bf16_peak": 100.0 * rec["tflops"] / world / peak_burst,
             "kernel": {"name": head_kernel_name(rec["head_dim"]), "ms": rec["kernel_ms"],
                        "achieved": rec["kernel_tflops"], "frac": rec["kernel_tflops"] / peak_burst,
                        "peak": peak_burst, "peak_source": f"bf16_tflops ({peak_src}, burst)"},
             "clocks": rec.get("clocks")}
        f8 = rec.get("fp8")
        if f8:
            r["fp8_vs_bf16"] = {
                "what": "per call, interleaved step by step with the bf16 call (same clocks), L2 flushed",
                "bf16_ms": f8["bf16_ms"], "fp8_attention_ms": f8["attn_ms"],
                "quantiser_plus_attention_ms": f8["quant_attn_ms"],
                "delayed_quantiser_plus_attention_ms": f8["delayed_attn_ms"],
                "speedup_quantiser_plus_attention": f8["bf16_ms"] / f8["quant_attn_ms"],
                "speedup_delayed_quantiser_plus_attention": f8["bf16_ms"] / f8["delayed_attn_ms"]}
        if name in workloads.SHORT_PACK_NAMES or name == "tiny":
            # short-segment regime: bound by HBM (per-segment intensity about L/2 FLOP per byte, below
            # the ridge of about 259 FLOP/B for L < ~520); unique bytes / time
            r["hbm"] = {"bound": "hbm", "unique_bytes": rec["unique_bytes"], "achieved": rec["gbs"],
                        "kernel_achieved": rec["kernel_gbs"], "peak": hbm, "unit": "GB/s",
                        "frac": rec["gbs"] / world / hbm, "kernel_frac": rec["kernel_gbs"] / hbm,
                        "peak_source": f"hbm_gbs ({peak_src}, copy bandwidth)"}
            off = rec.get("packing_off")
            if off:
                r["packing_off"] = {"ms_per_call": off["ms_per_call"], "value": off["tflops"], "unit": "TFLOP/s",
                                    "gbs": off["gbs"], "kernel_gbs": off["kernel_gbs"],
                                    "tile_utilisation": off["ledger"]["tile_utilisation"],
                                    "score_tiles": off["ledger"]["score_tiles"], "clocks": off.get("clocks")}
                r["packing_speedup"] = off["ms_per_call"] / rec["ms_per_call"]
            short_rec[name] = r
        else:
            configs_rec[name] = r
    line = {
        "metric": HEADLINE_METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": dict(workload_desc(cfg), l2="flushed between timed steps (256 MiB write, untimed)",
                       gpu_state=(f"{args.steps} calls right after {args.warmup} warm-up calls, L2 flushed "
                                  f"before each: a burst of about {sum(step_ms):.1f} ms of GPU time; the "
                                  "power-limited steady state is the `steady_state` record"),
                       parallelism=f"{world} independent replica(s), no collective"),
        "pct_of_bf16_peak": 100.0 * value / world / peak_burst,
        "pct_of_bf16_sustained": 100.0 * value / world / float(
            peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"])),
        "pct_of_bf16_datasheet_dense": 100.0 * value / world / 2250.0,  # vendor figure, not measured here
        "step_ms_p10_p50_p90": [q10, q50, q90],
        "tile_ledger": {"score_tiles": head_ledger["score_tiles"], "useful_pairs": head_ledger["useful_pairs"],
                        "tile_utilisation": head_ledger["tile_utilisation"],
                        "note": "useful (query, key) pairs / (128 x 128 score tiles computed x 16384), all heads"},
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                     "frac": achieved / peak,
                     "peak_source": (f"bf16_tflops_sustained ({peak_src}; kernel timed inside {t_prof:.2f} s "
                                     "of back-to-back steps)") if sustained
                                    else f"bf16_tflops ({peak_src}, burst; kernel timed over {t_prof:.3f} s)",
                     "kernel": head_kernel_name(d),
                     "traffic": (trec or {}).get("dram_bytes_per_launch"),
                     "traffic_unit": "bytes per launch (ncu dram__bytes_read.sum + dram__bytes_write.sum)"},
        "e2e": {"value": flops * world / (e2e_ms * 1e-3) / 1e12, "unit": "TFLOP/s", "ms_per_step": e2e_ms,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "pipelining": "two device buffer sets, three streams: the copies of steps i-1 and i+1 "
                              "overlap the kernels of step i; one region timed over all steps",
                "l2": "not flushed: each step's inputs arrive by host-to-device copy"},
        "backward": {
            "metric": "varlen attn bwd effective TFLOP/s (valid FLOPs: 5 GEMMs = 10 * sum(L_i^2) * d * H)",
            "value": bwd_flops * world / (bwd_ms * 1e-3) / 1e12, "unit": "TFLOP/s", "ms_per_step": bwd_ms,
            "step_ms_p10_p50_p90": [bq10, bq50, bq90], "valid_flops_per_step": bwd_flops,
            "roofline": {"bound": "tensor", "kernel": "attn_bwd_kernel<%d>" % d,
                         "achieved": bwd_flops / (bkern_ms * 1e-3) / 1e12,
                         "peak": bpeak, "unit": "TFLOP/s",
                         "frac": bwd_flops / (bkern_ms * 1e-3) / 1e12 / bpeak,
                         "peak_source": bpeak_src,
                         "traffic": (btrec or {}).get("dram_bytes_per_launch"),
                         "traffic_unit": "bytes per launch (ncu dram__bytes_read.sum + dram__bytes_write.sum)"},
            "gpu_launches": 4 * args.steps,  # prep, schedule, main, dq conversion per step
        },
        "projections": {
            "hidden": C, "note": "synthetic x and weights at this pack's shape; same steps, warm-up and L2 flush",
            "qkv_rope": {"value": qkv_flops * world / (qkv_ms * 1e-3) / 1e12, "unit": "TFLOP/s", "ms_per_step": qkv_ms,
                         "flops_per_step": qkv_flops, "kernel": "gemm_kernel<QKV+RoPE>"},
            "out_proj": {"value": out_flops * world / (out_ms * 1e-3) / 1e12, "unit": "TFLOP/s", "ms_per_step": out_ms,
                         "flops_per_step": out_flops, "kernel": "gemm_kernel<plain>"},
        },
        "fp8": None if fp8_rec is None else {
            "metric": "FP8 (E4M3) varlen attn fwd effective TFLOP/s (same valid FLOPs as the headline)",
            "note": "q, k per-tensor, v per-channel, P per-tensor E4M3; tcgen05 kind::f8f6f4 MMAs",
            "attention": {"value": flops * world / (fp8_rec["fp8_ms"] * 1e-3) / 1e12, "unit": "TFLOP/s",
                          "ms_per_step": fp8_rec["fp8_ms"], "launches_per_step": 2},
            "quantiser": {"ms_per_step": fp8_rec["quant_ms"], "launches_per_step": 3,
                          "roofline": {"bound": "hbm", "unit": "GB/s", "bytes_per_call": fp8_rec["quant_bytes"],
                                       "bytes_note": "algorithmic: q, k, v read once + E4M3 codes written "
                                                     "(9 B per element); the two-pass kernels move "
                                                     "%.0f B per call" % fp8_rec["quant_bytes_moved"],
                                       "achieved": fp8_rec["quant_bytes"] / (fp8_rec["quant_ms"] * 1e-3) / 1e9,
                                       "peak": float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"])),
                                       "frac": fp8_rec["quant_bytes"] / (fp8_rec["quant_ms"] * 1e-3) / 1e9 /
                                       float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"])),
                                       "kernels": "memset + fp8_amax_kernel + fp8_quantize_kernel"}},
            "quantiser_plus_attention": {"value": flops * world / (fp8_rec["both_ms"] * 1e-3) / 1e12,
                                         "unit": "TFLOP/s", "ms_per_step": fp8_rec["both_ms"]},
            "delayed_quantiser": {"ms_per_step": fp8_rec["dquant_ms"], "launches_per_step": 2,
                                  "note": "one pass: scales from a previous step's maxima, this call's maxima "
                                          "returned (pa_fp8_quantize_qkv_delayed)",
                                  "roofline": {"bound": "hbm", "unit": "GB/s", "bytes_per_call": fp8_rec["quant_bytes"],
                                               "achieved": fp8_rec["quant_bytes"] / (fp8_rec["dquant_ms"] * 1e-3) / 1e9,
                                               "peak": float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"])),
                                               "frac": fp8_rec["quant_bytes"] / (fp8_rec["dquant_ms"] * 1e-3) / 1e9 /
                                               float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"])),
                                               "kernels": "memset of amax_out + fp8_quantize_kernel<true>"}},
            "delayed_quantiser_plus_attention": {"value": flops * world / (fp8_rec["dboth_ms"] * 1e-3) / 1e12,
                                                 "unit": "TFLOP/s", "ms_per_step": fp8_rec["dboth_ms"]},
            "bf16_same_stretch": {"value": flops * world / (fp8_rec["bf16_ms"] * 1e-3) / 1e12, "unit": "TFLOP/s",
                                  "ms_per_step": fp8_rec["bf16_ms"],
                                  "note": "the bf16 call timed again next to the FP8 timings (same clocks)"},
            "roofline": {"bound": "tensor", "kernel": "attn_fwd_fp8_kernel",
                         "achieved": flops / fp8_rec["kern_s"] / 1e12,
                         "peak": 2.0 * (float(peaks.get("bf16_tflops_sustained",
                                                        FALLBACK_PEAKS["bf16_tflops_sustained"]))
                                        if fp8_rec["t_prof"] >= 0.25 else peak_burst),
                         "frac": flops / fp8_rec["kern_s"] / 1e12 / (2.0 * (float(
                             peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"]))
                             if fp8_rec["t_prof"] >= 0.25 else peak_burst)),
                         "unit": "TFLOP/s",
                         "peak_source": "2 x the measured bf16 cuBLAS figure (%s; the nominal dense FP8 / BF16 "
                                        "ratio 4.5 / 2.25 PFLOP/s)" % (
                                            "sustained" if fp8_rec["t_prof"] >= 0.25 else "burst"),
                         "traffic": None},
        },
        "gpu_launches": 2 * args.steps,  # schedule + attention kernel per step, headline timed region
        "clocks": clock_rec,
        "steady_state": steady,
        "per_config": configs_rec or None,
        "short_segments": short_rec or None,
    }
    if world == 1 and not args.no_cpu_baseline:
        r, rows, secs, threads = oracle_sample_rate(p, cfg, args.cpu_seconds)
        line["cpu_baseline"] = {"value": r, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
                                "sample": f"{rows} random (token, head) rows of the same pack, {secs:.1f} s; "
                                          "rate = valid FLOPs of those rows / wall time"}
    print(json.dumps(line))
    return 0


def run_packing_study(args, local):
    """Padded vs bucketed vs packed (Mage-Flow page, the table after "Packing + Flash Attention
    varlen"): the training pack's images through the forward + backward of the packed kernel,
    laid out three ways.  The padded and bucketed layouts run every padded sequence as a
    segment of its padded length: the work of a dense kernel over padded sequences (their
    outputs are a timing vehicle, not compared).  Prints one JSON line."""
    import dit_resolution_packed_b200 as pa
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    cfg = workloads.load_config(args.config if args.config != "mixed" else "training")
    H, d = cfg["heads"], cfg["head_dim"]
    real = [int(n) for n in cfg["segments"]]
    valid = workloads.valid_flops(real, H, d)
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=device)
    stream = torch.cuda.current_stream()
    res = {}
    for name, lay in workloads.packing_layouts(real).items():
        p = workloads.random_pack(lay["segments"], H, d, seed=int(cfg["seed"]), scale=cfg["scale"])
        q, k, v = (p[n].to(device) for n in ("q", "k", "v"))
        cu = p["cu_seqlens"].to(device)
        out, lse = torch.empty_like(q), torch.empty(q.shape[0], H, dtype=torch.float32, device=device)
        dout = workloads.random_dout(q.shape, 11).to(device)
        dq, dk, dv = (torch.empty_like(q) for _ in range(3))

        def step():
            rc = pa.pa_varlen_attn_fwd(q, k, v, cu, p["max_seqlen"], p["scale"], out, lse, stream)
            rc = rc or pa.pa_varlen_attn_bwd(q, k, v, out, lse, dout, cu, p["max_seqlen"], p["scale"], dq, dk, dv,
                                             stream)
            if rc != pa.PA_OK:
                raise pa.PackAttnError(rc, name)

        n_steps = max(10, args.steps // 30)
        for _ in range(max(3, args.warmup // 30)):
            flush.fill_(1.0)
            step()
        torch.cuda.synchronize()
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n_steps)]
        for a, b in ev:
            flush.fill_(1.0)
            a.record(stream)
            step()
            b.record(stream)
        torch.cuda.synchronize()
        rc = pa.pa_get_error(stream)
        if rc != pa.PA_OK:
            raise pa.PackAttnError(rc, name)
        ms = statistics.median(a.elapsed_time(b) for a, b in ev)
        res[name] = {"processed_tokens": int(sum(lay["segments"])), "real_tokens": int(sum(real)),
                     "token_utilisation": lay["token_utilisation"], "ms_fwd_bwd": ms,
                     "valid_tflops_fwd_bwd": 3.5 * valid / (ms * 1e-3) / 1e12}
    base = res["padded"]["ms_fwd_bwd"]
    for r in res.values():
        r["relative_throughput"] = base / r["ms_fwd_bwd"]
    print(json.dumps({"study": "padded vs bucketed (groups of 4) vs packed: forward + backward attention",
                      "workload": workload_desc(cfg)["workload"], "heads": H, "head_dim": d,
                      "valid_flops_fwd_bwd": 3.5 * valid, "schemes": res,
                      "pages_table_a100": {"padded": [0.45, 1.0], "bucketed": [0.78, 1.3], "packed": [0.97, 2.1]},
                      "note": "the pages' figures are whole training throughput on an A100, for context only"}))
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1500)
    ap.add_argument("--warmup", type=int, default=200)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--config", default="mixed", choices=workloads.CONFIG_NAMES + workloads.SHORT_PACK_NAMES)
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-configs", action="store_true", help="skip the per-configuration and short-segment records")
    ap.add_argument("--steady-s", type=float, default=0.6,
                    help="seconds of back-to-back calls in the steady-state record")
    ap.add_argument("--packing-study", action="store_true",
                    help="padded vs bucketed vs packed layouts of the training image mix (one GPU)")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)  # at least three untimed warm-up steps
    world, rank, local = dist_setup(args.gpus)
    try:
        if args.impl == "reference":
            return run_reference(args, world, rank)
        if args.packing_study:
            return run_packing_study(args, local)
        return run_ours(args, world, rank, local)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    sys.exit(main())
