"""Benchmark of the SageAttention2 forward pass on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl sage2|reference]
                    [--config C5] [--no-e2e] [--no-cpu-baseline]

One step = one whole forward pass (smoothing + INT4 of Q/K, the correction,
FP8 V, the fused attention kernel) over one batch of the workload, through the
C ABI's three stage calls (sage2_smooth_quant_qk, sage2_quant_v on a second
stream since it is independent of Q and K, then sage2_attn_fwd_quantized: the
kernels sage2_attn_fwd runs, into caller-owned payload buffers), with CUDA
events around each attention launch; the e2e leg
calls sage2_attn_fwd_host with pinned host buffers: every step copies the
inputs in and the output back (pipelined by heads inside the call).  The default workload is the causal bf16 prefill case
B=1, H=32, N=32768, d=128 (the long-sequence d=128 point at which the tensor
roofline target is stated).  Metric: TOPS = 4*B*H*N^2*d / t, halved for causal.
Under torchrun each rank runs its own full copy of the workload (heads are
independent: no collective on the data path), so scaling is weak.  Rank 0
prints one JSON line.

--impl reference times the CPU oracle (the plain C restatement of the method,
oracle/sage2_oracle.c, OpenMP on every host core) on a bounded sample of the
same workload; the cpu_baseline leg times the same sample.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from quantized_attention_04_b200.inputs import CONFIGS, make_qkv, sweep_config  # noqa: E402

METRIC = "quantized attention TOPS (4*B*H*N^2*d/t, halved if causal)"
KERNELS_PER_STEP = 8   # k_mean_partial, k_smooth_quant (K blocks, Q blocks), k_qbar_split,
                       # k_qk_corr_tc, k_v_amax, k_v_quant, k_attn_fwd


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d["bf16_tflops"], d.get("bf16_tflops_sustained"), d["hbm_gbs"], "measured"
    return 1590.0, 1400.0, 6650.0, "fallback"


# ---------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 100 ms around a
    timed region (`with ClockSampler(i) as clk: <timed region>`).  Entering
    waits (at most 5 s) until the sampler has written its first row, so the
    region cannot end before sampling starts; only rows stamped inside the
    region are summarised."""
    FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    STAMP = "%Y/%m/%d %H:%M:%S.%f"

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None
        self.t0 = self.t1 = None

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-i", str(self.gpu), "-lms", "100"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except (FileNotFoundError, OSError):
            self.proc = None
        deadline = time.time() + 5.0
        while self.proc is not None and self.proc.poll() is None and time.time() < deadline:
            if os.path.getsize(self.path) > 0:
                break
            time.sleep(0.02)
        self.t0 = time.time()
        return self

    def __exit__(self, *exc):
        self.t1 = time.time()
        if self.proc is not None:
            time.sleep(0.15)                     # the row that covers the region's end
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    @classmethod
    def parse(cls, lines, t0=None, t1=None):
        """(sm MHz, max sm MHz, [hw_slowdown, hw_thermal, sw_thermal, sw_power_cap])
        for each row stamped within [t0, t1 + 0.1 s] (all rows without bounds)."""
        import datetime
        rows = []
        for line in lines:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 10:
                continue
            try:
                stamp = datetime.datetime.strptime(parts[0], cls.STAMP).timestamp()
                row = (float(parts[2]), float(parts[3]), parts[6:10])
            except ValueError:
                continue
            if t0 is not None and not (t0 - 0.1 <= stamp <= t1 + 0.1):
                continue
            rows.append(row)
        return rows

    def summary(self):
        rows = []
        if self.path and os.path.exists(self.path):
            with open(self.path) as f:
                rows = self.parse(f, self.t0, self.t1)
            os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for _, _, flags in rows for i, f in enumerate(flags)
                          if f.lower().startswith("active")})
        return {"sm_mhz": statistics.median(r[0] for r in rows),
                "sm_max_mhz": max(r[1] for r in rows), "reasons": reasons,
                "samples": len(rows)}


# ---------------------------------------------------------------- dist
def dist_setup(n_gpus: int, backend: str | None = None, timeout_s: float = 120.0):
    """One process per GPU (torchrun's env): NCCL on GPUs, gloo without (the
    CPU tests of this plumbing).  Returns (world, rank, local_rank)."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = backend or ("nccl" if torch.cuda.is_available() else "gloo")
        kw = {}
        if backend == "nccl":
            torch.cuda.set_device(local)
            kw["device_id"] = torch.device("cuda", local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=timeout_s), **kw)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, world: int) -> float:
    """The slowest rank's time: every multi-GPU number is the max over ranks."""
    if world == 1:
        return x
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate(ops_per_rank: float, ms: float, world: int) -> float:
    """Whole-job throughput (TOPS): every rank runs its own copy of the
    workload (weak scaling), timed by the slowest rank."""
    return ops_per_rank * world / (ms * 1e-3) / 1e12


# ---------------------------------------------------------------- recorded DRAM traffic
TRAFFIC_RECORD = os.path.join(ROOT, "profiles", "k_attn_fwd_traffic.txt")
# every source the attention kernel is compiled from
ATTN_SOURCES = [os.path.join(ROOT, "quantized_attention_04_b200", "csrc", f)
                for f in ("attn.cu", "sm100_ptx.cuh", "sage2_internal.h")]


def attn_sources_sha256() -> str:
    import hashlib
    h = hashlib.sha256()
    for path in ATTN_SOURCES:
        h.update(open(path, "rb").read())
    return h.hexdigest()


def recorded_traffic(workload: str):
    """DRAM bytes (read + write) of one k_attn_fwd launch on `workload`, from
    the ncu record under profiles/, or None when there is none for this
    workload or the kernel's sources changed since it was taken (the record
    carries the SHA-256 of attn.cu, sm100_ptx.cuh and sage2_internal.h, read
    in that order)."""
    if not os.path.exists(TRAFFIC_RECORD):
        return None
    sha = attn_sources_sha256()
    rec = {}
    for line in open(TRAFFIC_RECORD):
        line = line.strip()
        if line.startswith("- ") and ":" in line:
            key, val = line[2:].split(":", 1)
            rec[key.strip()] = val.strip().strip("`")
    if rec.get("workload") != workload or rec.get("kernel sources sha256") != sha:
        return None
    try:
        return float(rec["dram bytes per launch"])
    except (KeyError, ValueError):
        return None


# ---------------------------------------------------------------- oracle leg
REF_BLOCKS = 8   # query blocks of head (0,0) in one CPU sample


def sample_blocks(cfg, n_blocks: int = REF_BLOCKS):
    nb = (cfg.N + 127) // 128
    return sorted(set(int(x) for x in np.linspace(0, nb - 1, n_blocks)))


def oracle_sample(cfg, q, k, v, qk_bits: int = 4):
    """One CPU sample: the plain C oracle (oracle/sage2_oracle.c) on head (0,0)
    of the workload: the head's smoothing, INT4/INT8 and FP8 payloads, then
    the correction and the quantized attention of REF_BLOCKS query blocks
    spread over the sequence, the blocks in parallel on every host core
    (OpenMP).  Returns (ops, seconds, description); ops counts 4 d per
    (query, visible key) of the sampled rows, the metric's own unit."""
    from oracle import c_oracle as corc
    blocks = sample_blocks(cfg)
    Q = q[0, 0].float().numpy()
    K = k[0, 0].float().numpy()
    V = v[0, 0].float().numpy()
    sm = 1.0 / math.sqrt(cfg.d)
    t0 = time.perf_counter()
    _, ops = corc.sample_forward(Q, K, V, cfg.causal, sm, blocks, qk_bits)
    dt = time.perf_counter() - t0
    nb = (cfg.N + 127) // 128
    desc = (f"plain C oracle, head (0,0) of {cfg.name}: smoothing/quantization of the whole "
            f"head + correction and attention of {len(blocks)} of {nb} query blocks "
            f"{blocks[:2]}..{blocks[-1:]} (OpenMP over blocks)")
    return ops, dt, desc


def host_cores() -> int:
    """Threads the C oracle runs on: OpenMP's default, the host cores this
    process may use (os.cpu_count() counts every CPU of the machine)."""
    from oracle import c_oracle as corc
    return corc.threads()


def run_reference(args, cfg, world, rank):
    if rank != 0:
        return
    q, k, v = make_qkv(cfg)
    times, opss = [], []
    desc = ""
    for _ in range(args.warmup):
        oracle_sample(cfg, q, k, v, args.qk_bits)
    for _ in range(args.steps):
        ops, dt, desc = oracle_sample(cfg, q, k, v, args.qk_bits)
        times.append(dt)
        opss.append(ops)
    value = sum(opss) / sum(times) / 1e12
    cores = host_cores()
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TOPS",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * statistics.mean(times), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded; distributions of the workload)",
        "config": {"workload": cfg.name, "B": cfg.B, "H": cfg.H, "N": cfg.N, "d": cfg.d,
                   "causal": cfg.causal, "input_dtype": cfg.dtype, "sample": desc},
        "cpu_baseline": {"value": value, "unit": "TOPS", "cores": cores,
                         "host_cpus": os.cpu_count(), "kind": "oracle", "sample": desc},
        "e2e": {"value": value, "unit": "TOPS", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------- main leg
def run_sage2(args, cfg, world, rank, local):
    import quantized_attention_04_b200 as qa
    from quantized_attention_04_b200 import build as _build
    if not os.path.exists(qa.LIB_PATH):
        _build.build()
    qa.lib()
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    q, k, v = make_qkv(cfg)
    sm = 1.0 / math.sqrt(cfg.d)
    qd, kd, vd = q.to(dev), k.to(dev), v.to(dev)
    od = torch.empty_like(qd)
    stream = torch.cuda.current_stream(dev)

    variant = ("int4" if args.qk_bits == 4 else "int8") + ("-packed" if args.packed else "") \
        + ("+smooth_v" if args.smooth_v else "")
    # Payload buffers are allocated once, by the caller, as the C ABI allows.
    pay = qa.sage2_smooth_quant_qk(qd, kd, qk_bits=args.qk_bits, packed=args.packed)
    vpay = qa.sage2_quant_v(vd, smooth=args.smooth_v)
    # The timed step runs the three stage calls of the C ABI (the same kernels,
    # in the same order, as sage2_attn_fwd) so that the attention launch can be
    # bracketed by its own events on the launching stream.
    attn_ev = []
    # V's quantization is independent of Q's and K's: it runs on a second
    # stream, as it does inside sage2_attn_fwd, and the attention waits for it
    vstream = torch.cuda.Stream(dev)
    fork_ev, v_done = torch.cuda.Event(), torch.cuda.Event()

    def step(record: bool):
        fork_ev.record(stream)
        vstream.wait_event(fork_ev)
        with torch.cuda.stream(vstream):
            qa.sage2_quant_v(vd, out=vpay, smooth=args.smooth_v)
        v_done.record(vstream)
        qa.sage2_smooth_quant_qk(qd, kd, out=pay, qk_bits=args.qk_bits, packed=args.packed,
                                 causal_corr=cfg.causal)
        stream.wait_event(v_done)
        if record:
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
        qa.sage2_attn_fwd_quantized(pay, vpay[0], vpay[1], cfg.N, cfg.causal, sm, out=od,
                                    v_mean=vpay[2] if args.smooth_v else None)
        if record:
            e1.record(stream)
            attn_ev.append((e0, e1))

    for _ in range(args.warmup):
        step(False)
    torch.cuda.synchronize()
    if qa.sage2_check_device_error(dev) != 0:
        raise RuntimeError("device error during warm-up")

    # ---- timed region: whole hot path, inputs resident in HBM
    barrier(world)
    torch.cuda.synchronize()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clk:
        ev0.record(stream)
        for _ in range(args.steps):
            step(True)
        ev1.record(stream)
        torch.cuda.synchronize()
    barrier(world)
    if qa.sage2_check_device_error(dev) != 0:
        raise RuntimeError("device error during the timed steps")
    ms_local = ev0.elapsed_time(ev1) / args.steps
    ms = max_over_ranks(ms_local, world)
    clocks = clk.summary()
    total_ops = cfg.ops() * world
    value = aggregate(cfg.ops(), ms, world)

    # ---- dominant kernel: its average launch inside the timed region
    attn_ms = max_over_ranks(statistics.mean(a.elapsed_time(b) for a, b in attn_ev), world)
    del pay, vpay
    bf16_peak, bf16_sus, hbm, peak_src = load_peaks()
    fp8_peak = bf16_peak * 2.0   # dense fp8/int8 : bf16 nominal ratio 4.5 : 2.25
    attn_tflops = cfg.ops() / (attn_ms * 1e-3) / 1e12
    roofline = {"bound": "tensor", "achieved": attn_tflops, "peak": fp8_peak, "unit": "TFLOP/s",
                "frac": attn_tflops / fp8_peak,
                "traffic": recorded_traffic(cfg.name) if variant == "int4" else None,
                "kernel": "k_attn_fwd", "kernel_ms": attn_ms,
                "peak_source": f"{peak_src} bf16 burst x 2 (fp8/int8 dense : bf16 dense)"}

    # ---- end to end through the public API with host buffers
    e2e = None
    if not args.no_e2e:
        qh, kh, vh = q.pin_memory(), k.pin_memory(), v.pin_memory()
        oh = torch.empty(od.shape, dtype=od.dtype).pin_memory()

        # the public host-buffer entry: chunks of heads are copied in, run and
        # copied back on library streams, overlapping copies with kernels
        def e2e_step():
            qa.sage2_attn_fwd_host(qh, kh, vh, oh, causal=cfg.causal, sm_scale=sm,
                                   qk_bits=args.qk_bits, smooth_v=args.smooth_v, device=dev)

        for _ in range(2):
            e2e_step()
        torch.cuda.synchronize()
        barrier(world)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.steps):
            e2e_step()
        e1.record(stream)
        torch.cuda.synchronize()
        barrier(world)
        e_ms = max_over_ranks(e0.elapsed_time(e1) / args.steps, world)
        e2e = {"value": total_ops / (e_ms * 1e-3) / 1e12, "unit": "TOPS",
               "ms_per_step": e_ms,
               "h2d_bytes_per_step": int(3 * qh.numel() * qh.element_size()),
               "d2h_bytes_per_step": int(oh.numel() * oh.element_size())}

    # ---- CPU oracle baseline (rank 0, N = 1 only): the reference arm's
    # sample, repeated for about ten seconds of CPU work
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        tot_ops = tot_s = 0.0
        reps = 0
        while reps < 20 and (tot_s < 10.0 or reps < 2):
            ops, dt, desc = oracle_sample(cfg, q, k, v, args.qk_bits)
            tot_ops += ops
            tot_s += dt
            reps += 1
        cpu = {"value": tot_ops / tot_s / 1e12, "unit": "TOPS", "cores": host_cores(),
               "host_cpus": os.cpu_count(), "kind": "oracle",
               "sample": f"{desc}; {reps} samples", "seconds": tot_s}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "TOPS", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "int8/e4m3 (INT4 values)" if args.qk_bits == 4 else "int8/e4m3 (INT8 values)",
            "data": "synthetic (seeded; distributions of the workload)",
            "config": {"workload": cfg.name, "B": cfg.B, "H": cfg.H, "N": cfg.N, "d": cfg.d,
                       "causal": cfg.causal, "input_dtype": cfg.dtype, "variant": variant,
                       "parallelism": f"replicas x{world} (independent heads, no collective)",
                       "l2": "inputs larger than L2 (3 x %d MB per step)" %
                             (q.numel() * q.element_size() // 2 ** 20)},
            "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e,
            "gpu_launches": KERNELS_PER_STEP * args.steps, "clocks": clocks,
        }
        print(json.dumps(line), flush=True)


# ---------------------------------------------------------------- packed sequences
def varlen_lengths(S: int):
    """The packed workload: S causal bf16 sequences, H=32, d=128, with seeded
    lengths uniform on [256, 4096] (a serving-style mix)."""
    rng = np.random.default_rng(2000 + S)
    return [int(x) for x in rng.integers(256, 4097, S)]


def run_varlen(args, world, rank, local):
    import quantized_attention_04_b200 as qa
    from quantized_attention_04_b200.inputs import Config, Dist
    lens = varlen_lengths(args.varlen)
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(int).tolist()
    T, H, d = cu[-1], 32, 128
    cfg = Config(f"VL{args.varlen}", 1, H, T, d, True, "bf16",
                 q=Dist(2.0), k=Dist(2.0, outliers=4, outlier_scale=20.0),
                 v=Dist(2.0, outliers=4, outlier_scale=20.0), index=40 + args.varlen)
    q, k, v = (t[0] for t in make_qkv(cfg))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    qd, kd, vd = q.to(dev), k.to(dev), v.to(dev)
    od = torch.empty_like(qd)
    sm = 1.0 / math.sqrt(d)
    stream = torch.cuda.current_stream(dev)

    def step():
        qa.sage2_attn_fwd_varlen(qd, kd, vd, cu, causal=True, sm_scale=sm, out=od,
                                 qk_bits=args.qk_bits, smooth_v=args.smooth_v)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if qa.sage2_check_device_error(dev) != 0:
        raise RuntimeError("device error during warm-up")
    barrier(world)
    torch.cuda.synchronize()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clk:
        ev0.record(stream)
        for _ in range(args.steps):
            step()
        ev1.record(stream)
        torch.cuda.synchronize()
    barrier(world)
    ms = max_over_ranks(ev0.elapsed_time(ev1) / args.steps, world)
    ops = sum(4.0 * H * n * n * d / 2 for n in lens) * world
    value = ops / (ms * 1e-3) / 1e12
    bf16_peak, _, _, peak_src = load_peaks()
    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "TOPS", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "int8/e4m3 (INT4 values)" if args.qk_bits == 4 else "int8/e4m3 (INT8 values)",
            "data": "synthetic (seeded; distributions of the workload)",
            "config": {"workload": cfg.name, "sequences": len(lens), "tokens": T, "H": H, "d": d,
                       "causal": True, "input_dtype": "bf16", "lengths": lens,
                       "variant": ("int4" if args.qk_bits == 4 else "int8")
                                  + ("+smooth_v" if args.smooth_v else ""),
                       "parallelism": f"replicas x{world} (independent heads, no collective)"},
            # one C call runs every kernel of every sequence: the whole step is measured
            "roofline": {"bound": "tensor", "achieved": value, "peak": 2.0 * bf16_peak,
                         "unit": "TFLOP/s", "frac": value / (2.0 * bf16_peak), "traffic": None,
                         "kernel": "whole varlen step (all kernels, every sequence)",
                         "peak_source": f"{peak_src} bf16 burst x 2"},
            "cpu_baseline": None, "e2e": None, "clocks": clk.summary(),
            # per sequence: K mean (2), smoothing+INT4, q-mean split, correction, V amax,
            # V quant, attention; V smoothing adds the V mean (2)
            "gpu_launches": (10 if args.smooth_v else 8) * sum(1 for n in lens if n) * args.steps,
        }
        print(json.dumps(line), flush=True)


# ---------------------------------------------------------------- roofline sweep
def run_sweep(args, world, rank, local):
    """The causal bf16 sweep d in {64, 128} x N in {4096, 16384, 32768} at B=1,
    H=32: per point, the whole step and the attention launch (CUDA events around
    it inside the timed steps), one JSON line each."""
    import quantized_attention_04_b200 as qa
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    bf16_peak, _, _, peak_src = load_peaks()
    for d in (64, 128):
        for N in (4096, 16384, 32768):
            cfg = sweep_config(N, d)
            q, k, v = make_qkv(cfg)
            qd, kd, vd = q.to(dev), k.to(dev), v.to(dev)
            od = torch.empty_like(qd)
            sm = 1.0 / math.sqrt(d)
            stream = torch.cuda.current_stream(dev)
            pay = qa.sage2_smooth_quant_qk(qd, kd)
            vpay = qa.sage2_quant_v(vd)
            attn_ev = []

            def step(record):
                qa.sage2_smooth_quant_qk(qd, kd, out=pay, causal_corr=True)
                qa.sage2_quant_v(vd, out=vpay)
                if record:
                    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                    e0.record(stream)
                qa.sage2_attn_fwd_quantized(pay, vpay[0], vpay[1], N, True, sm, out=od)
                if record:
                    e1.record(stream)
                    attn_ev.append((e0, e1))

            for _ in range(args.warmup):
                step(False)
            torch.cuda.synchronize()
            barrier(world)
            ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            with ClockSampler(local) as clk:
                ev0.record(stream)
                for _ in range(args.steps):
                    step(True)
                ev1.record(stream)
                torch.cuda.synchronize()
            barrier(world)
            if qa.sage2_check_device_error(dev) != 0:
                raise RuntimeError("device error in the sweep")
            ms = max_over_ranks(ev0.elapsed_time(ev1) / args.steps, world)
            attn_ms = max_over_ranks(statistics.mean(a.elapsed_time(b) for a, b in attn_ev), world)
            ops = cfg.ops()
            if rank == 0:
                print(json.dumps({
                    "metric": METRIC, "value": ops * world / (ms * 1e-3) / 1e12, "unit": "TOPS",
                    "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
                    "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
                    "dtype": "int8/e4m3 (INT4 values)", "data": "synthetic (seeded; LLM-like)",
                    "config": {"workload": cfg.name, "B": 1, "H": 32, "N": N, "d": d,
                               "causal": True, "input_dtype": "bf16"},
                    "roofline": {"bound": "tensor", "achieved": ops / (attn_ms * 1e-3) / 1e12,
                                 "peak": 2.0 * bf16_peak, "unit": "TFLOP/s",
                                 "frac": ops / (attn_ms * 1e-3) / 1e12 / (2.0 * bf16_peak),
                                 "traffic": None, "kernel": "k_attn_fwd", "kernel_ms": attn_ms,
                                 "peak_source": f"{peak_src} bf16 burst x 2"},
                    "clocks": clk.summary(), "gpu_launches": KERNELS_PER_STEP * args.steps,
                }), flush=True)
            del qd, kd, vd, od, pay, vpay


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="sage2", choices=["sage2", "reference"])
    ap.add_argument("--config", default="C5", choices=sorted(CONFIGS))
    ap.add_argument("--qk-bits", type=int, default=4, choices=[4, 8],
                    help="4: the method (INT4 Q/K); 8: the INT8 variant")
    ap.add_argument("--smooth-v", action="store_true", help="the V-smoothing variant")
    ap.add_argument("--packed", action="store_true",
                    help="INT4 payloads stored two per byte (expanded before the attention kernel)")
    ap.add_argument("--sweep", action="store_true",
                    help="the causal bf16 sweep d x N at B=1, H=32 (one line per point)")
    ap.add_argument("--varlen", type=int, default=0,
                    help="time the packed-sequence entry on this many seeded sequences instead")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    cfg = CONFIGS[args.config]
    if args.impl == "reference":
        world = int(os.environ.get("WORLD_SIZE", "1"))
        rank = int(os.environ.get("RANK", "0"))
        run_reference(args, cfg, world, rank)
        return
    world, rank, local = dist_setup(args.gpus)
    try:
        if args.sweep:
            run_sweep(args, world, rank, local)
        elif args.varlen:
            run_varlen(args, world, rank, local)
        else:
            run_sage2(args, cfg, world, rank, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
