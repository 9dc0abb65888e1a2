"""Benchmark of the KDA hot path on B200: chunked prefill and recurrent decode.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload t8k_h12|b16_t512_d64|packed_16k|t32k_h96]

One JSON line on rank 0.  `value` is prefill tokens/s over all ranks for the
headline prefill shape (B=1, T=8192, H=12, dk=dv=128, bf16; workload "t8k_h12"),
measured over K timed calls of kda_chunk_fwd with the inputs already in HBM.
Each rank runs its own shard (independent sequences, no collective: weak
scaling).  The `decode` object is the second half of the metric: K timed
kda_decode_step calls on the config-4 shape (N=256 sequences x H=96 heads,
d=128, 1.61 GB of fp32 state), reported as GB/s of algorithmic traffic and as a
fraction of the measured HBM peak.

`prefill_noalloc` times the same prefill through kda_chunk_fwd_noalloc (the single-kernel
path on the library's fixed scratch array; its parity is checked in the tests).
`prefill_bwd` times the backward (kda_chunk_bwd: the chunked form on the tensor cores)
with its per-kernel times, and the fp32 recurrent sweep (kda_chunk_bwd_recurrent) beside it.
`configs` times the other prefill workloads the same way (configs 0-3 of the
workload table: fp32_t256, b16_t512_d64, packed_16k, t32k_h96), each with its
fraction of the HBM roofline and the oracle timed on a bounded sample of it;
`decode.cpu_baseline` is the oracle's decode step on 8 of the 256 sequences,
scaled to whole steps/s.

L2: every prefill step reads a different one of three resident input sets
(3 x 152 MB > 126 MB L2), so no step finds its inputs in L2; the decode state
(1.61 GB) is far larger than L2.

`--impl reference` times the float64 CPU oracle on a bounded sample of the same
workload (rank 0 only) and prints the same metric and unit with "impl":
"reference".
"""
from __future__ import annotations

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

METRIC = "KDA prefill tokens/s (H=12,d=128,T=8192); decode state GB/s vs HBM peak"
UNIT = "tokens/s"


def _peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), float(p["bf16_tflops"]), float(p["bf16_tflops_sustained"]), "measured"
    except Exception:
        return 6650.0, 1590.0, 1400.0, "fallback"


# ---------------------------------------------------------------------------
# algorithmic work per call (bytes the method must move at minimum; flops of
# the chunked form counted as dense tensor-core work)
# ---------------------------------------------------------------------------
def prefill_bytes(T_rows: int, H: int, dk: int, dv: int, s_in: int, nseq: int,
                  h0: bool, hT: bool) -> int:
    per_tok = (2 * dk + dv) * s_in + 4 * dk + 4 + dv * s_in
    return T_rows * H * per_tok + nseq * H * 4 * dk * dv * (int(h0) + int(hT))


def prefill_flops(T_rows: int, H: int, dk: int, dv: int, C: int = 64) -> int:
    return T_rows * H * (2 * C * (3 * dk + 2 * dv) + 6 * dk * dv)


def decode_bytes(N: int, H: int, dk: int, dv: int, s_in: int) -> int:
    return N * H * (8 * dk * dv + (2 * dk + dv) * s_in + 4 * dk + 4 + dv * s_in)


# ---------------------------------------------------------------------------
# clocks sampled during the timed region
# ---------------------------------------------------------------------------
class NvmlClockSampler:
    """Polls the GPU's SM clock, max clock, power and clock-event reasons every 2 ms
    through NVML (read-only queries) and keeps them as ClockSampler-style rows."""
    FIELDS = None

    def __init__(self, gpu_index: int):
        import pynvml
        self.nv = pynvml
        pynvml.nvmlInit()
        self.h = pynvml.nvmlDeviceGetHandleByIndex(gpu_index)
        self.max_sm = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        g = lambda *names, d: next((getattr(pynvml, n) for n in names if hasattr(pynvml, n)), d)
        self.bits = [g("nvmlClocksEventReasonHwSlowdown", "nvmlClocksThrottleReasonHwSlowdown",
                       d=0x8),
                     g("nvmlClocksEventReasonHwThermalSlowdown",
                       "nvmlClocksThrottleReasonHwThermalSlowdown", d=0x40),
                     g("nvmlClocksEventReasonSwThermalSlowdown",
                       "nvmlClocksThrottleReasonSwThermalSlowdown", d=0x20),
                     g("nvmlClocksEventReasonSwPowerCap", "nvmlClocksThrottleReasonSwPowerCap",
                       d=0x4)]
        self.lines: list[str] = []
        self.stop_ev = threading.Event()
        self.t = None

    def start(self):
        self.t = threading.Thread(target=self._poll, daemon=True)
        self.t.start()

    def _poll(self):
        nv = self.nv
        get_reasons = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            nv.nvmlDeviceGetCurrentClocksThrottleReasons
        while not self.stop_ev.is_set():
            try:
                sm = nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM)
                pw = nv.nvmlDeviceGetPowerUsage(self.h) / 1000.0
                rs = get_reasons(self.h)
                flags = ["Active" if rs & b else "Not Active" for b in self.bits]
                self.lines.append(", ".join([str(sm), str(self.max_sm), f"{pw:.1f}"] + flags))
            except Exception:
                pass
            time.sleep(0.002)

    def mark(self) -> int:
        return len(self.lines)

    def stop(self):
        self.stop_ev.set()
        if self.t is not None:
            self.t.join(timeout=2)

    def summary(self, lo: int, hi: int) -> dict:
        return ClockSampler.summarize(self.lines[lo:hi] or self.lines[-3:])


def make_clock_sampler(gpu_index: int):
    """NVML polling when available (dense samples even in short timed regions), else
    nvidia-smi's loop mode."""
    try:
        return NvmlClockSampler(gpu_index)
    except Exception:
        return ClockSampler(gpu_index)


class ClockSampler:
    FIELDS = ["clocks.sm", "clocks.max.sm", "power.draw",
              "clocks_event_reasons.hw_slowdown", "clocks_event_reasons.hw_thermal_slowdown",
              "clocks_event_reasons.sw_thermal_slowdown", "clocks_event_reasons.sw_power_cap"]

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines: list[str] = []
        self.t = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), "--query-gpu=" + ",".join(self.FIELDS),
                 "--format=csv,noheader,nounits", "-lms", "20"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
            return
        self.t = threading.Thread(target=self._read, daemon=True)
        self.t.start()

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def mark(self) -> int:
        return len(self.lines)

    def stop(self):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
            if self.t is not None:
                self.t.join(timeout=2)

    def summary(self, lo: int, hi: int) -> dict:
        return ClockSampler.summarize(self.lines[lo:hi] or self.lines[-3:])

    @staticmethod
    def summarize(lines) -> dict:
        rows = []
        for line in lines:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) == len(ClockSampler.FIELDS):
                rows.append(parts)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
        sm = [float(r[0]) for r in rows if r[0].replace(".", "", 1).isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[3 + i] == "Active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": float(rows[0][1]) if rows[0][1].replace(".", "", 1).isdigit() else None,
                "reasons": reasons, "samples": len(rows)}


# ---------------------------------------------------------------------------
def _dist():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def run_reference(args, world, rank):
    """The float64 oracle on the host cores: W untimed and K timed steps, each step one
    pass over a bounded sample of the workload (its first --ref-tokens tokens, default
    1024, all heads), so that the whole run ends within minutes."""
    if rank != 0:
        return 0
    import kda_inputs as ki
    import oracle
    oracle.build()
    x = ki.make_prefill(args.workload)
    Tb = min(x["T"], args.ref_tokens if args.ref_tokens > 0 else 1024)
    q, k, v, g, b = (x[n][:, :Tb] for n in ("q", "k", "v", "g", "beta"))
    cu = None
    if x["cu_seqlens"] is not None:
        import torch
        cu = torch.clamp(x["cu_seqlens"], max=Tb)
    pairs = (q.shape[0] if cu is None else cu.numel() - 1) * x["H"]
    threads = max(1, min(oracle.max_threads(), pairs))
    step = lambda: oracle.prefill(q, k, v, g, b, None, cu, nthreads=threads)
    for _ in range(args.warmup):
        step()
    times = []
    for _ in range(args.steps):
        t0 = time.perf_counter()
        step()
        times.append(time.perf_counter() - t0)
    tok = Tb * q.shape[0]
    val = tok * len(times) / sum(times)
    desc = (f"first {Tb} tokens x {x['H']} heads of the {args.workload} workload per step, "
            f"float64 recurrence, {threads} threads")
    line = {
        "impl": "reference", "metric": METRIC, "value": val, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * sum(times) / len(times),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": _config(args, x, world),
        "cpu_baseline": {"value": val, "unit": UNIT, "cores": threads, "kind": "oracle",
                         "sample": desc},
        "e2e": {"value": val, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def _config(args, x, world):
    return {"workload": f"{args.workload}: B={x['B']} T={x['T']} H={x['H']} dk={x['dk']} "
                        f"dv={x['dv']} {x['dtype']} (seeded synthetic)",
            "global_batch": x["B"] * world, "seq_len": x["T"], "heads": x["H"],
            "head_dim": x["dk"], "parallelism": f"dp{world} (independent sequences per rank)",
            "l2": "prefill rotates 3 resident input sets (3 x inputs > 126 MB L2); decode "
                  "state 1.61 GB > L2",
            "decode_workload": "decode_n256_h96: N=256 H=96 d=128 bf16, fp32 state 1.61 GB"}


def _oracle_timing(args):
    """Float64 oracle over the whole workload (or its first --ref-tokens tokens),
    repeated until about --ref-seconds of CPU time have passed.  Returns
    (tokens/s of the median pass, threads used, sample description, pass times)."""
    import kda_inputs as ki
    import oracle
    oracle.build()
    x = ki.make_prefill(args.workload)
    Tb = min(x["T"], args.ref_tokens) if args.ref_tokens > 0 else x["T"]
    q, k, v, g, b = (x[n][:, :Tb] for n in ("q", "k", "v", "g", "beta"))
    cu = None
    if x["cu_seqlens"] is not None:
        import torch
        cu = torch.clamp(x["cu_seqlens"], max=Tb)
    pairs = (q.shape[0] if cu is None else cu.numel() - 1) * x["H"]
    threads = max(1, min(oracle.max_threads(), pairs))
    times = []
    t_all = time.perf_counter()
    while True:
        t0 = time.perf_counter()
        oracle.prefill(q, k, v, g, b, None, cu, nthreads=threads)
        times.append(time.perf_counter() - t0)
        if time.perf_counter() - t_all >= args.ref_seconds or len(times) >= 50:
            break
    tok = Tb * q.shape[0]
    med = statistics.median(times)
    desc = (f"{'all' if Tb == x['T'] else 'first'} {Tb} tokens x {x['H']} heads of the "
            f"{args.workload} workload, float64 recurrence, {len(times)} passes "
            f"({sum(times):.1f} s)")
    return tok / med, threads, desc, times


def cpu_baseline(args):
    """Oracle timed on the host cores on a bounded sample (about 10-30 s)."""
    val, threads, desc, _ = _oracle_timing(args)
    return {"value": val, "unit": UNIT, "cores": threads, "kind": "oracle", "sample": desc}


def whole_job_rate(units_per_rank: int, world: int, steps: int, ms_max: float) -> float:
    """Units per second over all ranks: every rank processes units_per_rank per
    step (weak scaling); the job takes the slowest rank's time."""
    return units_per_rank * world * steps / (ms_max / 1e3)


def rank_seed(base: int, rank: int, i: int = 0) -> int:
    """Seed of input set i on a rank: every rank draws its own shard."""
    return base + 1000 * rank + i


def _max_over_ranks(val, world, dev):
    if world == 1:
        return val
    import torch
    import torch.distributed as dist
    t = torch.tensor([val], device=dev, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def prefill_leg(args, world, rank, dev, stream, barrier, clocks):
    """K timed kda_chunk_fwd calls on resident inputs, then the e2e leg."""
    import torch

    import gated_delta_rule_74_b200 as kda
    import kda_inputs as ki

    spec = ki.PREFILL_SPECS[args.workload]
    sets = []                       # 3 resident input sets (L2 rotation)
    for i in range(3):
        x = ki.make_prefill(spec, seed=rank_seed(spec.seed, rank, i))
        d = {n: (t.to(dev) if isinstance(t, torch.Tensor) else t) for n, t in x.items()}
        d["out"] = torch.empty_like(d["v"])
        d["hT"] = torch.empty(x["B"], x["H"], x["dk"], x["dv"], device=dev)
        sets.append(d)
    x0 = sets[0]
    rows = x0["T"] if x0["cu_seqlens"] is not None else x0["B"] * x0["T"]
    s_in = 2 if x0["dtype"] == "bf16" else 4
    bytes_call = prefill_bytes(rows, x0["H"], x0["dk"], x0["dv"], s_in, x0["B"],
                               x0["h0"] is not None, True)
    flops_call = prefill_flops(rows, x0["H"], x0["dk"], x0["dv"])

    def prefill(i):
        d = sets[i % 3]
        kda.kda_chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], h0=d["h0"],
                          cu_seqlens=d["cu_seqlens"], out=d["out"], hT=d["hT"], stream=stream)

    for i in range(args.warmup):
        prefill(i)
    torch.cuda.synchronize()
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    mark0 = clocks.mark()
    n0 = kda.kda_launch_count()
    t_start.record(stream)
    for i in range(args.steps):
        prefill(i)
    t_end.record(stream)
    torch.cuda.synchronize()
    barrier()
    launches = kda.kda_launch_count() - n0
    mark1 = clocks.mark()
    local_ms = t_start.elapsed_time(t_end)
    ms_max = _max_over_ranks(local_ms, world, dev)
    call_ms = local_ms / args.steps
    # Per-kernel durations: the same K steps once more with CUDA events around every
    # library launch.  The events keep consecutive kernels from overlapping (the
    # library lets a kernel start while its predecessor drains), so this pass gives
    # kernel times and shares, not the step time.
    kda.kda_timing_start()
    for i in range(args.steps):
        prefill(i)
    torch.cuda.synchronize()
    ktimes = kda.kda_timing_read()
    kda.kda_timing_stop()

    # e2e: pinned host buffers -> device -> kda_chunk_fwd -> host, all timed.  Steps are
    # pipelined over three streams with two device buffer sets: while step i computes,
    # step i+1's inputs are copied in and step i-1's outputs copied out (events order
    # every reuse of a buffer); every step's copies are inside the timed region.
    hx = {n: x0[n].cpu().pin_memory() for n in ("q", "k", "v", "g", "beta")}
    h_out = [torch.empty(x0["out"].shape, dtype=x0["out"].dtype).pin_memory() for _ in range(2)]
    h_hT = [torch.empty(x0["hT"].shape, dtype=torch.float32).pin_memory() for _ in range(2)]
    dx = [{n: torch.empty_like(x0[n]) for n in hx} for _ in range(2)]
    dout = [torch.empty_like(x0["out"]) for _ in range(2)]
    dhT = [torch.empty_like(x0["hT"]) for _ in range(2)]
    h2d = sum(t.numel() * t.element_size() for t in hx.values())
    d2h = h_out[0].numel() * h_out[0].element_size() + h_hT[0].numel() * 4
    e2e_steps = max(3, args.steps // 4)
    cp_in, cp_out = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_comp = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]
    for e in ev_comp + ev_out:
        e.record(stream)

    def e2e_step(i):
        b = i & 1
        cp_in.wait_event(ev_comp[b])            # step i-2 no longer reads dx[b]
        with torch.cuda.stream(cp_in):
            for n in hx:
                dx[b][n].copy_(hx[n], non_blocking=True)
        ev_in[b].record(cp_in)
        stream.wait_event(ev_in[b])
        stream.wait_event(ev_out[b])           # step i-2's outputs have left dout[b], dhT[b]
        kda.kda_chunk_fwd(dx[b]["q"], dx[b]["k"], dx[b]["v"], dx[b]["g"], dx[b]["beta"],
                          h0=x0["h0"], cu_seqlens=x0["cu_seqlens"], out=dout[b], hT=dhT[b],
                          stream=stream)
        ev_comp[b].record(stream)
        cp_out.wait_event(ev_comp[b])
        with torch.cuda.stream(cp_out):
            h_out[b].copy_(dout[b], non_blocking=True)
            h_hT[b].copy_(dhT[b], non_blocking=True)
        ev_out[b].record(cp_out)

    for i in range(2):
        e2e_step(i)
    torch.cuda.synchronize()
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    cp_in.wait_event(e0)
    for i in range(e2e_steps):
        e2e_step(i)
    stream.wait_event(ev_out[(e2e_steps - 1) & 1])
    stream.wait_event(ev_out[e2e_steps & 1])
    e1.record(stream)
    torch.cuda.synchronize()
    barrier()
    e2e_ms = _max_over_ranks(e0.elapsed_time(e1), world, dev)
    return dict(x0=x0, rows=rows, s_in=s_in, bytes_call=bytes_call, flops_call=flops_call,
                ktimes=ktimes,
                value=whole_job_rate(rows, world, args.steps, ms_max), ms_max=ms_max,
                call_ms=call_ms, launches=launches, clocks=clocks.summary(mark0, mark1),
                e2e={"value": whole_job_rate(rows, world, e2e_steps, e2e_ms), "unit": UNIT,
                     "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                     "steps": e2e_steps})


def grouped_leg(args, world, rank, dev, stream, barrier, hbm, G=64):
    """The headline prefill with one decay value per group of G key channels
    (the decay-granularity variant): K timed calls on three resident input sets."""
    import torch

    import gated_delta_rule_74_b200 as kda
    import kda_inputs as ki

    spec = ki.PREFILL_SPECS[args.workload]
    sets = []
    for i in range(3):
        x = ki.make_prefill(spec, seed=spec.seed + 1000 * rank + 500 + i)
        d = {n: (t.to(dev) if isinstance(t, torch.Tensor) else t) for n, t in x.items()}
        d["g"] = d["g"][..., ::G].contiguous()
        d["out"] = torch.empty_like(d["v"])
        d["hT"] = torch.empty(x["B"], x["H"], x["dk"], x["dv"], device=dev)
        sets.append(d)
    x0 = sets[0]
    if x0["dk"] % G:
        return None
    rows = x0["T"] if x0["cu_seqlens"] is not None else x0["B"] * x0["T"]
    s_in = 2 if x0["dtype"] == "bf16" else 4
    H, dk, dv = x0["H"], x0["dk"], x0["dv"]
    bytes_call = rows * H * ((2 * dk + dv) * s_in + 4 * (dk // G) + 4 + dv * s_in) + \
        x0["B"] * H * 4 * dk * dv * (int(x0["h0"] is not None) + 1)

    def call(i):
        d = sets[i % 3]
        kda.kda_chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], h0=d["h0"],
                          cu_seqlens=d["cu_seqlens"], out=d["out"], hT=d["hT"], stream=stream)

    for i in range(args.warmup):
        call(i)
    torch.cuda.synchronize()
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for i in range(args.steps):
        call(i)
    e1.record(stream)
    torch.cuda.synchronize()
    barrier()
    ms = _max_over_ranks(e0.elapsed_time(e1), world, dev) / args.steps
    gbs = bytes_call / (ms / 1e3) / 1e9
    return {"call": f"kda_chunk_fwd_grouped (G={G})", "decay_group": G,
            "tokens_per_s": rows * world / (ms / 1e3), "ms_per_call": ms,
            "algorithmic_bytes_per_call": bytes_call, "gbs": gbs, "frac_of_hbm_peak": gbs / hbm}


def fused_leg(args, world, rank, dev, stream, barrier, hbm, W=4):
    """The headline prefill with the q/k short convolution + L2 norm and the output
    gate fused (kda_chunk_fwd_fused): K timed calls on three resident input sets."""
    import torch

    import gated_delta_rule_74_b200 as kda
    import kda_inputs as ki

    spec = ki.PREFILL_SPECS[args.workload]
    if spec.dtype != "bf16":
        return None
    sets = []
    for i in range(3):
        x = ki.make_fused_prefill(spec, W=W, seed=spec.seed + 1000 * rank + 800 + i)
        d = {n: (t.to(dev) if isinstance(t, torch.Tensor) else t) for n, t in x.items()}
        d["out"] = torch.empty_like(d["v"])
        d["hT"] = torch.empty(x["B"], x["H"], x["dk"], x["dv"], device=dev)
        sets.append(d)
    x0 = sets[0]
    rows = x0["T"] if x0["cu_seqlens"] is not None else x0["B"] * x0["T"]
    H, dk, dv = x0["H"], x0["dk"], x0["dv"]
    # raw q, k, v, gate in; g, beta; out; taps and states
    bytes_call = rows * H * ((2 * dk + 2 * dv) * 2 + 4 * dk + 4 + dv * 2) + \
        2 * H * dk * W * 4 + x0["B"] * H * 4 * dk * dv * (int(x0["h0"] is not None) + 1)

    def call(i):
        d = sets[i % 3]
        kda.kda_chunk_fwd_fused(d["q_raw"], d["k_raw"], d["v"], d["g"], d["beta"],
                                conv_q=d["conv_q"], conv_k=d["conv_k"], gate=d["gate"],
                                h0=d["h0"], cu_seqlens=d["cu_seqlens"], out=d["out"], hT=d["hT"],
                                stream=stream)

    for i in range(args.warmup):
        call(i)
    torch.cuda.synchronize()
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for i in range(args.steps):
        call(i)
    e1.record(stream)
    torch.cuda.synchronize()
    barrier()
    ms = _max_over_ranks(e0.elapsed_time(e1), world, dev) / args.steps
    gbs = bytes_call / (ms / 1e3) / 1e9
    return {"call": f"kda_chunk_fwd_fused (conv W={W}, L2 norm, output gate)",
            "tokens_per_s": rows * world / (ms / 1e3), "ms_per_call": ms,
            "algorithmic_bytes_per_call": bytes_call, "gbs": gbs, "frac_of_hbm_peak": gbs / hbm}


def bwd_leg(args, world, rank, dev, stream, barrier, hbm):
    """The prefill backward (kda_chunk_bwd) on the headline workload: a few timed
    calls on two resident input sets, fp32 gradients of sum(out*dout) + sum(hT*dhT)."""
    import torch

    import gated_delta_rule_74_b200 as kda
    import kda_inputs as ki

    spec = ki.PREFILL_SPECS[args.workload]
    sets = []
    for i in range(2):
        x = ki.make_prefill(spec, seed=spec.seed + 1000 * rank + 700 + i)
        d = {n: (t.to(dev) if isinstance(t, torch.Tensor) else t) for n, t in x.items()}
        gen = torch.Generator().manual_seed(rank_seed(spec.seed + 900, rank, i))
        d["dout"] = torch.randn(x["v"].shape, generator=gen).to(x["v"].dtype).to(dev)
        d["dhT"] = (0.1 * torch.randn((x["B"], x["H"], x["dk"], x["dv"]), generator=gen)).to(dev)
        d["grads"] = {n: torch.empty(x[src].shape, dtype=torch.float32, device=dev)
                      for n, src in (("dq", "q"), ("dk", "k"), ("dv", "v"), ("dg", "g"),
                                     ("dbeta", "beta"))}
        if x["h0"] is not None:
            d["grads"]["dh0"] = torch.empty_like(d["h0"])
        sets.append(d)
    x0 = sets[0]
    rows = x0["T"] if x0["cu_seqlens"] is not None else x0["B"] * x0["T"]
    s_in = 2 if x0["dtype"] == "bf16" else 4
    H, dk, dv = x0["H"], x0["dk"], x0["dv"]
    nstate = int(x0["h0"] is not None) * 2 + 1
    bytes_call = rows * H * ((2 * dk + 2 * dv) * s_in + 4 * dk + 4 + 12 * dk + 4 * dv + 4) + \
        x0["B"] * H * 4 * dk * dv * nstate
    steps = max(1, min(args.steps, args.bwd_steps))

    def call(i, recurrent=False):
        d = sets[i % 2]
        kda.kda_chunk_bwd(d["q"], d["k"], d["v"], d["g"], d["beta"], d["dout"], h0=d["h0"],
                          dhT=d["dhT"], cu_seqlens=d["cu_seqlens"], grads=d["grads"],
                          stream=stream, recurrent=recurrent)

    def timed(n, recurrent=False):
        for i in range(min(args.warmup, 3)):
            call(i, recurrent)
        torch.cuda.synchronize()
        barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for i in range(n):
            call(i, recurrent)
        e1.record(stream)
        torch.cuda.synchronize()
        barrier()
        return _max_over_ranks(e0.elapsed_time(e1), world, dev) / n

    ms = timed(steps)
    # per-kernel times: a second pass with CUDA events around each launch
    kda.kda_timing_start()
    for i in range(steps):
        call(i)
    torch.cuda.synchronize()
    kt = kda.kda_timing_read()
    kda.kda_timing_stop()
    kernels = {name: {"launches_per_call": n / steps, "ms_per_call": t / steps}
               for name, (n, t) in kt.items() if name.startswith("bwd_") and n > 0}
    rec_ms = timed(2, recurrent=True)
    gbs = bytes_call / (ms / 1e3) / 1e9
    return {"call": "kda_chunk_bwd", "method": "chunked form, tensor cores", "steps": steps,
            "tokens_per_s": rows * world / (ms / 1e3), "ms_per_call": ms,
            "algorithmic_bytes_per_call": bytes_call, "gbs": gbs, "frac_of_hbm_peak": gbs / hbm,
            "kernels": kernels,
            "recurrent": {"call": "kda_chunk_bwd_recurrent", "ms_per_call": rec_ms,
                          "tokens_per_s": rows * world / (rec_ms / 1e3)}}


def decode_leg(args, world, rank, dev, stream, barrier, clocks, hbm, peak_kind):
    """K timed kda_decode_step calls on the config-4 shape (state in HBM)."""
    import torch

    import gated_delta_rule_74_b200 as kda
    import kda_inputs as ki

    dspec = ki.DECODE_SPECS["decode_n256_h96"]
    dd = ki.make_decode(dspec, steps=1, seed=dspec.seed + 1000 * rank, N=args.decode_n or None)
    S = dd["S0"].to(dev)
    q, k, v, g, b = (dd[n][0].to(dev) for n in ("q", "k", "v", "g", "beta"))
    out = torch.empty(dd["N"], dd["H"], dd["dv"], dtype=q.dtype, device=dev)
    for _ in range(args.warmup):
        kda.kda_decode_step(q, k, v, g, b, S, out=out, stream=stream)
    torch.cuda.synchronize()
    barrier()
    mark0 = clocks.mark()
    n0 = kda.kda_launch_count()
    d0, d1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    d0.record(stream)
    for _ in range(args.decode_steps):
        kda.kda_decode_step(q, k, v, g, b, S, out=out, stream=stream)
    d1.record(stream)
    torch.cuda.synchronize()
    barrier()
    launches = kda.kda_launch_count() - n0
    dms = _max_over_ranks(d0.elapsed_time(d1), world, dev)
    dbytes = decode_bytes(dd["N"], dd["H"], dd["dk"], dd["dv"], 2)
    step_ms = dms / args.decode_steps
    gbs = dbytes / (step_ms / 1e3) / 1e9
    # fused multi-token decode: all 16 tokens of the config-4 workload in one launch
    fused = None
    if not args.no_fused_decode:
        L = dspec.steps
        dt = ki.make_decode(dspec, steps=L, seed=dspec.seed + 1000 * rank, N=args.decode_n or None)
        tq = {n: dt[n].transpose(0, 1).contiguous().to(dev) for n in ("q", "k", "v", "g", "beta")}
        del dt
        tout = torch.empty(dd["N"], L, dd["H"], dd["dv"], dtype=q.dtype, device=dev)
        fbytes = dd["N"] * dd["H"] * (8 * dd["dk"] * dd["dv"] + L * ((2 * dd["dk"] + dd["dv"]) * 2
                                                                   + 4 * dd["dk"] + 4 + dd["dv"] * 2))

        def time_tokens(fn, name):
            for _ in range(3):
                fn(tq["q"], tq["k"], tq["v"], tq["g"], tq["beta"], S, out=tout, stream=stream)
            torch.cuda.synchronize()
            barrier()
            nf = max(3, args.decode_steps // 8)
            n1 = kda.kda_launch_count()
            f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            f0.record(stream)
            for _ in range(nf):
                fn(tq["q"], tq["k"], tq["v"], tq["g"], tq["beta"], S, out=tout, stream=stream)
            f1.record(stream)
            torch.cuda.synchronize()
            barrier()
            fl = kda.kda_launch_count() - n1
            fms = _max_over_ranks(f0.elapsed_time(f1), world, dev) / nf
            fgbs = fbytes / (fms / 1e3) / 1e9
            return {"call": name, "tokens_per_launch_per_sequence": L,
                    "ms_per_launch": fms, "tokens_per_s": dd["N"] * L * world * 1e3 / fms,
                    "bytes_per_launch": fbytes, "gbs": fgbs, "frac_of_hbm_peak": fgbs / hbm,
                    "speedup_vs_single_steps": (step_ms * L) / fms, "launches": fl}

        fused = time_tokens(kda.kda_decode_tokens, "kda_decode_tokens")
        if L <= 16 and dd["dk"] == 128 and dd["dv"] == 128 and q.dtype == torch.bfloat16:
            fused["chunk_form"] = time_tokens(
                kda.kda_decode_chunk, "kda_decode_chunk (one chunk on the tensor cores)")
        del tq, tout
    return {"metric": "decode state GB/s vs HBM peak", "fused_tokens": fused, "workload":
            f"decode_n256_h96 shape: N={dd['N']} H={dd['H']} dk=dv=128 bf16 q/k/v, fp32 state "
            f"{dd['N'] * dd['H'] * 65536 / 1e9:.2f} GB", "gbs": gbs,
            "frac_of_hbm_peak": gbs / hbm, "peak_gbs": hbm, "peak_kind": peak_kind,
            "steps_per_s": 1e3 / step_ms, "tokens_per_s": dd["N"] * world * 1e3 / step_ms,
            "ms_per_step": step_ms, "steps": args.decode_steps, "bytes_per_step": dbytes,
            "gpu_launches": launches, "clocks": clocks.summary(mark0, clocks.mark())}


def noalloc_leg(args, world, rank, dev, stream, barrier, hbm):
    """The headline prefill through kda_chunk_fwd_noalloc (the single-kernel prefill on the
    library's fixed scratch array): K timed calls on three resident input sets."""
    import torch

    import gated_delta_rule_74_b200 as kda
    import kda_inputs as ki

    spec = ki.PREFILL_SPECS[args.workload]
    sets = []
    for i in range(3):
        x = ki.make_prefill(spec, seed=rank_seed(spec.seed, rank, i))
        d = {n: (t.to(dev) if isinstance(t, torch.Tensor) else t) for n, t in x.items()}
        d["out"] = torch.empty_like(d["v"])
        d["hT"] = torch.empty(x["B"], x["H"], x["dk"], x["dv"], device=dev)
        sets.append(d)
    x0 = sets[0]
    rows = x0["T"] if x0["cu_seqlens"] is not None else x0["B"] * x0["T"]
    s_in = 2 if x0["dtype"] == "bf16" else 4
    bytes_call = prefill_bytes(rows, x0["H"], x0["dk"], x0["dv"], s_in, x0["B"],
                               x0["h0"] is not None, True)

    def call(i):
        d = sets[i % 3]
        kda.kda_chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], h0=d["h0"],
                          cu_seqlens=d["cu_seqlens"], out=d["out"], hT=d["hT"], stream=stream,
                          noalloc=True)

    for i in range(args.warmup):
        call(i)
    torch.cuda.synchronize()
    barrier()
    steps = max(3, min(args.steps, 50))
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for i in range(steps):
        call(i)
    e1.record(stream)
    torch.cuda.synchronize()
    barrier()
    ms = _max_over_ranks(e0.elapsed_time(e1), world, dev) / steps
    gbs = bytes_call / (ms / 1e3) / 1e9
    return {"call": "kda_chunk_fwd_noalloc", "tokens_per_s": rows * world / (ms / 1e3),
            "ms_per_call": ms, "algorithmic_bytes_per_call": bytes_call, "gbs": gbs,
            "frac_of_hbm_peak": gbs / hbm}


CONFIG_WORKLOADS = ("fp32_t256", "b16_t512_d64", "packed_16k", "t32k_h96")
L2_BYTES = 126 * 1024 * 1024


def configs_leg(args, world, rank, dev, stream, barrier, hbm, tf_sust):
    """Every other prefill workload: K timed kda_chunk_fwd calls each (three resident
    input sets when one set is smaller than twice the L2, else one set larger than
    L2), its fraction of the HBM roofline, and -- on rank 0 at N = 1 -- the float64
    oracle timed on a bounded sample of the same workload."""
    import torch

    import gated_delta_rule_74_b200 as kda
    import kda_inputs as ki

    res = {}
    for name in CONFIG_WORKLOADS:
        if name == args.workload:
            continue
        spec = ki.PREFILL_SPECS[name]
        x = ki.make_prefill(spec, seed=rank_seed(spec.seed, rank))
        s_in = 2 if x["dtype"] == "bf16" else 4
        rows = x["T"] if x["cu_seqlens"] is not None else x["B"] * x["T"]
        bytes_call = prefill_bytes(rows, x["H"], x["dk"], x["dv"], s_in, x["B"],
                                   x["h0"] is not None, True)
        nsets = 3 if bytes_call < 2 * L2_BYTES else 1
        sets = []
        for i in range(nsets):
            xi = x if i == 0 else ki.make_prefill(spec, seed=rank_seed(spec.seed, rank, i))
            d = {n: (t.to(dev) if isinstance(t, torch.Tensor) else t) for n, t in xi.items()}
            d["out"] = torch.empty_like(d["v"])
            d["hT"] = torch.empty(xi["B"], xi["H"], xi["dk"], xi["dv"], device=dev)
            sets.append(d)
        del x

        def call(i):
            d = sets[i % nsets]
            kda.kda_chunk_fwd(d["q"], d["k"], d["v"], d["g"], d["beta"], h0=d["h0"],
                              cu_seqlens=d["cu_seqlens"], out=d["out"], hT=d["hT"], stream=stream)

        steps = max(3, min(args.steps, 50))
        for i in range(args.warmup):
            call(i)
        torch.cuda.synchronize()
        barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for i in range(steps):
            call(i)
        e1.record(stream)
        torch.cuda.synchronize()
        barrier()
        ms = _max_over_ranks(e0.elapsed_time(e1), world, dev) / steps
        gbs = bytes_call / (ms / 1e3) / 1e9
        flops = prefill_flops(rows, sets[0]["H"], sets[0]["dk"], sets[0]["dv"])
        t_roof = max(bytes_call / (hbm * 1e9), flops / (tf_sust * 1e12) if s_in == 2 else 0.0)
        entry = {"workload": f"{name}: {spec.desc}", "tokens_per_s": rows * world / (ms / 1e3),
                 "ms_per_call": ms, "steps": steps, "algorithmic_bytes_per_call": bytes_call,
                 "gbs": gbs, "frac_of_hbm_peak": gbs / hbm,
                 "roofline_ms": 1e3 * t_roof, "frac_of_roofline": 1e3 * t_roof / ms,
                 "l2": (f"{nsets} resident input sets rotated" if nsets > 1 else
                        "one input set, larger than L2")}
        del sets
        torch.cuda.empty_cache()
        if world == 1 and not args.no_cpu_baseline and rank == 0:
            sub = argparse.Namespace(**vars(args))
            sub.workload = name
            sub.ref_tokens = {"t32k_h96": 256, "packed_16k": 2048}.get(name, 0)
            sub.ref_seconds = 3.0
            val, threads, desc, _ = _oracle_timing(sub)
            entry["cpu_baseline"] = {"value": val, "unit": UNIT, "cores": threads,
                                     "kind": "oracle", "sample": desc}
        res[name] = entry
    return res


def decode_oracle(args, N_sample=8):
    """The float64 oracle's decode step on a bounded sample of the config-4 shape
    (N_sample of the 256 sequences, all 96 heads), scaled to whole steps."""
    import kda_inputs as ki
    import oracle
    oracle.build()
    dspec = ki.DECODE_SPECS["decode_n256_h96"]
    dd = ki.make_decode(dspec, steps=1, N=N_sample)
    q, k, v, g, b = (dd[n][0] for n in ("q", "k", "v", "g", "beta"))
    threads = max(1, min(oracle.max_threads(), N_sample * dd["H"]))
    S = dd["S0"]
    times = []
    t_all = time.perf_counter()
    while time.perf_counter() - t_all < 3.0 and len(times) < 50:
        t0 = time.perf_counter()
        oracle.decode(q, k, v, g, b, S, nthreads=threads)
        times.append(time.perf_counter() - t0)
    med = statistics.median(times)
    scale = dspec.N / N_sample
    return {"value": 1.0 / (med * scale), "unit": "steps/s", "cores": threads, "kind": "oracle",
            "sample": f"{N_sample} of the {dspec.N} sequences x {dd['H']} heads per step, "
                      f"float64 recurrence, median of {len(times)} steps, scaled to all "
                      f"{dspec.N} sequences"}


KERNEL_NAMES = {"prep": "kda_chunk_prep_kernel", "state": "kda_state_pass_kernel",
                "fused": "kda_chunk_tc_kernel",
                "simt": "kda_chunk_simt_kernel"}


# the sources the split prefill's kernels (prep kernel, state pass) are compiled from
TRAFFIC_SOURCES = ("chunk_split.cu", "chunk_record.cuh", "decay_pairs.cuh", "kda_common.cuh",
                   "segments.cuh", "sm100.cuh", "tma.cuh")


def _source_hash() -> str:
    """Hash of the split prefill's kernel sources with comments and whitespace removed:
    DRAM traffic depends on that code, so a comment edit (or a change to another kernel)
    keeps a capture valid."""
    import hashlib
    import re
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "gated_delta_rule_74_b200", "csrc")
    for name in TRAFFIC_SOURCES:
        with open(os.path.join(csrc, name), encoding="utf-8") as f:
            text = f.read()
        text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)        # block comments
        text = re.sub(r"//[^\n]*", " ", text)                      # line comments
        text = re.sub(r"\s+", " ", text)
        h.update(name.encode() + text.encode())
    return h.hexdigest()[:16]


def _traffic(workload: str) -> dict:
    """DRAM bytes per launch per kernel from the committed ncu capture, if the
    kernels have not changed since it was taken."""
    tpath = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(tpath) as f:
            t = json.load(f)
    except Exception:
        return {}
    if t.get("source_hash") != _source_hash():
        return {}
    w = dict(t.get("workloads", {}).get(workload, {}))
    w.pop("launches_captured", None)
    return w


_BYTE_UNITS = {"byte": 1, "Kbyte": 1e3, "Mbyte": 1e6, "Gbyte": 1e9, "KB": 1e3, "MB": 1e6,
               "GB": 1e9, "": 1}


def _ncu_dram_bytes(csv_path: str) -> dict:
    """DRAM bytes (read + write) per captured launch of each kernel kind, from an
    ncu --csv export: either a launch list (one row per launch and metric) or the
    raw page of a report (`ncu -i rep --page raw --csv`: one row per launch, a
    column per metric, a row of units under the header)."""
    import csv
    rows = list(csv.reader(open(csv_path)))
    hdr = next(i for i, r in enumerate(rows) if r and r[0] == "ID")
    H = rows[hdr]
    ki = H.index("Kernel Name")
    per = {}
    if "Metric Name" in H:
        mi, vi, ui = H.index("Metric Name"), H.index("Metric Value"), H.index("Metric Unit")
        for r in rows[hdr + 1:]:
            if len(r) <= vi or r[mi] not in ("dram__bytes_read.sum", "dram__bytes_write.sum"):
                continue
            kind = next((k for k, n in KERNEL_NAMES.items() if n in r[ki]), None)
            if kind is not None:
                b = float(r[vi].replace(",", "")) * _BYTE_UNITS[r[ui]]
                per.setdefault(kind, {}).setdefault(r[0], 0.0)
                per[kind][r[0]] += b
        return per
    cols = [H.index(m) for m in ("dram__bytes_read.sum", "dram__bytes_write.sum")]
    units = rows[hdr + 1]
    for r in rows[hdr + 2:]:
        if len(r) <= max(cols):
            continue
        kind = next((k for k, n in KERNEL_NAMES.items() if n in r[ki]), None)
        if kind is not None:
            per.setdefault(kind, {})[csv_path + ":" + r[0]] = sum(
                float(r[c].replace(",", "")) * _BYTE_UNITS[units[c]] for c in cols)
    return per


def ingest_ncu(csv_paths, workload: str) -> int:
    """Write profiles/traffic.json from ncu --csv exports (launch lists or raw
    pages) that hold dram__bytes_read.sum and dram__bytes_write.sum per launch:
    the average DRAM bytes per launch of each kernel kind, tagged with the hash of
    the kernel sources it was taken on."""
    per = {}
    for path in csv_paths:
        for kind, launches in _ncu_dram_bytes(path).items():
            per.setdefault(kind, {}).update(launches)
    tpath = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(tpath) as f:
            t = json.load(f)
    except Exception:
        t = {}
    if t.get("source_hash") != _source_hash():
        t = {"source_hash": _source_hash(), "workloads": {}}
    t["workloads"][workload] = {k: sum(v.values()) / len(v) for k, v in per.items()}
    t["workloads"][workload]["launches_captured"] = {k: len(v) for k, v in per.items()}
    with open(tpath, "w") as f:
        json.dump(t, f, indent=1)
    print(json.dumps(t["workloads"][workload]))
    return 0


def _roofline(args, pf, hbm, tf_sust, peak_kind) -> dict:
    """Roofline of one kda_chunk_fwd call (all its launches) against the
    method's algorithmic bytes, and of its dominant kernel (largest share of the
    live-measured kernel time) against the part of those bytes it moves."""
    x0 = pf["x0"]
    rows, H, dk, dv, s_in = pf["rows"], x0["H"], x0["dk"], x0["dv"], pf["s_in"]
    nseq = x0["B"]
    states = nseq * H * 4 * dk * dv * (int(x0["h0"] is not None) + 1)
    reads = rows * H * ((2 * dk + dv) * s_in + 4 * dk + 4)          # q, k, v, g, beta
    writes = rows * H * dv * s_in                                   # out
    algo = {"prep": reads, "state": writes + states, "fused": pf["bytes_call"],
            "simt": pf["bytes_call"]}
    kt = {k: v for k, v in pf["ktimes"].items() if v[0] > 0 and k != "decode"}
    total_ms = sum(v[1] for v in kt.values()) or 1e-9
    traffic = _traffic(args.workload)
    kernels = {}
    for k, (n, ms) in kt.items():
        per_call = n / args.steps
        kernels[k] = {"kernel": KERNEL_NAMES.get(k, k), "launches_per_call": per_call,
                      "avg_launch_ms": ms / n, "share": ms / total_ms,
                      "algorithmic_bytes_per_launch": algo.get(k, 0) / per_call,
                      "traffic_per_launch": traffic.get(k)}
    dom = max(kernels, key=lambda k: kernels[k]["share"]) if kernels else None
    call_gbs = pf["bytes_call"] / (pf["call_ms"] / 1e3) / 1e9
    achieved_tf = pf["flops_call"] / (pf["call_ms"] / 1e3) / 1e12
    out = {"bound": "hbm", "unit": "GB/s", "peak": hbm, "peak_kind": peak_kind,
           "kernel": "kda_chunk_fwd (one call: " + " + ".join(
               f"{kernels[k]['launches_per_call']:g} x {kernels[k]['kernel']}" for k in kernels) + ")",
           "achieved": call_gbs, "frac": call_gbs / hbm,
           "algorithmic_bytes_per_launch": pf["bytes_call"], "avg_launch_ms": pf["call_ms"],
           "traffic": sum(traffic.get(k, 0) * kernels[k]["launches_per_call"] for k in kernels)
           if traffic and all(traffic.get(k) is not None for k in kernels) else None,
           "tensor": {"achieved_tflops": achieved_tf, "peak_sustained": tf_sust,
                      "frac_sustained": achieved_tf / tf_sust,
                      "flops_per_launch": pf["flops_call"]},
           "kernels": kernels,
           "kernel_times": "second pass over the K timed steps with CUDA events around each launch"}
    if dom is not None:
        d = kernels[dom]
        gbs = d["algorithmic_bytes_per_launch"] / (d["avg_launch_ms"] / 1e3) / 1e9
        out["dominant"] = {"kernel": d["kernel"], "share": d["share"], "bound": "hbm",
                           "achieved": gbs, "peak": hbm, "unit": "GB/s", "frac": gbs / hbm,
                           "algorithmic_bytes_per_launch": d["algorithmic_bytes_per_launch"],
                           "avg_launch_ms": d["avg_launch_ms"],
                           "traffic": d["traffic_per_launch"]}
    return out



def run_ours(args, world, rank, local):
    import torch
    import torch.distributed as dist

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)

    def barrier():
        if world > 1:
            dist.barrier()

    hbm, tf_burst, tf_sust, peak_kind = _peaks()
    stream = torch.cuda.current_stream()
    vis = os.environ.get("CUDA_VISIBLE_DEVICES")
    clocks = make_clock_sampler(int(vis.split(",")[local]) if vis else local)
    clocks.start()
    time.sleep(0.3)
    pf = None
    if not args.decode_only:
        pf = prefill_leg(args, world, rank, dev, stream, barrier, clocks)
    grp = None
    if not args.decode_only and not args.no_grouped:
        grp = grouped_leg(args, world, rank, dev, stream, barrier, hbm)
    fzd = None
    if not args.decode_only and not args.no_fused_prep:
        fzd = fused_leg(args, world, rank, dev, stream, barrier, hbm)
    bwd = None
    if not args.decode_only and not args.no_bwd:
        bwd = bwd_leg(args, world, rank, dev, stream, barrier, hbm)
    nal = None
    if not args.decode_only and not args.no_noalloc:
        nal = noalloc_leg(args, world, rank, dev, stream, barrier, hbm)
    cfg = None
    if not args.decode_only and not args.no_configs:
        cfg = configs_leg(args, world, rank, dev, stream, barrier, hbm, tf_sust)
    dec = None
    if not args.no_decode:
        dec = decode_leg(args, world, rank, dev, stream, barrier, clocks, hbm, peak_kind)
        if dec is not None and world == 1 and rank == 0 and not args.no_cpu_baseline:
            dec["cpu_baseline"] = decode_oracle(args)
    clocks.stop()

    if rank != 0:
        if world > 1:
            dist.destroy_process_group()
        return 0
    if pf is None:
        print(json.dumps({"metric": METRIC, "decode_only": True, "decode": dec}), flush=True)
        if world > 1:
            dist.destroy_process_group()
        return 0

    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(args)
    roof = _roofline(args, pf, hbm, tf_sust, peak_kind)
    line = {
        "metric": METRIC, "value": pf["value"], "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": pf["ms_max"] / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16" if pf["s_in"] == 2 else "f32",
        "data": "synthetic (seeded random inputs shaped like the pages' models)",
        "config": _config(args, pf["x0"], world),
        "roofline": roof,
        "prefill_decay_g64": grp,
        "prefill_fused_prep": fzd,
        "prefill_bwd": bwd,
        "prefill_noalloc": nal,
        "configs": cfg,
        "decode": dec, "e2e": pf["e2e"], "gpu_launches": pf["launches"],
        "clocks": pf["clocks"], "cpu_baseline": cpu,
    }
    print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="t8k_h12", choices=["t8k_h12", "b16_t512_d64", "packed_16k", "t32k_h96"])
    ap.add_argument("--decode-steps", type=int, default=100)
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-fused-prep", action="store_true",
                    help="skip the fused conv + norm + gate prefill (kda_chunk_fwd_fused) leg")
    ap.add_argument("--no-bwd", action="store_true",
                    help="skip the prefill backward (kda_chunk_bwd) leg")
    ap.add_argument("--bwd-steps", type=int, default=5,
                    help="timed kda_chunk_bwd calls (at most --steps)")
    ap.add_argument("--no-grouped", action="store_true",
                    help="skip the grouped-decay (G = 64) prefill leg")
    ap.add_argument("--no-fused-decode", action="store_true",
                    help="skip the multi-token decode (kda_decode_tokens) leg")
    ap.add_argument("--decode-only", action="store_true",
                    help="skip the prefill legs (for profiling the decode kernel)")
    ap.add_argument("--decode-n", type=int, default=0,
                    help="sequences in the decode leg (0 = the config-4 value, 256)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-noalloc", action="store_true",
                    help="skip the kda_chunk_fwd_noalloc leg")
    ap.add_argument("--no-configs", action="store_true",
                    help="skip the other prefill workloads (configs leg)")
    ap.add_argument("--ref-tokens", type=int, default=0,
                    help="tokens of the workload the oracle processes per pass (0: all for "
                         "the cpu_baseline leg, 1024 per step for --impl reference)")
    ap.add_argument("--ref-seconds", type=float, default=10.0,
                    help="cpu_baseline leg: repeat oracle passes until this much time has passed")
    ap.add_argument("--ingest-ncu", nargs="+", default=[],
                    help="write profiles/traffic.json from these ncu --csv exports (launch "
                         "lists or raw pages of reports; no GPU run)")
    args = ap.parse_args()
    if args.ingest_ncu:
        return ingest_ncu(args.ingest_ncu, args.workload)
    args.warmup = max(args.warmup, 3)     # at least 3 untimed warm-up steps
    world, rank, local = _dist()
    if args.impl == "reference":
        return run_reference(args, world, rank)
    return run_ours(args, world, rank, local)


if __name__ == "__main__":
    sys.exit(main())
