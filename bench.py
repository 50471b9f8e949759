"""Decode-attention benchmark: MLRA step-2 decode on synthetic inputs, one JSON line.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--workload NAME]

A step is one decode call (queries of N sequences against their resident latent/RoPE caches):
prep -> split-KV attention -> combine, all in libmlra.so.  ``value`` is whole-job decode
tokens/s (one token per sequence per step), device-timed with CUDA events over exactly K steps
between barriers, max over ranks.  Multi-GPU runs are weak scaling: every rank decodes its own
batch (seed + rank), with no collective on the data path.

``--impl reference`` times the CPU float64 oracle (the only other implementation of this path)
on a bounded sample of the same workload and prints the same line with ``"impl": "reference"``.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import math
import os
import pathlib
import statistics
import sys
import threading
import time

ROOT = pathlib.Path(__file__).resolve().parent
sys.path.insert(0, str(ROOT))

import torch  # noqa: E402

import workloads  # noqa: E402

METRIC = "decode tokens/s and latent-KV HBM GB/s (fraction of B200 peak), 1 GPU"
DEFAULT_WORKLOAD = "mlra4_n8_l32k"
L2_BYTES = 126 * 2 ** 20
PROFILE_DIR = ROOT / "profiles"
KERNEL_SOURCES = ["mlra_decode_kernel.cuh", "sm100_ptx.cuh", "mlra_plan.cuh", "mlra_internal.h"]
K1_SAMPLE = 8  # time the attention kernel on every 8th step of the timed region
# Warm-up runs at least the W steps asked for and at least this long, right before the timed
# region: a GPU that idled (input set-up, the oracle's timing) needs a few milliseconds of load
# before its clocks leave the idle state, and a short timed region would otherwise measure the
# ramp.  Much longer (a quarter of a second) and the 1 kW power cap engages during the warm-up:
# the sustained record measures that regime on purpose.
WARM_SECONDS = 0.02


# ----------------------------------------------------------------------------- work accounting
def cache_bytes(inp: workloads.Inputs) -> int:
    """Algorithmic bytes of one attention launch: every cached latent/RoPE element once."""
    w = inp.workload
    elem = 2  # the kernel streams bf16
    return int(inp.seq_lens.to(torch.int64).sum()) * (w.d_latent + w.d_rope) * elem


def algorithmic_flops(inp: workloads.Inputs) -> int:
    """2 H (d_c + d_R) for the scores (RoPE term once per head) + 2 H d_c for the outputs."""
    w = inp.workload
    return int(inp.seq_lens.to(torch.int64).sum()) * 2 * w.heads * (2 * w.d_latent + w.d_rope)


def measured_peaks() -> dict:
    p = ROOT / "MEASURED_PEAKS.json"
    if p.exists():
        d = json.loads(p.read_text())
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"], "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "source": "fallback"}


PROJECT_SOURCES = ["mlra_project_kernel.cuh", "sm100_ptx.cuh", "mlra_internal.h"]


def kernel_hash(sources=None) -> str:
    h = hashlib.sha256()
    for name in sources or KERNEL_SOURCES:
        h.update((ROOT / "latent_kv_cache_mlra_b200" / "csrc" / name).read_bytes())
    return h.hexdigest()[:16]


def recorded_traffic(workload: str, kind: str = "decode_kernel", sources=None):
    """DRAM bytes per launch of a kernel from the committed ncu summary
    profiles/<kind>_<workload>.md, if it matches the current kernel source; else None."""
    f = PROFILE_DIR / f"{kind}_{workload}.md"
    if not f.exists():
        return None
    vals = {}
    for line in f.read_text().splitlines():
        if line.startswith("- ") and ":" in line:
            k, v = line[2:].split(":", 1)
            vals[k.strip()] = v.strip()
    if vals.get("kernel_source_hash") != kernel_hash(sources):
        return None
    try:
        return int(float(vals["dram_bytes_per_launch"]))
    except (KeyError, ValueError):
        return None


# ----------------------------------------------------------------------------- clocks
class ClockSampler:
    """Samples SM clock, power and clock-event reasons with NVML every ``period`` seconds."""

    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown"}

    def __init__(self, device_index: int, period: float = 0.02):
        self.samples, self.period, self.ok = [], period, False
        self._stop = threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.handle = self._handle(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.handle, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:  # no NVML (CPU machine): the line carries clocks = null
            self.ok = False

    def _handle(self, idx):
        nv = self.nv
        try:
            uuid = str(torch.cuda.get_device_properties(idx).uuid)
            return nv.nvmlDeviceGetHandleByUUID(("GPU-" + uuid) if not uuid.startswith("GPU-") else uuid)
        except Exception:
            return nv.nvmlDeviceGetHandleByIndex(idx)

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                sm = nv.nvmlDeviceGetClockInfo(self.handle, nv.NVML_CLOCK_SM)
                try:
                    reasons = nv.nvmlDeviceGetCurrentClocksEventReasons(self.handle)
                except AttributeError:
                    reasons = nv.nvmlDeviceGetCurrentClocksThrottleReasons(self.handle)
                power = nv.nvmlDeviceGetPowerUsage(self.handle) / 1000.0
                self.samples.append((sm, reasons, power))
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        if self.ok:
            self._stop.set()
            self.t.join()

    def summary(self):
        if not self.ok or not self.samples:
            return None
        sms = [s[0] for s in self.samples]
        bits = 0
        for s in self.samples:
            bits |= s[1]
        return {"sm_mhz": statistics.median(sms), "sm_max_mhz": self.max_mhz,
                "reasons": [n for b, n in self.REASONS.items() if bits & b],
                "samples": len(self.samples), "power_w_median": statistics.median(s[2] for s in self.samples)}


# ----------------------------------------------------------------------------- distributed
def dist_setup(n_gpus: int):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if world > 1:
        import torch.distributed as dist
        rank, local = int(os.environ["RANK"]), int(os.environ.get("LOCAL_RANK", "0"))
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
        return rank, world, local
    return 0, 1, 0


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, world: int, device=None) -> float:
    if world == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def weak_scaling_value(batch_per_rank: int, world: int, ms_per_step: float) -> float:
    """Whole-job decode tokens/s: every rank decodes its own batch (one token per sequence) per
    step, and the step time is the maximum over ranks."""
    return batch_per_rank * world / (ms_per_step * 1e-3)


def rank_workload(name: str, rank: int) -> workloads.Workload:
    w = workloads.get(name)
    return workloads.Workload(**{**w.__dict__, "seed": w.seed + 7919 * rank})


# ----------------------------------------------------------------------------- CPU oracle
def host_threads() -> int:
    """Threads the oracle's BLAS calls use (else the cores this process may run on)."""
    threads = len(os.sched_getaffinity(0))
    try:
        from threadpoolctl import threadpool_info
        nums = [p.get("num_threads", 0) for p in threadpool_info() if p.get("user_api") == "blas"]
        if nums:
            threads = max(nums)
    except ImportError:
        pass
    return threads


def time_oracle(inp: workloads.Inputs, budget_s: float, max_seqs=None):
    """Runs the oracle on whole sequences (all heads), cycling over the batch, until the budget
    is spent; returns (seconds, sequences done, threads used)."""
    import oracle
    try:
        from threadpoolctl import threadpool_info
    except ImportError:
        threadpool_info = None
    w = inp.workload
    order = list(range(w.batch))[: max_seqs or w.batch]
    t0 = time.perf_counter()
    done = 0
    while order:
        s = order[done % len(order)]
        oracle.decode(inp.q_lat, inp.q_rope, inp.c_kv, inp.k_rope, inp.seq_lens, inp.page_table,
                      w.num_branches, w.sigma, w.gamma, page_size=w.page_size,
                      max_seq_len=inp.max_seq_len, seqs=[s])
        done += 1
        if time.perf_counter() - t0 > budget_s:
            break
    dt = time.perf_counter() - t0
    threads = len(os.sched_getaffinity(0))
    if threadpool_info:
        nums = [p.get("num_threads", 0) for p in threadpool_info() if p.get("user_api") == "blas"]
        if nums:
            threads = max(nums)
    return dt, done, threads


def time_oracle_heads(inp: workloads.Inputs, seq: int, heads: slice, length=None):
    """Oracle time for some heads of one sequence, over its first `length` positions (default:
    all of them)."""
    import oracle
    w = inp.workload
    lens = inp.seq_lens.clone()
    if length is not None:
        lens[seq] = min(int(lens[seq]), int(length))
    t0 = time.perf_counter()
    oracle.decode(inp.q_lat, inp.q_rope, inp.c_kv, inp.k_rope, lens, inp.page_table,
                  w.num_branches, w.sigma, w.gamma, page_size=w.page_size,
                  max_seq_len=inp.max_seq_len, seqs=[seq], heads=heads)
    return time.perf_counter() - t0


def workload_config(w: workloads.Workload, inp: workloads.Inputs) -> dict:
    return {"workload": w.name, "batch": w.batch, "heads": w.heads, "branches": w.num_branches,
            "d_latent": w.d_latent, "d_rope": w.d_rope,
            "seq_len": w.seq_len if not w.ragged else f"log-uniform[{w.min_seq_len},{w.seq_len}]",
            "tokens_in_cache": int(inp.seq_lens.sum()), "page_size": w.page_size,
            "softmax_scale": w.sigma, "branch_scale": w.gamma, "latent_scale": w.latent_scale,
            "seed": w.seed, "layers": 1,
            "l2": f"inputs larger than L2 ({cache_bytes(inp) / 1e6:.0f} MB of cache per step vs 126 MiB L2)"
            if cache_bytes(inp) > L2_BYTES else
            "L2 flushed (read of 2x L2) before each step; each step timed alone, the flush outside"}


# ----------------------------------------------------------------------------- reference arm
def run_reference(args):
    rank, world = int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1"))
    if rank != 0:
        return 0
    w = workloads.get(args.workload)
    inp = workloads.make_inputs(w)
    H = w.heads
    # one step = every head of sequence 0 over a prefix of its positions, the prefix sized so that
    # the whole warm-up + timed run stays within about two minutes (the gather of the cache rows
    # is shared by all heads, as in a full step).  Whole sequences run with the BLAS threads of the
    # host; short prefixes with one thread, where threading only adds overhead.
    from threadpoolctl import threadpool_limits
    L0 = int(inp.seq_lens[0])
    per_step = 120.0 / max(1, args.steps + args.warmup)
    sl = slice(None)
    probe = time_oracle_heads(inp, 0, sl)
    if per_step >= probe:
        npos, limit = L0, None
    else:
        with threadpool_limits(1):
            cal = min(2048, L0)
            time_oracle_heads(inp, 0, sl, cal)
            rate = cal / time_oracle_heads(inp, 0, sl, cal)      # positions per second, all heads
        npos, limit = int(max(16, min(L0, per_step * rate))), 1
    nh = H
    with threadpool_limits(limit):
        threads = host_threads()
        for _ in range(args.warmup):
            time_oracle_heads(inp, 0, sl, npos)
        ts = [time_oracle_heads(inp, 0, sl, npos) for _ in range(args.steps)]
    t_step = sum(ts) / len(ts)
    # share of one full decode step (head-positions of all sequences) that a timed step covers
    frac = nh * npos / (H * float(inp.seq_lens.sum()))
    value = w.batch * frac / t_step                # tokens/s of a full step at this rate
    sample = (f"all {H} heads of sequence 0 over its first {npos} of {L0} positions per timed "
              f"step ({frac:.2e} of one decode step)")
    line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": t_step * 1e3,
            "projected_ms_per_full_step": t_step / frac * 1e3,
            "note": "each timed step is the bounded sample below (ms_per_step is its measured "
                    "time); value scales it to decode tokens/s of a full step",
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "impl": "reference",
            "config": {**workload_config(w, inp), "parallelism": f"dp{world}"},
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": threads,
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line))
    return 0


# ----------------------------------------------------------------------------- our arm
def make_decoder(mlra, w, inp, dev, **kw):
    pt = None if inp.page_table is None else inp.page_table.to(dev)
    q, qr = inp.q_lat.to(dev), inp.q_rope.to(dev)
    c, kr = inp.c_kv.to(dev), inp.k_rope.to(dev)
    lens = inp.seq_lens.to(dev)
    dec = mlra.Decoder(q, qr, c, kr, lens, pt, num_branches=w.num_branches,
                       softmax_scale=w.sigma, branch_scale=w.gamma, max_seq_len=inp.max_seq_len,
                       page_size=w.page_size, with_lse=False, **kw)
    return dec, (q, qr, c, kr, lens, pt)


def time_decode(mlra, dec, inp, steps, warmup, world, dev, local):
    """Device time of `steps` decode calls after `warmup` untimed ones (CUDA events, max over
    ranks).  Caches larger than L2 run back to back between two events; smaller ones get an L2
    flush (a read of twice the L2) before each call, outside the events around it.  The attention
    kernel alone is timed on every K1_SAMPLE-th call."""
    stream = torch.cuda.current_stream(dev)
    nbytes = cache_bytes(inp)
    # inputs smaller than L2 are evicted before each step by reading a buffer twice the L2 size
    # (a read leaves clean lines: the timed kernels pay no write-back of the flush)
    flush = None if nbytes > L2_BYTES else torch.ones(2 * L2_BYTES // 4, dtype=torch.float32, device=dev)
    sink = torch.empty((), dtype=torch.float32, device=dev)
    dec()
    torch.cuda.synchronize()
    rc, flags = dec.status()
    if rc != 0:
        raise RuntimeError(f"device status after the first call: {mlra.status_string(rc)} (flags {flags})")

    def warm():
        """The W warm-up steps, continued until WARM_SECONDS of them ran (steps run returned)."""
        n, t0 = 0, time.perf_counter()
        while n < warmup or time.perf_counter() - t0 < WARM_SECONDS:
            if flush is not None:
                torch.sum(flush, dim=0, out=sink)
            dec()
            n += 1
            if n % 64 == 0:
                torch.cuda.synchronize()  # keep the host's clock tied to the device's progress
        return n

    # The attention kernel is timed on one step in K1_SAMPLE: an event recorded between two
    # kernels stops the next one from starting early (programmatic dependent launch), so the
    # other steps run undisturbed.
    n_k1 = (steps + K1_SAMPLE - 1) // K1_SAMPLE
    k1 = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(n_k1)]
    for a, b in k1:  # torch creates the CUDA event on its first record; the library re-records it
        a.record(stream)
        b.record(stream)
    torch.cuda.synchronize()
    t_start, t_stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    per_step = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                for _ in range(steps if flush is not None else 0)]
    with ClockSampler(local) as clk:
        warm_run = warm()
        barrier(world)
        torch.cuda.synchronize()
        t_start.record(stream)
        for i in range(steps):
            ev = k1[i // K1_SAMPLE] if i % K1_SAMPLE == 0 else None
            if flush is None:
                dec(k1_events=ev)
            else:
                torch.sum(flush, dim=0, out=sink)
                per_step[i][0].record(stream)
                dec(k1_events=ev)
                per_step[i][1].record(stream)
        t_stop.record(stream)
        torch.cuda.synchronize()
        barrier(world)
    ms_total = (t_start.elapsed_time(t_stop) if flush is None
                else sum(a.elapsed_time(b) for a, b in per_step))
    k1_ms = [a.elapsed_time(b) for a, b in k1]
    ms_step = max_over_ranks(ms_total, world, dev) / steps
    k1_avg_ms = max_over_ranks(sum(k1_ms) / len(k1_ms), world, dev)
    rc, flags = dec.status()
    if rc != 0:
        raise RuntimeError(f"device status after timing: {mlra.status_string(rc)} (flags {flags})")
    return {"ms_step": ms_step, "k1_ms": k1_avg_ms, "clocks": clk.summary(),
            "flushed": flush is not None, "warmup_run": warm_run}


def workload_record(w, inp, t, peaks) -> dict:
    """A sub-record of the JSON line: one workload's step time and its attention kernel's rate."""
    nbytes = cache_bytes(inp)
    gbs = nbytes / (t["k1_ms"] * 1e-3) / 1e9
    return {"ms_per_step": t["ms_step"], "tokens_per_s": w.batch / (t["ms_step"] * 1e-3),
            "k1_us": t["k1_ms"] * 1e3, "k1_gbs": gbs, "frac": gbs / peaks["hbm_gbs"],
            "frac_of_8tbs": gbs / 8000.0,
            "step_gbs": nbytes / (t["ms_step"] * 1e-3) / 1e9,
            "cache_bytes": nbytes, "l2": "L2 flushed before each step" if t["flushed"] else
            "inputs larger than L2, back to back", "warmup_run": t["warmup_run"],
            "clocks": t["clocks"]}


SIDE_WORKLOADS = ["mla_n8_l32k", "long_mlra4_l128k", "long_mlra2_l128k", "serving_mlra4_n64_paged"]
SIDE_STEPS = 400            # timed steps of each side workload (a fraction of a second each)
SUSTAINED_SECONDS = 1.5     # back-to-back load of the headline workload, under the power cap


def run_ours(args):
    from latent_kv_cache_mlra_b200 import mlra

    rank, world, local = dist_setup(args.gpus)
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    w = rank_workload(args.workload, rank)
    inp = workloads.make_inputs(w)
    dec, (q, qr, c, kr, lens, pt) = make_decoder(mlra, w, inp, dev)
    stream = torch.cuda.current_stream(dev)
    launches_per_step = dec.plan.launches
    nbytes, nflops = cache_bytes(inp), algorithmic_flops(inp)
    flush = None if nbytes > L2_BYTES else torch.ones(2 * L2_BYTES // 4, dtype=torch.float32, device=dev)
    sink = torch.empty((), dtype=torch.float32, device=dev)
    t = time_decode(mlra, dec, inp, args.steps, args.warmup, world, dev, local)
    ms_step, k1_avg_ms = t["ms_step"], t["k1_ms"]

    # End to end through the public API, pinned host queries/lengths in and the output back to the
    # host every step, double-buffered over three streams: step i's inputs are copied in while
    # step i-1 computes and step i's output is copied out while step i+1 computes.  The step's
    # inputs (queries, RoPE queries, lengths) sit side by side in one pinned staging buffer and go
    # in with one copy; the decoder reads them through views of its device copy.
    parts = [inp.q_lat.to(q.dtype), inp.q_rope.to(qr.dtype), inp.seq_lens.to(lens.dtype)]
    offs, off = [], 0
    for x in parts:
        offs.append(off)
        off += (x.numel() * x.element_size() + 255) // 256 * 256
    h_in = torch.empty(off, dtype=torch.uint8).pin_memory()
    for x, o in zip(parts, offs):
        h_in[o:o + x.numel() * x.element_size()].view(x.dtype).copy_(x.reshape(-1))
    h_outs = [torch.empty(dec.out.shape, dtype=dec.out.dtype).pin_memory() for _ in range(2)]
    h2d = h_in.numel()  # the staging buffer, alignment padding included
    d2h = h_outs[0].numel() * h_outs[0].element_size()
    bufs = []
    for _ in range(2):
        d_in = torch.empty(off, dtype=torch.uint8, device=dev)
        qk, qrk, lk = (d_in[o:o + x.numel() * x.element_size()].view(x.dtype).view(x.shape)
                       for x, o in zip(parts, offs))
        deck = mlra.Decoder(qk, qrk, c, kr, lk, pt, num_branches=w.num_branches,
                            softmax_scale=w.sigma, branch_scale=w.gamma,
                            max_seq_len=inp.max_seq_len, page_size=w.page_size, with_lse=False)
        bufs.append((d_in, deck))
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_done = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]

    def e2e_step(i):
        k = i % 2
        d_in, deck = bufs[k]
        if i >= 2:
            s_in.wait_event(ev_done[k])         # decode i-2 has read buffer k's inputs
        with torch.cuda.stream(s_in):
            d_in.copy_(h_in, non_blocking=True)
            ev_in[k].record(s_in)
        stream.wait_event(ev_in[k])
        if i >= 2:
            stream.wait_event(ev_out[k])        # buffer k's previous output has left the device
        if flush is not None:
            torch.sum(flush, dim=0, out=sink)
        deck()
        ev_done[k].record(stream)
        s_out.wait_event(ev_done[k])
        with torch.cuda.stream(s_out):
            h_outs[k].copy_(deck.out, non_blocking=True)
            ev_out[k].record(s_out)

    for i in range(min(args.warmup, 10)):
        e2e_step(i)
    torch.cuda.synchronize()
    e_start, e_stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    e_start.record(stream)
    s_in.wait_event(e_start)
    for i in range(args.steps):
        e2e_step(i)
    stream.wait_event(ev_out[(args.steps - 1) % 2])
    stream.wait_event(ev_out[args.steps % 2])
    e_stop.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    e2e_ms = max_over_ranks(e_start.elapsed_time(e_stop), world, dev) / args.steps
    for _, deck in bufs:
        rc, flags = deck.status()
        if rc != 0:
            raise RuntimeError(f"device status after the end-to-end run: {mlra.status_string(rc)}")

    peaks = measured_peaks()
    achieved_gbs = nbytes / (k1_avg_ms * 1e-3) / 1e9
    step_gbs = nbytes / (ms_step * 1e-3) / 1e9
    tflops = nflops / (k1_avg_ms * 1e-3) / 1e12
    total_seqs = w.batch * world
    line = {
        "metric": METRIC, "value": weak_scaling_value(w.batch, world, ms_step), "unit": "tokens/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic", "config": {**workload_config(w, inp), "parallelism": f"dp{world}"},
        "latent_gbs": step_gbs * world,
        "latent_gbs_frac_of_measured": step_gbs / peaks["hbm_gbs"],
        "latent_gbs_frac_of_8tbs": step_gbs / 8000.0,
        "roofline": {"bound": "hbm", "achieved": achieved_gbs, "peak": peaks["hbm_gbs"],
                     "unit": "GB/s", "frac": achieved_gbs / peaks["hbm_gbs"],
                     "traffic": recorded_traffic(w.name), "kernel": "mlra_decode_kernel",
                     "kernel_ms": k1_avg_ms, "algorithmic_bytes_per_launch": nbytes,
                     "peak_source": f"{peaks['source']} hbm_gbs (copy test)",
                     "frac_of_8tbs": achieved_gbs / 8000.0,
                     "tensor_tflops": tflops, "tensor_frac": tflops / peaks["bf16_tflops"]},
        "e2e": {"value": total_seqs / (e2e_ms * 1e-3), "unit": "tokens/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "note": "queries and lengths copied in, output copied out each step, double-"
                        "buffered on copy streams; the latent/RoPE cache stays resident like "
                        "model state" + ("" if flush is None else
                                         "; the L2 flush before each step is inside this loop")},
        "gpu_launches": launches_per_step * args.steps,
        "warmup_run": t["warmup_run"],
        "clocks": t["clocks"],
    }
    line["roofline"]["note"] = (
        "kernel_ms is the attention kernel alone, timed with events around it on every "
        f"{K1_SAMPLE}th step; an event between two kernels cancels the programmatic early start, "
        "so kernel_ms can exceed the back-to-back ms_per_step, in which each kernel's prologue "
        "overlaps the previous one")
    if world == 1 and not args.no_side:
        # the headline workload under sustained load (the power cap lowers the SM clock), then
        # every other single-GPU workload of the study, each timed the same way
        sus_steps = max(args.steps, int(SUSTAINED_SECONDS / (ms_step * 1e-3)))
        ts = time_decode(mlra, dec, inp, sus_steps, args.warmup, world, dev, local)
        line["sustained"] = {**workload_record(w, inp, ts, peaks), "steps": sus_steps,
                             "seconds": sus_steps * ts["ms_step"] * 1e-3}
        side = {}
        del dec, bufs, q, qr, c, kr, lens, pt
        torch.cuda.empty_cache()
        for name in SIDE_WORKLOADS:
            if name == w.name:
                continue
            wk = workloads.get(name)
            ink = workloads.make_inputs(wk)
            deck, _ = make_decoder(mlra, wk, ink, dev)
            tk = time_decode(mlra, deck, ink, SIDE_STEPS, args.warmup, world, dev, local)
            side[name] = workload_record(wk, ink, tk, peaks)
            del deck, ink
            torch.cuda.empty_cache()
        line["workloads"] = side
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        dt, done, threads = time_oracle(inp, budget_s=12.0)
        line["cpu_baseline"] = {"value": done / dt, "unit": "tokens/s", "cores": threads,
                                "kind": "oracle",
                                "sample": f"{done} whole sequences (all heads, full length), cycling "
                                          f"over the {w.batch} of the batch, {dt:.1f} s on the host "
                                          f"cores"}
    if rank == 0:
        print(json.dumps(line))
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


# ----------------------------------------------------------------------------- branch parallelism
def branch_layout(num_branches: int, world: int, rank: int):
    """(shard, shards, branches per device) of `rank` when the layer's B branches are spread over
    `world` devices: device g keeps the g-th of `world` equal column blocks of the latent, i.e.
    B / world adjacent branches ("Multi-Head Low-Rank Attention", section 3.2)."""
    if world < 1 or world > num_branches or num_branches % world or not 0 <= rank < world:
        raise ValueError(f"{num_branches} branches cannot be spread evenly over {world} devices")
    return rank, world, num_branches // world


def branch_step(w: workloads.Workload, inp: workloads.Inputs, dev, world: int, rank: int,
                d_head: int = 128):
    """This device's share of a branch-parallel layer step: steps 2 and 3 of its branches (CUDA)
    and, with more than one device, the all-reduce of y over the devices.  The inputs and W^UV are
    the same on every device (one layer, split by branches); each device cuts its blocks."""
    from latent_kv_cache_mlra_b200 import tp
    shard, shards, per_device = branch_layout(w.num_branches, world, rank)
    g = torch.Generator().manual_seed(w.seed + 77)
    w_uv = (torch.randn(w.heads, d_head, w.d_latent, generator=g) / w.d_latent ** 0.5).to(torch.bfloat16)
    pt = None if inp.page_table is None else inp.page_table.to(dev)
    step = tp.BranchShardStep(
        tp.shard_queries(inp.q_lat, shard, shards).to(dev), inp.q_rope.to(dev),
        tp.shard_latent(inp.c_kv, shard, shards).to(dev), inp.k_rope.to(dev), inp.seq_lens.to(dev),
        pt, tp.shard_wuv(w_uv, shard, shards).to(dev), num_branches=w.num_branches,
        branches_per_device=per_device, softmax_scale=w.sigma, max_seq_len=inp.max_seq_len,
        page_size=w.page_size, reduce=world > 1)
    return step, w_uv, per_device


def run_branch(args):
    """One attention layer's decode step with the branches spread over the devices (the pages'
    tensor-parallel setting): each device runs steps 2 and 3 of its B / world branches on its
    column block of the cache, then one NCCL all-reduce of y [N, H, d_head] sums the branches.
    The same layer is split, so scaling is strong; the step time is the maximum over ranks."""
    rank, world, local = dist_setup(args.gpus)
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    w = workloads.get(args.workload)
    inp = workloads.make_inputs(w)
    step, _, per_device = branch_step(w, inp, dev, world, rank)
    stream = torch.cuda.current_stream(dev)
    dc_dev = w.d_latent * per_device // w.num_branches
    dev_bytes = int(inp.seq_lens.to(torch.int64).sum()) * (dc_dev + w.d_rope) * 2
    flush = None if dev_bytes > L2_BYTES else torch.ones(2 * L2_BYTES // 4, dtype=torch.float32, device=dev)
    sink = torch.empty((), dtype=torch.float32, device=dev)
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    with ClockSampler(local) as clk:
        barrier(world)
        torch.cuda.synchronize()
        for i in range(args.steps):
            if flush is not None:
                torch.sum(flush, dim=0, out=sink)
            ev[i][0].record(stream)
            y = step.local()
            ev[i][1].record(stream)
            if world > 1:
                import torch.distributed as dist
                dist.all_reduce(y, op=dist.ReduceOp.SUM, group=step.group)
            ev[i][2].record(stream)
        torch.cuda.synchronize()
        barrier(world)
    local_ms = max_over_ranks(sum(a.elapsed_time(b) for a, b, _ in ev) / args.steps, world, dev)
    ar_ms = max_over_ranks(sum(b.elapsed_time(c) for _, b, c in ev) / args.steps, world, dev)
    ms = max_over_ranks(sum(a.elapsed_time(c) for a, _, c in ev) / args.steps, world, dev)
    rc, flags = step.decoder.status()
    if rc != 0:
        raise RuntimeError(f"device status after timing: {rc} (flags {flags})")
    peaks = measured_peaks()
    line = {"metric": "attention layer decode (steps 2-3), branch-parallel", "value": w.batch / (ms * 1e-3),
            "unit": "tokens/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": ms, "higher_is_better": True, "scaling": "strong", "vs_baseline": None,
            "dtype": "bf16", "data": "synthetic",
            "config": {**workload_config(w, inp), "parallelism": f"branch{world}",
                       "branches_per_device": per_device, "d_head": 128},
            "branch_shard": {"local_us": local_ms * 1e3, "allreduce_us": ar_ms * 1e3,
                             "allreduce_bytes": w.batch * w.heads * 128 * 4,
                             "cache_bytes_per_device": dev_bytes,
                             "cache_elements_per_token_per_device": dc_dev + w.d_rope,
                             "local_gbs": dev_bytes / (local_ms * 1e-3) / 1e9,
                             "local_frac": dev_bytes / (local_ms * 1e-3) / 1e9 / peaks["hbm_gbs"],
                             "note": "local = decode + step 3 of this device's branches (events "
                                     "around them, the L2 flush outside); the all-reduce is NCCL "
                                     "over the devices (none on one device)"},
            "gpu_launches": (step.decoder.plan.launches + 1) * args.steps,
            "clocks": clk.summary()}
    if rank == 0:
        print(json.dumps(line))
    del step
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


# ----------------------------------------------------------------------------- steps 1 and 3
def graph_time(body, steps, pre=None):
    """Mean device time (ms) of body() over `steps` calls replayed from one CUDA graph (no host
    launch work between an event and its kernels); pre() runs before each call, untimed."""
    evs = [(torch.cuda.Event(enable_timing=True, external=True),
            torch.cuda.Event(enable_timing=True, external=True)) for _ in range(steps)]
    dev = torch.cuda.current_device()
    side = torch.cuda.Stream(dev)
    side.wait_stream(torch.cuda.current_stream(dev))
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.stream(side), torch.cuda.graph(graph, stream=side):
        for a, b in evs:
            if pre is not None:
                pre()
            a.record()
            body()
            b.record()
    torch.cuda.synchronize()
    graph.replay()
    torch.cuda.synchronize()
    return sum(a.elapsed_time(b) for a, b in evs) / len(evs)


def run_stage(args):
    """Times the steps around the attention path on the workload's shapes (d_head = 128 per head):
      project: step 3 (value up-projection + branch sum) alone, W^UV evicted from L2 each call;
      absorb:  step 1 (query absorption of W^UK) alone, W^UK evicted from L2 each call;
      layer:   one attention layer's whole decode step -- step 1, the new token's RoPE and cache
               append, step 2 (the path's two kernels) and step 3 -- with L2 evicted before each
               step (and, for reference, back to back);
      multi:   step 2 for --q-len query tokens per sequence (mlra_decode_multi).
    Weights are N(0, 1/fan-in) bf16 draws, packed once.  Prints one JSON line."""
    from latent_kv_cache_mlra_b200 import mlra

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    w = workloads.get(args.workload)
    inp = workloads.make_inputs(w)
    d_head, N, H, d_c, d_R = 128, w.batch, w.heads, w.d_latent, w.d_rope
    g = torch.Generator().manual_seed(w.seed + 77)
    w_uv = mlra.pack_wuv((torch.randn(H, d_head, d_c, generator=g) / d_c ** 0.5).to(torch.bfloat16).to(dev))
    w_uk = mlra.pack_wuk((torch.randn(H, d_head, d_c, generator=g) / d_head ** 0.5).to(torch.bfloat16).to(dev))
    pt = None if inp.page_table is None else inp.page_table.to(dev)
    c, kr, lens = inp.c_kv.to(dev), inp.k_rope.to(dev), inp.seq_lens.to(dev)
    q_lat, q_rope = inp.q_lat.to(dev), inp.q_rope.to(dev)
    flush = torch.ones(2 * L2_BYTES // 4, dtype=torch.float32, device=dev)
    sink = torch.empty((), dtype=torch.float32, device=dev)
    evict = lambda: torch.sum(flush, dim=0, out=sink)  # noqa: E731  (a read: clean lines)
    q_nope = torch.randn(N, H, d_head, generator=g).to(dev)
    peaks = measured_peaks()
    if args.stage in ("project", "absorb"):
        if args.stage == "project":
            dec = mlra.Decoder(q_lat, q_rope, c, kr, lens, pt, num_branches=w.num_branches,
                               softmax_scale=w.sigma, branch_scale=w.gamma,
                               max_seq_len=inp.max_seq_len, page_size=w.page_size)
            x, wt = dec().contiguous(), w_uv
            y = torch.empty(N, H, d_head, dtype=torch.float32, device=dev)
            body = lambda: mlra.project(x, wt, y)  # noqa: E731
            kernel, what = "mlra_project_kernel", "step-3 projection (W^UV, branch sum)"
        else:
            x, wt = q_nope, w_uk
            y = torch.empty(N, H, d_c, dtype=torch.bfloat16, device=dev)
            body = lambda: mlra.absorb(x, wt, y)  # noqa: E731
            kernel, what = "mlra_project_kernel", "step-1 absorption (W^UK)"
        for _ in range(args.warmup):
            evict()
            body()
        with ClockSampler(0) as clk:
            ms = graph_time(body, args.steps, pre=evict)
        nbytes = wt.numel() * 2 + x.numel() * x.element_size() + y.numel() * y.element_size()
        flops = 2 * N * H * d_head * d_c
        gbs = nbytes / (ms * 1e-3) / 1e9
        line = {"metric": f"{what} time per decode step", "value": ms * 1e3, "unit": "us",
                "higher_is_better": False,
                "roofline": {"bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"],
                             "unit": "GB/s", "frac": gbs / peaks["hbm_gbs"], "kernel": kernel,
                             "algorithmic_bytes_per_launch": nbytes,
                             "traffic": recorded_traffic(w.name, f"{args.stage}_kernel",
                                                         PROJECT_SOURCES),
                             "tensor_tflops": flops / (ms * 1e-3) / 1e12},
                "l2": "L2 flushed (read of 2x L2) before each launch"}
    elif args.stage == "multi":
        # q query tokens per sequence (speculative / chunked-prefill step), causal among them
        q = args.q_len
        gq = torch.Generator().manual_seed(w.seed + 78)
        qm = torch.randn(N, q, H, d_c, generator=gq).to(torch.bfloat16).to(dev)
        qrm = torch.randn(N, q, H, d_R, generator=gq).to(torch.bfloat16).to(dev)
        dims = mlra.dims_for(qm[:, 0], qrm[:, 0], c, kr, lens, pt, w.num_branches,
                             max_seq_len=inp.max_seq_len, page_size=w.page_size)
        ws = torch.empty(mlra.workspace_size_multi(dims, q), dtype=torch.uint8, device=dev)
        outm = torch.empty(N, q, H, d_c, dtype=torch.float32, device=dev)
        body = lambda: mlra.decode_multi(qm, qrm, c, kr, lens, pt, num_branches=w.num_branches,  # noqa: E731
                                         softmax_scale=w.sigma, branch_scale=w.gamma,
                                         max_seq_len=inp.max_seq_len, page_size=w.page_size,
                                         out=outm, workspace=ws)
        # the single-token call timed the same way (events around every call), for the ratio
        q1, qr1 = qm[:, :1].contiguous(), qrm[:, :1].contiguous()
        ws1 = torch.empty(mlra.workspace_size_multi(dims, 1), dtype=torch.uint8, device=dev)
        out1 = torch.empty(N, 1, H, d_c, dtype=torch.float32, device=dev)
        body1 = lambda: mlra.decode_multi(q1, qr1, c, kr, lens, pt, num_branches=w.num_branches,  # noqa: E731
                                          softmax_scale=w.sigma, branch_scale=w.gamma,
                                          max_seq_len=inp.max_seq_len, page_size=w.page_size,
                                          out=out1, workspace=ws1)
        for _ in range(args.warmup):
            body()
            body1()
        big = cache_bytes(inp) > L2_BYTES
        with ClockSampler(0) as clk:
            ms = graph_time(body, args.steps, pre=None if big else evict)
            ms1 = graph_time(body1, args.steps, pre=None if big else evict)
        once = cache_bytes(inp)  # the cache read once: what a fused multi-token kernel needs
        token_bytes = once // max(1, int(inp.seq_lens.sum()))
        read = sum(max(0, int(L) - (q - 1 - t)) for L in inp.seq_lens.tolist()
                   for t in range(q)) * token_bytes
        gbs = once / (ms * 1e-3) / 1e9
        line = {"metric": f"multi-token decode ({q} query tokens per sequence) query tokens/s",
                "value": N * q / (ms * 1e-3), "unit": "tokens/s", "higher_is_better": True,
                "ms_per_step": ms, "q_len": q,
                "ms_per_step_one_token": ms1, "ratio_to_one_token": ms / ms1,
                "path": "two tokens per CTA (128 query rows)" if (q % 2 == 0 and H == 64 and
                                                                 w.d_latent // w.num_branches == 128)
                        else "one token per CTA",
                "roofline": {"bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"],
                             "unit": "GB/s", "frac": gbs / peaks["hbm_gbs"],
                             "kernel": "mlra_decode_kernel (whole call)",
                             "algorithmic_bytes_per_launch": once,
                             "bytes_read_per_step": read,
                             "note": "algorithmic = the cache read once; this path reads each "
                                     "token's causal prefix, about q times the cache"},
                "l2": "inputs larger than L2" if big else
                      "L2 flushed (read of 2x L2) before each step, outside the timed region"}
    else:  # layer
        q_rope_in = torch.randn(N, H, d_R, generator=g).to(dev)
        k_new, c_new = torch.randn(N, d_R, generator=g).to(dev), torch.randn(N, d_c, generator=g).to(dev)
        q_lat2 = torch.empty(N, H, d_c, dtype=torch.bfloat16, device=dev)
        q_rope2 = torch.empty(N, H, d_R, dtype=torch.bfloat16, device=dev)
        lens_in = (lens - 1).clamp(min=0).to(torch.int32)   # the new token is the last position
        dec = mlra.Decoder(q_lat2, q_rope2, c, kr, lens, pt, num_branches=w.num_branches,
                           softmax_scale=w.sigma, branch_scale=w.gamma,
                           max_seq_len=inp.max_seq_len, page_size=w.page_size)
        y = torch.empty(N, H, d_head, dtype=torch.float32, device=dev)
        dims_l = mlra.dims_for(q_lat2, q_rope2, c, kr, lens, pt, w.num_branches,
                               max_seq_len=inp.max_seq_len, page_size=w.page_size)
        ws_l = torch.empty(mlra.workspace_size_project(dims_l), dtype=torch.uint8, device=dev)

        def front():
            # RoPE/append first: the absorption's weight copies then start under its tail
            # (they precede the absorption kernel's dependency wait)
            mlra.rope_append(q_rope_in, k_new, c_new, lens_in, pt, c, kr,
                             max_seq_len=inp.max_seq_len if pt is None else None,
                             page_size=w.page_size, q_rope_out=q_rope2)
            mlra.absorb(q_nope, w_uk, q_lat2)

        def body():  # steps 2 and 3 in one call: step 3 merges the split sequences itself
            front()
            mlra.decode_project(q_lat2, q_rope2, c, kr, lens, pt, w_uv, num_branches=w.num_branches,
                                softmax_scale=w.sigma, branch_scale=w.gamma,
                                max_seq_len=inp.max_seq_len, page_size=w.page_size, y=y,
                                workspace=ws_l)

        def body_unfused():  # the attention path's combine kernel, then step 3
            front()
            mlra.project(dec(), w_uv, y)

        for _ in range(args.warmup):
            body()
            body_unfused()
        with ClockSampler(0) as clk:
            # L2 evicted before every step, as after the model's other layers: this layer's
            # weights and queries come from HBM (the timed region is the step alone)
            ms = graph_time(body, args.steps, pre=evict)
            ms_unfused = graph_time(body_unfused, args.steps, pre=evict)
            # back to back, the 16 MB of this layer's weights may stay in L2 (the cache stream is
            # evict-first): a single-layer best case, reported beside the value
            ms_kept = graph_time(body, args.steps)
        line = {"metric": "attention layer decode step (steps 1-3, RoPE and cache append)",
                "value": N / (ms * 1e-3), "unit": "tokens/s", "higher_is_better": True,
                "ms_per_step": ms, "ms_per_step_back_to_back": ms_kept,
                "ms_per_step_unfused": ms_unfused,
                "kernels_per_step": 4 + (0 if dec.plan.launches == 2 else 1),
                "note": "steps 2-3 through mlra_decode_project (no combine kernel); "
                        "ms_per_step_unfused: mlra_decode (with its combine) then mlra_project",
                "l2": "L2 flushed (read of 2x L2) before each step, outside the timed region"}
    line.update({"steps": args.steps, "warmup": args.warmup, "dtype": "bf16", "data": "synthetic",
                 "config": {"workload": w.name, "batch": N, "heads": H, "d_latent": d_c,
                            "d_rope": d_R, "d_head": d_head},
                 "clocks": clk.summary()})
    print(json.dumps(line))
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=400)
    ap.add_argument("--warmup", type=int, default=50)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(workloads.WORKLOADS))
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--parallel", choices=["dp", "branch"], default="dp",
                    help="dp: every device decodes its own batch (weak scaling, the default line); "
                         "branch: one layer's branches spread over the devices, steps 2-3 and an "
                         "all-reduce (strong scaling)")
    ap.add_argument("--no-side", action="store_true",
                    help="skip the sustained leg and the other workloads' sub-records")
    ap.add_argument("--q-len", type=int, default=2,
                    help="query tokens per sequence for --stage multi")
    ap.add_argument("--stage", choices=["decode", "project", "absorb", "layer", "multi"],
                    default="decode",
                    help="decode: the attention path (the default line); project / absorb: step 3 "
                         "/ step 1 alone; layer: steps 1-3 with RoPE and the cache append; multi: "
                         "--q-len query tokens per sequence")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        return run_reference(args)
    if args.parallel == "branch":
        return run_branch(args)
    if args.stage != "decode":
        return run_stage(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
