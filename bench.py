#!/usr/bin/env python3
"""Benchmark of the fused rotate + int4-quantise hot path (and the W4A4 linear) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--no-extra]

One step = one pass of the hot path over one batch: the fused randomized-Hadamard
rotate + int4 group-quantise + pack of the Llama-3.2-1B-shaped activation batch
A[8192, 2048] bf16 (Student-t(4) x 0.5, 0.5% channels x100, G = 32). ``value`` is the
whole-job throughput in GB/s of algorithmic bytes (bf16 read + packed codes + fp16
scales written), with inputs resident in HBM; inputs and outputs rotate through six
buffer sets (258 MB > the 126 MB L2) so every step reads from DRAM. Every timed step is
replayed from CUDA graphs; after the synchronize that opens the timed region an untimed
~2 ms device-side spacer and one untimed replay run ahead of the start event, so the host
has queued the replays and the graph is running when the GPU reaches them (exactly K
steps lie between the two events).

Also reported: the roofline of that kernel against the measured HBM copy bandwidth, the
same metric end to end through the C ABI from pinned host memory, the fp64 oracle timed
on the host cores, SM clocks sampled during the timed region, and (unless --no-extra)
the other workloads: down_proj K = 8192 int4/int2, HARP K = 11008, and the W4A4 linear
(prefill TOPS against the int8 tensor peak, decode GB/s).

``--impl reference`` times the fp64 CPU oracle on the same workload (a bounded sample of
rows per step) and prints the same JSON line with "impl": "reference".
Under torchrun (N > 1) every rank runs the full batch on its own GPU (weak scaling,
no data-path collective); time is the max over ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "rotate+int4-quant GB/s (fraction of HBM peak); W4A4 linear TOPS vs int8 peak"
WORKLOAD = "llama32_1b"
INT8_DENSE_SPEC_TOPS = 4500.0
SPACER_CYCLES = 4_000_000   # ~2 ms at 1.965 GHz


WORKLOAD_DESC = ("llama32_1b: A[8192,2048] bf16, RHT K=2048 (signs + FWHT + 1/sqrt(K)), int4 G=32, "
                 "packed codes + fp16 scales")


def max_over_ranks(x: float, device=None) -> float:
    """Max of a per-rank scalar over the process group (identity without one). Measurement
    only: the data path has no collective."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput_gbs(bytes_per_step: int, steps: int, world: int, ms: float) -> float:
    """Whole-job GB/s: every rank processes its own full batch (weak scaling)."""
    return bytes_per_step * steps * world / (ms / 1e3) / 1e9


def algorithmic_bytes(M: int, K: int, bits: int, G: int, in_bytes: int = 2) -> int:
    return M * K * in_bytes + M * K * bits // 8 + M * (K // G) * 2


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


def kernel_sources_sha() -> str:
    """Hash of the timed rotation kernel's device code: rot_fwht.cu up to the few-row kernel (the
    helpers, the generic fused kernel and the tensor-core kernel the bench times) and the device
    helpers of rot_internal.cuh (host code does not change the kernel)."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "hadamard_butterfly_rotation_b200", "csrc")
    src = open(os.path.join(csrc, "rot_fwht.cu"), "rb").read()
    h.update(src[:src.find(b"\n// Few-row kernel for 4096-coordinate chunks")])
    hdr = open(os.path.join(csrc, "rot_internal.cuh"), "rb").read()
    h.update(hdr[hdr.find(b"device helpers"):])
    return h.hexdigest()[:16]


def profiled_traffic(name: str):
    """Per-launch DRAM bytes from a committed ncu summary, if it was taken on the current kernel."""
    p = os.path.join(ROOT, "profiles", f"{name}.json")
    if not os.path.exists(p):
        return None
    d = json.load(open(p))
    if d.get("source_sha") != kernel_sources_sha():
        return None
    return d.get("dram_bytes_per_launch")


class ClockSampler:
    """Samples SM clock and throttle reasons with NVML while the timed region runs."""

    def __init__(self, dev_index: int, period: float = 0.01):
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self.period = period
        self._stop = threading.Event()
        self._t = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(dev_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self.nv = None

    def _run(self):
        nv = self.nv
        names = {
            "hw_slowdown": getattr(nv, "nvmlClocksEventReasonHwSlowdown", 0x8),
            "hw_thermal_slowdown": getattr(nv, "nvmlClocksEventReasonHwThermalSlowdown", 0x40),
            "sw_thermal_slowdown": getattr(nv, "nvmlClocksEventReasonSwThermalSlowdown", 0x20),
            "sw_power_cap": getattr(nv, "nvmlClocksEventReasonSwPowerCap", 0x4),
            "hw_power_brake_slowdown": getattr(nv, "nvmlClocksEventReasonHwPowerBrakeSlowdown", 0x80),
        }
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
                r = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                for k, bit in names.items():
                    if r & bit:
                        self.reasons.add(k)
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.nv is not None:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self._t:
            self._t.join()

    def summary(self):
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons), "samples": len(self.samples)}


# ----------------------------------------------------------------------------- reference arm

def cpu_oracle_throughput(wl, bits, G, seconds: float):
    """fp64 oracle (dense RHT + quantisation) on the host cores: GB/s of algorithmic bytes."""
    from oracle import hadamard as Hd
    from oracle import quant as Q
    try:
        from threadpoolctl import threadpool_info
        cores = max(i.get("num_threads", 1) for i in threadpool_info()) if threadpool_info() else os.cpu_count()
    except Exception:
        cores = os.cpu_count()
    rows = 512
    done_rows, t0 = 0, time.perf_counter()
    r0 = 0
    while True:
        blk = wl.A[r0:r0 + rows]
        Q.quantize(Hd.rht_apply(blk, wl.signs), bits, G)
        done_rows += blk.shape[0]
        r0 = (r0 + rows) % wl.M
        if time.perf_counter() - t0 >= seconds:
            break
    dt = time.perf_counter() - t0
    gbs = algorithmic_bytes(done_rows, wl.K, bits, G) / dt / 1e9
    return gbs, cores, done_rows, dt


def cpu_plain_throughput(wl, bits, G, seconds: float):
    """The plain scalar O(K log K) C loop (signs, in-place FWHT, x 1/sqrt(K), group quantisation,
    packing; OpenMP over rows) on the host cores: GB/s of algorithmic bytes."""
    from oracle import plain
    rows = 2048
    threads = plain.max_threads()
    done_rows, r0 = 0, 0
    t0 = time.perf_counter()
    while True:
        blk = wl.A[r0:r0 + rows]
        plain.rht_quant(blk, wl.signs, bits, G, threads=threads)
        done_rows += blk.shape[0]
        r0 = (r0 + rows) % wl.M
        if time.perf_counter() - t0 >= seconds:
            break
    dt = time.perf_counter() - t0
    return algorithmic_bytes(done_rows, wl.K, bits, G) / dt / 1e9, threads, done_rows, dt


def parity_sample(wl, bits, G, codes_dev, scales_dev, rows: int = 256):
    """The bench's own output against the fp64 oracle on a sample of rows: codes and scales
    must be bit-exact outside the 1e-5 rounding-boundary windows; the excluded elements are
    counted and reported."""
    from oracle import hadamard as Hd
    from oracle import quant as Q
    idx = np.linspace(0, wl.M - 1, rows).astype(np.int64)
    y = Hd.rht_apply(wl.A[idx], wl.signs)
    q_ref, s_ref = Q.quantize(y, bits, G)
    cflag, gflag = Q.boundary_flags(y, bits, G)
    q = Q.unpack(codes_dev[idx.tolist()].cpu().numpy(), bits, wl.K)
    s16 = scales_dev[idx.tolist()].cpu().numpy().view(np.uint16)
    return {"rows": int(rows), "codes_compared": int(q.size), "codes_excluded": int(cflag.sum()),
            "groups_excluded": int(gflag.sum()),
            "codes_differing_outside_windows": int(((q != q_ref) & ~cflag).sum()),
            "scales_differing_outside_windows": int(((s16 != s_ref.view(np.uint16)) & ~gflag).sum()),
            "codes_differing_inside_windows": int(((q != q_ref) & cflag).sum())}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    import workloads as W
    wl = W.make_workload(WORKLOAD)
    bits, G = wl.quant[0]
    step_times = []
    from oracle import hadamard as Hd
    from oracle import quant as Q
    rows = 512
    for i in range(args.warmup + args.steps):
        r0 = (i * rows) % wl.M
        t0 = time.perf_counter()
        Q.quantize(Hd.rht_apply(wl.A[r0:r0 + rows], wl.signs), bits, G)
        if i >= args.warmup:
            step_times.append(time.perf_counter() - t0)
    tot = sum(step_times)
    gbs = algorithmic_bytes(rows * len(step_times), wl.K, bits, G) / tot / 1e9
    try:
        from threadpoolctl import threadpool_info
        cores = max(i.get("num_threads", 1) for i in threadpool_info())
    except Exception:
        cores = os.cpu_count()
    sample = f"{rows} of {wl.M} rows per step (fp64 dense Sylvester RHT + fp32-decision quantiser)"
    line = {
        "impl": "reference", "metric": METRIC, "value": round(gbs, 4), "unit": "GB/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(1000 * tot / len(step_times), 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": WORKLOAD_DESC, "global_batch": wl.M, "rows_per_step": rows},
        "cpu_baseline": {"value": round(gbs, 4), "unit": "GB/s", "cores": cores, "kind": "oracle", "sample": sample},
        "e2e": {"value": round(gbs, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line))
    return 0


# ----------------------------------------------------------------------------- our arm

def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50000)
    ap.add_argument("--warmup", type=int, default=200)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-extra", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--profile", default=None,
                    choices=["rot_quant", "q_proj_act_int4", "down_proj_int4", "down_proj_int2", "harp_init",
                             "harp_random", "w4a4_prefill", "w4a4_decode"],
                    help="launch only this kernel --steps times (for ncu captures); prints timing only")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        return run_reference(args)
    if args.profile:
        return run_profile(args)

    import torch
    import torch.distributed as dist
    import workloads as W
    import hadamard_butterfly_rotation_b200 as hbr

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        torch.cuda.set_device(local)
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    dev = torch.device("cuda", local if world > 1 else 0)
    torch.cuda.set_device(dev)

    wl = W.make_workload(WORKLOAD, seed=0)
    bits, G = wl.quant[0]
    M, K = wl.M, wl.K
    plan = hbr.Plan.rht(K, wl.signs)
    A_host = torch.from_numpy(wl.A).to(torch.bfloat16)
    NSETS = 6
    A_sets = [A_host.to(dev) for _ in range(NSETS)]
    outs = [(torch.empty((M, K * bits // 8), dtype=torch.uint8, device=dev),
             torch.empty((M, K // G), dtype=torch.float16, device=dev)) for _ in range(NSETS)]
    stream = torch.cuda.current_stream(dev)

    def step(i):
        c, s = outs[i % NSETS]
        hbr.rot_quant(A_sets[i % NSETS], plan, bits, G, codes=c, scales=s)

    # one period of the buffer rotation in a CUDA graph (warm-up steps run before capture)
    steps_graph = StepGraph(step, NSETS, warm=args.warmup)
    steps_graph.prepare(args.steps)
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(dev.index) as clk:
        # untimed lead-in ahead of the start event: a device-side spacer (the host queues everything
        # behind it) and one replay of the step graph, so the timed replays follow a running graph
        # and neither the first launch's host latency nor its device-side start-up is timed (together
        # ~7 % of a 20-step run)
        torch.cuda._sleep(SPACER_CYCLES)
        steps_graph.run(NSETS)
        ev0.record(stream)
        steps_graph.run(args.steps)
        ev1.record(stream)
        torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    ms = max_over_ranks(ev0.elapsed_time(ev1), dev)
    bytes_step = algorithmic_bytes(M, K, bits, G)
    gbs = job_throughput_gbs(bytes_step, args.steps, world, ms)
    per_launch_s = ms / 1e3 / args.steps
    achieved = bytes_step / per_launch_s / 1e9
    peaks, peak_kind = load_peaks()

    # end to end through the public API from pinned host memory: every step copies its A in
    # (H2D), rotates + quantises, and copies codes + scales out (D2H). Steps are pipelined over
    # three buffer sets and three streams (copy in / compute / copy out), so the copies of one
    # step overlap the kernel and the copies of its neighbours.
    A_pin = A_host.pin_memory()
    E_SETS = 3
    c_pins = [torch.empty((M, K * bits // 8), dtype=torch.uint8).pin_memory() for _ in range(E_SETS)]
    s_pins = [torch.empty((M, K // G), dtype=torch.float16).pin_memory() for _ in range(E_SETS)]
    s_in, s_comp, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev_in = [torch.cuda.Event() for _ in range(E_SETS)]
    ev_comp = [torch.cuda.Event() for _ in range(E_SETS)]
    ev_out = [torch.cuda.Event() for _ in range(E_SETS)]

    def e2e_step(i):
        k = i % E_SETS
        dA, (dc, ds) = A_sets[k], outs[k]
        if i >= E_SETS:
            s_in.wait_event(ev_comp[k])            # the kernel of step i - 3 has read dA
        with torch.cuda.stream(s_in):
            dA.copy_(A_pin, non_blocking=True)
        ev_in[k].record(s_in)
        s_comp.wait_event(ev_in[k])
        if i >= E_SETS:
            s_comp.wait_event(ev_out[k])           # step i - 3's outputs have been copied out
        hbr.rot_quant(dA, plan, bits, G, codes=dc, scales=ds, stream=s_comp)
        ev_comp[k].record(s_comp)
        s_out.wait_event(ev_comp[k])
        with torch.cuda.stream(s_out):
            c_pins[k].copy_(dc, non_blocking=True)
            s_pins[k].copy_(ds, non_blocking=True)
        ev_out[k].record(s_out)

    for i in range(2 * E_SETS):
        e2e_step(i)
    torch.cuda.synchronize(dev)
    e_steps = 30
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s_in)
    for i in range(e_steps):
        e2e_step(i + 2 * E_SETS)
    e1.record(s_out)
    torch.cuda.synchronize(dev)
    e_ms = max_over_ranks(e0.elapsed_time(e1) / e_steps, dev)
    e2e_gbs = bytes_step * world / (e_ms / 1e3) / 1e9

    extra = {}
    if not args.no_extra and rank == 0:
        extra = run_extra(hbr, W, dev, stream, peaks)

    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return 0

    cpu = None
    if world == 1:
        gb, cores, rows_done, dt = cpu_oracle_throughput(wl, bits, G, args.cpu_seconds)
        cpu = {"value": round(gb, 4), "unit": "GB/s", "cores": cores, "kind": "oracle",
               "sample": f"{rows_done} rows of A[8192,2048] ({dt:.1f} s, blocks of 512 rows): fp64 dense "
                         "Sylvester RHT + quantiser"}
        pg, pth, prow, pdt = cpu_plain_throughput(wl, bits, G, max(1.0, args.cpu_seconds / 2))
        cpu["plain"] = {"value": round(pg, 3), "unit": "GB/s", "cores": pth,
                        "kind": "plain scalar O(K log K) C loop (fp32 FWHT + group quantisation, OpenMP)",
                        "sample": f"{prow} rows of A[8192,2048] ({pdt:.1f} s, blocks of 2048 rows)"}
    psample = parity_sample(wl, bits, G, outs[0][0], outs[0][1]) if rank == 0 else None
    line = {
        "metric": METRIC, "value": round(gbs, 2), "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms / args.steps, 6), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": WORKLOAD_DESC,
                   "global_batch": M * world, "l2": "6 rotating input/output sets (258 MB > 126 MB L2)",
                   "launch": "every timed step replayed from CUDA graphs (6-step periods plus one remainder graph), "
                             "queued behind an untimed ~2 ms device-side spacer and one untimed replay",
                   "parallelism": f"dp{world} (independent rows)"},
        "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
                     "frac": round(achieved / peaks["hbm_gbs"], 4), "traffic": profiled_traffic("rot_quant_llama32_1b"),
                     "peak_source": f"{peak_kind} HBM copy bandwidth (MEASURED_PEAKS.json hbm_gbs)"},
        "cpu_baseline": cpu,
        "e2e": {"value": round(e2e_gbs, 2), "unit": "GB/s", "pipeline": "3 streams (copy in / compute / copy out)",
                "h2d_bytes_per_step": M * K * 2,
                "d2h_bytes_per_step": M * K * bits // 8 + M * (K // G) * 2},
        "gpu_launches": args.steps,
        "clocks": clk.summary(),
        "boundary_excluded": psample,
    }
    if extra:
        line["roofline_w4a4"] = extra.pop("roofline_w4a4", None)
        line["extra"] = extra
    print(json.dumps(line))
    return 0


def _time_loop(fn, n, stream, warm=5):
    """Seconds per call of fn(i) over n direct launches (host launch cost included)."""
    import torch
    for i in range(warm):
        fn(i)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for i in range(n):
        fn(i)
    e1.record(stream)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / n / 1e3  # seconds per call


class StepGraph:
    """Steps 0 .. period-1 of fn(i) (launching on the current stream) captured in one CUDA
    graph, so that back-to-back steps are timed on the device without per-launch host cost.
    run(n) issues exactly n steps: n // period replays of that graph, then one replay of a
    graph holding steps 0 .. (n % period) - 1 (captured by prepare(n), before timing)."""

    def __init__(self, fn, period, warm=3):
        import torch
        self.fn, self.period = fn, period
        for i in range(warm):
            fn(i)
        torch.cuda.synchronize()
        self.g = self._capture(period)
        self.tail = {}

    def _capture(self, k):
        import torch
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for i in range(k):
                self.fn(i)
        g.replay()
        torch.cuda.synchronize()
        return g

    def prepare(self, n):
        rem = n % self.period
        if rem and rem not in self.tail:
            self.tail[rem] = self._capture(rem)

    def run(self, n):
        self.prepare(n)
        reps, rem = divmod(n, self.period)
        for _ in range(reps):
            self.g.replay()
        if rem:
            self.tail[rem].replay()


def _graph_time(fn, n, period, warm=3):
    """Seconds per step of fn(i), n steps replayed from a CUDA graph of `period` steps (queued behind
    an untimed device-side spacer, as in the main measurement)."""
    import torch
    sg = StepGraph(fn, period, warm)
    sg.prepare(n)
    stream = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    torch.cuda._sleep(SPACER_CYCLES)
    e0.record(stream)
    sg.run(n)
    e1.record(stream)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / n / 1e3


L2_FLUSH_BYTES = 256_000_000   # twice the 126 MB L2


def _rotating(tensors, min_sets=3):
    """Copies of a step's operands (the first set is the tensors themselves), enough that the sets
    together exceed twice the L2: replaying them in turn, no step finds its operands in L2 (the
    layer-by-layer case of a model larger than L2)."""
    nbytes = sum(t.numel() * t.element_size() for t in tensors)
    nsets = max(min_sets, -(-L2_FLUSH_BYTES // max(1, nbytes)))
    return [tuple(tensors)] + [tuple(t.clone() for t in tensors) for _ in range(nsets - 1)]


def run_extra(hbr, W, dev, stream, peaks):
    import torch
    out = {}
    hbm = peaks["hbm_gbs"]
    # rotate + quantise on the other workloads
    for name, variant in (("q_proj_prefill", None), ("down_proj", None), ("harp11008", "init_identity"),
                          ("harp11008", "random")):
        wl = W.make_workload(name)
        if variant is None:
            plan = hbr.Plan.rht(wl.K, wl.signs)
        else:
            plan = hbr.harp_plan(W.harp_draws(2, wl.extra["radices"]), wl.signs, variant)
        # enough rotating input/output sets to exceed twice the 126 MB L2
        nsets = max(3, -(-256_000_000 // (wl.M * wl.K * 2 + wl.M * wl.K // 2)))
        As = [torch.from_numpy(wl.A).to(torch.bfloat16).to(dev) for _ in range(nsets)]
        for bits, G in wl.quant:
            outs = [(torch.empty((wl.M, wl.K * bits // 8), dtype=torch.uint8, device=dev),
                     torch.empty((wl.M, wl.K // G), dtype=torch.float16, device=dev)) for _ in range(nsets)]
            n = 200 if variant != "random" else 20

            def f(i):
                c, s = outs[i % nsets]
                hbr.rot_quant(As[i % nsets], plan, bits, G, codes=c, scales=s)
            t = _graph_time(f, n, nsets)
            b = algorithmic_bytes(wl.M, wl.K, bits, G)
            key = f"{name}{'_' + variant if variant else ''}_int{bits}_G{G}"
            out[key] = {"us": round(t * 1e6, 2), "GB/s": round(b / t / 1e9, 1), "frac_hbm": round(b / t / 1e9 / hbm, 4)}
        del As
    # W4A4 linear: prefill TOPS and decode GB/s
    int8_peak = measure_int8_peak(dev)
    for name in ("q_proj_prefill", "up_proj_prefill", "q_proj_decode", "up_proj_decode"):
        wl = W.make_workload(name)
        bits, G = wl.quant[0]
        plan = hbr.Plan.rht(wl.K, wl.signs)
        Aq, As_ = hbr.rot_quant(torch.from_numpy(wl.A).to(torch.bfloat16).to(dev), plan, bits, G)
        Wq, Ws = hbr.rot_quant(torch.from_numpy(np.ascontiguousarray(wl.W.T)).to(dev), plan, bits, G)
        N = Wq.shape[0]
        C = torch.empty((wl.M, N), dtype=torch.bfloat16, device=dev)
        n = 50 if wl.M > 16 else 200
        sets = _rotating((Aq, As_, Wq, Ws, C))

        def lin(i, sets=sets):
            a, sa, w, sw, c = sets[i % len(sets)]
            hbr.w4a4_linear(a, sa, w, sw, G, out=c)
        t = _graph_time(lin, n, len(sets))
        del sets
        ops = 2.0 * wl.M * N * wl.K
        wbytes = Wq.numel() + Ws.numel() * 2 + Aq.numel() + As_.numel() * 2 + C.numel() * 2
        out[f"w4a4_{name}"] = {"us": round(t * 1e6, 2), "TOPS": round(ops / t / 1e12, 1),
                               "frac_int8_spec": round(ops / t / 1e12 / INT8_DENSE_SPEC_TOPS, 4),
                               "frac_int8_measured": round(ops / t / 1e12 / int8_peak, 4) if int8_peak else None,
                               "GB/s": round(wbytes / t / 1e9, 1)}
    out.update(run_extra_next(hbr, W, dev, hbm, int8_peak))
    out["int8_peak_measured_TOPS"] = round(int8_peak, 1) if int8_peak else None
    # roofline of the prefill linear: int8 dense peak = the measured bf16 burst peak x 2 (the
    # nominal int8 : bf16 dense ratio, 4.5 : 2.25 PFLOP/s)
    qp = out.get("w4a4_q_proj_prefill")
    if qp:
        int8_from_bf16 = peaks["bf16_tflops"] * 2.0
        out["roofline_w4a4"] = {
            "bound": "tensor", "kernel": "w4a4_kernel (tcgen05 kind::i8), q_proj prefill M=2048 N=K=4096 G=128",
            "achieved": qp["TOPS"], "peak": round(int8_from_bf16, 1), "unit": "TOPS",
            "frac": round(qp["TOPS"] / int8_from_bf16, 4),
            "peak_source": "measured bf16 burst (MEASURED_PEAKS.json bf16_tflops) x 2, the nominal int8:bf16 ratio",
            "same_run_torch_int_mm_TOPS": out["int8_peak_measured_TOPS"],
            "spec_dense_int8_TOPS": INT8_DENSE_SPEC_TOPS}
    return out


def run_extra_next(hbr, W, dev, hbm, int8_peak):
    """Timings of the paths beyond the headline: the W4A8 linear, the two-sided linear, the
    one-call online path, int8-stored and per-block HARP processors, and K = 5120."""
    import torch
    out = {}
    for name in ("q_proj_prefill", "q_proj_decode"):
        wl = W.make_workload(name)
        bits, G = wl.quant[0]
        plan = hbr.Plan.rht(wl.K, wl.signs)
        dA = torch.from_numpy(wl.A).to(torch.bfloat16).to(dev)
        Wq, Ws = hbr.rot_quant(torch.from_numpy(np.ascontiguousarray(wl.W.T)).to(dev), plan, bits, G)
        N = Wq.shape[0]
        C = torch.empty((wl.M, N), dtype=torch.bfloat16, device=dev)
        n = 50 if wl.M > 16 else 200
        ops = 2.0 * wl.M * N * wl.K
        # every timing replays rotating operand sets (together above twice the L2)
        # W4A8: int8 activation codes
        A8, S8 = hbr.rot_quant(dA, plan, 8, G)
        sets = _rotating((A8.view(torch.int8), S8, Wq, Ws, C))

        def w8(i, sets=sets):
            a, sa, w, sw, c = sets[i % len(sets)]
            hbr.w4a8_linear(a, sa, w, sw, G, out=c)
        t = _graph_time(w8, n, len(sets))
        del sets
        out[f"w4a8_{name}"] = {"us": round(t * 1e6, 2), "TOPS": round(ops / t / 1e12, 1),
                               "frac_int8_measured": round(ops / t / 1e12 / int8_peak, 4) if int8_peak else None}
        # one call: rotate + quantise the bf16 activations, then the linear
        ws = torch.empty(hbr.w4a4_linear_act_workspace(wl.M, wl.K, G), dtype=torch.uint8, device=dev)
        A4, S4 = hbr.rot_quant(dA, plan, 4, G)
        sets = _rotating((dA, A4, S4, Wq, Ws, C, ws))

        def act(i, sets=sets):
            a, _, _, w, sw, c, wsp = sets[i % len(sets)]
            hbr.w4a4_linear_act(a, plan, w, sw, G, out=c, workspace=wsp)

        def sep(i, sets=sets):
            a, a4, s4, w, sw, c, _ = sets[i % len(sets)]
            hbr.rot_quant(a, plan, 4, G, codes=a4, scales=s4)
            hbr.w4a4_linear(a4, s4, w, sw, G, out=c)
        t = _graph_time(act, n, len(sets))
        t2 = _graph_time(sep, n, len(sets))
        out[f"act_path_{name}"] = {"us": round(t * 1e6, 2), "separate_calls_us": round(t2 * 1e6, 2)}
        # two-sided: the output rows returned through an RHT of size N
        U = hbr.Plan.rht(N, W.signs(W.rng(77), N))

        def two(i, sets=sets):
            _, a4, s4, w, sw, c, _ = sets[i % len(sets)]
            hbr.w4a4_linear_rot(a4, s4, w, sw, G, U, out=c)
        t = _graph_time(two, n, len(sets))
        del sets
        out[f"two_sided_{name}"] = {"us": round(t * 1e6, 2)}
    # HARP K = 11008 with int8-stored parameters (256 Cayley blocks of radix 43), the fp32
    # per-block QR variant, and 5120 = (8, 8, 8, 5, 2)
    wl = W.make_workload("harp11008")
    dA = torch.from_numpy(wl.A).to(torch.bfloat16).to(dev)
    codes = torch.empty((wl.M, wl.K // 2), dtype=torch.uint8, device=dev)
    scales = torch.empty((wl.M, wl.K // 128), dtype=torch.float16, device=dev)
    plans = {"harp11008_q8_cayley_per_block": hbr.harp_q8_plan(W.harp_q8_draws(4, wl.extra["radices"]), wl.signs),
             "harp11008_random_per_block_qr": hbr.harp_plan(W.harp_draws(2, wl.extra["radices"], per_block_gaussian=True),
                                                            wl.signs, "random")}
    for key, plan in plans.items():
        t = _graph_time(lambda i: hbr.rot_quant(dA, plan, 4, 128, codes=codes, scales=scales), 10, 5)
        b = algorithmic_bytes(wl.M, wl.K, 4, 128)
        out[f"{key}_int4_G128"] = {"us": round(t * 1e6, 2), "GB/s": round(b / t / 1e9, 1)}
    K = 5120
    g = W.rng(10)
    A = torch.from_numpy(W.activations(g, 4096, K, outlier_frac=0.01, outlier_scale=20.0)).to(torch.bfloat16).to(dev)
    plan = hbr.harp_q8_plan(W.harp_q8_draws(9, [8, 8, 8, 5, 2]), W.signs(g, K))
    codes = torch.empty((4096, K // 2), dtype=torch.uint8, device=dev)
    scales = torch.empty((4096, K // 128), dtype=torch.float16, device=dev)
    t = _graph_time(lambda i: hbr.rot_quant(A, plan, 4, 128, codes=codes, scales=scales), 10, 5)
    b = algorithmic_bytes(4096, K, 4, 128)
    out["harp5120_q8_A4096_int4_G128"] = {"us": round(t * 1e6, 2), "GB/s": round(b / t / 1e9, 1)}
    return out


def run_profile(args):
    """One kernel, one workload, --warmup + --steps launches; for ncu captures."""
    import torch
    import workloads as W
    import hadamard_butterfly_rotation_b200 as hbr
    dev = torch.device("cuda", 0)
    stream = torch.cuda.current_stream(dev)
    name = args.profile
    if name.startswith("w4a4"):
        wl = W.make_workload("q_proj_prefill" if name == "w4a4_prefill" else "q_proj_decode")
        bits, G = wl.quant[0]
        plan = hbr.Plan.rht(wl.K, wl.signs)
        Aq, As = hbr.rot_quant(torch.from_numpy(wl.A).to(torch.bfloat16).to(dev), plan, bits, G)
        Wq, Ws = hbr.rot_quant(torch.from_numpy(np.ascontiguousarray(wl.W.T)).to(dev), plan, bits, G)
        C = torch.empty((wl.M, Wq.shape[0]), dtype=torch.bfloat16, device=dev)
        sets = _rotating((Aq, As, Wq, Ws, C))
        nsets = len(sets)

        def fn(i):
            a, sa, w, sw, c = sets[i % nsets]
            hbr.w4a4_linear(a, sa, w, sw, G, out=c)
        work = 2.0 * wl.M * Wq.shape[0] * wl.K
        unit = "TOPS"
    else:
        wname = {"rot_quant": "llama32_1b", "q_proj_act_int4": "q_proj_prefill",
                 "down_proj_int4": "down_proj", "down_proj_int2": "down_proj",
                 "harp_init": "harp11008", "harp_random": "harp11008"}[name]
        wl = W.make_workload(wname)
        bits, G = wl.quant[1] if name == "down_proj_int2" else wl.quant[0]
        if name.startswith("harp"):
            plan = hbr.harp_plan(W.harp_draws(2, wl.extra["radices"]), wl.signs,
                                 "init_identity" if name == "harp_init" else "random")
        else:
            plan = hbr.Plan.rht(wl.K, wl.signs)
        # rotating input/output sets (together above twice the 126 MB L2), so that consecutive
        # launches captured with --cache-control none see steady-state DRAM reads and write-backs
        nsets = max(3, -(-256_000_000 // (wl.M * wl.K * 2 + wl.M * wl.K // 2)))
        A0 = torch.from_numpy(wl.A).to(torch.bfloat16).to(dev)
        As_ = [A0.clone() for _ in range(nsets)]
        outs = [(torch.empty((wl.M, wl.K * bits // 8), dtype=torch.uint8, device=dev),
                 torch.empty((wl.M, wl.K // G), dtype=torch.float16, device=dev)) for _ in range(nsets)]
        fn = lambda i: hbr.rot_quant(As_[i % nsets], plan, bits, G, codes=outs[i % nsets][0],
                                     scales=outs[i % nsets][1])
        work = algorithmic_bytes(wl.M, wl.K, bits, G)
        unit = "GB/s"
    t = _graph_time(fn, args.steps, nsets, warm=args.warmup)
    print(json.dumps({"profile": name, "us_per_launch": round(t * 1e6, 3),
                      unit: round(work / t / 1e9 if unit == "GB/s" else work / t / 1e12, 2)}))
    return 0


def measure_int8_peak(dev):
    """Same-run int8 tensor ceiling: torch._int_mm 8192^3 (library GEMM, reference only)."""
    import torch
    try:
        a = torch.randint(-8, 8, (8192, 8192), dtype=torch.int8, device=dev)
        b = torch.randint(-8, 8, (8192, 8192), dtype=torch.int8, device=dev).t()
        t = _time_loop(lambda i: torch._int_mm(a, b), 10, torch.cuda.current_stream(dev), warm=2)
        return 2 * 8192 ** 3 / t / 1e12
    except Exception:
        return None


if __name__ == "__main__":
    sys.exit(main())
