"""Benchmark of paged-KV long-history prefill attention on B200.

One step = the whole hot path over one synthetic workload: for every piece, pa_prefill (paged
K/V through the page table, split history) and pa_combine. Default workload: the full
32,768-token prefill in 2,048-token chunks (16 Q / 2 KV heads, D256, fp16, page size 16),
the pages' headline shape (BaseRT issue #51: paged vs contiguous KV at 32K).

Prints one JSON line (rank 0): query tokens/s over all GPUs, TFLOP/s, the paged/contiguous
ratio, the roofline of the prefill kernel, an end-to-end number through host buffers, and the
fp64 CPU oracle timed on a bounded sample as a baseline. `--impl reference` times the oracle
alone as the reference arm. Multi-GPU runs are independent replicas (no data exchange).
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "prefill-attn query tok/s & TFLOP/s vs BF16 peak; paged/contiguous ratio"
UNIT = "query tok/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0}
L2_FLUSH_BYTES = 512 << 20


# DRAM traffic of the roofline kernel, per launch: dram__bytes_read.sum + dram__bytes_write.sum
# of one-launch ncu captures of the c5 step's prefill kernel (chunks spread over the history,
# combined over the 16 chunks as stated in "chunks" and "how"). It stands for the kernel whose
# sources hash to `sources`; after any change to them the bench reports null until the
# captures are taken again.
TRAFFIC_CAPTURE = {
    "workload": "c5", "sources": "fa8f8d4e9d5b6d04", "bytes_per_launch": 108.12e6,
    "how": ("ncu dram__bytes_read.sum + dram__bytes_write.sum of one launch each of chunks 0, 3, "
            "6, 9, 12 and 15 (21.2, 39.3, 65.0, 94.2, 149.9, 321.2 MB; three launches per capture "
            "of bench.py --section piece), linear in between, mean over the 16 chunks")}


def kernel_sources_hash() -> str:
    """Hash of the prefill kernels' device code and of the schedule that feeds them, comments
    and blank lines left out (a comment edit does not change the kernel)."""
    import hashlib
    import re
    csrc = os.path.join(ROOT, "paged_kv_long_b200", "csrc")
    files = [os.path.join(csrc, f) for f in ("pa_geometry.h", "pa_kernels.cu", "pa_plan.cpp",
                                             "pa_schedule.h", "prefill_pair.cuh", "sm100.cuh")]
    h = hashlib.sha256()
    for f in files:
        with open(f) as fh:
            text = fh.read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        code = [ln.split("//")[0].rstrip() for ln in text.splitlines()]
        h.update(os.path.basename(f).encode())
        h.update("\n".join(ln for ln in code if ln.strip()).encode())
    return h.hexdigest()[:16]


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        d = json.load(open(path))
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                "source": "measured"}
    except Exception:
        return dict(FALLBACK_PEAKS, bf16_tflops_sustained=FALLBACK_PEAKS["bf16_tflops"],
                    source="fallback")


def roofline_peak(clocks: dict, peaks: dict) -> tuple[float, bool]:
    """The bf16 denominator of an in-step kernel and whether the timed steps ran power-capped.
    The measured burst GEMM rate applies to a kernel that runs at full clock, the sustained
    (power-capped) one to a kernel timed inside back-to-back steps long enough to reach the power
    cap, read from the timed window's clocks: median SM clock below 95 % of its maximum with
    sw_power_cap active (c5's 20 steps: ~7 ms each, capped after ~4 steps). Without clock
    samples the burst figure (the stricter one) applies."""
    capped = bool(clocks.get("sm_mhz") and clocks.get("sm_max_mhz")
                  and "sw_power_cap" in clocks.get("reasons", [])
                  and clocks["sm_mhz"] < 0.95 * clocks["sm_max_mhz"])
    return (peaks["bf16_tflops_sustained"] if capped else peaks["bf16_tflops"]), capped


class ClockSampler:
    """Clocks and throttle reasons while running: nvidia-smi every 20 ms (the sampler is given a
    moment to start before the timed region) and, where NVML is importable, the SM clock, power
    and clock-event reasons every ~2 ms with timestamps, so that the clock under load is the
    median over the timed window alone (`start()` .. `stop()`)."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    # NVML clock-event reason bits
    NV_REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
                  0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown"}

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None
        self.nv = []          # (time, sm MHz, power W, reason bits)
        self.window = [None, None]
        self._stop = None
        self._thread = None

    def _nvml_handle(self):
        import pynvml
        pynvml.nvmlInit()
        try:  # the device torch calls cuda:<gpu>, found by its PCI address
            import torch
            pr = torch.cuda.get_device_properties(self.gpu)
            bus = f"{pr.pci_domain_id:08x}:{pr.pci_bus_id:02x}:{pr.pci_device_id:02x}.0"
            return pynvml, pynvml.nvmlDeviceGetHandleByPciBusId(bus)
        except Exception:
            return pynvml, pynvml.nvmlDeviceGetHandleByIndex(self.gpu)

    def _poll(self):
        try:
            nv, h = self._nvml_handle()
        except Exception:
            return
        while not self._stop.is_set():
            try:
                self.nv.append((time.perf_counter(),
                                nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM),
                                nv.nvmlDeviceGetPowerUsage(h) / 1000.0,
                                nv.nvmlDeviceGetCurrentClocksEventReasons(h)))
            except Exception:
                return
            time.sleep(0.002)

    def __enter__(self):
        import threading
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                 "-lms", "20"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
        self._stop = threading.Event()
        self._thread = threading.Thread(target=self._poll, daemon=True)
        self._thread.start()
        time.sleep(0.5)
        return self

    def start(self):
        self.window[0] = time.perf_counter()

    def stop(self):
        self.window[1] = time.perf_counter()

    def __exit__(self, *exc):
        if self._stop is not None:
            self._stop.set()
            self._thread.join(timeout=5)
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        rows = []
        try:
            for line in open(self.path):
                f = [x.strip() for x in line.split(",")]
                if len(f) >= 9:
                    rows.append(f)
        except Exception:
            pass
        finally:
            try:
                os.unlink(self.path)
            except Exception:
                pass
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = {names[i] for r in rows for i in range(4) if r[5 + i] == "Active"}
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        smax = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        pw = [float(r[3]) for r in rows if r[3].replace(".", "").isdigit()]
        out = {"sm_mhz": statistics.median(sm) if sm else None,
               "sm_max_mhz": max(smax) if smax else None, "samples": len(rows),
               "power_w_max": max(pw, default=None), "source": "nvidia-smi, 20 ms"}
        t0, t1 = self.window
        win = [x for x in self.nv if t0 is not None and t1 is not None and t0 <= x[0] <= t1]
        if win:
            for x in win:
                reasons |= {n for bit, n in self.NV_REASONS.items() if x[3] & bit}
            out.update({"sm_mhz": statistics.median(x[1] for x in win),
                        "sm_mhz_min": min(x[1] for x in win),
                        "power_w_max": max(x[2] for x in win), "samples_timed": len(win),
                        "source": "NVML every ~2 ms over the timed steps (median); "
                                  "reasons: nvidia-smi and NVML"})
        if not rows and not win:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"], "samples": 0}
        out["reasons"] = sorted(reasons)
        return out


def cpu_model() -> str:
    """The host CPU's model name (first "model name" line of /proc/cpuinfo)."""
    try:
        for line in open("/proc/cpuinfo"):
            if line.lower().startswith("model name"):
                return line.split(":", 1)[1].strip()
    except Exception:
        pass
    import platform
    return platform.processor() or "unknown"


def bench_config(wl, args, world: int) -> dict:
    """The workload configuration both arms report (the same dict, so that the two lines can be
    compared key for key)."""
    return {"workload": wl.name, "seq_len": wl.total_keys, "chunk_rows": wl.pieces[0][1],
            "pieces": len(wl.pieces), "n_q_heads": wl.n_q_heads, "n_kv_heads": wl.n_kv_heads,
            "head_dim": wl.head_dim, "page_size": wl.page_size, "kv_layout": args.layout,
            "split_policy": args.policy if args.splits is None else f"{args.splits} splits",
            "l2": f"flushed between steps ({args.l2_flush_mb} MiB write outside the timed events)",
            "parallelism": f"replicas x{world}"}


def dist_env():
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def max_over_ranks(x: float, device=None) -> float:
    """The largest of every rank's x (a time: the job ends when its slowest replica does); x
    itself without a process group. Every rank must call it, in the same order."""
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(x)
    import torch
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(world: int, units_per_rank: float, t_ms: float) -> float:
    """Whole-job rate of `world` replicas that each process units_per_rank units in at most
    t_ms (the max over ranks)."""
    return world * units_per_rank / (t_ms / 1e3)


# ----------------------------------------------------------------------------- CPU oracle legs
class OracleSampler:
    """The fp64 CPU oracle timed on a stride sample of (row, head) pairs spread over the whole
    workload (one random head per sampled row), scaled to query tokens/s."""

    def __init__(self, wl, inp, threads: int = 0):
        from oracle import oracle
        self.oracle, self.wl, self.inp = oracle, wl, inp
        self.threads = threads if threads > 0 else oracle.max_threads()

    def run(self, n: int, seed: int = 17):
        import numpy as np
        wl, inp, oracle = self.wl, self.inp, self.oracle
        pieces = wl.pieces
        rng = np.random.default_rng(seed)
        t_sum, pairs = 0.0, 0
        total_rows = sum(r for _, r in pieces)
        gidx = np.linspace(0, total_rows - 1, n).astype(np.int64)
        starts = np.cumsum([0] + [r for _, r in pieces])
        for i, (h, r) in enumerate(pieces):
            sel = gidx[(gidx >= starts[i]) & (gidx < starts[i + 1])] - starts[i]
            if len(sel) == 0:
                continue
            heads = rng.integers(0, wl.n_q_heads, size=len(sel)).astype(np.int32)
            pb = oracle.Problem(q=inp.piece_q(i), k=inp.k_pool, v=inp.v_pool, hist_len=h,
                                dtype=wl.dtype, page_table=inp.page_table, scale=wl.scale)
            t0 = time.perf_counter()
            oracle.attend(pb, sel, heads, threads=self.threads)
            t_sum += time.perf_counter() - t0
            pairs += len(sel)
        # one (row, head) pair is 1/Hq of a query token's attention
        return (pairs / wl.n_q_heads) / t_sum, pairs, t_sum

    def calibrate(self, seconds: float) -> int:
        """Sample size that costs about `seconds` of CPU time."""
        n = max(8, self.threads)
        while True:
            _, pairs, t = self.run(n)
            if t >= seconds / 4 or n >= 200000:
                break
            n *= 2
        return int(max(8, min(200000, n * seconds / max(t, 1e-6))))


def reference_arm(args):
    """The oracle as the reference arm, on the host cores of rank 0. A step is one bounded
    stride sample of the workload's (row, head) pairs; `ms_per_step` is that sample's measured
    wall time and `value` the query tokens of attention it covers per second."""
    rank, world, _ = dist_env()
    if rank != 0:
        return 0
    from paged_kv_long_b200.inputs import WORKLOADS, generate
    wl = WORKLOADS[args.workload]
    inp = generate(wl, poison=False)
    steps, warmup = args.steps, args.warmup
    per_step = max(1.0, min(10.0, 80.0 / max(steps + warmup, 1)))
    sampler = OracleSampler(wl, inp, args.cpu_threads)
    n = sampler.calibrate(per_step)
    for k in range(warmup):
        sampler.run(max(8, n // 4), seed=50 + k)
    rates, secs, pairs = [], [], 0
    for k in range(steps):
        r, pairs, t = sampler.run(n, seed=100 + k)
        rates.append(r)
        secs.append(t)
    cores = sampler.threads
    value = statistics.median(rates)
    step_tokens = pairs / wl.n_q_heads
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": steps, "warmup": warmup,
        "ms_per_step": statistics.median(secs) * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": bench_config(wl, args, world),
        "step": (f"one stride sample of {pairs} (row, head) pairs over the workload's "
                 f"{wl.query_rows} query rows = {step_tokens:.1f} query tokens of attention; "
                 f"ms_per_step is its measured wall time"),
        "timed_seconds": sum(secs),
        "workload_ms_extrapolated": wl.query_rows / value * 1e3,
        "reference_parallelism": f"rank 0 only, {cores} host threads (OpenMP)",
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "cpu_model": cpu_model(),
                         "sample": f"{pairs} (row, head) pairs per step, stride-sampled over the "
                                   f"workload's {wl.query_rows} query rows; {statistics.median(secs):.2f} s "
                                   f"per step measured"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------------------- GPU arm
def time_steps(dw, steps, warmup, flush, stream, record_kernels=False, clocks=None):
    """Per-step CUDA-event timing with an L2 flush between steps (outside the timed events).
    Returns (per-step ms list, prefill-kernel ms list per step). `clocks` (a ClockSampler)
    gets the timed window."""
    import torch
    from paged_kv_long_b200 import binding
    for _ in range(warmup):
        with torch.cuda.stream(stream):
            flush.zero_()
        dw.run(stream)
    torch.cuda.synchronize()
    if clocks is not None:
        clocks.start()
    step_ms, kern_ms = [], []
    evs = []
    for _ in range(steps):
        with torch.cuda.stream(stream):  # on the timed stream: done before the step's events
            flush.zero_()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        kev = []
        torch.cuda.nvtx.range_push("prefill step")  # for profilers that filter on NVTX ranges
        e0.record(stream)
        for i in range(len(dw.wl.pieces)):
            if record_kernels:
                a = torch.cuda.Event(enable_timing=True)
                b = torch.cuda.Event(enable_timing=True)
                a.record(stream)
                q, k, v, tab = dw.piece_inputs(i)
                binding.prefill(dw.plans[i], q, k, v, tab, dw.outs[i], dw.ws, stream)
                b.record(stream)
                binding.combine(dw.plans[i], dw.ws, dw.outs[i], stream)
                kev.append((a, b))
            else:
                dw.run_piece(i, stream)
        e1.record(stream)
        torch.cuda.nvtx.range_pop()
        evs.append((e0, e1, kev))
    torch.cuda.synchronize()
    if clocks is not None:
        clocks.stop()
    for e0, e1, kev in evs:
        step_ms.append(e0.elapsed_time(e1))
        kern_ms.append([a.elapsed_time(b) for a, b in kev])
    return step_ms, kern_ms


def kv_append_measure(inp, dev, stream, peaks, reps=20):
    """pa_kv_append on the workload's rows: all of them in one call (HBM-bound; the roofline is
    the measured copy bandwidth), and chunk by chunk as a prefill engine issues them."""
    import numpy as np
    import torch
    from paged_kv_long_b200 import binding
    wl = inp.wl
    dt = torch.bfloat16 if wl.dtype == "bf16" else torch.float16

    def dev_bits(bits):
        return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).to(dev).view(dt)

    h0 = wl.first_pos
    rows = wl.total_keys - h0
    kn, vn = dev_bits(inp.k_logical[h0:h0 + rows]), dev_bits(inp.v_logical[h0:h0 + rows])
    kp, vp = dev_bits(inp.k_pool), dev_bits(inp.v_pool)
    tab = torch.from_numpy(inp.page_table).to(dev)
    with torch.cuda.stream(stream):
        def timed(fn):
            """Per call: an event pair around each call on the stream, median over reps (the
            host's time between calls is not the kernel's)."""
            for _ in range(3):
                fn()
            evs = []
            for _ in range(reps):
                e0 = torch.cuda.Event(enable_timing=True)
                e1 = torch.cuda.Event(enable_timing=True)
                e0.record(stream)
                fn()
                e1.record(stream)
                evs.append((e0, e1))
            torch.cuda.synchronize()
            return statistics.median(a.elapsed_time(b) for a, b in evs)

        def timed_back_to_back(fn):
            for _ in range(3):
                fn()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            for _ in range(reps):
                fn()
            e1.record(stream)
            torch.cuda.synchronize()
            return e0.elapsed_time(e1) / reps

        t_pair = timed(lambda: binding.kv_append(kn, vn, kp, vp, tab, h0, stream))

        def graphed(fn, n):
            """n calls captured in one CUDA graph, replayed between one event pair: the kernel's
            time per call with the launch gaps of a graph, not the event-to-kernel latency."""
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                for _ in range(n):
                    fn(torch.cuda.current_stream())
            for _ in range(2):
                g.replay()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            g.replay()
            e1.record(stream)
            torch.cuda.synchronize()
            return e0.elapsed_time(e1) / n

        t_all = graphed(lambda st: binding.kv_append(kn, vn, kp, vp, tab, h0, st), reps)

        def chunks():
            for h, r in wl.pieces:
                binding.kv_append(kn[h - h0:h - h0 + r], vn[h - h0:h - h0 + r], kp, vp, tab, h,
                                  stream)
        t_chunks = timed_back_to_back(chunks)
    nbytes = 2 * rows * wl.n_kv_heads * wl.head_dim * 2 * 2   # K and V, read once, written once
    gbs = nbytes / (t_all * 1e-3) / 1e9
    return {"workload": f"{rows} rows of K and V (all the workload's positions) in one call",
            "timing": (f"{reps} calls replayed as one CUDA graph between an event pair, per call; "
                       "ms_event_pair: an event pair around each eager call, median (it adds "
                       "the event-to-kernel latency)"),
            "ms": t_all, "ms_event_pair": t_pair, "GB_per_s": gbs,
            "peak_GB_per_s": peaks["hbm_gbs"],
            "frac": gbs / peaks["hbm_gbs"], "bytes": nbytes,
            "us_per_chunk_call_host_bound": t_chunks * 1e3 / len(wl.pieces),
            "chunk_calls": len(wl.pieces)}


DECODE_BATCH = 32          # sequences of one decode step
DECODE_LENS = (1024, 32768)  # key counts drawn uniformly from this range (the prompt sweep's)


def decode_measure(wl, dev, stream, peaks, reps=20, seed=6000):
    """pa_decode (+ pa_combine) on a batch of sequences over one shared page pool, with the
    workload's heads, head dim, page size and dtype: HBM-bound (every key's K and V row read
    once), so the roofline is the measured copy bandwidth."""
    import numpy as np
    import torch
    from paged_kv_long_b200 import binding
    from paged_kv_long_b200.inputs import decode_batch
    lens = np.random.default_rng(seed).integers(DECODE_LENS[0], DECODE_LENS[1] + 1,
                                               size=DECODE_BATCH)
    db = decode_batch(seed + 1, lens, wl.n_q_heads, wl.n_kv_heads, wl.head_dim, wl.page_size,
                      wl.dtype, poison=False)
    dt = torch.bfloat16 if wl.dtype == "bf16" else torch.float16

    def dev_bits(bits):
        return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).to(dev).view(dt)

    q, kp, vp = dev_bits(db.q), dev_bits(db.k_pool), dev_bits(db.v_pool)
    tab = torch.from_numpy(db.block_table).to(dev)
    sl = torch.from_numpy(db.seq_lens).to(dev)
    p = binding.decode_plan(wl.n_q_heads, wl.n_kv_heads, wl.head_dim, wl.page_size,
                            DECODE_BATCH, int(lens.max()), wl.dtype)
    out = torch.empty((DECODE_BATCH, wl.n_q_heads, wl.head_dim), dtype=torch.float32,
                      device=dev)
    ws = binding.workspace(p, dev)
    # the same step as a batch of one-row chunks: host lengths, balanced items
    bp = binding.batch_plan(wl.n_q_heads, wl.n_kv_heads, wl.head_dim, wl.page_size,
                            np.ones(DECODE_BATCH, dtype=np.int32), lens - 1, wl.dtype)
    ws_b = binding.workspace(bp.plan, dev)

    def timed(fn):
        with torch.cuda.stream(stream):
            for _ in range(3):
                fn()
            evs = []
            for _ in range(reps):
                e0 = torch.cuda.Event(enable_timing=True)
                e1 = torch.cuda.Event(enable_timing=True)
                e0.record(stream)
                fn()
                e1.record(stream)
                evs.append((e0, e1))
            torch.cuda.synchronize()
        return statistics.median(a.elapsed_time(b) for a, b in evs)

    ms = timed(lambda: binding.decode(p, q, kp, vp, tab, sl, out, ws, stream))
    ms_b = timed(lambda: binding.batch_prefill(bp, q.view(DECODE_BATCH, wl.n_q_heads,
                                                          wl.head_dim), kp, vp, tab, out, ws_b,
                                               stream))
    keys = int(lens.sum())
    nbytes = (2 * keys * wl.n_kv_heads * wl.head_dim * 2            # K and V rows
              + DECODE_BATCH * wl.n_q_heads * wl.head_dim * (2 + 4))  # Q in, fp32 out
    gbs = nbytes / (ms * 1e-3) / 1e9
    return {"workload": f"{DECODE_BATCH} sequences, {keys} keys in all (lengths uniform in "
                        f"{DECODE_LENS[0]}..{DECODE_LENS[1]}), one query token each, "
                        f"{wl.n_q_heads}q/{wl.n_kv_heads}kv D{wl.head_dim} PS{wl.page_size} "
                        f"{wl.dtype}; K/V {nbytes / 1e9:.2f} GB > L2",
            "splits": p.splits, "ms": ms, "GB_per_s": gbs, "peak_GB_per_s": peaks["hbm_gbs"],
            "frac": gbs / peaks["hbm_gbs"], "bytes": nbytes,
            "tokens_per_s": DECODE_BATCH / (ms * 1e-3),
            "balanced": {"how": "pa_batch_prefill with one row per sequence (host lengths)",
                         "items": int(bp.plan.units), "ms": ms_b,
                         "GB_per_s": nbytes / (ms_b * 1e-3) / 1e9,
                         "frac": nbytes / (ms_b * 1e-3) / 1e9 / peaks["hbm_gbs"]}}


def routes_measure(inp, dev, stream, flush, reps=8):
    """The cold prompt's two bulk-prefill routes, each a whole step (every chunk): paged (append
    the chunk's K/V to pages, prefill through the table) and contiguous staging + page publish
    (prefill on the staging buffer, publish the chunk's rows). L2 flushed before each step; the
    two routes' steps alternate and each route reports its median."""
    import torch
    from paged_kv_long_b200.runner import PrefillRoutes
    rt = PrefillRoutes(inp, dev)
    routes = (("paged", rt.run_paged), ("staged", rt.run_staged))
    evs = {r: [] for r, _ in routes}
    with torch.cuda.stream(stream):
        for _ in range(3):
            for _, fn in routes:
                fn(stream)
        for _ in range(reps):  # interleaved, so that drift hits both routes alike
            for route, fn in routes:
                flush.zero_()
                e0 = torch.cuda.Event(enable_timing=True)
                e1 = torch.cuda.Event(enable_timing=True)
                e0.record(stream)
                fn(stream)
                e1.record(stream)
                evs[route].append((e0, e1))
        torch.cuda.synchronize()
    res = {r: statistics.median(a.elapsed_time(b) for a, b in e) for r, e in evs.items()}
    same = all(torch.equal(a, b) for a, b in zip(rt.outs["paged"], rt.outs["staged"]))
    del rt
    return {"workload": "cold prompt of the bench workload, chunk by chunk",
            "paged_route_ms": res["paged"], "staged_route_ms": res["staged"],
            "staged_over_paged_time": res["staged"] / res["paged"],
            "outputs_identical": bool(same)}


def e2e_steps(inp, dw, steps, stream):
    """End to end through the public API: pinned host inputs -> device, prefill + combine for
    every piece, outputs -> pinned host, every step (DeviceWorkload.run_streamed: the pools
    first, then each chunk's Q copy, compute and output copy on three streams, overlapped).
    Returns (per-step ms, h2d, d2h bytes)."""
    import numpy as np
    import torch
    wl = inp.wl
    tdt = torch.bfloat16 if wl.dtype == "bf16" else torch.float16

    def pinned(a, dt=None):
        t = torch.from_numpy(np.ascontiguousarray(a))
        if dt is not None:
            t = t.view(torch.int16).view(dt)
        return t.pin_memory()

    hq = pinned(inp.q.view(np.int16), tdt)
    hk = pinned(inp.k_pool.view(np.int16), tdt)
    hv = pinned(inp.v_pool.view(np.int16), tdt)
    ht = pinned(inp.page_table)
    houts = [torch.empty(tuple(o.shape), dtype=torch.float32).pin_memory() for o in dw.outs]
    h2d = sum(t.numel() * t.element_size() for t in (hq, hk, hv, ht))
    d2h = sum(t.numel() * t.element_size() for t in houts)
    ms = []
    copy_in = torch.cuda.Stream(stream.device)
    copy_out = torch.cuda.Stream(stream.device)
    for k in range(steps + 1):
        e0 = torch.cuda.Event(enable_timing=True)
        e0.record(copy_in)
        e1 = dw.run_streamed(hq, hk, hv, ht, houts, copy_in, stream, copy_out)
        e1.synchronize()
        torch.cuda.synchronize()
        if k > 0:  # the first is a warm-up
            ms.append(e0.elapsed_time(e1))
    return ms, h2d, d2h


# The pages' long-history attention sweep (splash PR #33, "Results"): a 2048-row chunk at 32K
# history in 512-row pieces with 4 splits (c3), and a 128-row piece at 128K history with 16
# splits and with 1 split (c4); each also with the planner's own choice.
SIDE_WORKLOADS = (("c3", (4, 0)), ("c4", (16, 1, 0)))


_GENERATED = {}


def generated(name: str):
    """Seeded timing inputs of a workload (unused pool slots zero), made once per process."""
    from paged_kv_long_b200.inputs import generate
    if name not in _GENERATED:
        _GENERATED[name] = generate(name, poison=False)
    return _GENERATED[name]


def workloads_measure(dev, stream, flush, peaks, reps=10):
    """The 32K-128K configurations beside the headline: for each split setting, paged and
    contiguous steps alternate (L2 flushed before each); per step the prefill launches are timed
    with an event pair each on the launching stream. Reported medians: the step, the prefill
    launches' summed time, their algorithmic TFLOP/s and fraction of the measured bf16 peak, and
    the K/V bytes the pieces must read (every visible key's K and V row once) per second of
    prefill-kernel time."""
    import torch
    from paged_kv_long_b200.inputs import WORKLOADS
    from paged_kv_long_b200.runner import DeviceWorkload
    res = {}
    peak = peaks["bf16_tflops"]
    for name, split_settings in SIDE_WORKLOADS:
        wl = WORKLOADS[name]
        inp = generated(name)
        flops, kvb = wl.flops(), wl.kv_bytes()
        t_roof = max(flops / (peak * 1e12), kvb / (peaks["hbm_gbs"] * 1e9))
        rows = []
        for sp in split_settings:
            dw = DeviceWorkload(inp, dev, paged=True, splits=sp)
            dwc = DeviceWorkload(inp, dev, paged=False, splits=sp)
            time_steps(dw, 0, 3, flush, stream)
            time_steps(dwc, 0, 3, flush, stream)
            pp, cc, pk, ck = [], [], [], []
            for _ in range(reps):
                a_ms, a_k = time_steps(dw, 1, 0, flush, stream, record_kernels=True)
                b_ms, b_k = time_steps(dwc, 1, 0, flush, stream, record_kernels=True)
                pp += a_ms
                cc += b_ms
                pk.append(sum(a_k[0]))
                ck.append(sum(b_k[0]))
            torch.cuda.synchronize()
            same = all(torch.equal(x, y) for x, y in zip(dw.outs, dwc.outs))
            t_p, t_c = statistics.median(pp), statistics.median(cc)
            k_p, k_c = statistics.median(pk), statistics.median(ck)
            tf = flops / (k_p / 1e3) / 1e12
            rows.append({
                "splits": "planner" if sp == 0 else sp,
                "plans": [{"policy": int(p.policy), "splits": int(p.splits), "units": int(p.units)}
                          for p in dw.plans],
                "paged_ms": t_p, "contiguous_ms": t_c, "paged_contiguous_ratio": t_c / t_p,
                "query_tok_per_s": wl.query_rows / (t_p / 1e3),
                "kernel_ms": k_p, "kernel_ms_contiguous": k_c,
                "kernel_tflops": tf, "frac": tf / peak,
                "frac_of_sustained_peak": tf / peaks["bf16_tflops_sustained"],
                "kv_GB_per_s": kvb / (k_p * 1e-3) / 1e9,
                "step_frac_of_roofline": t_roof / (t_p / 1e3),
                "paged_contiguous_outputs_identical": bool(same)})
            del dw, dwc
        res[name] = {"workload": wl.name, "algorithmic_flops": flops, "algorithmic_kv_bytes": kvb,
                     "peak_tflops": peak, "runs": rows,
                     "how": (f"{reps} paged and {reps} contiguous steps alternating, L2 flushed "
                             "before each; medians; kernel = the prefill launches' summed event "
                             "time; frac = flops / kernel time / peak; kv_GB_per_s = algorithmic "
                             "K+V bytes / kernel time")}
        torch.cuda.empty_cache()
    return res


def pieces_run(wl, dev, stream, args):
    """Some pieces of a workload alone (for one-launch profiler captures): every listed piece's
    prefill + combine `--steps` times in turn (L2 flushed before each), in the chosen layout and
    split setting. Launch order: piece p0's prefill, its merge (if split), piece p1's ...; the
    first (steps - 1) rounds are warm-up for a capture of the last round."""
    import torch
    from paged_kv_long_b200.runner import DeviceWorkload
    inp = generated(args.workload)
    dw = DeviceWorkload(inp, dev, paged=args.layout == "paged", splits=args.splits,
                        policy=args.policy)
    idx = [int(x) for x in args.pieces.split(",")] if args.pieces else list(range(len(wl.pieces)))
    flush = torch.empty(max(args.l2_flush_mb, 1) * (1 << 20) // 4, dtype=torch.float32,
                        device=dev)
    ms = {i: [] for i in idx}
    for _ in range(args.steps):
        for i in idx:
            with torch.cuda.stream(stream):
                flush.zero_()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            dw.run_piece(i, stream)
            e1.record(stream)
            ms[i].append((e0, e1))
    torch.cuda.synchronize()
    return {"workload": wl.name, "layout": args.layout,
            "pieces": {str(i): {"hist_len": wl.pieces[i][0], "rows": wl.pieces[i][1],
                                "splits": int(dw.plans[i].splits), "policy": int(dw.plans[i].policy),
                                "units": int(dw.plans[i].units),
                                "ms": [a.elapsed_time(b) for a, b in ms[i]]} for i in idx}}


def section_arm(args):
    """One side measurement alone (for profiling it): prints its JSON object on one line."""
    import torch
    from paged_kv_long_b200.inputs import WORKLOADS, generate
    wl = WORKLOADS[args.workload]
    dev = torch.device("cuda", 0)
    stream = torch.cuda.Stream(dev)
    peaks = load_peaks()
    if args.section == "piece":
        res = pieces_run(wl, dev, stream, args)
    elif args.section == "decode":
        res = decode_measure(wl, dev, stream, peaks, reps=args.steps)
    else:
        inp = generate(wl, poison=False)
        if args.section == "kv_append":
            res = kv_append_measure(inp, dev, stream, peaks, reps=args.steps)
        else:
            flush = torch.empty((L2_FLUSH_BYTES) // 4, dtype=torch.float32, device=dev)
            res = routes_measure(inp, dev, stream, flush, reps=args.steps)
    print(json.dumps({"section": args.section, **res}), flush=True)
    return 0


def gpu_arm(args):
    import torch
    import torch.distributed as dist
    from paged_kv_long_b200.inputs import WORKLOADS, generate
    from paged_kv_long_b200.runner import DeviceWorkload

    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    wl = WORKLOADS[args.workload]
    inp = generate(wl, poison=False)
    dev = torch.device("cuda", local)
    stream = torch.cuda.Stream(dev)
    split_arg = args.splits if args.splits is not None else None
    paged = args.layout == "paged"
    dw = DeviceWorkload(inp, dev, paged=paged, splits=split_arg, policy=args.policy)
    flush = torch.empty(max(args.l2_flush_mb, 1) * (1 << 20) // 4, dtype=torch.float32, device=dev)
    peaks = load_peaks()

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    # ---- timed region: K steps of the paged path
    barrier()
    with ClockSampler(local) as clk:
        wall0 = time.perf_counter()
        step_ms, kern_ms = time_steps(dw, args.steps, args.warmup, flush, stream,
                                      record_kernels=True, clocks=clk)
        barrier()
        wall = time.perf_counter() - wall0
    clocks = clk.summary()
    t_step = max_over_ranks(sum(step_ms) / len(step_ms), dev)
    tokens = wl.query_rows
    value = job_throughput(world, tokens, t_step)
    flops = wl.flops()
    tflops = flops / (t_step / 1e3) / 1e12

    # ---- prefill kernel roofline: algorithmic FLOPs over its summed launch durations
    kern_total_ms = sum(sum(k) for k in kern_ms) / len(kern_ms)
    kern_tflops = flops / (kern_total_ms / 1e3) / 1e12
    peak, power_capped = roofline_peak(clocks, peaks)
    t_roof = max(flops / (peak * 1e12), wl.kv_bytes() / (peaks["hbm_gbs"] * 1e9))

    traffic, traffic_note = None, "no capture of this kernel build"
    cap = TRAFFIC_CAPTURE
    if (cap and paged and args.workload == cap["workload"] and args.policy == "makespan"
            and args.splits is None and kernel_sources_hash() == cap["sources"]):
        traffic = cap["bytes_per_launch"]
        traffic_note = cap["how"]

    # ---- contiguous control at the same split counts (the ratio's denominator)
    t_contig = t_paged_pairs = last_paged = last_contig = same_bits = None
    if paged and not args.no_contiguous:
        from paged_kv_long_b200 import binding
        # the same schedule per piece as the paged run (the planner does not look at the layout)
        dwc = DeviceWorkload(inp, dev, paged=False, splits=split_arg, policy=args.policy)
        for p, pc in zip(dw.plans, dwc.plans):
            assert (p.policy, p.splits, p.units, p.ws_bytes) == (pc.policy, pc.splits, pc.units,
                                                                pc.ws_bytes)
        # paged and contiguous steps alternate, so that clock or neighbour drift hits both
        time_steps(dwc, 0, args.warmup, flush, stream)
        pp, cc, pk, ck = [], [], [], []
        for _ in range(max(6, args.steps // 2)):
            a_ms, a_k = time_steps(dw, 1, 0, flush, stream, record_kernels=True)
            b_ms, b_k = time_steps(dwc, 1, 0, flush, stream, record_kernels=True)
            pp += a_ms
            cc += b_ms
            pk.append(a_k[0][-1])
            ck.append(b_k[0][-1])
        t_paged_pairs = statistics.median(pp)
        t_contig = statistics.median(cc)
        last_paged = statistics.median(pk)
        last_contig = statistics.median(ck)
        # verify mode: the two layouts run the same schedule on the same keys, so their outputs
        # of the last step must be the same bits
        torch.cuda.synchronize()
        same_bits = all(torch.equal(a_, b_) for a_, b_ in zip(dw.outs, dwc.outs))
        del dwc

    # ---- KV append, the step before prefill (its own HBM roofline)
    kv = None
    if paged and not args.no_kv_append:
        kv = kv_append_measure(inp, dev, stream, peaks)

    # ---- contiguous staging + page publish against the paged route (cold prompts only)
    routes = None
    if paged and not args.no_routes and wl.first_pos == 0:
        routes = routes_measure(inp, dev, stream, flush)

    # ---- batched paged decode on a cache of the same shape (its own HBM roofline)
    dec = None
    if paged and not args.no_decode:
        dec = decode_measure(wl, dev, stream, peaks)

    # ---- the 32K-128K configurations (c3, c4) at the workload's and the planner's splits
    side = None
    if paged and not args.no_workloads and world == 1:
        side = workloads_measure(dev, stream, flush, peaks)

    # ---- end to end through the public API with host buffers
    e2e = None
    if not args.no_e2e and paged:
        e_ms, h2d, d2h = e2e_steps(inp, dw, max(2, min(args.steps, 5)), stream)
        t_e = max_over_ranks(sum(e_ms) / len(e_ms), dev)
        e2e = {"value": job_throughput(world, tokens, t_e), "unit": UNIT,
               "how": "pinned host -> device (pools, then each chunk's Q), prefill + combine, "
                      "each chunk's output -> pinned host; copies overlap compute on 3 streams",
               "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": d2h, "ms_per_step": t_e}

    launches = args.steps * sum(1 + (1 if p.splits > 1 else 0) for p in dw.plans)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        sampler = OracleSampler(wl, inp, args.cpu_threads)
        r, pairs, t = sampler.run(sampler.calibrate(args.cpu_seconds))
        cpu = {"value": r, "unit": UNIT, "cores": sampler.threads, "kind": "oracle",
               "cpu_model": cpu_model(),
               "sample": f"{pairs} (row, head) pairs stride-sampled over all {wl.query_rows} query "
                         f"rows of the workload, {t:.1f} s of fp64 CPU work, scaled to tok/s"}
        if not args.no_workloads:
            # the oracle on one thread, on the 128-row piece at 131,072 history (c4)
            from paged_kv_long_b200.inputs import WORKLOADS
            wl4 = WORKLOADS["c4"]
            s1 = OracleSampler(wl4, generated("c4"), threads=1)
            r1, p1, t1 = s1.run(s1.calibrate(3.0))
            cpu["single_thread_c4"] = {
                "value": r1, "unit": UNIT, "cores": 1, "gflops": r1 * wl4.flops() / wl4.query_rows / 1e9,
                "sample": f"{p1} (row, head) pairs of c4, {t1:.1f} s on one thread"}

    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return 0
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": t_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": wl.dtype, "data": "synthetic",
        "config": bench_config(wl, args, world),
        "splits_per_piece": [p.splits for p in dw.plans],
        "tflops": tflops,
        "paged_contiguous_ratio": (t_contig / t_paged_pairs) if t_contig else None,
        "paged_contiguous_ratio_last_chunk": (last_contig / last_paged) if t_contig else None,
        "contiguous_ms_per_step": t_contig,
        "ratio_method": "median of alternating paged / contiguous steps (L2 flushed before each)",
        "paged_contiguous_outputs_identical": same_bits,
        "roofline": {"bound": "tensor", "achieved": kern_tflops, "peak": peak,
                     "unit": "TFLOP/s", "frac": kern_tflops / peak, "traffic": traffic,
                     "traffic_source": traffic_note,
                     "peak_source": (f"{peaks['source']} bf16 dense, sustained (seconds of "
                                     "back-to-back GEMMs under the power cap): the timed steps "
                                     "ran power-capped (clocks: median SM clock below 95 % of "
                                     "max, sw_power_cap)" if power_capped else
                                     f"{peaks['source']} bf16 dense, burst: the timed steps ran "
                                     "at full clock"),
                     # the same kernel against the measured burst GEMM rate (full clock)
                     "frac_of_burst_peak": kern_tflops / peaks["bf16_tflops"],
                     "frac_of_sustained_peak": kern_tflops / peaks["bf16_tflops_sustained"],
                     "burst_peak": peaks["bf16_tflops"],
                     "sustained_peak": peaks["bf16_tflops_sustained"],
                     "kernel_ms_each_step": [round(sum(k), 4) for k in kern_ms],
                     "step_frac_of_roofline": t_roof / (t_step / 1e3),
                     # the step split: the prefill launches' summed event time, and the rest
                     # (the merges of split pieces and the gaps between launches)
                     "kernel_ms_per_step": kern_total_ms,
                     "outside_kernel_ms_per_step": t_step - kern_total_ms,
                     "kernel": "prefill_pair_kernel (pa_prefill, head dim 256)" if wl.head_dim == 256 else "prefill_kernel (pa_prefill)",
                     "algorithmic_flops_per_step": flops},
        "e2e": e2e,
        "kv_append": kv,
        "decode": dec,
        "workloads": side,
        "staging_route": routes,
        "cpu_baseline": cpu,
        "gpu_launches": launches,
        "clocks": clocks,
        "wall_s": wall,
    }
    print(json.dumps(line), flush=True)
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="c5", choices=["c1", "c2", "c3", "c4", "c5"])
    ap.add_argument("--splits", type=int, default=None,
                    help="split count for every piece (default: the workload's, else the planner)")
    ap.add_argument("--policy", default="makespan", choices=["makespan", "cores", "legacy", "balanced"])
    ap.add_argument("--layout", default="paged", choices=["paged", "contiguous"])
    ap.add_argument("--no-contiguous", action="store_true", help="skip the contiguous control")
    ap.add_argument("--l2-flush-mb", type=int, default=L2_FLUSH_BYTES >> 20)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-kv-append", action="store_true")
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-routes", action="store_true")
    ap.add_argument("--no-workloads", action="store_true",
                    help="skip the c3/c4 side measurements (and the 1-thread oracle on c4)")
    ap.add_argument("--section", default="all",
                    choices=["all", "decode", "kv_append", "routes", "piece"],
                    help="run one side measurement alone (1 GPU; --steps = its repetitions); "
                         "'piece' runs the pieces listed by --pieces")
    ap.add_argument("--pieces", default="", help="piece indices for --section piece, e.g. 0,7,15")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--cpu-threads", type=int, default=0,
                    help="host threads of the oracle legs (0: all cores)")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        return reference_arm(args)
    if args.section != "all":
        return section_arm(args)
    return gpu_arm(args)


if __name__ == "__main__":
    sys.exit(main())
