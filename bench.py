"""Benchmark: sliding-window causal attention on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl {ours,reference}]

A step is one swa_forward over the Mistral-shaped workload (B=1, H=32, T=16384,
D=128, W=4096, bf16), inputs resident in HBM. The same run then times, each in a timed
region of its own: the window sweep (B=2, H=16, T=8192, D=128, W in {1, 256, 1024, 4096,
8192}) under "sweep"; the small workload (B=1, H=8, T=512, D=64, W=128) with L2 hot and
with L2 flushed between steps under "small"; swa_decode over the streaming workload (B=64
streams, H=32, D=128, W=4096 ring, positions uniform in [0, 100000)) under "decode"; the
chunked streaming prefill (the same streams each taking 128 new tokens,
swa_chunk_forward) under "chunk"; the multi-head module (cuBLASLt projections around the
attention, B1 T16384 d_model 4096, 32 heads, W4096) under "module"; the backward of
the Mistral-shaped prefill under "backward"; and the prefill on inputs whose rows a few
keys dominate (falling scores, B1 H8 T16384 D128 W4096) with adaptive P under "peaked".
Useful prefill FLOPs count the band only:
4*B*H*D*sum_i min(i+1, W). Decode bytes are the K/V slots read plus q, out and pos;
chunk bytes are the ring slots the chunk needs, its q, k, v, out, the appended rows and
pos.

Under torchrun each rank runs the same workload on its own GPU (weak scaling, no
collective on the data path); times are the max over ranks. `--impl reference` times
the float64 CPU oracle on bounded samples of the same workload (rank 0 only).
"""
import argparse
import json
import os
import statistics
import sys
import threading
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from sliding_window_causal_b200 import inputs  # noqa: E402

METRIC = "SWA prefill TFLOP/s (band FLOPs, % bf16 TC peak); decode HBM GB/s"
L2_BYTES = 126 * 2**20


# DRAM traffic per launch of each kernel on the bench workload, from one ncu capture
# (dram__bytes_read.sum + dram__bytes_write.sum; the captures are summarised in profiles/).
# Reported only while the kernel's sources are unchanged since the capture.
KERNEL_SOURCES = {"prefill": ["prefill_pp.cuh", "ptx.cuh", "umma.h", "plan.h"],
                  "decode": ["decode.cuh", "ptx.cuh"],
                  "chunk": ["chunk.cuh", "prefill_pp.cuh", "ptx.cuh", "umma.h", "plan.h"]}
# Decode and chunk were captured with 16 of the 64 streams (1.07 GB of rings). Each stream
# reads only its own ring, so traffic grows with the units processed (ring slots, chunk rows),
# but the positions are random and 16 streams are not a quarter of them. The capture is
# scaled by the kernel's algorithmic bytes, full workload over the 16-stream sample (the
# chunk kernel's count leaves out the append's ring writes): (sample, full) below.
SAMPLE_ALGORITHMIC_BYTES = {"decode": (951_025_792, 4_296_016_384),
                            "chunk": (1_121_042_560, 4_508_746_240)}


def _scaled(kind, captured):
    sample, full = SAMPLE_ALGORITHMIC_BYTES[kind]
    return captured * full / sample


MEASURED_TRAFFIC = {
    # Mistral-shaped workload, captured at full size (prefill only on the device)
    "prefill": {"bytes": 548.4e6 + 116.5e6, "sources": "c826ea2319336f9b"},
    "decode": {"bytes": _scaled("decode", 951.0e6 + 3.7e6), "sources": "5d66f52c4894035b"},
    "chunk": {"bytes": _scaled("chunk", 1105.4e6 + 17.4e6), "sources": "11efae5968553e54"},
}


def measured_traffic(kind):
    import hashlib
    m = hashlib.sha256()
    for f in KERNEL_SOURCES[kind]:
        with open(os.path.join(ROOT, "sliding_window_causal_b200", "csrc", f), "rb") as fh:
            m.update(fh.read())
    rec = MEASURED_TRAFFIC[kind]
    return rec["bytes"] if m.hexdigest()[:16] == rec["sources"] else None


def band_flops(B, H, T, D, W):
    # sum_{i<T} min(i+1, W) = W(W+1)/2 + (T-W)W for T >= W, else T(T+1)/2
    w = min(W, T)
    s = w * (w + 1) // 2 + (T - w) * w
    return 4 * B * H * D * s


def decode_bytes(B, H, D, W, pos):
    n = torch.clamp(pos + 1, max=W).sum().item()
    return int(n * H * D * 2 * 2 + 2 * B * H * D * 2 + 8 * B)


def chunk_work(B, H, C, D, W, pos):
    """(band FLOPs, algorithmic bytes) of one chunked streaming step: row c of stream b
    (position P = pos[b] + c) scores min(P+1, W) keys; the bytes are the ring slots the
    chunk needs (positions max(0, pos-W+1) .. pos-1, K and V), the chunk's q, k, v and
    out, the appended K and V rows and pos."""
    flops = 0
    ring_slots = 0
    for p in pos.tolist():
        P = torch.arange(p, p + C, dtype=torch.int64)
        flops += int(torch.clamp(P + 1, max=W).sum().item())
        ring_slots += min(p, W - 1)
    flops *= 4 * H * D
    nbytes = H * ring_slots * D * 2 * 2 + B * H * C * D * 2 * 4 + B * H * min(C, W) * D * 2 * 2 + 8 * B
    return flops, nbytes


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d["bf16_tflops"], d["hbm_gbs"], "measured"
    return 1590.0, 6650.0, "fallback"


class ClockSampler:
    """Samples the SM clock and the clock-event reasons with NVML while running."""

    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
               0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x100: "display_clock_setting"}

    def __init__(self, index, period=0.005):
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self.period, self.index = period, index
        self._stop = threading.Event()
        self._t = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self.nv = None

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
                r = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                for bit, name in self.REASONS.items():
                    if r & bit:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.nv is not None:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *a):
        if self._t is not None:
            self._stop.set()
            self._t.join()

    def summary(self):
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons - {"gpu_idle"}),
                "samples": len(self.samples)}


def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    pg = None
    if world > 1:
        import torch.distributed as dist
        import datetime
        backend = "nccl" if args.impl == "ours" else "gloo"
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
        pg = dist
    return world, rank, local, pg


def max_over_ranks(x, pg, device):
    """The largest of every rank's x (x itself without a process group); all ranks must
    call it, in the same order."""
    if pg is None:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    pg.all_reduce(t, op=pg.ReduceOp.MAX)
    pg.barrier()
    return t.item()


def whole_job(units_per_rank, ms_per_step, world):
    """Whole-job throughput under weak scaling: every rank processes units_per_rank per
    step, and the step takes ms_per_step (the max over ranks)."""
    return world * units_per_rank / (ms_per_step * 1e-3)


def timed(fn, steps, stream, pg, device):
    """Run fn() `steps` times between a barrier + synchronize on both sides; returns
    the elapsed device time in ms (CUDA events on `stream`), max over ranks."""
    if pg is not None:
        pg.barrier()
    torch.cuda.synchronize(device)
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record(stream)
    for _ in range(steps):
        fn()
    end.record(stream)
    torch.cuda.synchronize(device)
    return max_over_ranks(start.elapsed_time(end), pg, device)


def cpu_baseline_prefill(wl, budget_s, q, k, v):
    """Time the float64 oracle on query rows of the workload (batch 0), 2048 rows per call,
    head after head in order (starting again from head 0 after the last), until about
    budget_s of wall time has passed. Only the oracle calls are timed: widening a head's
    inputs to float64 is input preparation. Returns (TFLOP/s, description, threads)."""
    import numpy as np
    import oracle
    T, D, W = wl.T, wl.D, wl.W
    chunk = 2048
    flops = rows_done = 0
    t_oracle = 0.0
    head = None
    t0 = time.perf_counter()
    while time.perf_counter() - t0 < budget_s:
        hh = (rows_done // T) % wl.H
        if hh != head:
            qh, kh, vh = (t[0:1, hh:hh + 1].to(torch.float64).numpy() for t in (q, k, v))
            head = hh
        r0 = rows_done % T
        rows = np.arange(r0, min(T, r0 + chunk), dtype=np.int64)
        t1 = time.perf_counter()
        oracle.forward_rows(qh, kh, vh, W, rows)
        t_oracle += time.perf_counter() - t1
        flops += int(sum(4 * D * min(i + 1, W) for i in rows))
        rows_done += len(rows)
    full, rest = divmod(rows_done, T)
    if full + (rest > 0) <= wl.H:
        parts = ([f"head 0 in full" if full == 1 else f"heads 0..{full - 1} in full"] if full else []) + \
                ([f"rows 0..{rest - 1} of head {full}"] if rest else [])
        where = ", then ".join(parts)
    else:
        where = f"{rows_done / T:.2f} heads' rows, heads 0..{wl.H - 1} in order and round again"
    desc = (f"{rows_done} query rows of batch 0: {where}; {t_oracle:.1f} s in the oracle "
            f"of {time.perf_counter() - t0:.1f} s")
    return flops / t_oracle / 1e12, desc, oracle.max_threads()


def run_reference(args, world, rank):
    """Reference arm: the float64 CPU oracle on bounded samples of the prefill workload."""
    if rank != 0:
        return
    wl = inputs.MISTRAL
    q, k, v = inputs.for_workload(wl)
    per_step = float(os.environ.get("SWA_REF_STEP_S", "4"))
    for _ in range(args.warmup):
        cpu_baseline_prefill(wl, per_step / 4, q, k, v)
    vals = []
    t0 = time.perf_counter()
    desc, threads = "", 1
    for _ in range(args.steps):
        val, desc, threads = cpu_baseline_prefill(wl, per_step, q, k, v)
        vals.append(val)
    dt = time.perf_counter() - t0
    value = statistics.mean(vals)
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": dt * 1e3 / max(1, args.steps), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": wl.name, "B": wl.B, "H": wl.H, "T": wl.T, "D": wl.D, "W": wl.W,
                   "seed": wl.seed},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
                         "sample": f"per step: {desc}"},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def roofline_point(F, nbytes, ms, peak_tf, peak_gbs, peak_kind):
    """Roofline of one prefill launch: F band FLOPs and nbytes algorithmic bytes (q, k, v
    read once, out written once) in ms. The bound is the tensor core when the arithmetic
    intensity F / nbytes is at or above the ridge (peak FLOP/s over peak bytes/s), HBM
    below it; `attainable` is min(tensor peak, intensity x HBM peak)."""
    tf = F / (ms * 1e-3) / 1e12
    gbs = nbytes / (ms * 1e-3) / 1e9
    ai = F / nbytes
    ridge = peak_tf * 1e3 / peak_gbs
    attainable = min(peak_tf, ai * peak_gbs / 1e3)
    if ai >= ridge:
        r = {"bound": "tensor", "achieved": tf, "peak": peak_tf, "unit": "TFLOP/s", "frac": tf / peak_tf}
    else:
        r = {"bound": "hbm", "achieved": gbs, "peak": peak_gbs, "unit": "GB/s", "frac": gbs / peak_gbs}
    r.update({"peak_kind": peak_kind, "intensity_flop_per_byte": ai, "ridge_flop_per_byte": ridge,
              "attainable_tflops": attainable, "frac_of_attainable": tf / attainable, "tflops": tf,
              "gbs": gbs, "algorithmic_bytes": nbytes, "traffic": None})
    return r


def cpu_info():
    """(CPU model name, logical CPU count) of this host."""
    model = None
    try:
        with open("/proc/cpuinfo") as fh:
            for line in fh:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    return model, os.cpu_count()


def cpu_one_thread_small(budget_s):
    """The float64 oracle on the small workload (B1 H8 T512 D64 W128) on one thread, whole
    calls repeated for about budget_s: (GFLOP/s, calls)."""
    import oracle
    wl = inputs.SMALL
    q, k, v = (t.to(torch.float64).numpy() for t in inputs.for_workload(wl))
    F = band_flops(wl.B, wl.H, wl.T, wl.D, wl.W)
    n0 = oracle.max_threads()
    oracle.set_threads(1)
    try:
        calls, t_or = 0, 0.0
        while t_or < budget_s:
            t1 = time.perf_counter()
            oracle.forward(q, k, v, wl.W)
            t_or += time.perf_counter() - t1
            calls += 1
    finally:
        oracle.set_threads(n0)
    return calls * F / t_or / 1e9, calls


def prefill_workload(name):
    if name == "mistral":
        return inputs.MISTRAL
    if name == "small":
        return inputs.SMALL
    for w in inputs.SWEEP:
        if name == f"sweep-w{w.W}":
            return w
    raise SystemExit(f"unknown workload {name}")


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-peaked", action="store_true",
                    help="skip the prefill on inputs whose rows a few keys dominate (adaptive P)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-chunk", action="store_true")
    ap.add_argument("--no-module", action="store_true")
    ap.add_argument("--no-backward", action="store_true")
    ap.add_argument("--no-sweep", action="store_true")
    ap.add_argument("--no-small", action="store_true")
    ap.add_argument("--backward-workload", default="mistral",
                    help="prefill workload whose backward the backward leg times (as --workload)")
    ap.add_argument("--chunk-streams", type=int, default=None,
                    help="override the chunk workload's stream count (smaller profiling runs)")
    ap.add_argument("--workload", default="mistral",
                    help="prefill workload of the main line: mistral (default), small, "
                         "sweep-w{1,256,1024,4096,8192}")
    ap.add_argument("--decode-streams", type=int, default=None,
                    help="override the decode workload's stream count (smaller profiling runs)")
    args = ap.parse_args()
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")
    world, rank, local, pg = dist_setup(args)
    if args.impl == "reference":
        run_reference(args, world, rank)
        if pg is not None:
            pg.destroy_process_group()
        return

    import sliding_window_causal_b200 as swa
    from sliding_window_causal_b200 import _native

    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    stream = torch.cuda.current_stream(device)
    peak_tf, peak_gbs, peak_kind = load_peaks()

    # ------------------------------------------------------------ prefill
    wl = prefill_workload(args.workload)
    qh, kh, vh = inputs.for_workload(wl)
    q, k, v = (t.to(device) for t in (qh, kh, vh))
    out = torch.empty_like(q)
    F = band_flops(wl.B, wl.H, wl.T, wl.D, wl.W)
    fwd = lambda: swa.forward(q, k, v, wl.W, out=out)
    for _ in range(args.warmup):
        fwd()
    swa.device_status()
    dev_index = int(os.environ.get("CUDA_VISIBLE_DEVICES", str(local)).split(",")[local]) \
        if os.environ.get("CUDA_VISIBLE_DEVICES", "").replace(",", "").isdigit() else local
    with ClockSampler(dev_index) as clk:
        ms = timed(fwd, args.steps, stream, pg, device)
    swa.device_status()
    ms_step = ms / args.steps
    value = whole_job(F, ms_step, world) / 1e12
    achieved = F / (ms_step * 1e-3) / 1e12

    # ------------------------------------------------------------ e2e (host buffers)
    e2e = None
    staging = (q, k, v, out)
    if not args.no_e2e:
        pin = lambda t: t.pin_memory()
        qp, kp, vp = pin(qh), pin(kh), pin(vh)
        outp = torch.empty(qh.shape, dtype=qh.dtype).pin_memory()
        e2e_fn = lambda: swa.forward_host(qp, kp, vp, wl.W, out=outp, device=device, staging=staging)
        for _ in range(3):
            e2e_fn()
        e2e_steps = max(3, min(args.steps, 20))
        e2e_ms = timed(e2e_fn, e2e_steps, stream, pg, device) / e2e_steps
        swa.device_status()
        e2e = {"value": world * F / (e2e_ms * 1e-3) / 1e12, "unit": "TFLOP/s",
               "h2d_bytes_per_step": 3 * qh.numel() * qh.element_size(),
               "d2h_bytes_per_step": outp.numel() * outp.element_size(), "steps": e2e_steps}
        del qp, kp, vp, outp

    # ------------------------------------------------------------ window sweep
    sweep = None
    if not args.no_sweep:
        sweep = []
        for sw in inputs.SWEEP:
            sq, sk, sv = (t.to(device) for t in inputs.for_workload(sw))
            sout = torch.empty_like(sq)
            sfn = lambda sq=sq, sk=sk, sv=sv, sout=sout, W=sw.W: swa.forward(sq, sk, sv, W, out=sout)
            for _ in range(args.warmup):
                sfn()
            swa.device_status()
            with ClockSampler(dev_index) as sclk:
                sms = timed(sfn, args.steps, stream, pg, device) / args.steps
            swa.device_status()
            sF = band_flops(sw.B, sw.H, sw.T, sw.D, sw.W)
            snb = 4 * sw.B * sw.H * sw.T * sw.D * 2
            sweep.append({
                "workload": sw.name, "W": sw.W, "band_flops": sF, "ms_per_step": sms,
                "value": world * sF / (sms * 1e-3) / 1e12, "unit": "TFLOP/s",
                "roofline": roofline_point(sF, snb, sms, peak_tf, peak_gbs, f"{peak_kind} bf16 burst / HBM copy"),
                "l2": f"inputs larger than L2 (q, k, v {3 * sq.numel() * 2 / 2**20:.0f} MiB), no flush",
                "clocks": sclk.summary(), "gpu_launches": args.steps, "seed": sw.seed})
            del sq, sk, sv, sout, sfn
        torch.cuda.empty_cache()

    # ------------------------------------------------------------ small workload (hot and cold L2)
    small = None
    if not args.no_small:
        sw = inputs.SMALL
        sq, sk, sv = (t.to(device) for t in inputs.for_workload(sw))
        sout = torch.empty_like(sq)
        sfn = lambda: swa.forward(sq, sk, sv, sw.W, out=sout)
        for _ in range(args.warmup):
            sfn()
        swa.device_status()
        with ClockSampler(dev_index) as hclk:
            hot_ms = timed(sfn, args.steps, stream, pg, device) / args.steps
        # cold L2: a 256 MiB buffer is written between steps, outside the timed events
        flush = torch.empty(256 * 2**20 // 4, dtype=torch.float32, device=device)
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
        with ClockSampler(dev_index) as cclk2:
            for a, b in ev:
                flush.zero_()
                a.record(stream)
                sfn()
                b.record(stream)
            torch.cuda.synchronize(device)
        cold_ms = max_over_ranks(sum(a.elapsed_time(b) for a, b in ev) / args.steps, pg, device)
        swa.device_status()
        # The same call back to back from one CUDA graph (50 calls captured once, replayed
        # `steps` times): the device time of a call without the host's per-call launch
        # overhead, which the two figures above include at this size.
        graph_hot = None
        try:
            reps = 50
            gstream = torch.cuda.Stream(device)
            gstream.wait_stream(stream)
            with torch.cuda.stream(gstream):
                sfn()
            torch.cuda.synchronize(device)
            graph = torch.cuda.CUDAGraph()
            with torch.cuda.graph(graph, stream=gstream):
                for _ in range(reps):
                    sfn()
            with torch.cuda.stream(stream):
                graph.replay()
                torch.cuda.synchronize(device)
                with ClockSampler(dev_index) as gclk:
                    g_ms = timed(graph.replay, args.steps, stream, pg, device) / (args.steps * reps)
            swa.device_status()
            graph_hot = {"ms_per_call": g_ms, "value": world * band_flops(sw.B, sw.H, sw.T, sw.D, sw.W) / (g_ms * 1e-3) / 1e12,
                         "unit": "TFLOP/s", "calls_per_graph": reps, "gpu_launches": args.steps * reps,
                         "clocks": gclk.summary(),
                         "l2": "inputs smaller than L2: L2-resident"}
            del graph
        except Exception as e:  # capture is an extra view of the same call; report, do not fail
            graph_hot = {"unavailable": f"{type(e).__name__}: {e}"}
        sF = band_flops(sw.B, sw.H, sw.T, sw.D, sw.W)
        snb = 4 * sw.B * sw.H * sw.T * sw.D * 2
        small = {
            "workload": sw.name, "band_flops": sF, "seed": sw.seed,
            "hot_l2": {"ms_per_step": hot_ms, "value": world * sF / (hot_ms * 1e-3) / 1e12, "unit": "TFLOP/s",
                       "l2": "inputs smaller than L2 (1.5 MiB): L2-resident between steps",
                       "roofline": roofline_point(sF, snb, hot_ms, peak_tf, peak_gbs, f"{peak_kind} bf16 burst / HBM copy"),
                       "clocks": hclk.summary()},
            "cold_l2": {"ms_per_step": cold_ms, "value": world * sF / (cold_ms * 1e-3) / 1e12, "unit": "TFLOP/s",
                        "l2": "a 256 MiB buffer written between steps, outside the timed events",
                        "roofline": roofline_point(sF, snb, cold_ms, peak_tf, peak_gbs, f"{peak_kind} bf16 burst / HBM copy"),
                        "clocks": cclk2.summary()},
            "graph_hot": graph_hot,
            "gpu_launches": 2 * args.steps,
            "note": "latency-bound: 32 query tiles on 148 SMs"}
        del sq, sk, sv, sout, sfn, flush
        torch.cuda.empty_cache()

    # ------------------------------------------------------------ decode
    decode_line = None
    if not args.no_decode:
        del q, k, v, out, staging
        torch.cuda.empty_cache()
        dw = inputs.DECODE
        if args.decode_streams:
            import dataclasses
            dw = dataclasses.replace(dw, B=args.decode_streams,
                                     name=dw.name.replace("B64", f"B{args.decode_streams}"))
        dq, dkr, dvr, dpos = inputs.for_workload(dw)
        nbytes = decode_bytes(dw.B, dw.H, dw.D, dw.W, dpos)
        dq, dkr, dvr, dpos = (t.to(device) for t in (dq, dkr, dvr, dpos))
        dout = torch.empty_like(dq)
        dec = lambda: swa.decode(dq, dkr, dvr, dpos, dw.W, out=dout)
        for _ in range(args.warmup):
            dec()
        swa.device_status()
        with ClockSampler(dev_index) as dclk:
            dms = timed(dec, args.steps, stream, pg, device) / args.steps
        swa.device_status()
        gbs = nbytes / (dms * 1e-3) / 1e9
        S, chunk = swa.split_plan(dw.B, dw.H, dw.D, dw.W)
        decode_line = {
            "metric": "decode HBM GB/s", "value": world * gbs, "unit": "GB/s", "ms_per_step": dms,
            "config": {"workload": dw.name, "B": dw.B, "H": dw.H, "D": dw.D, "W": dw.W,
                       "pos": "uniform [0, 100000)", "seed": dw.seed, "splits": S, "chunk": chunk,
                       "l2": f"inputs larger than L2 ({2 * dkr.numel() * 2 / 1e9:.2f} GB of rings)"},
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": peak_gbs, "unit": "GB/s",
                         "frac": gbs / peak_gbs, "peak_kind": peak_kind,
                         "traffic": measured_traffic("decode") if dw.B == 64 else None,
                         "algorithmic_bytes": nbytes},
            "clocks": dclk.summary(), "gpu_launches": args.steps,
        }

    # ------------------------------------------------------------ peaked inputs, adaptive P
    # Rows that a few keys dominate (falling scores: the oldest key of each band) make the
    # fast prefill recompute nearly every row; the default mode switches a device to
    # adaptive P after such a launch. Timed here in the adaptive mode directly.
    peaked_line = None
    if not args.no_peaked:
        torch.cuda.empty_cache()
        PB, PH, PT, PD, PW, pseed = 1, 8, 16384, 128, 4096, 77
        pq, pk, pv = (t.to(device) for t in inputs.peaked_prefill_inputs(PB, PH, PT, PD, pseed, "falling"))
        pout = torch.empty_like(pq)
        prev_mode = swa.set_prefill_mode(swa.PREFILL_ADAPTIVE)
        try:
            pstep = lambda: swa.forward(pq, pk, pv, PW, out=pout)
            for _ in range(args.warmup):
                pstep()
            swa.device_status()
            psteps = max(3, min(args.steps, 20))
            with ClockSampler(dev_index) as pclk:
                pms = timed(pstep, psteps, stream, pg, device) / psteps
            swa.device_status()
        finally:
            swa.set_prefill_mode(prev_mode)
        pF = band_flops(PB, PH, PT, PD, PW)
        peaked_line = {
            "metric": "prefill TFLOP/s, rows dominated by a few keys, adaptive P", "unit": "TFLOP/s",
            "value": world * pF / (pms * 1e-3) / 1e12, "ms_per_step": pms, "steps": psteps,
            "config": {"workload": f"falling scores B{PB} H{PH} T{PT} D{PD} W{PW}", "seed": pseed,
                       "inputs": "q all ones, k_t = -0.05 t + N(0, 0.01^2), v ~ N(0,1), bf16",
                       "mode": "adaptive"},
            "clocks": pclk.summary(), "gpu_launches": psteps,
        }
        del pq, pk, pv, pout

    # ------------------------------------------------------------ chunked streaming prefill
    chunk_line = None
    if not args.no_chunk:
        torch.cuda.empty_cache()
        cw = inputs.CHUNKED
        if args.chunk_streams:
            import dataclasses
            cw = dataclasses.replace(cw, B=args.chunk_streams,
                                     name=cw.name.replace("B64", f"B{args.chunk_streams}"))
        cq, ck, cv, ckr, cvr, cpos = inputs.for_workload(cw)
        cflops, cbytes = chunk_work(cw.B, cw.H, cw.C, cw.D, cw.W, cpos)
        cq, ck, cv, ckr, cvr, cpos = (t.to(device) for t in (cq, ck, cv, ckr, cvr, cpos))
        cout = torch.empty_like(cq)
        # Every step processes the same chunk at the same positions (the append rewrites the
        # same slots), so every step does the same work.
        stepc = lambda: swa.chunk_forward(cq, ck, cv, ckr, cvr, cpos, cw.W, out=cout)
        for _ in range(args.warmup):
            stepc()
        swa.device_status()
        with ClockSampler(dev_index) as cclk:
            cms = timed(stepc, args.steps, stream, pg, device) / args.steps
        swa.device_status()
        cgbs = cbytes / (cms * 1e-3) / 1e9
        ctf = cflops / (cms * 1e-3) / 1e12
        chunk_line = {
            "metric": "chunked streaming prefill HBM GB/s", "value": world * cgbs, "unit": "GB/s",
            "ms_per_step": cms, "tflops": world * ctf,
            "config": {"workload": cw.name, "B": cw.B, "H": cw.H, "C": cw.C, "D": cw.D, "W": cw.W,
                       "pos": "uniform [0, 100000)", "seed": cw.seed, "band_flops": cflops,
                       "l2": f"inputs larger than L2 ({2 * ckr.numel() * 2 / 1e9:.2f} GB of rings)"},
            "roofline": {"bound": "hbm", "achieved": cgbs, "peak": peak_gbs, "unit": "GB/s",
                         "frac": cgbs / peak_gbs, "peak_kind": peak_kind,
                         "traffic": measured_traffic("chunk") if cw.B == 64 else None,
                         "algorithmic_bytes": cbytes, "tensor_frac": ctf / peak_tf},
            "clocks": cclk.summary(), "gpu_launches": 2 * args.steps,
        }
        del cq, ck, cv, ckr, cvr, cpos, cout

    # ------------------------------------------------------------ multi-head module
    module_line = None
    if not args.no_module:
        torch.cuda.empty_cache()
        mB, mT, md, mH, mW = 1, 16384, 4096, 32, 4096
        gm = torch.Generator().manual_seed(1006)
        mx = torch.randn(mB, mT, md, generator=gm).to(torch.bfloat16).to(device)
        mws = [(torch.randn(md, md, generator=gm) / md ** 0.5).to(torch.bfloat16).to(device) for _ in range(4)]
        mbs = [(torch.randn(md, generator=gm) * 0.1).to(torch.bfloat16).to(device) for _ in range(4)]
        mout = torch.empty_like(mx)
        mwork = torch.empty(swa.mha_workspace_bytes(mB, mT, md, torch.bfloat16), dtype=torch.uint8, device=device)
        mstep = lambda: swa.mha_forward(mx, mws[0], mbs[0], mws[1], mbs[1], mws[2], mbs[2], mws[3], mbs[3],
                                        mH, mW, out=mout, workspace=mwork)
        for _ in range(args.warmup):
            mstep()
        swa.device_status()
        with ClockSampler(dev_index) as mclk:
            mms = timed(mstep, args.steps, stream, pg, device) / args.steps
        swa.device_status()
        gemm_flops = 4 * 2 * mB * mT * md * md
        attn_flops = band_flops(mB, mH, mT, md // mH, mW)
        mtf = (gemm_flops + attn_flops) / (mms * 1e-3) / 1e12
        module_line = {
            "metric": "sliding-window MHA module TFLOP/s (projection + band FLOPs)", "value": world * mtf,
            "unit": "TFLOP/s", "ms_per_step": mms,
            "config": {"workload": f"mha module bf16 B{mB} T{mT} d{md} H{mH} W{mW}", "B": mB, "T": mT,
                       "d_model": md, "H": mH, "W": mW, "seed": 1006, "gemm_flops": gemm_flops,
                       "band_flops": attn_flops,
                       "l2": f"inputs larger than L2 (x {mB * mT * md * 2 / 2**20:.0f} MiB, kernels "
                             f"{4 * md * md * 2 / 2**20:.0f} MiB), no flush"},
            "roofline": {"bound": "tensor", "achieved": mtf, "peak": peak_tf, "unit": "TFLOP/s",
                         "frac": mtf / peak_tf, "peak_kind": f"{peak_kind} bf16 burst", "traffic": None},
            "clocks": mclk.summary(), "gpu_launches": args.steps,
        }
        del mx, mws, mbs, mout, mwork

    # ------------------------------------------------------------ backward (gradients)
    backward_line = None
    if not args.no_backward:
        torch.cuda.empty_cache()
        bw = prefill_workload(args.backward_workload)
        bq, bk, bv = (t.to(device) for t in inputs.for_workload(bw))
        gb = torch.Generator().manual_seed(1007)
        bdo = torch.randn(bw.B, bw.H, bw.T, bw.D, generator=gb).to(bw.dtype).to(device)
        bsteps = max(3, args.steps // 5)
        bout, blse = swa.forward_lse(bq, bk, bv, bw.W)  # the forward's output and statistics
        bstep = lambda: swa.backward(bq, bk, bv, bdo, bw.W, out=bout, lse=blse)
        for _ in range(3):
            bstep()
        swa.device_status()
        with ClockSampler(dev_index) as bclk:
            bms = timed(bstep, bsteps, stream, pg, device) / bsteps
        swa.device_status()
        bflops = 5 * band_flops(bw.B, bw.H, bw.T, bw.D, bw.W) // 2  # five band products
        b_in = 5 * bw.B * bw.H * bw.T * bw.D * 2  # bytes of q, k, v, out, dout (bf16)
        btf = bflops / (bms * 1e-3) / 1e12
        backward_line = {
            "metric": "backward TFLOP/s (2.5 x band FLOPs)", "value": world * btf, "unit": "TFLOP/s",
            "ms_per_step": bms, "steps": bsteps,
            "config": {"workload": bw.name + " backward", "B": bw.B, "H": bw.H, "T": bw.T, "D": bw.D,
                       "W": bw.W, "seed": bw.seed, "dout_seed": 1007, "useful_flops": bflops,
                       "l2": f"inputs larger than L2 (q, k, v, out, dout {b_in / 2**20:.0f} MiB), no flush"
                       if b_in > L2_BYTES else "inputs smaller than L2: L2-resident"},
            "roofline": {"bound": "tensor", "achieved": btf, "peak": peak_tf, "unit": "TFLOP/s",
                         "frac": btf / peak_tf, "peak_kind": f"{peak_kind} bf16 burst", "traffic": None,
                         "products_issued_per_useful": 7 / 5},
            "clocks": bclk.summary(), "gpu_launches": 3 * bsteps,
        }
        del bq, bk, bv, bdo, bout, blse

    # ------------------------------------------------------------ CPU baseline (rank 0, N = 1)
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        val, desc, threads = cpu_baseline_prefill(wl, float(os.environ.get("SWA_CPU_BUDGET_S", "15")),
                                                  qh, kh, vh)
        model, ncpu = cpu_info()
        one, calls = cpu_one_thread_small(2.0)
        cpu = {"value": val, "unit": "TFLOP/s", "cores": threads, "kind": "oracle", "sample": desc,
               "cpu_model": model, "nproc": ncpu,
               "one_thread": {"value": one, "unit": "GFLOP/s", "workload": inputs.SMALL.name,
                              "sample": f"{calls} whole calls of the oracle on one thread"}}

    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": wl.name, "B": wl.B, "H": wl.H, "T": wl.T, "D": wl.D, "W": wl.W,
                   "seed": wl.seed, "band_flops": F,
                   "l2": f"inputs larger than L2 (q, k, v {3 * qh.numel() * 2 / 2**20:.0f} MiB), no flush"
                   if 3 * qh.numel() * 2 > L2_BYTES else "inputs smaller than L2: L2-resident"},
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak_tf, "unit": "TFLOP/s",
                     "frac": achieved / peak_tf, "peak_kind": f"{peak_kind} bf16 burst",
                     "traffic": measured_traffic("prefill") if args.workload == "mistral" else None,
                     "algorithmic_bytes": 4 * wl.B * wl.H * wl.T * wl.D * 2,
                     "frac_of_spec_2250": achieved / 2250.0},
        "e2e": e2e,
        "gpu_launches": args.steps,
        "clocks": clk.summary(),
        "cpu_baseline": cpu,
        "sweep": sweep,
        "small": small,
        "decode": decode_line,
        "chunk": chunk_line,
        "module": module_line,
        "backward": backward_line,
        "peaked": peaked_line,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    if pg is not None:
        pg.destroy_process_group()


if __name__ == "__main__":
    main()
