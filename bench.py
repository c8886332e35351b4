#!/usr/bin/env python
"""MoE-layer throughput on B200: tokens/s and TFLOP/s against the roofline,
overlapped vs sequential.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]

One step = one pass of the whole layer (route, permute, grouped SwiGLU FFN,
combine) over one batch of synthetic tokens through moe_layer_forward.  The
default workload is the Mixtral-8x7B-shaped layer (T=4096, d=4096, E=8, top-2,
d_ff=14336).  Under torchrun with N > 1 every rank runs an independent replica
on its own GPU and token shard (the layer has no cross-token exchange), and the
job value is N*T tokens over the slowest rank's time (weak scaling).

--impl reference times the CPU oracle (plain C++) on the host cores, a bounded
token sample per step; it is a deliberately slow baseline, not a target.

Besides the benchmark line: --sweep times every cell of the d=4096/E=32 grid
(overlapped vs sequential per consumer-SM setting), and --oracle-timings times
the CPU oracle on each configuration; each prints one JSON line per case.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

from combine_overlap_b200 import synth  # noqa: E402

PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}

# ncu DRAM traffic (dram__bytes_read.sum + dram__bytes_write.sum) of one launch of
# the persistent FFN kernel, keyed by workload, valid only for the kernel sources
# whose hash is recorded with it (see profiles/).
TRAFFIC = {"mixtral": {"bytes": 4202588000 + 312804096, "kernel_hash": "dd7fc0020a58"}}


def kernel_source_hash() -> str:
    """Hash of the code (comments and whitespace removed) of the files that make
    and launch the persistent FFN kernel."""
    import re
    h = hashlib.sha1()
    for rel in ("combine_overlap_b200/csrc/ffn.cu", "combine_overlap_b200/csrc/common.cuh",
                "combine_overlap_b200/csrc/combine.cuh", "combine_overlap_b200/csrc/kernels.h",
                "combine_overlap_b200/csrc/api.cu"):
        with open(os.path.join(ROOT, rel), encoding="utf-8") as fh:
            src = fh.read()
        src = re.sub(r"/\*.*?\*/", " ", src, flags=re.S)   # block comments
        src = re.sub(r"//[^\n]*", " ", src)                 # line comments
        h.update(" ".join(src.split()).encode())
    return h.hexdigest()[:12]


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as fh:
            p = json.load(fh)
        return p, "measured"
    except (OSError, ValueError):
        return dict(PEAKS_FALLBACK), "fallback"


def parse():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--workload", default="mixtral", choices=sorted(synth.WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=("ours", "reference"))
    ap.add_argument("--consumer-sms", type=int, default=0, help="0 = cost model")
    ap.add_argument("--mgb", type=int, default=1)
    ap.add_argument("--no-join", action="store_true", help="producers do not join the combine")
    ap.add_argument("--one-cta", action="store_true", help="force 128-row tiles on single CTAs")
    ap.add_argument("--b-per-atom", action="store_true",
                    help="load weight tiles with one TMA copy per 64-column atom")
    ap.add_argument("--cta-pair", action="store_true", help="force 256-row tiles on CTA pairs")
    ap.add_argument("--wide-cta", action="store_true",
                    help="force 256-row tiles on single CTAs (two 128-row MMAs per K step)")
    ap.add_argument("--flags", default="0",
                    help="extra moe_layer_args.flags bits (e.g. 0x400 = MOE_SCHED_INTERLEAVE)")
    ap.add_argument("--cpu-seconds", type=float, default=10.0, help="CPU oracle baseline budget")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-clocks", action="store_true")
    ap.add_argument("--cool-down", type=float, default=0.5,
                    help="seconds the GPU idles before each timed region (same starting power state)")
    ap.add_argument("--sweep", action="store_true",
                    help="d=4096/E=32/top-4 sweep: T x router x consumer SMs, overlapped vs "
                         "sequential; one JSON line per cell (not the benchmark line)")
    ap.add_argument("--sweep-layers", default="",
                    help="comma-separated workloads for --sweep (default: the d=4096/E=32 grid)")
    ap.add_argument("--sweep-cells", default="seq,0,2,4,8,16",
                    help="--sweep cells: 'seq' or 'C[/mgb]' (overlapped, C consumer SMs, 0 = cost model)")
    ap.add_argument("--ep-sweep", action="store_true",
                    help="fused expert-parallel return on 2 and 4 virtual ranks: owners' step "
                         "overlapped vs sequential, and the homes' combine; one JSON line each")
    ap.add_argument("--oracle-timings", action="store_true",
                    help="time the CPU oracle on each benchmark configuration; one JSON line "
                         "per configuration (not the benchmark line)")
    return ap.parse_args()


# ----------------------------------------------------------------- clocks ---
class Clocks:
    """nvidia-smi samples of the SM clock, power and throttle reasons, every 50 ms,
    from before the warm-up to the end of the GPU work.  Each sample carries
    nvidia-smi's own wall-clock timestamp (its output reaches this process in
    bursts, so the time of arrival is not the time of the sample), and a timed
    region takes the samples whose timestamps fall inside its wall-clock window."""
    FIELDS = ("timestamp,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    REASONS = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")

    def __init__(self, device: int, enabled: bool = True, period_ms: int = 50):
        import threading
        self.proc = None
        self.samples = []          # (t_wall, sm_mhz, max_mhz, power_w, reasons)
        self.windows = {}
        if not enabled:
            return
        try:
            uuid = str(torch.cuda.get_device_properties(device).uuid)
            sel = uuid if uuid.startswith("GPU-") else f"GPU-{uuid}"
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", str(period_ms), "-i", sel], stdout=subprocess.PIPE,
                stderr=subprocess.DEVNULL, text=True)
        except (OSError, RuntimeError):
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()
        import atexit
        atexit.register(self.stop)   # never leave the sampler running after an error

    def _read(self):
        for line in self.proc.stdout:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm, smax = float(parts[1]), float(parts[2])
                ts = datetime.datetime.strptime(parts[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
            except ValueError:
                continue
            try:
                pw = float(parts[3])
            except ValueError:
                pw = None
            reasons = {n for n, v in zip(self.REASONS, parts[5:9]) if v.lower().startswith("active")}
            self.samples.append((ts, sm, smax, pw, reasons))

    def mark(self, name: str, t0: float, t1: float):
        """Record the wall-clock window [t0, t1] (time.time()) of a timed region."""
        self.windows[name] = (t0, t1)

    def stop(self):
        if self.proc is None or self.proc.returncode is not None:
            return
        time.sleep(0.2)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.thread.join(timeout=5)

    def summary(self, name: str | None = None, pad_s: float = 0.06):
        """Median SM clock, max clock and the throttle reasons seen, over the samples
        inside region `name` (widened by one sampling period on each side, so a region
        shorter than the period still gets its neighbours), or over every sample."""
        if name is not None and name in self.windows:
            t0, t1 = self.windows[name]
            sel = [s for s in self.samples if t0 - pad_s <= s[0] <= t1 + pad_s]
        else:
            sel = list(self.samples)
        if not sel:
            return None
        reasons = set()
        for s in sel:
            reasons |= s[4]
        pw = [s[3] for s in sel if s[3] is not None]
        return {"sm_mhz": statistics.median(s[1] for s in sel), "sm_max_mhz": max(s[2] for s in sel),
                "samples": len(sel), "power_w_max": max(pw) if pw else None,
                "reasons": sorted(reasons)}


# ------------------------------------------------------------ distributed ---
def dist_setup(n_gpus: int):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != n_gpus:
        raise SystemExit(f"--gpus {n_gpus} but WORLD_SIZE={world}: launch N>1 under torchrun")
    return world, rank, local


def shard_workload(wl: synth.Workload, rank: int) -> synth.Workload:
    """Rank r's token shard of a replicated layer: same shapes and expert weights
    (the weights keep wl's seed), its own tokens and gate logits."""
    if rank == 0:
        return wl
    return synth.Workload(wl.name, wl.T, wl.d, wl.f, wl.E, wl.k, wl.router, wl.seed + 1000 * rank)


def rank_inputs(wl: synth.Workload, rank: int, device="cpu"):
    """x, logits of rank r's token shard and the replicated expert weights."""
    shard = shard_workload(wl, rank)
    W1, W3, W2 = synth.make_weights(wl, device)
    return synth.make_x(shard, device), synth.make_logits(shard, device), W1, W3, W2


def max_over_ranks(values, world: int, device=None):
    """Element-wise max of a list of floats over all ranks (device-timed numbers:
    the job is as slow as its slowest rank)."""
    t = torch.tensor(list(values), dtype=torch.float64, device=device)
    if world > 1:
        import torch.distributed as dist
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def job_tokens_per_s(T: int, world: int, ms_per_step: float) -> float:
    """Whole-job throughput: every rank processes T tokens per step."""
    return T * world / (ms_per_step * 1e-3)


def flops_and_bytes(wl: synth.Workload, counts):
    """Algorithmic FLOPs (6 R d f, no masked rows) and minimum HBM bytes (active
    experts' weights + x + logits + out + routing indices) of one layer."""
    F = 6 * wl.R * wl.d * wl.f
    active = sum(1 for c in counts if c > 0)
    B = active * 3 * wl.d * wl.f * 2 + wl.T * wl.d * 2 * 2 + wl.T * wl.E * 4 + 16 * wl.R
    return F, B


# --------------------------------------------------------------- our arm ---
def run_ours(args):
    world, rank, local = dist_setup(args.gpus)
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=dev)
    from combine_overlap_b200 import moe

    wl = synth.WORKLOADS[args.workload]
    # each rank its own token shard; the same expert weights on every rank
    x, logits, W1, W3, W2 = rank_inputs(wl, rank, dev)
    ws = moe.alloc_workspace(wl.T, wl.d, wl.f, wl.E, wl.k, dev)
    out = torch.empty((wl.T, wl.d), dtype=torch.bfloat16, device=dev)
    kw = dict(consumer_sms=args.consumer_sms, mgb=args.mgb,
              flags=(moe.SCHED_NO_JOIN if args.no_join else 0) | (moe.SCHED_ONE_CTA if args.one_cta else 0)
              | (moe.SCHED_CTA_PAIR if args.cta_pair else 0)
              | (moe.SCHED_B_PER_ATOM if args.b_per_atom else 0)
              | (moe.SCHED_WIDE_CTA if args.wide_cta else 0) | int(args.flags, 0))

    def step(mode, evb=None, eve=None):
        moe.layer_forward(x, logits, W1, W3, W2, wl.k, ws, mode, out=out, ev_begin=evb, ev_end=eve, **kw)

    def barrier():
        if world > 1:
            torch.distributed.barrier()

    stream = torch.cuda.current_stream()
    # the clock sampler starts before the warm-up, so starting it costs the timed
    # regions nothing; each region marks its host-clock window
    clk = Clocks(local, not args.no_clocks)
    for _ in range(args.warmup):
        step(moe.MODE_OVERLAPPED)
        step(moe.MODE_SEQUENTIAL)
    torch.cuda.synchronize()
    code, consumer_sms, n_bands = moe.get_status(ws)
    if code != moe.MOE_OK:
        raise RuntimeError(f"warm-up: {moe.status_string(code)}")
    counts = moe.layer_forward(x, logits, W1, W3, W2, wl.k, ws, moe.MODE_OVERLAPPED, outputs=True,
                               **kw)[1]["counts"].cpu().tolist()

    def cool_down():
        # every timed region starts from the same power state: the part is capped at
        # 1 kW and lowers its clock after ~0.1 s of dense MMA work, so without a pause
        # a region would inherit the clock the previous regions left
        torch.cuda.synchronize()
        time.sleep(args.cool_down)

    def timed(mode, name, hooks=False):
        K = args.steps
        evb = [torch.cuda.Event(enable_timing=True) for _ in range(K)] if hooks else [None] * K
        eve = [torch.cuda.Event(enable_timing=True) for _ in range(K)] if hooks else [None] * K
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        cool_down()
        # a few untimed steps right before the region, so it starts in the steady
        # state rather than after the host-side pause above
        for _ in range(3):
            step(mode)
        barrier()
        torch.cuda.synchronize()
        h0 = time.time()
        e0.record(stream)
        for i in range(K):
            step(mode, evb[i], eve[i])
        e1.record(stream)
        torch.cuda.synchronize()
        clk.mark(name, h0, time.time())
        barrier()
        total = e0.elapsed_time(e1) / K
        ffn = sum(b.elapsed_time(e) for b, e in zip(evb, eve)) / K if hooks else None
        return total, ffn

    # The contract's timed region: K overlapped steps.  It runs without the
    # library's timing hooks: a recorded event between two launches costs them
    # their programmatic overlap.
    t_ovl, _ = timed(moe.MODE_OVERLAPPED, "contract")
    # The persistent FFN kernel's average launch duration, from K more overlapped
    # steps with the hooks (events recorded on the launching stream around it).
    t_ovl_hooked, ffn_ovl = timed(moe.MODE_OVERLAPPED, "hooked", hooks=True)
    # overlapped vs sequential: the two modes alternate step by step (paired
    # samples under the same clock and power state), each step timed with events
    # on the stream; medians per mode
    K = args.steps
    ev = {m: [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True),
               torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(K)] for m in ("seq", "ovl")}
    cool_down()
    barrier()
    torch.cuda.synchronize()
    h0 = time.time()
    for i in range(K):
        # alternate which mode goes first, so neither always follows the other
        order = (("seq", moe.MODE_SEQUENTIAL), ("ovl", moe.MODE_OVERLAPPED))
        for m, mode in (order if i % 2 == 0 else order[::-1]):
            e0, e1, fb, fe = ev[m][i]
            e0.record(stream)
            step(mode, fb, fe)
            e1.record(stream)
    torch.cuda.synchronize()
    clk.mark("paired", h0, time.time())
    barrier()
    step_ms = {m: [e0.elapsed_time(e1) for e0, e1, _, _ in ev[m]] for m in ev}
    ffn_ms = {m: [fb.elapsed_time(fe) for _, _, fb, fe in ev[m]] for m in ev}
    # the combine after the expert FFN: the full pass (sequential) or the remainder
    # pass (overlapped)
    post_ms = {m: [fe.elapsed_time(e1) for _, e1, _, fe in ev[m]] for m in ev}
    t_seq = statistics.median(step_ms["seq"])
    ffn_seq = statistics.median(ffn_ms["seq"])
    t_ovl_med = statistics.median(step_ms["ovl"])
    ffn_ovl_med = statistics.median(ffn_ms["ovl"])
    post_seq = statistics.median(post_ms["seq"])
    post_ovl = statistics.median(post_ms["ovl"])

    # The same overlapped call captured once in a CUDA graph and replayed K times.
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        step(moe.MODE_OVERLAPPED)
    cool_down()
    for _ in range(max(3, args.warmup)):
        g.replay()
    barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    h0 = time.time()
    e0.record(stream)
    for _ in range(args.steps):
        g.replay()
    e1.record(stream)
    torch.cuda.synchronize()
    clk.mark("graph", h0, time.time())
    barrier()
    t_graph = e0.elapsed_time(e1) / args.steps
    del g

    # End to end through the public call: every step copies its inputs (x, logits)
    # from pinned host memory and reads its output back to pinned host memory.
    # Device buffers are double-buffered and the copies run on a second stream,
    # so step i's copies overlap steps i-1 and i+1's compute (as a serving loop
    # would); the timed region runs from the first H2D to the last D2H.
    x_h = x.cpu().pin_memory()
    l_h = logits.cpu().pin_memory()
    out_h = [torch.empty(out.shape, dtype=out.dtype).pin_memory() for _ in range(2)]
    x_d = [torch.empty_like(x) for _ in range(2)]
    l_d = [torch.empty_like(logits) for _ in range(2)]
    o_d = [torch.empty_like(out) for _ in range(2)]
    h2d, d2h = torch.cuda.Stream(), torch.cuda.Stream()
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]
    ev_d2h = [torch.cuda.Event() for _ in range(2)]

    def e2e_steps(n):
        # H2D on one stream, D2H on another: step i+1's inputs upload while step i
        # computes, and step i's output downloads while step i+1 computes.
        for i in range(n):
            b = i & 1
            with torch.cuda.stream(h2d):
                if i >= 2:
                    h2d.wait_event(ev_out[b])          # step i-2 has consumed x_d[b]
                x_d[b].copy_(x_h, non_blocking=True)
                l_d[b].copy_(l_h, non_blocking=True)
                ev_in[b].record(h2d)
            stream.wait_event(ev_in[b])
            if i >= 2:
                stream.wait_event(ev_d2h[b])           # step i-2's output is downloaded
            moe.layer_forward(x_d[b], l_d[b], W1, W3, W2, wl.k, ws, moe.MODE_OVERLAPPED, out=o_d[b], **kw)
            ev_out[b].record(stream)
            with torch.cuda.stream(d2h):
                d2h.wait_event(ev_out[b])
                out_h[b].copy_(o_d[b], non_blocking=True)
                ev_d2h[b].record(d2h)
        stream.wait_stream(d2h)

    cool_down()
    e2e_steps(max(2, args.warmup))
    barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    h0 = time.time()
    e0.record(stream)
    h2d.wait_event(e0)
    e2e_steps(args.steps)
    e1.record(stream)
    torch.cuda.synchronize()
    clk.mark("e2e", h0, time.time())
    barrier()
    t_e2e = e0.elapsed_time(e1) / args.steps
    clk.stop()
    clocks = clk.summary("contract")
    clocks_by_region = {n: clk.summary(n) for n in ("contract", "hooked", "paired", "graph", "e2e")}
    clocks_run = clk.summary()
    if not torch.equal(out_h[(args.steps - 1) & 1].to(out.device), out):
        raise RuntimeError("end-to-end output differs from the device-resident run")
    code, _, _ = moe.get_status(ws)
    if code != moe.MOE_OK:
        raise RuntimeError(f"timed runs: {moe.status_string(code)}")
    # one more overlapped call, untimed: how many tokens the persistent kernel
    # combined itself (the combine pass after it did the rest)
    step(moe.MODE_OVERLAPPED)
    in_kernel = moe.debug_tokens_combined(ws, wl.T, wl.d, wl.f, wl.E, wl.k, stream)

    (t_ovl, t_seq, ffn_ovl, ffn_seq, t_e2e, t_ovl_med, ffn_ovl_med, post_seq, post_ovl,
     t_graph, t_ovl_hooked) = max_over_ranks([t_ovl, t_seq, ffn_ovl, ffn_seq, t_e2e, t_ovl_med,
                                              ffn_ovl_med, post_seq, post_ovl, t_graph,
                                              t_ovl_hooked], world, dev)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(wl, x, logits, W1, W3, W2, args.cpu_seconds)

    if rank == 0:
        peaks, src = load_peaks()
        F, B = flops_and_bytes(wl, counts)
        # the FFN launch and the layer step last milliseconds: the burst cuBLAS
        # figure is their peak (the sustained one, under the power cap after
        # seconds of back-to-back GEMMs, is reported beside it)
        peak_tf = peaks["bf16_tflops"]
        peak_tf_sus = peaks.get("bf16_tflops_sustained")
        hbm = peaks["hbm_gbs"]
        t_roof_ms = max(F / (peak_tf * 1e12), B / (hbm * 1e9)) * 1e3
        ach = F / (ffn_ovl * 1e-3) / 1e12
        h = kernel_source_hash()
        tr = TRAFFIC.get(wl.name)
        traffic = tr["bytes"] if tr and tr.get("kernel_hash") == h else None
        T_all = wl.T * world
        res = {
            "metric": "MoE-layer tokens/s",
            "value": job_tokens_per_s(wl.T, world, t_ovl),
            "unit": "tokens/s",
            "n_gpus": world,
            "steps": args.steps,
            "warmup": args.warmup,
            "ms_per_step": t_ovl,
            "higher_is_better": True,
            "scaling": "weak",
            "vs_baseline": None,
            "dtype": "bf16",
            "data": "synthetic: seeded counter-based N(0,1) tokens and gate logits, random-init N(0,0.02) bf16 expert weights",
            "config": {"workload": wl.name, "T": wl.T, "d_model": wl.d, "d_ff": wl.f, "E": wl.E,
                       "top_k": wl.k, "router": wl.router, "mode": "overlapped",
                       "mma_tile": moe.TILE_VARIANTS[moe.tile_variant(wl.T, wl.f, wl.E, wl.k,
                                                                      kw["flags"])],
                       "parallelism": f"replicas x{world} (token shards, no collective)",
                       "l2": "inputs larger than L2: active expert weights %.2f GB per step" % (B / 1e9)},
            "tflops": world * F / (t_ovl * 1e-3) / 1e12,
            "roofline_frac_layer": t_roof_ms / t_ovl,
            "roofline_layer": {"bound": "tensor" if F / (peak_tf * 1e12) >= B / (hbm * 1e9) else "hbm",
                               "time_ms": t_roof_ms, "flops": F, "min_bytes": B,
                               "peak_tflops": peak_tf, "peak_hbm_gbs": hbm,
                               "peaks": f"{src} (bf16 burst, HBM copy)",
                               "frac_vs_sustained_peak": (max(F / (peak_tf_sus * 1e12), B / (hbm * 1e9)) * 1e3
                                                          / t_ovl) if peak_tf_sus else None},
            "sequential": {"value": T_all / (t_seq * 1e-3), "ms_per_step": t_seq,
                           "ffn_ms": ffn_seq, "tflops": world * F / (t_seq * 1e-3) / 1e12,
                           "overlapped_ms_per_step": t_ovl_med, "overlapped_ffn_ms": ffn_ovl_med,
                           "method": "K steps of each mode, alternating step by step; medians"},
            "speedup_vs_sequential": t_seq / t_ovl_med,
            # Overlap accounting from the paired steps (medians):
            #   producer only = the sequential mode's GEMM1 and GEMM2 launches,
            #   combine only  = the sequential mode's combine pass,
            #   overlapped    = the overlapped mode's persistent launch + remainder pass;
            #   ratio = 1 - (overlapped - producer only) / combine only  (1: the combine
            #   is fully hidden; above 1: the single launch also saves the GEMM1 -> GEMM2
            #   launch boundary); op_speedup = (producer only + combine only) / overlapped.
            "overlap": {"producer_only_ms": ffn_seq, "combine_only_ms": post_seq,
                        "overlapped_ms": ffn_ovl_med + post_ovl, "remainder_combine_ms": post_ovl,
                        "ratio": 1.0 - (ffn_ovl_med + post_ovl - ffn_seq) / post_seq,
                        "op_speedup": (ffn_seq + post_seq) / (ffn_ovl_med + post_ovl),
                        "tokens_combined_in_kernel": in_kernel,
                        "tokens": wl.T},
            "graph": {"ms_per_step": t_graph, "eager_ms_per_step": t_ovl,
                      "method": "the overlapped call captured once in a CUDA graph, K replays"},
            "consumer_sms": consumer_sms,
            "n_bands": n_bands,
            "masked_row_waste": (n_bands * 128 - wl.R) / (n_bands * 128),
            "roofline": {"kernel": "ffn_kernel (persistent GEMM1+GEMM2+combine)", "bound": "tensor",
                         "achieved": ach, "peak": peak_tf, "unit": "TFLOP/s", "frac": ach / peak_tf,
                         "traffic": traffic, "launch_ms": ffn_ovl,
                         "launch_timing": "CUDA events on the launching stream around the "
                                          "persistent kernel, K overlapped steps after the "
                                          "contract region (%.4f ms per step there)" % t_ovl_hooked,
                         "peak_kind": f"{src} burst bf16 (cuBLAS 8192^3, best of 10): the kernel is "
                                      "a ms-long launch",
                         "frac_vs_sustained_peak": ach / peak_tf_sus if peak_tf_sus else None},
            "e2e": {"value": job_tokens_per_s(wl.T, world, t_e2e), "unit": "tokens/s", "ms_per_step": t_e2e,
                    "h2d_bytes_per_step": x.numel() * 2 + logits.numel() * 4,
                    "d2h_bytes_per_step": out.numel() * 2,
                    "method": "pinned host buffers; double-buffered device buffers; H2D and D2H on their own streams, overlapping the neighbouring steps' compute"},
            "gpu_launches": 6 * args.steps,   # route, plan, scatter, gather, persistent FFN, combine
            "clocks": clocks,
            "clocks_by_region": clocks_by_region,
            "clocks_whole_run": clocks_run,
            "kernel_hash": h,
        }
        if cpu is not None:
            res["cpu_baseline"] = cpu
        print(json.dumps(res), flush=True)
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()


# ------------------------------------------------------------ CPU oracle ---
def _oracle_tokens_per_s(o, xh, idx, gate, W, n, T, seed):
    import numpy as np
    rng = np.random.default_rng(seed)
    toks = rng.choice(T, size=min(n, T), replace=False).astype(np.int32)
    t0 = time.perf_counter()
    o.tokens(xh, idx, gate, W[0], W[1], W[2], toks)
    return len(toks), time.perf_counter() - t0


def _host_inputs(wl, x, logits, W1, W3, W2):
    import oracle
    o = oracle.get()
    threads = o.set_threads(os.cpu_count() or 1)
    xh = synth.bf16_bits(x)
    lh = logits.detach().cpu().numpy()
    W = [synth.bf16_bits(w) for w in (W1, W3, W2)]
    idx, gate = o.route(lh, wl.k)
    return o, threads, xh, idx, gate, W


def cpu_baseline(wl, x, logits, W1, W3, W2, seconds):
    """The oracle, as it stands, on a bounded token sample of the same workload."""
    o, threads, xh, idx, gate, W = _host_inputs(wl, x, logits, W1, W3, W2)
    n0 = max(threads, 4)
    n, dt = _oracle_tokens_per_s(o, xh, idx, gate, W, n0, wl.T, 1)
    n = int(min(wl.T, max(n0, n * seconds / max(dt, 1e-6))))
    n, dt = _oracle_tokens_per_s(o, xh, idx, gate, W, n, wl.T, 2)
    return {"value": n / dt, "unit": "tokens/s", "cores": threads, "kind": "oracle",
            "sample": f"{n} of {wl.T} tokens (routing in full), token-by-token oracle path, {dt:.1f} s"}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if rank != 0:
        return
    wl = synth.WORKLOADS[args.workload]
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    inp = synth.make_inputs(wl, dev)
    o, threads, xh, idx, gate, W = _host_inputs(wl, inp["x"], inp["logits"], inp["W1"], inp["W3"], inp["W2"])
    del inp
    if dev == "cuda":
        torch.cuda.empty_cache()
    # size each step to ~3 s of oracle work
    n, dt = _oracle_tokens_per_s(o, xh, idx, gate, W, max(threads, 4), wl.T, 0)
    n = int(min(wl.T, max(threads, n * 3.0 / max(dt, 1e-6))))
    for i in range(args.warmup):
        _oracle_tokens_per_s(o, xh, idx, gate, W, max(threads, 4), wl.T, 100 + i)
    tot_n, tot_t = 0, 0.0
    for i in range(args.steps):
        m, t = _oracle_tokens_per_s(o, xh, idx, gate, W, n, wl.T, 1000 + i)
        tot_n += m
        tot_t += t
    v = tot_n / tot_t
    sample = f"{n} of {wl.T} tokens per step, token-by-token oracle path, {threads} threads"
    res = {
        "impl": "reference",
        "metric": "MoE-layer tokens/s", "value": v, "unit": "tokens/s", "n_gpus": world,
        # a step is the timed token sample, not the whole layer (which would take
        # layer_ms_extrapolated below)
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": tot_t / args.steps * 1e3,
        "tokens_per_step": tot_n / args.steps,
        "layer_ms_extrapolated": wl.T / v * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic: seeded counter-based inputs, random-init weights",
        "config": {"workload": wl.name, "T": wl.T, "d_model": wl.d, "d_ff": wl.f, "E": wl.E,
                   "top_k": wl.k, "router": wl.router, "mode": "cpu oracle",
                   "parallelism": "host cores"},
        "cpu_baseline": {"value": v, "unit": "tokens/s", "cores": threads, "kind": "oracle", "sample": sample},
        "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(res), flush=True)


def _cpu_model():
    try:
        with open("/proc/cpuinfo") as fh:
            for line in fh:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def run_oracle_timings(args):
    """The CPU oracle's own speed on each benchmark configuration, as it stands:
    single-threaded on the tiny layer (whole layer, permuted path) and on the T=512
    sweep layer; on every host thread for the Mixtral-shaped, fine-grained and
    imbalanced layers.  Beyond the tiny layer a token sample of about
    `--cpu-seconds` of work is timed through the token-by-token definition path and
    the whole layer is extrapolated from it (marked so)."""
    import oracle
    o = oracle.get()
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    nproc = os.cpu_count() or 1
    cpu = _cpu_model()
    for name, threads in (("tiny", 1), ("sweep_T512_uniform", 1), ("mixtral", nproc),
                          ("fine_grained", nproc), ("imbalanced", nproc)):
        wl = synth.WORKLOADS[name]
        inp = synth.make_inputs(wl, dev)
        xh = synth.bf16_bits(inp["x"])
        lh = inp["logits"].detach().cpu().numpy()
        W = [synth.bf16_bits(inp[n]) for n in ("W1", "W3", "W2")]
        del inp
        used = o.set_threads(threads)
        if name == "tiny":
            t0 = time.perf_counter()
            o.forward(xh, lh, W[0], W[1], W[2], wl.k)
            dt = time.perf_counter() - t0
            n, extrap = wl.T, False
        else:
            idx, gate = o.route(lh, wl.k)
            n, dt = _oracle_tokens_per_s(o, xh, idx, gate, W, max(used, 2), wl.T, 1)
            n = int(min(wl.T, max(used, n * args.cpu_seconds / max(dt, 1e-6))))
            n, dt = _oracle_tokens_per_s(o, xh, idx, gate, W, n, wl.T, 2)
            extrap = n < wl.T
        tps = n / dt
        print(json.dumps({"oracle_timing": name, "threads": used, "nproc": nproc, "cpu": cpu,
                          "tokens_timed": n, "seconds": dt, "tokens_per_s": tps,
                          "layer_seconds": wl.T / tps, "extrapolated": extrap,
                          "path": "whole layer (permuted)" if name == "tiny"
                          else "token-by-token definition path"}), flush=True)


def _sweep_cells(spec: str):
    """Cells of a paired sweep: "seq[+flags]" (sequential mode) or "C[/mgb][+flags]"
    (overlapped mode, C consumer SMs, 0 = the cost model; mgb row bands per consumer
    item; flags = extra moe_layer_args.flags bits, e.g. +0x400)."""
    cells = []
    for tok in spec.split(","):
        tok = tok.strip()
        body, _, fl = tok.partition("+")
        flags = int(fl, 0) if fl else 0
        if body == "seq":
            cells.append((tok, None, 0, 1, flags))
        else:
            c, _, m = body.partition("/")
            cells.append((tok, "ovl", int(c), int(m) if m else 1, flags))
    return cells


def run_sweep(args):
    """Paired sweep of layers x cells.  Per layer, every cell (the sequential mode,
    the overlapped mode at the cost model's split, at fixed consumer-SM counts, or at
    other segment sizes mgb) runs once per round, the order rotated from round to
    round, each step timed with CUDA events on the stream; medians per cell.  So the
    cells of a layer see the same clock and power history, and none always runs
    first.  One JSON line per layer, with the clocks sampled during it."""
    from combine_overlap_b200 import moe
    torch.cuda.set_device(0)
    peaks, src = load_peaks()
    peak_tf = peaks["bf16_tflops"]
    names = args.sweep_layers.split(",") if args.sweep_layers else \
        [n for n in synth.WORKLOADS if n.startswith("sweep_")]
    cells = _sweep_cells(args.sweep_cells)
    clk = Clocks(0, not args.no_clocks)
    for name in names:
        wl = synth.WORKLOADS[name]
        x, logits, W1, W3, W2 = rank_inputs(wl, 0, "cuda")
        ws = moe.alloc_workspace(wl.T, wl.d, wl.f, wl.E, wl.k)
        out = torch.empty((wl.T, wl.d), dtype=torch.bfloat16, device="cuda")
        counts = moe.layer_forward(x, logits, W1, W3, W2, wl.k, ws, outputs=True)[1]["counts"].cpu().tolist()
        F, B = flops_and_bytes(wl, counts)
        t_roof = max(F / (peak_tf * 1e12), B / (peaks["hbm_gbs"] * 1e9)) * 1e3

        def step(cell):
            _, mode, C, mgb, fl = cell
            m = moe.MODE_SEQUENTIAL if mode is None else moe.MODE_OVERLAPPED
            moe.layer_forward(x, logits, W1, W3, W2, wl.k, ws, m, out=out, consumer_sms=C, mgb=mgb,
                              flags=fl)

        used = {}
        for cell in cells:
            for _ in range(max(1, args.warmup)):
                step(cell)
            if cell[1] is not None:
                torch.cuda.synchronize()
                code, c_used, _ = moe.get_status(ws)
                if code != moe.MOE_OK:
                    raise RuntimeError(f"{name} {cell[0]}: {moe.status_string(code)}")
                used[cell[0]] = c_used
        evs = {c[0]: [] for c in cells}
        torch.cuda.synchronize()
        h0 = time.time()
        n = len(cells)
        for i in range(args.steps):
            for j in range(n):
                cell = cells[(i + j) % n]
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record()
                step(cell)
                e1.record()
                evs[cell[0]].append((e0, e1))
        torch.cuda.synchronize()
        clk.mark(name, h0, time.time())
        code, _, _ = moe.get_status(ws)
        if code != moe.MOE_OK:
            raise RuntimeError(f"{name}: {moe.status_string(code)}")
        # per overlapped cell, one more untimed call: tokens the persistent kernel
        # combined itself
        in_kernel = {}
        for cell in cells:
            if cell[1] is not None:
                step(cell)
                in_kernel[cell[0]] = moe.debug_tokens_combined(ws, wl.T, wl.d, wl.f, wl.E, wl.k)
        ms = {c: sorted(a.elapsed_time(b) for a, b in v) for c, v in evs.items()}
        med = {c: statistics.median(v) for c, v in ms.items()}
        q = {c: (v[len(v) // 4], v[(3 * len(v)) // 4]) for c, v in ms.items()}
        res = {"sweep": name, "T": wl.T, "router": wl.router, "steps": args.steps,
               "mma_tile": moe.TILE_VARIANTS[moe.tile_variant(wl.T, wl.f, wl.E, wl.k)],
               "roofline_ms": t_roof, "flops": F, "min_bytes": B,
               "roofline_bound": "tensor" if F / (peak_tf * 1e12) >= B / (peaks["hbm_gbs"] * 1e9) else "hbm",
               "peaks": f"{src}: bf16 burst {peak_tf} TFLOP/s, HBM {peaks['hbm_gbs']} GB/s",
               "cells": {}}
        for c in ms:
            cell = {"ms": med[c], "q25_ms": q[c][0], "q75_ms": q[c][1],
                    "tokens_per_s": wl.T / (med[c] * 1e-3), "tflops": F / (med[c] * 1e-3) / 1e12,
                    "roofline_frac": t_roof / med[c]}
            if c in used:
                cell["consumer_sms_used"] = used[c]
            if c in in_kernel:
                cell["tokens_combined_in_kernel"] = in_kernel[c]
            if "seq" in med and c != "seq":
                cell["speedup_vs_sequential"] = med["seq"] / med[c]
            base = cells[0][0]
            if c != base:
                cell[f"ratio_vs_{base}"] = med[base] / med[c]
            res["cells"][c] = cell
        res["clocks"] = clk.summary(name)
        print(json.dumps(res), flush=True)
        del x, logits, W1, W3, W2, ws, out
        torch.cuda.empty_cache()
    clk.stop()


def run_ep_sweep(args):
    """The fused expert-parallel return on W virtual ranks of one GPU: per layer and
    W, the owners' step (moe_ep_owner_forward: expert GEMMs plus the return of every
    row band into its home rank's buffer) in the overlapped mode (consumer CTAs
    return bands while the GEMM runs) against the sequential mode (GEMMs, then the
    return as its own pass), and the homes' combine.  Each owner's two modes run as
    paired steps, the order alternating, each timed with CUDA events; medians,
    summed over the owners.  One JSON line per (layer, W)."""
    from combine_overlap_b200 import ep, moe
    torch.cuda.set_device(0)
    names = args.sweep_layers.split(",") if args.sweep_layers else ["sweep_T8192_uniform", "mixtral"]
    for name in names:
        wl = synth.WORKLOADS[name]
        for W in (2, 4):
            if wl.E % W:
                continue
            T_r = wl.T // W
            shards = [synth.Workload(f"{name}_r{r}", T_r, wl.d, wl.f, wl.E, wl.k, wl.router,
                                     wl.seed + 1000 * r) for r in range(W)]
            xs = [synth.make_x(sw, "cuda") for sw in shards]
            ls = [synth.make_logits(sw, "cuda") for sw in shards]
            W1, W3, W2 = synth.make_weights(wl, "cuda")
            outs, st = ep.virtual_ranks_forward(xs, ls, W1, W3, W2, wl.k)
            torch.cuda.synchronize()
            El = wl.E // W
            homes = st["homes"]
            t_ovl, t_seq, t_home = 0.0, 0.0, 0.0
            for o, own in enumerate(st["owners"]):
                if own["N"] == 0:
                    continue
                lo, hi = o * El, (o + 1) * El
                base = [int(h["offsets"][lo].item()) for h in homes]

                def owner(mode):
                    moe.ep_owner_forward(own["x_recv"], own["slot_recv"], own["recv_counts"], W1[lo:hi],
                                         W3[lo:hi], W2[lo:hi], wl.k, o, base, [h["y"] for h in homes],
                                         [h["arrive"] for h in homes], own["ws"], mode)
                ev = {m: [] for m in ("ovl", "seq")}
                for _ in range(max(1, args.warmup)):
                    owner(moe.MODE_OVERLAPPED)
                    owner(moe.MODE_SEQUENTIAL)
                torch.cuda.synchronize()
                for i in range(args.steps):
                    order = (("ovl", moe.MODE_OVERLAPPED), ("seq", moe.MODE_SEQUENTIAL))
                    for m, mode in (order if i % 2 == 0 else order[::-1]):
                        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                        e0.record()
                        owner(mode)
                        e1.record()
                        ev[m].append((e0, e1))
                torch.cuda.synchronize()
                code, c_used, nb = moe.get_status(own["ws"])
                if code != moe.MOE_OK:
                    raise RuntimeError(f"owner {o}: {moe.status_string(code)}")
                t_ovl += statistics.median(a.elapsed_time(b) for a, b in ev["ovl"])
                t_seq += statistics.median(a.elapsed_time(b) for a, b in ev["seq"])
            # every owner ran its steps: each token's arrival word is now a multiple
            # of k; one home combine per rank consumes the last round of rows
            for h in homes:
                h["arrive"].fill_(wl.k)
            torch.cuda.synchronize()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            for h in homes:
                moe.ep_home_combine(h["y"], h["arrive"], h["row_of"], h["gate"])
            e1.record()
            torch.cuda.synchronize()
            t_home = e0.elapsed_time(e1)
            ret_bytes = 2 * wl.T * wl.k * wl.d * 2
            print(json.dumps({"ep_sweep": name, "W": W, "tokens_per_rank": T_r, "steps": args.steps,
                              "owners_overlapped_ms": t_ovl, "owners_sequential_ms": t_seq,
                              "speedup_vs_sequential": t_seq / t_ovl, "homes_combine_ms": t_home,
                              "return_bytes": ret_bytes,
                              "method": "per owner: overlapped and sequential steps alternating, "
                                        "CUDA events, medians; summed over owners (run one after "
                                        "another on one GPU)"}), flush=True)
            del xs, ls, W1, W3, W2, outs, st
            torch.cuda.empty_cache()


def main():
    args = parse()
    if args.sweep:
        run_sweep(args)
        return
    if args.ep_sweep:
        run_ep_sweep(args)
        return
    if args.oracle_timings:
        run_oracle_timings(args)
        return
    if args.steps < 1 or args.warmup < 0:
        raise SystemExit("--steps must be >= 1 and --warmup >= 0")
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
