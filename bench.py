"""Benchmark of the Parallax attention hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

One step is one pass of the hot path over one batch: a decode call (single
pass over the KV cache plus the split combine, one kernel launch) for the
decode workloads, a causal prefill call for ``prefill``.  The default
workload is decode_bf16: batch 8, 16 query / 8 KV heads, head_dim 128, KV
length 4096, bf16 cache.

Timing: W untimed warm-up steps, then exactly K steps between a barrier plus
torch.cuda.synchronize() on both sides, timed with CUDA events on the stream
the kernels run on; the max over ranks is reported.  Decode steps run as
CUDA-graph replays (the library's kernels, captured once) so host launch cost
does not hide the device time; every step reads a different copy of the KV
cache, the copies totalling more than the 126 MB L2.  The ``e2e`` figure
goes through the public Python API call by call, with the step's query and
probe copied from pinned host memory and the output read back every step.

Multi-GPU (torchrun, one process per GPU): every rank runs its own copy of
the workload (independent sequences, no collective on the data path), so
scaling is weak and ``value`` is the total over ranks divided by the slowest
rank's time.

The default run (decode_bf16) then times every other workload the same way
(``per_config`` in the JSON line: decode_f32, decode_long, decode_paged,
prefill, prefill_paged, prefill_train, decode_projected), each with its
roofline against the measured and the nominal peak, its clocks and its
oracle baseline; ``--no-per-config`` skips them.

``--impl reference`` times the float64 CPU oracle on the host cores instead
(rank 0 only), on a bounded sample of the same workload per step.
"""

from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import torch  # noqa: E402

from parallax_local_linear_b200 import workloads as W  # noqa: E402

METRIC = "decode KV GB/s & tokens/s (% of HBM peak); prefill TFLOP/s (% of bf16 peak)"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
KERNEL_SOURCES = {
    "decode": ["parallax_local_linear_b200/csrc/decode.cuh", "parallax_local_linear_b200/csrc/ptx.cuh"],
    "prefill": ["parallax_local_linear_b200/csrc/prefill.cuh", "parallax_local_linear_b200/csrc/ptx.cuh"],
    "prefill_pair": ["parallax_local_linear_b200/csrc/prefill2.cuh", "parallax_local_linear_b200/csrc/prefill.cuh",
                     "parallax_local_linear_b200/csrc/ptx.cuh"],
    "prefill_paged": ["parallax_local_linear_b200/csrc/prefill.cuh", "parallax_local_linear_b200/csrc/ptx.cuh"],
    "prefill_bwd": ["parallax_local_linear_b200/csrc/prefill_bwd.cuh", "parallax_local_linear_b200/csrc/prefill.cuh",
                    "parallax_local_linear_b200/csrc/ptx.cuh"],
    "decode_projected": ["parallax_local_linear_b200/csrc/project.cuh", "parallax_local_linear_b200/csrc/decode.cuh",
                         "parallax_local_linear_b200/csrc/ptx.cuh"],
    "lla": ["parallax_local_linear_b200/csrc/lla.cuh", "parallax_local_linear_b200/csrc/prefill.cuh",
            "parallax_local_linear_b200/csrc/ptx.cuh"],
}
KV_COPIES = 4          # decode_bf16: 4 x 128 MiB of KV, more than L2
L2_SWEEP_BYTES = 128 << 20   # at least the 126 MB L2
GRAPH_STEPS = 64       # decode calls per captured graph


# ---------------------------------------------------------------- helpers

def parse_args(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None)
    ap.add_argument("--warmup", type=int, default=None)
    ap.add_argument("--workload", default="decode_bf16", choices=sorted(W.WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--num-ctas", type=int, default=0)
    ap.add_argument("--batch", type=int, default=0,
                    help="override the workload's batch (smaller cases for profiling)")
    ap.add_argument("--cta-pair", action="store_true",
                    help="prefill workloads: run the two-SM (cta_group::2) dense prefill kernel")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=12.0,
                    help="target CPU time of the oracle baseline sample")
    ap.add_argument("--cpu-seconds-per-config", type=float, default=4.0,
                    help="target CPU time of each other workload's oracle baseline sample")
    ap.add_argument("--no-per-config", dest="per_config", action="store_false",
                    help="time only --workload (by default the decode_bf16 run also times every other workload)")
    return ap.parse_args(argv)


def default_steps(workload):
    return {"decode_f32": 20000, "decode_bf16": 8192, "decode_projected": 8192, "lla_decode": 2048, "decode_long": 200,
            "decode_paged": 200, "prefill": 20, "prefill_paged": 20, "prefill_train": 10}[workload]


def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


def source_sha(kind):
    h = hashlib.sha256()
    for rel in KERNEL_SOURCES[kind]:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def profiled_traffic(kind, workload):
    """DRAM bytes per launch from the committed ncu summary, if it was taken
    on the current kernel source.  Returns (bytes or None, provenance)."""
    rel = os.path.join("profiles", f"{kind}-{workload}.md")
    path = os.path.join(ROOT, rel)
    if not os.path.exists(path):
        return None, f"no ncu summary at {rel}"
    fields = {}
    with open(path) as f:
        for line in f:
            if ":" in line and line.startswith("- "):
                k, v = line[2:].split(":", 1)
                fields[k.strip()] = v.strip().strip("`")
    sha = source_sha(kind)
    if fields.get("source_sha256") != sha:
        return None, (f"{rel} was captured on kernel source {fields.get('source_sha256')}, "
                      f"not the current {sha}: no counters for this source")
    try:
        return float(fields["dram_bytes_per_launch"]), (
            f"read from {rel} (ncu dram__bytes_read.sum + dram__bytes_write.sum, kernel source {sha}); "
            "not measured in this run")
    except (KeyError, ValueError):
        return None, f"{rel} holds no dram_bytes_per_launch"


def traffic_fields(kind, workload):
    t, src = profiled_traffic(kind, workload)
    return {"traffic": t, "traffic_source": src}


class ClockSampler:
    """Samples SM clock and throttle reasons through NVML while running."""

    REASONS = {
        0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
        0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
    }

    def __init__(self, device_index, period=0.005):
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self.period = period
        self._stop = threading.Event()
        self._thr = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception:   # NVML missing: report no clocks rather than guess
            self.nv = None

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
                bits = self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                for b, name in self.REASONS.items():
                    if bits & b and b != 0x1:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.nv is not None:
            self._thr = threading.Thread(target=self._run, daemon=True)
            self._thr.start()
        return self

    def __exit__(self, *exc):
        if self._thr is not None:
            self._stop.set()
            self._thr.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                    "samples": 0}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


class _F64View:
    """float64 numpy slices of a (device) tensor, copied on indexing."""

    def __init__(self, t):
        self.t = t
        self.shape = tuple(t.shape)

    def __getitem__(self, idx):
        return self.t[idx].double().cpu().numpy()


def reduce_over_ranks(ms, total, device, world):
    """Max of the per-rank times and sum of the per-rank work, over all ranks.

    Every rank calls this with the same arguments shape (a collective);
    world == 1 returns the inputs unchanged."""
    if world == 1:
        return float(ms), float(total)
    t = torch.tensor([float(ms), float(total)], dtype=torch.float64, device=device)
    tmax = t[:1].clone()
    tsum = t[1:].clone()
    torch.distributed.all_reduce(tmax, op=torch.distributed.ReduceOp.MAX)
    torch.distributed.all_reduce(tsum, op=torch.distributed.ReduceOp.SUM)
    return float(tmax[0]), float(tsum[0])


def blas_threads():
    try:
        import threadpoolctl
        info = threadpoolctl.threadpool_info()
        n = [i["num_threads"] for i in info if i.get("user_api") == "blas"]
        if n:
            return max(n)
    except Exception:
        pass
    return os.cpu_count()


# ------------------------------------------------------------------ decode

def decode_config(w, args, ctas):
    cfg = {"workload": w.name, "batch": w.batch, "num_q_heads": w.num_q_heads,
           "num_kv_heads": w.num_kv_heads, "head_dim": w.head_dim, "kv_len": w.kv_len,
           "kv_dtype": w.dtype, "paged": w.paged, "num_ctas": ctas}
    if w.paged:
        cfg["seq_lens"] = f"uniform in [{w.min_len}, {w.kv_len}], 64-token pages, seeded permutation"
    if w.key_offset_std:
        cfg["key_offset_std"] = w.key_offset_std
    return cfg


def bench_decode(args, w, rank, world, dev, peaks, peaks_kind):
    from parallax_local_linear_b200 import binding as px

    copies = KV_COPIES if w.name in ("decode_bf16", "decode_f32") else 1
    if w.name == "decode_f32":
        # one call's KV (128 KiB) is far below L2: enough copies that one pass
        # over them is twice its size, each graph replay visiting every copy once
        copies = max(copies, -(-2 * L2_SWEEP_BYTES // W.kv_bytes(w, None)))
    insts = [W.decode_inputs(w, device=dev, seed=w.seed + 1000 * rank + i) for i in range(copies)]
    lens = [None if x["seq_lens"] is None else x["seq_lens"].cpu().numpy() for x in insts]
    bytes_per_step = [W.kv_bytes(w, l) for l in lens]
    outs = [torch.empty_like(x["q"]) for x in insts]
    out_dtype = insts[0]["q"].dtype

    def step(i):
        x = insts[i % copies]
        px.decode(x["q"], x["rho"], x["k_cache"], x["v_cache"], x["scale"], seq_lens=x["seq_lens"],
                  page_table=x["page_table"], out=outs[i % copies], out_dtype=out_dtype,
                  num_ctas=args.num_ctas)

    p = px.decode_params(insts[0]["q"], insts[0]["k_cache"], page_table=insts[0]["page_table"],
                         num_ctas=args.num_ctas)
    ctas = px.decode_num_ctas(p)
    stream = torch.cuda.current_stream()

    # warm-up (also initialises the library and the workspace before capture)
    for i in range(max(args.warmup, 3)):
        step(i)
    torch.cuda.synchronize()
    assert px.last_device_error() == 0, "device error during warm-up"

    K = args.steps
    graphs = []
    if w.name in ("decode_bf16", "decode_f32"):
        g = torch.cuda.CUDAGraph()
        n = min(max(GRAPH_STEPS, copies), K)
        with torch.cuda.graph(g):
            for i in range(n):
                step(i)
        rem = K % n
        gr = None
        if rem:
            gr = torch.cuda.CUDAGraph()
            with torch.cuda.graph(gr):
                for i in range(rem):
                    step(i)
        graphs = [(g, K // n), (gr, 1)] if gr is not None else [(g, K // n)]
        for gg, _ in graphs:
            gg.replay()
        torch.cuda.synchronize()

    def run_timed():
        if graphs:
            for gg, reps in graphs:
                for _ in range(reps):
                    gg.replay()
        else:
            for i in range(K):
                step(i)

    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    with ClockSampler(dev.index) as clk:
        start.record(stream)
        run_timed()
        end.record(stream)
        torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    ms = start.elapsed_time(end)
    assert px.last_device_error() == 0, "device error during the timed steps"
    total_bytes = sum(bytes_per_step[i % copies] for i in range(K))
    ms_max, total_bytes = reduce_over_ranks(ms, total_bytes, dev, world)
    gbs = total_bytes / (ms_max * 1e-3) / 1e9
    tokens_per_s = w.batch * K * world / (ms_max * 1e-3)

    # e2e: public API, q/rho from pinned host memory each step, output read back
    e2e = e2e_decode(px, insts, outs, args, w, dev, bytes_per_step, world)

    per_launch_bytes = sum(bytes_per_step) / copies
    avg_launch_s = (ms * 1e-3) / K
    achieved = per_launch_bytes / avg_launch_s / 1e9
    peak = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    roofline = {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                "frac": round(achieved / peak, 4), **traffic_fields("decode", w.name),
                "peak_source": f"{peaks_kind} hbm_gbs", "kernel": "decode_tc_kernel" if w.dtype == "bf16"
                else "decode_f32_kernel", "algorithmic_bytes_per_launch": int(per_launch_bytes)}
    res = {
        "metric": METRIC, "value": round(gbs, 2), "unit": "GB/s", "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": round(ms_max / K, 6), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": w.dtype, "data": "synthetic",
        "config": dict(decode_config(w, args, ctas),
                       l2=("each step reads one of %d KV copies in turn (%.0f MiB total > 126 MB L2)"
                           % (copies, copies * per_launch_bytes / 2**20)) if copies > 1
                       else "KV larger than L2", timing="CUDA-graph replay" if graphs else "stream"),
        "tokens_per_s": round(tokens_per_s, 1),
        "pct_of_hbm_peak": round(100 * gbs / world / peak, 2),
        "roofline": roofline, "e2e": e2e, "gpu_launches": K, "clocks": clk.summary(),
    }
    return res, insts


def e2e_decode(px, insts, outs, args, w, dev, bytes_per_step, world):
    """End to end through the public API: each step copies the step's q and
    rho from pinned host memory, runs the decode and reads the output back.
    The headline figure is one call per step of a prepared decode
    (DecodePlan.run_io: one launch that reads q and rho from pinned host
    memory and writes the output there; the plan is made once per buffer
    set, as a serving loop with fixed buffers would);
    the one-shot decode() call with torch copies around it is timed the same
    way beside it."""
    copies = len(insts)
    host = []
    for x in insts:
        host.append({"q": x["q"].cpu().pin_memory(), "rho": x["rho"].cpu().pin_memory()})
    out_host = [torch.empty(o.shape, dtype=o.dtype).pin_memory() for o in outs]
    K = min(args.steps, 2048)
    dq = [torch.empty_like(x["q"]) for x in insts]
    dr = [torch.empty_like(x["rho"]) for x in insts]
    plans = [px.DecodePlan(dq[c], dr[c], x["k_cache"], x["v_cache"], x["scale"], out=outs[c],
                           seq_lens=x["seq_lens"], page_table=x["page_table"], num_ctas=args.num_ctas)
             for c, x in enumerate(insts)]

    def one_plan(i):
        c = i % copies
        plans[c].run_io(host[c]["q"], host[c]["rho"], out_host[c])

    def one_call(i):
        c = i % copies
        x = insts[c]
        dq[c].copy_(host[c]["q"], non_blocking=True)
        dr[c].copy_(host[c]["rho"], non_blocking=True)
        px.decode(dq[c], dr[c], x["k_cache"], x["v_cache"], x["scale"], seq_lens=x["seq_lens"],
                  page_table=x["page_table"], out=outs[c], out_dtype=outs[c].dtype, num_ctas=args.num_ctas)
        out_host[c].copy_(outs[c], non_blocking=True)

    def timed(fn):
        for i in range(3):
            fn(i)
        torch.cuda.synchronize()
        if world > 1:
            torch.distributed.barrier()
        t0 = time.perf_counter()
        start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        start.record()
        for i in range(K):
            fn(i)
        end.record()
        torch.cuda.synchronize()
        wall = time.perf_counter() - t0
        ms, total = reduce_over_ranks(start.elapsed_time(end), sum(bytes_per_step[i % copies] for i in range(K)),
                                      dev, world)
        return total / (ms * 1e-3) / 1e9, ms / K, 1e3 * wall / K

    gbs, ms, wall = timed(one_plan)
    gbs_call, ms_call, wall_call = timed(one_call)
    h2d = insts[0]["q"].numel() * insts[0]["q"].element_size() * 2
    d2h = outs[0].numel() * outs[0].element_size()
    return {"value": round(gbs, 2), "unit": "GB/s", "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "steps": K, "ms_per_step": round(ms, 6),
            "host_wall_ms_per_step": round(wall, 6), "api": "DecodePlan.run_io (parallax_decode_plan_run_io)",
            "one_shot_call": {"value": round(gbs_call, 2), "ms_per_step": round(ms_call, 6),
                              "host_wall_ms_per_step": round(wall_call, 6), "api": "decode (parallax_decode)"},
            "note": "every step the kernel reads the query and probe from pinned host memory and writes "
                    "the output into pinned host memory, across PCIe; the KV cache stays resident on the device"}


def pipelined_e2e(hx, outs_like, call, dev, steps):
    """`steps` calls through the public API, each with its inputs copied in
    from pinned host memory (`hx`) and its outputs read back into pinned host
    memory, run as a serving or training loop would: two device buffer sets,
    the host-to-device copies on one stream, the calls on the current one,
    the read-backs on a third, so that step i + 1's copies and step i - 1's
    read-back overlap step i's kernels.  Every copy of every step is inside
    the timed region.  `call(inputs, b)` runs one step on buffer set b (0 or
    1) and returns the step's output tensors, shaped like `outs_like`.
    Returns the milliseconds for all steps (events on the current stream,
    after it has waited for the other two)."""
    comp = torch.cuda.current_stream(dev)
    h2d, d2h = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    dx = [{k: torch.empty(t.shape, dtype=t.dtype, device=dev) for k, t in hx.items()} for _ in range(2)]
    oh = [[torch.empty(t.shape, dtype=t.dtype).pin_memory() for t in outs_like] for _ in range(2)]
    copied = [torch.cuda.Event() for _ in range(2)]
    used = [torch.cuda.Event() for _ in range(2)]
    read = [torch.cuda.Event() for _ in range(2)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    start.record(comp)
    h2d.wait_event(start)
    d2h.wait_event(start)
    for i in range(steps):
        b = i % 2
        if i >= 2:
            h2d.wait_event(used[b])   # step i - 2 has consumed this buffer set
        with torch.cuda.stream(h2d):
            for k in hx:
                dx[b][k].copy_(hx[k], non_blocking=True)
        copied[b].record(h2d)
        comp.wait_event(copied[b])
        if i >= 2:
            comp.wait_event(read[b])  # step i - 2's outputs have been read back
        outs = call(dx[b], b)
        used[b].record(comp)
        d2h.wait_event(used[b])
        with torch.cuda.stream(d2h):
            for o, t in zip(oh[b], outs):
                o.copy_(t, non_blocking=True)
                t.record_stream(d2h)   # the allocator keeps it until the read-back is done
        read[b].record(d2h)
    comp.wait_stream(h2d)
    comp.wait_stream(d2h)
    end.record(comp)
    torch.cuda.synchronize()
    return start.elapsed_time(end)


def bench_decode_projected(args, w, rank, world, dev, peaks, peaks_kind):
    """Decode with q and rho projected from the layer input in the same call
    (projection kernel, then the decode kernel with a programmatic dependency
    on it).  The plain decode of the same projections is timed beside it."""
    from parallax_local_linear_b200 import binding as px

    copies = KV_COPIES
    insts = [W.projected_decode_inputs(w, device=dev, seed=w.seed + 1000 * rank + i) for i in range(copies)]
    B, Hq, d = w.batch, w.num_q_heads, w.head_dim
    kv = W.kv_bytes(w)
    proj = W.projection_bytes(B, Hq, d, w.hidden)
    step_bytes = kv + proj
    qo = [torch.empty((B, Hq, d), dtype=torch.bfloat16, device=dev) for _ in range(copies)]
    ro = [torch.empty_like(t) for t in qo]
    outs = [torch.empty_like(t) for t in qo]

    def step(i):
        c = i % copies
        x = insts[c]
        px.decode_projected(x["x"], x["w_q"], x["w_rho"], x["k_cache"], x["v_cache"], x["scale"],
                            q_out=qo[c], rho_out=ro[c], out=outs[c], num_ctas=args.num_ctas)

    def plain(i):
        c = i % copies
        x = insts[c]
        px.decode(qo[c], ro[c], x["k_cache"], x["v_cache"], x["scale"], out=outs[c], num_ctas=args.num_ctas)

    ctas = px.decode_num_ctas(px.decode_params(qo[0], insts[0]["k_cache"], num_ctas=args.num_ctas))
    stream = torch.cuda.current_stream()
    for i in range(max(args.warmup, 3)):
        step(i)
        plain(i)
    torch.cuda.synchronize()
    assert px.last_device_error() == 0, "device error during warm-up"

    K = args.steps
    n = min(GRAPH_STEPS, K)

    def capture(fn, count):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for i in range(count):
                fn(i)
        return g

    def timed(fn):
        graphs = [(capture(fn, n), K // n)]
        if K % n:
            graphs.append((capture(fn, K % n), 1))
        for gg, _ in graphs:
            gg.replay()
        torch.cuda.synchronize()
        start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        if world > 1:
            torch.distributed.barrier()
        torch.cuda.synchronize()
        with ClockSampler(dev.index) as clk:
            start.record(stream)
            for gg, reps in graphs:
                for _ in range(reps):
                    gg.replay()
            end.record(stream)
            torch.cuda.synchronize()
        if world > 1:
            torch.distributed.barrier()
        return start.elapsed_time(end), clk

    ms, clk = timed(step)
    ms_plain, _ = timed(plain)
    assert px.last_device_error() == 0, "device error during the timed steps"
    ms_max, total_bytes = reduce_over_ranks(ms, step_bytes * K, dev, world)
    gbs = total_bytes / (ms_max * 1e-3) / 1e9
    achieved = step_bytes / (ms * 1e-3 / K) / 1e9
    peak = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))

    # e2e: x from pinned host memory each step, output read back; cache and weights resident
    x_host = [x["x"].cpu().pin_memory() for x in insts]
    out_host = [torch.empty(o.shape, dtype=o.dtype).pin_memory() for o in outs]
    x_dev = [torch.empty_like(x["x"]) for x in insts]
    Ke = min(K, 2048)

    def one(i):
        c = i % copies
        x = insts[c]
        x_dev[c].copy_(x_host[c], non_blocking=True)
        px.decode_projected(x_dev[c], x["w_q"], x["w_rho"], x["k_cache"], x["v_cache"], x["scale"],
                            q_out=qo[c], rho_out=ro[c], out=outs[c], num_ctas=args.num_ctas)
        out_host[c].copy_(outs[c], non_blocking=True)

    for i in range(3):
        one(i)
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    t0 = time.perf_counter()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record()
    for i in range(Ke):
        one(i)
    end.record()
    torch.cuda.synchronize()
    wall = time.perf_counter() - t0
    ms_e, tot_e = reduce_over_ranks(start.elapsed_time(end), step_bytes * Ke, dev, world)
    e2e = {"value": round(tot_e / (ms_e * 1e-3) / 1e9, 2), "unit": "GB/s",
           "h2d_bytes_per_step": insts[0]["x"].numel() * 2, "d2h_bytes_per_step": outs[0].numel() * 2,
           "steps": Ke, "ms_per_step": round(ms_e / Ke, 6), "host_wall_ms_per_step": round(1e3 * wall / Ke, 6),
           "note": "the layer input copied from pinned host memory and the output read back every step; "
                   "cache and weights stay resident on the device"}

    roofline = {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                "frac": round(achieved / peak, 4), **traffic_fields("decode_projected", w.name),
                "peak_source": f"{peaks_kind} hbm_gbs",
                "kernel": "project_qr_kernel + decode_tc_kernel (one call)",
                "algorithmic_bytes_per_launch": int(step_bytes)}
    cfg = dict(decode_config(w, args, ctas), hidden=w.hidden,
               l2="each step reads one of %d copies of cache and weights (%.0f MiB total > 126 MB L2)"
                  % (copies, copies * step_bytes / 2**20),
               timing="CUDA-graph replay", bytes="K + V + W_Q + W_R + x read, q and rho written",
               kv_bytes_per_step=int(kv), projection_bytes_per_step=int(proj),
               plain_decode_ms_per_step=round(ms_plain / K, 6),
               added_ms_per_step=round((ms - ms_plain) / K, 6))
    res = {
        "metric": METRIC, "value": round(gbs, 2), "unit": "GB/s", "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": round(ms_max / K, 6), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic", "config": cfg,
        "tokens_per_s": round(B * K * world / (ms_max * 1e-3), 1),
        "pct_of_hbm_peak": round(100 * gbs / world / peak, 2),
        "roofline": roofline, "e2e": e2e, "gpu_launches": 2 * K, "clocks": clk.summary(),
    }
    return res, insts


def bench_lla(args, w, rank, world, dev, peaks, peaks_kind):
    """Local Linear Attention with the solved probe over decode_bf16's inputs:
    the moments pass over K and V, then the per-head solve (two launches)."""
    from parallax_local_linear_b200 import binding as px

    ridge = 0.0
    copies = KV_COPIES
    insts = [W.decode_inputs(w, device=dev, seed=w.seed + 1000 * rank + i) for i in range(copies)]
    outs = [torch.empty_like(x["q"]) for x in insts]
    rhos = [torch.empty(x["q"].shape, dtype=torch.float32, device=dev) for x in insts]
    kv = W.kv_bytes(w)
    flops = W.lla_decode_flops(w)

    def step(i):
        c = i % copies
        x = insts[c]
        px.lla_decode(x["q"], x["k_cache"], x["v_cache"], x["scale"], ridge, out=outs[c], rho_out=rhos[c],
                      num_ctas=args.num_ctas)

    stream = torch.cuda.current_stream()
    for i in range(max(args.warmup, 3)):
        step(i)
    torch.cuda.synchronize()
    assert px.last_device_error() == 0, "device error during warm-up"
    K = args.steps
    n = min(GRAPH_STEPS, K)

    def capture(count):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for i in range(count):
                step(i)
        return g

    graphs = [(capture(n), K // n)]
    if K % n:
        graphs.append((capture(K % n), 1))
    for gg, _ in graphs:
        gg.replay()
    torch.cuda.synchronize()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    with ClockSampler(dev.index) as clk:
        start.record(stream)
        for gg, reps in graphs:
            for _ in range(reps):
                gg.replay()
        end.record(stream)
        torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    ms = start.elapsed_time(end)
    assert px.last_device_error() == 0, "device error during the timed steps"
    ms_max, total_bytes = reduce_over_ranks(ms, kv * K, dev, world)
    gbs = total_bytes / (ms_max * 1e-3) / 1e9
    step_s = ms * 1e-3 / K
    tflops = flops / step_s / 1e12
    hbm_peak = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    tc_peak = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    hbm_frac, tc_frac = kv / step_s / 1e9 / hbm_peak, tflops / tc_peak
    if tc_frac >= hbm_frac:
        roofline = {"bound": "tensor", "achieved": round(tflops, 1), "peak": tc_peak, "unit": "TFLOP/s",
                    "frac": round(tc_frac, 4), "peak_source": f"{peaks_kind} bf16_tflops",
                    "algorithmic_flops_per_launch": flops}
    else:
        roofline = {"bound": "hbm", "achieved": round(kv / step_s / 1e9, 1), "peak": hbm_peak, "unit": "GB/s",
                    "frac": round(hbm_frac, 4), "peak_source": f"{peaks_kind} hbm_gbs",
                    "algorithmic_bytes_per_launch": kv}
    roofline.update(traffic_fields("lla", w.name))
    roofline["kernel"] = ("lla_moments_kernel with the solve in place (one piece per head: one launch per call); "
                          "lla_moments_kernel + lla_solve_kernel when heads are cut into pieces")
    roofline["other_bound"] = ({"unit": "GB/s", "achieved": round(kv / step_s / 1e9, 1), "frac": round(hbm_frac, 4)}
                               if roofline["bound"] == "tensor" else
                               {"unit": "TFLOP/s", "achieved": round(tflops, 1), "frac": round(tc_frac, 4)})

    # e2e: q from pinned host memory each step, output read back; cache resident
    host_q = [x["q"].cpu().pin_memory() for x in insts]
    out_host = [torch.empty(o.shape, dtype=o.dtype).pin_memory() for o in outs]
    dq = [torch.empty_like(x["q"]) for x in insts]
    Ke = min(K, 2048)

    def one(i):
        c = i % copies
        x = insts[c]
        dq[c].copy_(host_q[c], non_blocking=True)
        px.lla_decode(dq[c], x["k_cache"], x["v_cache"], x["scale"], ridge, out=outs[c], rho_out=rhos[c],
                      num_ctas=args.num_ctas)
        out_host[c].copy_(outs[c], non_blocking=True)

    for i in range(3):
        one(i)
    torch.cuda.synchronize()
    s2, e2 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s2.record()
    for i in range(Ke):
        one(i)
    e2.record()
    torch.cuda.synchronize()
    ms_e, tot_e = reduce_over_ranks(s2.elapsed_time(e2), kv * Ke, dev, world)
    e2e = {"value": round(tot_e / (ms_e * 1e-3) / 1e9, 2), "unit": "GB/s",
           "h2d_bytes_per_step": insts[0]["q"].numel() * 2, "d2h_bytes_per_step": outs[0].numel() * 2,
           "steps": Ke, "ms_per_step": round(ms_e / Ke, 6)}
    cfg = dict(decode_config(w, args, None), ridge=ridge,
        l2="each step reads one of %d KV copies (%.0f MiB total > 126 MB L2)" % (copies, copies * kv / 2**20),
        timing="CUDA-graph replay", tflops=round(tflops, 1), algorithmic_flops_per_step=flops)
    cfg.pop("num_ctas", None)
    res = {
        "metric": METRIC, "value": round(gbs, 2), "unit": "GB/s", "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": round(ms_max / K, 6), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic", "config": cfg,
        "tokens_per_s": round(w.batch * K * world / (ms_max * 1e-3), 1),
        "roofline": roofline, "e2e": e2e, "gpu_launches": 2 * K, "clocks": clk.summary(),
    }
    return res, insts


def oracle_lla_sample(w, inp, budget_s):
    """Times the float64 LLA oracle on whole (sequence, query head) pairs;
    returns (GB/s of their K+V, seconds, pairs, description)."""
    import oracle
    B, Hq, Hkv = w.batch, w.num_q_heads, w.num_kv_heads
    g = Hq // Hkv
    pairs = [(b, h) for b in range(B) for h in range(Hq)]
    np.random.default_rng(0).shuffle(pairs)
    q = inp["q"].double().cpu().numpy()
    secs, nbytes, done = 0.0, 0, 0
    for b, h in pairs:
        K = inp["k_cache"][b, h // g].double().cpu().numpy()
        V = inp["v_cache"][b, h // g].double().cpu().numpy()
        t0 = time.perf_counter()
        oracle.lla_query(q[b, h], K, V, w.scale, 0.0)
        secs += time.perf_counter() - t0
        nbytes += K.shape[0] * 2 * w.head_dim * 2
        done += 1
        if secs >= budget_s:
            break
    desc = (f"{done} of {len(pairs)} (sequence, query head) pairs of {w.name} ({nbytes / 2**20:.1f} MiB of K+V), "
            "float64 numpy LLA oracle (explicit S_KK, S_KV, numpy.linalg.solve)")
    return nbytes / secs / 1e9, secs, done, desc


# ----------------------------------------------------------------- prefill

def bench_prefill(args, w, rank, world, dev, peaks, peaks_kind):
    from parallax_local_linear_b200 import binding as px

    x = W.prefill_inputs(w, device=dev, seed=w.seed + 1000 * rank)
    out = torch.empty_like(x["q"])

    def step():
        px.prefill(x["q"], x["rho"], x["k"], x["v"], causal=w.causal, scale=x["scale"], out=out,
                   cta_pair=args.cta_pair)

    for _ in range(max(args.warmup, 3)):
        step()
    torch.cuda.synchronize()
    assert px.last_device_error() == 0
    K = args.steps
    stream = torch.cuda.current_stream()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    with ClockSampler(dev.index) as clk:
        start.record(stream)
        for _ in range(K):
            step()
        end.record(stream)
        torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    ms = start.elapsed_time(end)
    flops = W.prefill_flops(w)
    ms_max, total_flops = reduce_over_ranks(ms, flops * K, dev, world)
    tflops = total_flops / (ms_max * 1e-3) / 1e12
    peak = float(peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"]))
    achieved = flops / (ms * 1e-3 / K) / 1e12

    # e2e through the public API: inputs copied from pinned host memory and
    # the output read back every step (copies overlapped across steps)
    hx = {k: x[k].cpu().pin_memory() for k in ("q", "rho", "k", "v")}
    Ke = max(1, min(K, 10))
    e2e_out = [torch.empty_like(out), torch.empty_like(out)]

    def e2e_call(d, b):
        px.prefill(d["q"], d["rho"], d["k"], d["v"], causal=w.causal, scale=x["scale"], out=e2e_out[b],
                   cta_pair=args.cta_pair)
        return [e2e_out[b]]
    ems = pipelined_e2e(hx, [out], e2e_call, dev, Ke)
    e2e = {"value": round(flops * Ke / (ems * 1e-3) / 1e12, 2), "unit": "TFLOP/s",
           "h2d_bytes_per_step": sum(t.numel() * t.element_size() for t in hx.values()),
           "d2h_bytes_per_step": out.numel() * out.element_size(), "steps": Ke,
           "overlap": "two buffer sets; step i+1's copies and step i-1's read-back run beside step i"}
    res = {
        "metric": METRIC, "value": round(tflops, 2), "unit": "TFLOP/s", "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": round(ms_max / K, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": w.name, "batch": w.batch, "num_heads": w.num_heads, "seq_len": w.seq_len,
                   "head_dim": w.head_dim, "causal": w.causal, "rho_scale": w.rho_scale,
                   "cta_pair": bool(args.cta_pair), "l2": "inputs 537 MB > 126 MB L2"},
        "pct_of_bf16_peak": round(100 * tflops / world / peak, 2),
        "roofline": {"bound": "tensor", "achieved": round(achieved, 1), "peak": peak, "unit": "TFLOP/s",
                     "frac": round(achieved / peak, 4),
                     **traffic_fields("prefill_pair" if args.cta_pair else "prefill", w.name),
                     "peak_source": f"{peaks_kind} bf16_tflops_sustained",
                     "kernel": "prefill_tc2_kernel (cta_pair)" if args.cta_pair else "prefill_tc_kernel",
                     "algorithmic_flops_per_launch": flops},
        "e2e": e2e, "gpu_launches": K, "clocks": clk.summary(),
    }
    return res, x


def bench_prefill_paged(args, w, rank, world, dev, peaks, peaks_kind):
    """Chunked prefill over the paged cache: one call per step."""
    from parallax_local_linear_b200 import binding as px

    x = W.chunked_prefill_inputs(w, device=dev, seed=w.seed + 1000 * rank)
    out = torch.empty_like(x["q"])
    meta = ("page_table", "cu_seqlens_q", "seq_lens")

    def call(src):
        px.prefill_paged(src["q"], src["rho"], x["k_cache"], x["v_cache"], src["page_table"],
                         src["cu_seqlens_q"], src["seq_lens"], max_q_len=x["max_q_len"], scale=x["scale"],
                         causal=w.causal, out=out)

    for _ in range(max(args.warmup, 3)):
        call(x)
    torch.cuda.synchronize()
    assert px.last_device_error() == 0
    K = args.steps
    stream = torch.cuda.current_stream()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    with ClockSampler(dev.index) as clk:
        start.record(stream)
        for _ in range(K):
            call(x)
        end.record(stream)
        torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    ms = start.elapsed_time(end)
    flops = W.chunked_prefill_flops(x["q_lens"], x["seq_lens_host"], w.num_heads, w.head_dim, w.causal)
    ms_max, total_flops = reduce_over_ranks(ms, flops * K, dev, world)
    tflops = total_flops / (ms_max * 1e-3) / 1e12
    peak = float(peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"]))
    achieved = flops / (ms * 1e-3 / K) / 1e12

    # e2e through the public API: each step copies the chunk's queries, probes
    # and the batch's page table / lengths from pinned host memory and reads
    # the output back; the KV cache is resident device state.
    hx = {k: x[k].cpu().pin_memory() for k in ("q", "rho") + meta}
    Ke = max(1, min(K, 10))
    e2e_out = [torch.empty_like(out), torch.empty_like(out)]

    def e2e_call(d, b):
        px.prefill_paged(d["q"], d["rho"], x["k_cache"], x["v_cache"], d["page_table"], d["cu_seqlens_q"],
                         d["seq_lens"], max_q_len=x["max_q_len"], scale=x["scale"], causal=w.causal,
                         out=e2e_out[b])
        return [e2e_out[b]]
    ems = pipelined_e2e(hx, [out], e2e_call, dev, Ke)
    e2e = {"value": round(flops * Ke / (ems * 1e-3) / 1e12, 2), "unit": "TFLOP/s",
           "h2d_bytes_per_step": sum(t.numel() * t.element_size() for t in hx.values()),
           "d2h_bytes_per_step": out.numel() * out.element_size(), "steps": Ke,
           "resident": "paged KV cache",
           "overlap": "two buffer sets; step i+1's copies and step i-1's read-back run beside step i"}
    kv_mb = 2 * x["k_cache"].numel() * 2 / 1e6
    qr_mb = 2 * x["q"].numel() * 2 / 1e6
    res = {
        "metric": METRIC, "value": round(tflops, 2), "unit": "TFLOP/s", "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": round(ms_max / K, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": w.name, "batch": w.batch, "num_heads": w.num_heads,
                   "num_kv_heads": w.num_kv_heads, "head_dim": w.head_dim, "causal": w.causal,
                   "q_lens": [int(v) for v in x["q_lens"]], "seq_lens": [int(v) for v in x["seq_lens_host"]],
                   "page_size": W.PAGE_SIZE, "rho_scale": w.rho_scale,
                   "l2": f"q+rho {qr_mb:.0f} MB + KV pages {kv_mb:.0f} MB > 126 MB L2"},
        "pct_of_bf16_peak": round(100 * tflops / world / peak, 2),
        "roofline": {"bound": "tensor", "achieved": round(achieved, 1), "peak": peak, "unit": "TFLOP/s",
                     "frac": round(achieved / peak, 4), **traffic_fields("prefill_paged", w.name),
                     "peak_source": f"{peaks_kind} bf16_tflops_sustained", "kernel": "prefill_tc_kernel (paged)",
                     "algorithmic_flops_per_launch": flops},
        "e2e": e2e, "gpu_launches": K, "clocks": clk.summary(),
    }
    return res, x


def bench_prefill_train(args, w, rank, world, dev, peaks, peaks_kind):
    """Training step of the attention layer: forward with the backward's
    row records, then the backward (4 launches per step)."""
    from parallax_local_linear_b200 import binding as px

    x = W.prefill_inputs(w, device=dev, seed=w.seed + 1000 * rank)
    dout = W.dout_like(x["q"], w.seed + 2000 + rank)

    def step(src, g):
        out, vbar, stats = px.prefill_train(src["q"], src["rho"], src["k"], src["v"], w.causal, x["scale"])
        return px.prefill_backward(src["q"], src["rho"], src["k"], src["v"], out, vbar, stats, g, w.causal,
                                   x["scale"])

    for _ in range(max(args.warmup, 3)):
        step(x, dout)
    torch.cuda.synchronize()
    assert px.last_device_error() == 0
    K = args.steps
    stream = torch.cuda.current_stream()
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(K)]
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    with ClockSampler(dev.index) as clk:
        for i in range(K):
            ev[i][0].record(stream)
            out, vbar, stats = px.prefill_train(x["q"], x["rho"], x["k"], x["v"], w.causal, x["scale"])
            ev[i][1].record(stream)
            px.prefill_backward(x["q"], x["rho"], x["k"], x["v"], out, vbar, stats, dout, w.causal, x["scale"])
            ev[i][2].record(stream)
        torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    ms = ev[0][0].elapsed_time(ev[-1][2])
    fwd_ms = sum(e[0].elapsed_time(e[1]) for e in ev) / K
    bwd_ms = sum(e[1].elapsed_time(e[2]) for e in ev) / K
    f_fwd, f_bwd = W.prefill_flops(w), W.prefill_backward_flops(w)
    flops = f_fwd + f_bwd
    ms_max, total_flops = reduce_over_ranks(ms, flops * K, dev, world)
    tflops = total_flops / (ms_max * 1e-3) / 1e12
    peak = float(peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"]))
    achieved = f_bwd / (bwd_ms * 1e-3) / 1e12

    # e2e through the public API: q, rho, k, v and dout copied in from pinned
    # host memory each step, the four gradients read back.
    hx = {k: x[k].cpu().pin_memory() for k in ("q", "rho", "k", "v")}
    hx["dout"] = dout.cpu().pin_memory()
    grads_like = [x["q"], x["rho"], x["k"], x["v"]]
    Ke = max(1, min(K, 5))
    ems = pipelined_e2e(hx, grads_like, lambda d, b: list(step(d, d["dout"])), dev, Ke)
    e2e = {"value": round(flops * Ke / (ems * 1e-3) / 1e12, 2), "unit": "TFLOP/s",
           "h2d_bytes_per_step": sum(t.numel() * t.element_size() for t in hx.values()),
           "d2h_bytes_per_step": sum(t.numel() * t.element_size() for t in grads_like), "steps": Ke,
           "overlap": "two buffer sets; step i+1's copies and step i-1's read-back run beside step i"}
    res = {
        "metric": METRIC, "value": round(tflops, 2), "unit": "TFLOP/s", "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": round(ms_max / K, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": w.name, "batch": w.batch, "num_heads": w.num_heads, "seq_len": w.seq_len,
                   "head_dim": w.head_dim, "causal": w.causal, "rho_scale": w.rho_scale,
                   "flop_per_pair": "forward 8*d + backward 16*d", "fwd_ms": round(fwd_ms, 4),
                   "bwd_ms": round(bwd_ms, 4), "l2": "inputs 671 MB > 126 MB L2"},
        "pct_of_bf16_peak": round(100 * tflops / world / peak, 2),
        "roofline": {"bound": "tensor", "achieved": round(achieved, 1), "peak": peak, "unit": "TFLOP/s",
                     "frac": round(achieved / peak, 4), **traffic_fields("prefill_bwd", w.name),
                     "peak_source": f"{peaks_kind} bf16_tflops_sustained",
                     "kernel": "prefill backward: rows + dq + dkv kernels (one call)",
                     "algorithmic_flops_per_launch": f_bwd},
        "e2e": e2e, "gpu_launches": 4 * K, "clocks": clk.summary(),
    }
    return res, x


# ------------------------------------------------------------- CPU oracle

def oracle_decode_sample(w, inp, budget_s, max_steps=None):
    """Times the float64 oracle on whole KV-head units of the workload.

    Returns (GB/s, seconds, units timed, description)."""
    import oracle

    B, Hq, Hkv = w.batch, w.num_q_heads, w.num_kv_heads
    g = Hq // Hkv
    units = [(b, kvh) for b in range(B) for kvh in range(Hkv)]
    rng = np.random.default_rng(0)
    rng.shuffle(units)
    q = inp["q"].double().cpu().numpy()
    rho = inp["rho"].double().cpu().numpy()
    projected = w.hidden > 0
    if projected:
        x = inp["x"].double().cpu().numpy()
        wq = _F64View(inp["w_q"])
        wr = _F64View(inp["w_rho"])
    lens = None if inp["seq_lens"] is None else inp["seq_lens"].cpu().numpy()
    table = None if inp["page_table"] is None else inp["page_table"].cpu().numpy()
    done, secs, nbytes = 0, 0.0, 0
    elt = 4 if w.dtype == "f32" else 2
    for b, kvh in units:
        n = w.kv_len if lens is None else int(lens[b])
        if table is None:
            K = inp["k_cache"][b, kvh, :n].double().cpu().numpy()
            V = inp["v_cache"][b, kvh, :n].double().cpu().numpy()
            kc = K[None, None]
            vc = V[None, None]
            heads = [(0, h) for h in range(g)]
            qq, rr = q[b:b + 1, kvh * g:(kvh + 1) * g], rho[b:b + 1, kvh * g:(kvh + 1) * g]
            if projected:
                rows = slice(kvh * g * w.head_dim, (kvh + 1) * g * w.head_dim)
                wqu, wru = wq[rows], wr[rows]
                t0 = time.perf_counter()
                oracle.decode_projected(x[b:b + 1], wqu, wru, kc, vc, w.scale, heads=heads)
                secs += time.perf_counter() - t0
            else:
                t0 = time.perf_counter()
                oracle.decode(qq, rr, kc, vc, w.scale, heads=heads)
                secs += time.perf_counter() - t0
        else:
            kv = _F64View(inp["k_cache"])
            vv = _F64View(inp["v_cache"])
            t0 = time.perf_counter()
            for h in range(kvh * g, (kvh + 1) * g):
                oracle.decode(q, rho, kv, vv, w.scale, seq_lens=lens, page_table=table, heads=[(b, h)])
            secs += time.perf_counter() - t0
        nbytes += n * 2 * w.head_dim * elt
        done += 1
        if secs >= budget_s or (max_steps and done >= max_steps):
            break
    if projected:
        # the workload's metric counts the weights once per step: credit the
        # sample with the fraction of the step's projection bytes it covers
        nbytes += W.projection_bytes(B, Hq, w.head_dim, w.hidden) * done // len(units)
    what = "K+V, plus its share of the projection bytes" if projected else "K+V"
    desc = (f"{done} of {len(units)} (sequence, KV head) units of {w.name}, all {g} query heads each "
            f"({nbytes / 2**20:.1f} MiB of {what}), float64 numpy oracle")
    return nbytes / secs / 1e9, secs, done, desc


def cpu_baseline(w, inp, budget_s):
    if w.name == "prefill":
        return cpu_baseline_prefill(w, inp, budget_s)
    if w.name == "prefill_paged":
        return cpu_baseline_prefill_paged(w, inp, budget_s)
    if w.name == "prefill_train":
        return cpu_baseline_prefill_train(w, inp, budget_s)
    if w.name == "lla_decode":
        gbs, secs, done, desc = oracle_lla_sample(w, inp, budget_s)
        return {"value": round(gbs, 4), "unit": "GB/s", "cores": blas_threads(), "kind": "oracle",
                "sample": desc, "seconds": round(secs, 2)}
    gbs, secs, done, desc = oracle_decode_sample(w, inp, budget_s)
    return {"value": round(gbs, 4), "unit": "GB/s", "cores": blas_threads(), "kind": "oracle",
            "sample": desc, "seconds": round(secs, 2)}


def cpu_baseline_prefill(w, inp, budget_s):
    import oracle
    B, H, T = w.batch, w.num_heads, w.seq_len
    rng = np.random.default_rng(1)
    rows = [(int(rng.integers(B)), int(rng.integers(H)), int(t)) for t in rng.integers(0, T, size=4096)]
    views = {k: _F64View(inp[k]) for k in ("q", "rho", "k", "v")}
    secs, flops, n = 0.0, 0, 0
    for r in rows:
        t0 = time.perf_counter()
        oracle.prefill_rows(views["q"], views["rho"], views["k"], views["v"], [r], w.scale, causal=True)
        secs += time.perf_counter() - t0
        flops += 8 * w.head_dim * (r[2] + 1)
        n += 1
        if secs >= budget_s:
            break
    return {"value": round(flops / secs / 1e12, 6), "unit": "TFLOP/s", "cores": blas_threads(),
            "kind": "oracle", "sample": f"{n} random rows of {w.name} (algorithmic FLOP of those rows)",
            "seconds": round(secs, 2)}


def cpu_baseline_prefill_paged(w, inp, budget_s):
    """The oracle on groups of 16 random rows of one (sequence, head); FLOP
    counted for those rows.  Inputs are read from host copies."""
    import oracle
    host = {k: (inp[k].cpu() if inp[k].is_cuda else inp[k]) for k in ("q", "rho", "k_cache", "v_cache")}
    views = {k: _F64View(v) for k, v in host.items()}
    table = inp["page_table"].cpu().numpy()
    cu = inp["cu_seqlens_q"].cpu().numpy()
    lens, q_lens = inp["seq_lens_host"], inp["q_lens"]
    rng = np.random.default_rng(1)
    secs, flops, n = 0.0, 0, 0
    while secs < budget_s:
        b = int(rng.integers(w.batch))
        if q_lens[b] == 0:
            continue
        h = int(rng.integers(w.num_heads))
        rows = [(b, int(i), h) for i in rng.integers(0, q_lens[b], size=16)]
        t0 = time.perf_counter()
        oracle.prefill_paged_rows(views["q"], views["rho"], views["k_cache"], views["v_cache"], table, cu, lens,
                                  rows, w.scale, causal=w.causal)
        secs += time.perf_counter() - t0
        flops += sum(8 * w.head_dim * (int(lens[b]) - int(q_lens[b]) + i + 1 if w.causal else int(lens[b]))
                     for _, i, _ in rows)
        n += len(rows)
    return {"value": round(flops / secs / 1e12, 6), "unit": "TFLOP/s", "cores": blas_threads(),
            "kind": "oracle", "sample": f"{n} random rows of {w.name}, in groups of 16 per (sequence, head) "
                                        "(algorithmic FLOP of those rows)",
            "seconds": round(secs, 2)}


def cpu_baseline_prefill_train(w, inp, budget_s):
    """The oracle's forward rows plus its float64 autograd gradients on
    (sequence, head) slices of the workload's first T' positions (T' = 256):
    algorithmic FLOP 24*d per visible pair of those slices."""
    import oracle
    Tp = 256
    rng = np.random.default_rng(2)
    secs, flops, n = 0.0, 0, 0
    while secs < budget_s:
        b, h = int(rng.integers(w.batch)), int(rng.integers(w.num_heads))
        sl = {k: inp[k][b:b + 1, h:h + 1, :Tp].double().cpu().numpy() for k in ("q", "rho", "k", "v")}
        g = np.random.default_rng(n).standard_normal(sl["q"].shape)
        t0 = time.perf_counter()
        rows = [(0, 0, t) for t in range(Tp)]
        oracle.prefill_rows(sl["q"], sl["rho"], sl["k"], sl["v"], rows, w.scale, causal=True)
        oracle.prefill_grads(sl["q"], sl["rho"], sl["k"], sl["v"], g, w.scale, causal=True)
        secs += time.perf_counter() - t0
        flops += 24 * w.head_dim * Tp * (Tp + 1) // 2
        n += 1
    return {"value": round(flops / secs / 1e12, 6), "unit": "TFLOP/s", "cores": blas_threads(), "kind": "oracle",
            "sample": f"{n} (sequence, head) slices of the first {Tp} positions: forward rows + float64 autograd "
                      "gradients (algorithmic FLOP 24*d per visible pair)",
            "seconds": round(secs, 2)}


def workload_shape(w, args):
    """The keys of this arm's `config` that name the workload itself (shapes,
    dtypes, lengths), without the ones about how the GPU arm launches and
    times it (grid size, L2 note, graph replay)."""
    if w.name in ("prefill", "prefill_train"):
        return {"workload": w.name, "batch": w.batch, "num_heads": w.num_heads, "seq_len": w.seq_len,
                "head_dim": w.head_dim, "causal": w.causal, "rho_scale": w.rho_scale}
    if w.name == "prefill_paged":
        return {"workload": w.name, "batch": w.batch, "num_heads": w.num_heads, "num_kv_heads": w.num_kv_heads,
                "head_dim": w.head_dim, "causal": w.causal, "page_size": W.PAGE_SIZE, "rho_scale": w.rho_scale}
    cfg = decode_config(w, args, None)
    cfg.pop("num_ctas", None)
    if w.hidden:
        cfg["hidden"] = w.hidden
    if w.name == "lla_decode":
        cfg["ridge"] = 0.0
    return cfg


def reference_arm(args, w, rank, world):
    """The float64 oracle on the host cores, on this workload's metric.

    Each step times the oracle on a bounded sample of the workload (whole
    (sequence, KV head) units for decode, random rows for prefill), sized so
    that warm-up plus all steps take about two minutes."""
    if rank != 0:
        return None
    budget = max(0.05, 120.0 / max(1, args.steps + args.warmup))
    if w.name in ("prefill", "prefill_train"):
        sub = W.PrefillWorkload(w.name, 1, 1, w.seq_len, w.head_dim, rho_scale=w.rho_scale, seed=w.seed)
        inp = W.prefill_inputs(sub, device="cpu")
    elif w.name == "prefill_paged":
        inp = W.chunked_prefill_inputs(w, device="cpu")
    elif w.hidden:
        inp = W.projected_decode_inputs(w, device="cpu")
    elif w.batch * w.kv_len <= 2**20:
        inp = W.decode_inputs(w, device="cpu")
    else:
        inp = _host_decode_sample(w)
    vals, secs_all, desc = [], 0.0, ""
    for i in range(args.warmup + args.steps):
        if w.name in ("prefill", "prefill_paged", "prefill_train"):
            sub_w = w if w.name != "prefill_train" else W.PrefillWorkload(w.name, 1, 1, w.seq_len, w.head_dim,
                                                                          rho_scale=w.rho_scale, seed=w.seed)
            cb = cpu_baseline(sub_w, inp, budget)
            v, secs, desc = cb["value"], cb["seconds"], cb["sample"]
        else:
            sub_w = w if inp["q"].shape[0] == w.batch else W.DecodeWorkload(
                w.name, inp["q"].shape[0], w.num_q_heads, w.num_kv_heads, w.head_dim, w.kv_len,
                dtype=w.dtype, paged=w.paged, min_len=w.min_len, hidden=w.hidden)
            sample = oracle_lla_sample if w.name == "lla_decode" else oracle_decode_sample
            v, secs, _, desc = sample(sub_w, inp, budget)
        if i >= args.warmup:
            vals.append(v)
            secs_all += secs
    value = statistics.median(vals)
    unit = "TFLOP/s" if w.name.startswith("prefill") else "GB/s"
    return {"impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": unit, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(1e3 * secs_all / args.steps, 3),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic",
            "config": dict(workload_shape(w, args), timing="host wall clock of the float64 oracle on a bounded sample"),
            "cpu_baseline": {"value": round(value, 6), "unit": unit, "kind": "oracle", "cores": blas_threads(),
                             "sample": "per step: " + desc},
            "e2e": {"value": round(value, 6), "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def _host_decode_sample(w):
    """Host-side inputs for a few sequences of a large decode workload (the
    oracle's timing does not depend on which sequences are drawn)."""
    n_seq = 2
    sub = W.DecodeWorkload(w.name, n_seq, w.num_q_heads, w.num_kv_heads, w.head_dim, w.kv_len,
                           dtype=w.dtype, key_offset_std=w.key_offset_std, paged=w.paged,
                           min_len=w.min_len, seed=w.seed)
    return W.decode_inputs(sub, device="cpu")


# -------------------------------------------------------------------- main

# Workloads timed after the headline one in the default run, each with its
# own roofline, clocks and oracle baseline (the four other configurations of
# the method's targets first, then the serving and training steps beyond them).
PER_CONFIG = ("decode_f32", "decode_long", "decode_paged", "prefill", "prefill_cta_pair", "prefill_paged",
              "prefill_train", "decode_projected", "lla_decode")
NOMINAL_PEAKS = {"GB/s": 8000.0, "TFLOP/s": 2250.0}   # B200 HBM3e and dense bf16, NVIDIA's figures


def run_workload(args, w, rank, world, dev, peaks, kind):
    if w.name == "prefill":
        return bench_prefill(args, w, rank, world, dev, peaks, kind)
    if w.name == "prefill_paged":
        return bench_prefill_paged(args, w, rank, world, dev, peaks, kind)
    if w.name == "prefill_train":
        return bench_prefill_train(args, w, rank, world, dev, peaks, kind)
    if w.hidden:
        res, inp = bench_decode_projected(args, w, rank, world, dev, peaks, kind)
        return res, inp[0]
    if w.name == "lla_decode":
        res, inp = bench_lla(args, w, rank, world, dev, peaks, kind)
        return res, inp[0]
    res, inp = bench_decode(args, w, rank, world, dev, peaks, kind)
    return res, inp[0]


def config_summary(res):
    """The per-workload record of the default run: throughput, its roofline
    against the measured and the nominal peak, clocks, e2e and the oracle."""
    rf = dict(res["roofline"])
    nominal = NOMINAL_PEAKS[rf["unit"]]
    rf["nominal_peak"] = nominal
    rf["frac_of_nominal"] = round(rf["achieved"] / nominal, 4)
    out = {k: res[k] for k in ("value", "unit", "ms_per_step", "steps", "warmup", "dtype", "config", "clocks",
                               "gpu_launches") if k in res}
    out["roofline"] = rf
    if "tokens_per_s" in res:
        out["tokens_per_s"] = res["tokens_per_s"]
    if "e2e" in res:
        out["e2e"] = {k: res["e2e"][k] for k in ("value", "unit", "h2d_bytes_per_step", "d2h_bytes_per_step")}
    if "cpu_baseline" in res:
        out["cpu_baseline"] = res["cpu_baseline"]
    return out


def main(argv=None):
    args = parse_args(argv)
    w = W.WORKLOADS[args.workload]
    if args.batch > 0:
        import dataclasses
        w = dataclasses.replace(w, batch=args.batch)
    steps_given, warmup_given = args.steps, args.warmup
    if args.steps is None:
        args.steps = default_steps(args.workload) if args.impl == "ours" else 10
    if args.warmup is None:
        args.warmup = 20 if args.impl == "ours" else 2
    rank, world, local = dist_env()

    if args.impl == "reference":
        res = reference_arm(args, w, rank, world)
        if res is not None:
            print(json.dumps(res), flush=True)
        return 0

    if not torch.cuda.is_available():
        print(json.dumps({"error": "bench.py needs a CUDA device"}), flush=True)
        return 1
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    if world > 1:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    peaks, kind = load_peaks()
    try:
        res, inp = run_workload(args, w, rank, world, dev, peaks, kind)
        if rank == 0 and world == 1 and not args.no_cpu_baseline:
            res["cpu_baseline"] = cpu_baseline(w, inp, args.cpu_seconds)
        del inp
        per_config = {}
        if args.per_config and args.workload == "decode_bf16" and args.batch == 0:
            import copy
            for key in PER_CONFIG:
                torch.cuda.empty_cache()
                name = "prefill" if key == "prefill_cta_pair" else key
                wc = W.WORKLOADS[name]
                ac = copy.copy(args)
                ac.cta_pair = key == "prefill_cta_pair"
                ac.steps = steps_given if steps_given is not None else default_steps(name)
                ac.warmup = warmup_given if warmup_given is not None else 5
                rc, ic = run_workload(ac, wc, rank, world, dev, peaks, kind)
                if rank == 0 and world == 1 and not args.no_cpu_baseline and not ac.cta_pair:
                    rc["cpu_baseline"] = cpu_baseline(wc, ic, args.cpu_seconds_per_config)
                del ic
                per_config[key] = config_summary(rc)
        if rank == 0:
            res["roofline"]["nominal_peak"] = NOMINAL_PEAKS[res["roofline"]["unit"]]
            res["roofline"]["frac_of_nominal"] = round(res["roofline"]["achieved"] /
                                                       res["roofline"]["nominal_peak"], 4)
            if per_config:
                res["per_config"] = per_config
                res["per_config_note"] = ("each workload timed in this same run on the same GPU after the "
                                          "headline, with its own timed region, launches, clocks and oracle "
                                          "sample; the top-level keys describe the headline alone")
            print(json.dumps(res), flush=True)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
