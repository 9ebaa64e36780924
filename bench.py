#!/usr/bin/env python
"""Benchmark of the BitNet b1.58 W1.58A8 linear layer on B200.

Default workload (one "step"): the BitNet-b1.58-2B decode sweep at M = 1 --
30 layers x 7 BitLinears (Q, K, V, O, gate, up, down) plus the LM head, 211
calls of the fused quantise + GEMV with fresh seeded weights per layer and a
fresh activation row per call. The calls are independent problems, so the
step issues them as one grouped call (bitnet_gemv_fused_grouped: one persistent
launch) and replays it as a CUDA graph; the JSON also reports the 211 separate
calls in three issue orders. Metric: GB/s of algorithmic bytes
(packed weights + bf16 activations + bf16 outputs + weight scales).

Also reported: the prefill workload (M in {2048, 8192} x four FFN shapes
through bitnet_linear) in INT8 TOPS against the dense INT8 tensor peak, the
LM-head GEMV alone, and the decode sweep in two dependent issue orders.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Multi-GPU (launched with torch.distributed.run): every rank runs its own
decode sweep (independent decode streams over replicated weights, no
collective on the data path); value = all ranks' bytes / max-over-ranks time.
"""
import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402
from synth import workloads as W  # noqa: E402

METRIC = "W1.58A8 linear: GB/s at M=1 decode, INT8 TOPS at M≥2048, vs B200 roofline"
UNIT = "GB/s"
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
INT8_OVER_BF16 = 2.0  # nominal dense ratio (4.5 / 2.25 PFLOP/s)
L2_BYTES = 126 * 1024 * 1024


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--no-prefill", action="store_true")
    ap.add_argument("--no-secondary", action="store_true",
                    help="skip the LLaMA GEMV (M <= 15) and mid-batch GEMM sections")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--branches", type=int, default=16,
                    help="graph branches for the independent calls of a step")
    ap.add_argument("--case", choices=("lm_head", "prefill", "decode_once", "midbatch", "gemv_m15",
                                       "rmsnorm"),
                    help="profiling aid: run one small case a few times and exit "
                         "(no JSON line); see profiles/ for the ncu commands")
    return ap.parse_args()


# ------------------------------------------------------------------ env

def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": float(p["hbm_gbs"]), "bf16_tflops": float(p["bf16_tflops"]),
                "bf16_tflops_sustained": float(p.get("bf16_tflops_sustained", p["bf16_tflops"])),
                "source": "measured"}
    return {"hbm_gbs": FALLBACK_HBM_GBS, "bf16_tflops": FALLBACK_BF16_TFLOPS,
            "bf16_tflops_sustained": 1400.0, "source": "fallback"}


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled during the timed region."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.Q}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *a):
        self.lines = []
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [l for l in out.splitlines() if l.strip()]

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for line in getattr(self, "lines", []):
            f = [c.strip() for c in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for name, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(name)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm)}


# the headers each kernel's translation unit reads (gemv.cuh includes the norm
# helpers of rmsnorm.cuh, which include ternarize.cuh)
_GEMV_HEADERS = ("common.cuh", "pack_quant.cuh", "ternarize.cuh", "rmsnorm.cuh", "gemv.cuh")
KERNEL_SOURCES = {
    "gemv_kernel": _GEMV_HEADERS,
    "gemv_grouped_kernel": _GEMV_HEADERS + ("gemv_grouped.cuh",),
    "gemm_i8_ts_kernel": ("common.cuh", "pack_quant.cuh", "gemm_ts.cuh"),
}


def source_hash(kernel):
    """Hash of the device sources a kernel is built from."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "bit_gemm_bitnet_b200", "csrc")
    for name in KERNEL_SOURCES[kernel]:
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(name.encode())
            h.update(f.read())
    return h.hexdigest()[:16]


def recorded_traffic(kernel):
    """DRAM bytes (read + write) of `kernel` from the committed ncu summary
    (profiles/ncu_traffic.json), if the kernel's sources are unchanged since
    the counters were taken; else None."""
    path = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        rec = json.load(f).get(kernel)
    if rec is None or rec.get("source_hash") != source_hash(kernel):
        return None
    return rec.get("bytes")


def max_over_ranks(values, device):
    """Element-wise max of per-rank device times over all ranks (the job is
    as slow as its slowest rank)."""
    import torch.distributed as dist
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t]


def whole_job_gbs(bytes_per_step, world, steps, max_ms):
    """Weak scaling: every rank moves bytes_per_step per step."""
    return bytes_per_step * world * steps / (max_ms / 1e3) / 1e9


def activation_variant(variant, rank):
    """Generator variant of a call's activation row on `rank`: each rank
    decodes its own tokens over the same weights."""
    return variant + 16 * rank


# ---------------------------------------------------------- decode sweep

def sweep_calls():
    names = [n for n, _, _ in W.DECODE_2B_LAYER]
    out = []
    for layer, name, K, N in W.decode_2b_sweep():
        variant = names.index(name) if name in names else len(names)
        out.append((layer, variant, K, N))
    return out


def call_bytes(M, K, N, sw_len=1):
    return N * K // 4 + 2 * M * K + 2 * M * N + 4 * sw_len


def build_decode(bn, dev, rank):
    calls = sweep_calls()
    packed, scales = [], []
    for layer, variant, K, N in calls:
        w = synth.ternary(synth.key(W.W_DECODE_2B, layer, synth.T_WEIGHT, variant), N, K)
        wd = torch.from_numpy(w).to(dev)
        packed.append(bn.bitnet_pack_weights(wd))
        del wd
        sw = synth.scale_wt(synth.key(W.W_DECODE_2B, layer, synth.T_SCALE_WT, variant))
        scales.append(torch.from_numpy(sw).to(dev))
    xs_total = sum(K for _, _, K, _ in calls)
    outs_total = sum(N for _, _, _, N in calls)
    x_host = torch.empty((xs_total,), dtype=torch.bfloat16).pin_memory()
    xv = x_host.view(torch.int16).numpy().view(np.uint16)
    off = 0
    for layer, variant, K, N in calls:
        xv[off:off + K] = synth.act_bf16(
            synth.key(W.W_DECODE_2B, layer, synth.T_ACT, activation_variant(variant, rank)),
            1, K)[0]
        off += K
    x_dev = x_host.to(dev)
    out_dev = torch.empty((outs_total,), dtype=torch.bfloat16, device=dev)
    out_host = torch.empty((outs_total,), dtype=torch.bfloat16).pin_memory()
    xs, outs = [], []
    xo = oo = 0
    for _, _, K, N in calls:
        xs.append(x_dev[xo:xo + K].view(1, K))
        outs.append(out_dev[oo:oo + N].view(1, N))
        xo += K
        oo += N
    nbytes = sum(call_bytes(1, K, N) for _, _, K, N in calls)
    return dict(calls=calls, packed=packed, scales=scales, xs=xs, outs=outs, x_host=x_host,
                x_dev=x_dev, out_dev=out_dev, out_host=out_host, bytes=nbytes)


def make_sweep(bn, d, order="independent", branches=8):
    """The step as raw C-ABI calls (pointers prepared once), issued in one of
    four orders:
      grouped      one bitnet_gemv_fused_grouped call over the 211 independent
                   problems (one persistent launch streams all their weights);
      independent  the 211 calls are independent problems (each has its own
                   activation row), issued round-robin on `branches` streams
                   forked from and joined back into the capturing stream;
      layer        the dependency order of a transformer layer: Q, K, V
                   concurrently, then O, then gate and up concurrently, then
                   down; layers one after another, the LM head last;
      stream       every call after the previous one on one stream;
      layer_grouped  the dependency order of a transformer layer on one
                   stream, with the stages a layer can group issued as one
                   grouped call: Q|K|V, then O, then gate|up, then down;
                   layers one after another, the LM head last (4 launches
                   per layer, 121 per step).
    Within a stream, consecutive kernels overlap through programmatic
    dependent launch; across streams they are ordered by events only."""
    import ctypes
    L = bn.lib()
    args = []
    for (layer, variant, K, N), p, s, x, o in zip(d["calls"], d["packed"], d["scales"],
                                                  d["xs"], d["outs"]):
        args.append((layer, variant, ctypes.c_void_p(o.data_ptr()),
                     ctypes.c_void_p(x.data_ptr()), ctypes.c_void_p(p.data_ptr()),
                     ctypes.c_void_p(s.data_ptr()), K, N))
    side = [torch.cuda.Stream() for _ in range(max(branches, 3))]
    grouped = bn.gemv_problems(d["xs"], d["packed"], d["scales"], d["outs"])
    # layer_grouped: per layer, the problem arrays of its Q|K|V and gate|up
    # stages (kept alive with the closure)
    stage_groups = []
    by_layer_idx = {}
    for i, (layer, variant, K, N) in enumerate(d["calls"]):
        by_layer_idx.setdefault(layer, {})[variant] = i
    for layer in sorted(by_layer_idx):
        idx = by_layer_idx[layer]
        if len(idx) == 1:
            stage_groups.append([[next(iter(idx.values()))]])
            continue
        stage_groups.append([[idx[0], idx[1], idx[2]], [idx[3]], [idx[4], idx[5]], [idx[6]]])
    stage_arrays = [[(bn.gemv_problems([d["xs"][i] for i in grp], [d["packed"][i] for i in grp],
                                       [d["scales"][i] for i in grp], [d["outs"][i] for i in grp]),
                      len(grp)) for grp in stages] for stages in stage_groups]

    def issue(a):
        _, _, o, x, p, s, K, N = a
        st = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
        r = L.bitnet_gemv_fused(o, x, 0, p, s, 1, 1, N, K, st)
        if r != 0:
            raise RuntimeError(f"bitnet_gemv_fused: {bn.status_string(r)}")

    def fan(groups):
        main = torch.cuda.current_stream()
        for i, grp in enumerate(groups):
            side[i].wait_stream(main)
            with torch.cuda.stream(side[i]):
                for a in grp:
                    issue(a)
        for i in range(len(groups)):
            main.wait_stream(side[i])

    def grouped_call(arr, n):
        st = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
        r = L.bitnet_gemv_fused_grouped(ctypes.cast(arr, ctypes.c_void_p), n, 1, 0, st)
        if r != 0:
            raise RuntimeError(f"bitnet_gemv_fused_grouped: {bn.status_string(r)}")

    def sweep():
        if order == "layer_grouped":
            for stages in stage_arrays:
                for arr, n in stages:
                    grouped_call(arr, n)
            return
        if order == "grouped":
            st = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
            r = L.bitnet_gemv_fused_grouped(ctypes.cast(grouped, ctypes.c_void_p), len(args), 1,
                                            0, st)
            if r != 0:
                raise RuntimeError(f"bitnet_gemv_fused_grouped: {bn.status_string(r)}")
        elif order == "stream":
            for a in args:
                issue(a)
        elif order == "independent":
            fan([args[i::branches] for i in range(branches)])
        else:
            by_layer = {}
            for a in args:
                by_layer.setdefault(a[0], []).append(a)
            for layer in sorted(by_layer):
                calls = {a[1]: a for a in by_layer[layer]}
                if len(calls) == 1:
                    issue(next(iter(calls.values())))
                    continue
                fan([[calls[0]], [calls[1]], [calls[2]]])   # Q, K, V
                issue(calls[3])                             # O
                fan([[calls[4]], [calls[5]]])               # gate, up
                issue(calls[6])                             # down
    return sweep


# A few milliseconds of device spin before the first timed event: the host
# then enqueues every timed step while the device is still busy, so a stall
# of the host (a context switch, the clock sampler starting) cannot leave
# the device idle between timed steps. The spin itself is outside the events.
HOST_LEAD_CYCLES = 6_000_000


# the issue orders timed beside the headline's single grouped launch
ORDERS = ("layer_grouped", "independent", "layer", "stream")


def time_graph(g, steps, warmup, barrier):
    for _ in range(warmup):
        g.replay()
    torch.cuda.synchronize()
    barrier()
    torch.cuda.synchronize()
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(steps + 1)]
    torch.cuda._sleep(HOST_LEAD_CYCLES)
    ev[0].record()
    for i in range(steps):
        g.replay()
        ev[i + 1].record()
    torch.cuda.synchronize()
    barrier()
    per = [ev[i].elapsed_time(ev[i + 1]) for i in range(steps)]
    return ev[0].elapsed_time(ev[-1]), per


def second_buffers(d, dev):
    """A copy of the decode set-up with its own device activation and output
    buffers (same weights), for double-buffered end-to-end steps."""
    d2 = dict(d)
    d2["x_dev"] = torch.empty_like(d["x_dev"])
    d2["out_dev"] = torch.empty_like(d["out_dev"])
    d2["out_host"] = torch.empty_like(d["out_host"]).pin_memory()
    xs, outs = [], []
    xo = oo = 0
    for _, _, K, N in d["calls"]:
        xs.append(d2["x_dev"][xo:xo + K].view(1, K))
        outs.append(d2["out_dev"][oo:oo + N].view(1, N))
        xo += K
        oo += N
    d2["xs"], d2["outs"] = xs, outs
    return d2


def time_e2e(graphs, ds, steps, warmup, barrier):
    """End to end through the C ABI, every step copying its activations from
    pinned host memory and its outputs back. Two buffer sets alternate, so
    the upload of step i+1 and the download of step i-1 run on their own
    streams while step i computes (a serving loop's double buffering)."""
    comp = torch.cuda.current_stream()
    up, down = torch.cuda.Stream(), torch.cuda.Stream()
    ev_up = [torch.cuda.Event() for _ in ds]
    ev_comp = [torch.cuda.Event() for _ in ds]
    ev_down = [torch.cuda.Event() for _ in ds]

    def step(i):
        b = i % len(ds)
        d = ds[b]
        up.wait_event(ev_comp[b])        # step i-2 has finished reading x_dev[b]
        with torch.cuda.stream(up):
            d["x_dev"].copy_(d["x_host"], non_blocking=True)
        ev_up[b].record(up)
        comp.wait_event(ev_up[b])
        comp.wait_event(ev_down[b])      # step i-2's outputs have been read back
        graphs[b].replay()
        ev_comp[b].record(comp)
        down.wait_event(ev_comp[b])
        with torch.cuda.stream(down):
            d["out_host"].copy_(d["out_dev"], non_blocking=True)
        ev_down[b].record(down)

    def drain():
        for b in range(len(ds)):
            comp.wait_event(ev_down[b])

    for i in range(warmup):
        step(i)
    drain()
    torch.cuda.synchronize()
    barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(comp)
    for i in range(steps):
        step(i)
    drain()
    e1.record(comp)
    torch.cuda.synchronize()
    barrier()
    return e0.elapsed_time(e1)


class L2Flush:
    """Flush L2 between timed repetitions: write one buffer twice the size of
    L2, then read another one of that size. The write evicts the timed
    call's data; the read then evicts the written (dirty) lines, so their
    write-back to HBM happens here rather than inside the timed call."""

    def __init__(self, dev):
        self.a = torch.empty((2 * L2_BYTES,), dtype=torch.uint8, device=dev)
        self.b = torch.ones((2 * L2_BYTES // 4,), dtype=torch.int32, device=dev)

    def __call__(self, r):
        self.a.fill_(r & 0xFF)
        self.b.amax()


def lm_head_alone(bn, d, dev, reps=20):
    """The LM-head GEMV (82 MB of packed weights) timed alone, L2 flushed:
    bitnet_gemv_fused as the product dispatches it, and for comparison the
    single-problem GEMV kernel (reached through bitnet_linear_bias with a
    zero bias, which that kernel alone takes)."""
    i = len(d["calls"]) - 1
    _, _, K, N = d["calls"][i]
    flush = L2Flush(dev)
    zero_bias = torch.zeros((N,), dtype=torch.bfloat16, device=dev)

    def timed(fn):
        times = []
        for r in range(reps + 3):
            flush(r)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            fn()
            e1.record()
            torch.cuda.synchronize()
            if r >= 3:
                times.append(e0.elapsed_time(e1))
        return statistics.median(times)

    ms = timed(lambda: bn.bitnet_gemv_fused(d["xs"][i], d["packed"][i], d["scales"][i],
                                            out=d["outs"][i]))
    ms_single = timed(lambda: bn.bitnet_linear(d["xs"][i], d["packed"][i], d["scales"][i],
                                               out=d["outs"][i], bias=zero_bias))
    # the pages' comparison: the same layer as a dense bf16 cuBLAS GEMV (the
    # time does not depend on the weight values)
    wb = torch.full((N, K), 0.5, dtype=torch.bfloat16, device=dev)
    ob = torch.empty((1, N), dtype=torch.bfloat16, device=dev)
    c_ms = timed(lambda: torch.mm(d["xs"][i], wb.t(), out=ob))
    del wb
    return {"K": K, "N": N, "ms": ms, "gbs": call_bytes(1, K, N) / ms / 1e6,
            "single_kernel_ms": ms_single,
            "single_kernel_gbs": call_bytes(1, K, N) / ms_single / 1e6,
            "cublas_bf16": {"ms": c_ms, "speedup": c_ms / ms}}


# ---------------------------------------------------------------- prefill

def time_flushed(fn, flush, reps=5, graph=True):
    """Median device ms of one fn() call with L2 flushed before each
    repetition. With graph=True the call is captured once in a CUDA graph and
    replayed, so the host's own cost of issuing it (which can outlast the
    flush) does not fall between the events."""
    run = fn
    if graph:
        fn()
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            fn()
        run = g.replay
    ts = []
    for r in range(reps + 2):
        flush(r)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        run()
        e1.record()
        torch.cuda.synchronize()
        if r >= 2:
            ts.append(e0.elapsed_time(e1))
    return statistics.median(ts)


def prefill(bn, dev, pk, reps=5):
    """The prefill workload: M in {2048, 8192} x four FFN shapes through
    bitnet_linear (per-token quantisation + tensor-core GEMM, bf16 out), each
    timed with CUDA events with L2 flushed between repetitions; and the GEMM
    alone (bitnet_gemm on activations quantised beforehand) for every case."""
    flush = L2Flush(dev)
    peak = pk["bf16_tflops"] * INT8_OVER_BF16

    def timed(fn):
        return time_flushed(fn, flush, reps)

    Mmax = max(W.PREFILL_M)
    cases, tot_ops, tot_ms, tot_gemm_ms = [], 0.0, 0.0, 0.0
    gemm_pub = None
    for K, N in W.PREFILL_SHAPES:
        x = synth.act_bf16(synth.key(W.W_PREFILL, Mmax, synth.T_ACT, K), Mmax, K)
        w = synth.ternary(synth.key(W.W_PREFILL, Mmax, synth.T_WEIGHT, K), N, K)
        sw = synth.scale_wt(synth.key(W.W_PREFILL, Mmax, synth.T_SCALE_WT, K))
        xd_all = torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).to(dev)
        del x
        wd = torch.from_numpy(w).to(dev)
        wp = bn.bitnet_pack_weights(wd)
        wb = wd.to(torch.bfloat16)
        del wd
        swd = torch.from_numpy(sw).to(dev)
        for M in W.PREFILL_M:
            xd = xd_all[:M]
            out = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
            ws = torch.empty((bn.bitnet_linear_workspace_bytes(M, K),), dtype=torch.uint8,
                             device=dev)
            ms = timed(lambda: bn.bitnet_linear(xd, wp, swd, out=out, workspace=ws))
            ops = 2.0 * M * N * K
            # the GEMM alone: bitnet_gemm on activations quantised beforehand
            xq, sa = bn.bitnet_quantize_act(xd)
            g_ms = timed(lambda: bn.bitnet_gemm(xq, wp, sa, swd, out=out))
            del xq, sa
            # the pages' comparison: the same layer as a dense bf16 cuBLAS GEMM
            c_ms = timed(lambda: torch.mm(xd, wb.t(), out=out))
            cases.append({"M": M, "K": K, "N": N, "ms": ms, "tops": ops / ms / 1e9,
                          "gemm_ms": g_ms, "gemm_tops": ops / g_ms / 1e9,
                          "cublas_bf16": {"ms": c_ms, "speedup": c_ms / ms}})
            tot_ops += ops
            tot_ms += ms
            tot_gemm_ms += g_ms
            if gemm_pub is None and M == Mmax:
                gemm_pub = {"M": M, "K": K, "N": N, "ms": g_ms, "tops": ops / g_ms / 1e9,
                            "frac": ops / g_ms / 1e9 / peak}
            del out, ws
        del xd_all, wp, wb
    bn.bitnet_device_status()
    tops = tot_ops / tot_ms / 1e9
    gemm_tops = tot_ops / tot_gemm_ms / 1e9
    return {"workload": "M in {2048, 8192} x (4096->11008, 11008->4096, 2560->6912, "
                        "6912->2560) through bitnet_linear (quantise + GEMM)",
            "tops": tops, "ms_total": tot_ms, "cases": cases,
            "gemm_only": {"tops": gemm_tops, "ms_total": tot_gemm_ms, "peak": peak,
                          "frac": gemm_tops / peak,
                          "kernel": "gemm_i8_ts_kernel via bitnet_gemm (pre-quantised)"},
            "roofline": {"bound": "tensor", "achieved": tops, "peak": peak, "unit": "TOPS",
                         "frac": tops / peak,
                         "peak_source": f"{pk['source']} bf16 burst x {INT8_OVER_BF16:g} "
                                        "(int8/bf16 nominal)",
                         "kernel": "quantize_rows_perm_kernel + gemm_i8_ts_kernel "
                                   "(timed together)",
                         "traffic": recorded_traffic("gemm_i8_ts_kernel")},
            "bitnet_gemm_natural_layout": gemm_pub}


# ------------------------------------------------- decode and mid-batch

def weight_rotation(wp):
    """Independent device copies of a packed weight tensor, together more than
    twice the L2 size, so that a loop over them reads the weights from HBM."""
    n = max(2, -(-2 * L2_BYTES // wp.numel()) + 1)
    return [wp.clone() for _ in range(n)]


def time_rotation(fns, reps=20, warmup=3):
    """Median ms per call of one CUDA graph that issues every call in `fns`
    (one call per weight copy), over `reps` replays."""
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        for fn in fns:
            fn()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=s):
            for fn in fns:
                fn()
        for _ in range(warmup):
            g.replay()
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(reps + 1)]
        torch.cuda._sleep(HOST_LEAD_CYCLES)
        ev[0].record(s)
        for i in range(reps):
            g.replay()
            ev[i + 1].record(s)
    torch.cuda.synchronize()
    per = [ev[i].elapsed_time(ev[i + 1]) for i in range(reps)]
    del g
    return statistics.median(per) / len(fns)


def bf16_rotation(w_int8):
    """Independent bf16 copies of a weight matrix (the dense layer cuBLAS
    would run), together more than twice the L2 size."""
    wb = w_int8.to(torch.bfloat16)
    n = max(2, -(-2 * L2_BYTES // (wb.numel() * 2)) + 1)
    return [wb.clone() for _ in range(n)]


def cublas_bf16(ms_ours, x_bf16, wb_copies, N):
    """The pages' kernel-level comparison: the same layer as a dense bf16
    GEMM through cuBLAS (torch.mm, y = x W^T), weights rotated like ours.
    A library reference point beside our kernel, not part of the path."""
    M = x_bf16.shape[0]
    out = torch.empty((M, N), dtype=torch.bfloat16, device=x_bf16.device)
    ms = time_rotation([lambda c=c: torch.mm(x_bf16, c.t(), out=out) for c in wb_copies])
    return {"ms": ms, "speedup": ms / ms_ours}


def llama_gemv(bn, dev, pk):
    """LLaMA-7B projections at M in {1, 4, 8, 15} through bitnet_gemv_fused
    (quantisation fused), weights rotated over copies larger than 2x L2."""
    hbm = pk["hbm_gbs"]
    cases = []
    for v, (name, K, N) in enumerate(W.LLAMA_GEMV_SHAPES):
        w = synth.ternary(synth.key(W.W_LLAMA_GEMV, 1, synth.T_WEIGHT, v), N, K)
        wd = torch.from_numpy(w).to(dev)
        copies = weight_rotation(bn.bitnet_pack_weights(wd))
        wb_copies = bf16_rotation(wd)
        del w, wd
        swd = torch.from_numpy(synth.scale_wt(synth.key(W.W_LLAMA_GEMV, 1, synth.T_SCALE_WT, v))).to(dev)
        for M in W.LLAMA_GEMV_M:
            x = synth.act_bf16(synth.key(W.W_LLAMA_GEMV, M, synth.T_ACT, v), M, K)
            xd = torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).to(dev)
            out = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
            ms = time_rotation([lambda c=c: bn.bitnet_gemv_fused(xd, c, swd, out=out)
                                for c in copies])
            gbs = call_bytes(M, K, N) / ms / 1e6
            # the same problems as one grouped call (independent projections
            # of a layer, such as Q, K and V, can be issued this way)
            gouts = [torch.empty((M, N), dtype=torch.bfloat16, device=dev) for _ in copies]
            g_ms = time_rotation([lambda: bn.bitnet_gemv_fused_grouped(
                [xd] * len(copies), copies, [swd] * len(copies), gouts)]) / len(copies)
            del gouts
            g_gbs = call_bytes(M, K, N) / g_ms / 1e6
            case = {"M": M, "K": K, "N": N, "ms": ms, "gbs": gbs, "frac_hbm": gbs / hbm,
                    "tops": 2.0 * M * N * K / ms / 1e9,
                    "grouped": {"problems": len(copies), "ms_per_problem": g_ms,
                                "gbs": g_gbs, "frac_hbm": g_gbs / hbm}}
            if M <= 2:
                # one problem per grouped call, the calls one after another
                s_ms = time_rotation([lambda c=c: bn.bitnet_gemv_fused_grouped(
                    [xd], [c], [swd], [out]) for c in copies])
                s_gbs = call_bytes(M, K, N) / s_ms / 1e6
                case["grouped_single"] = {"ms": s_ms, "gbs": s_gbs, "frac_hbm": s_gbs / hbm}
            case["cublas_bf16"] = cublas_bf16(ms, xd, wb_copies, N)
            cases.append(case)
        del copies, wb_copies
    bn.bitnet_device_status()
    return {"workload": "LLaMA-7B projections 4096->4096, 4096->11008, 11008->4096 at "
                        "M in {1, 4, 8, 15} through bitnet_gemv_fused, one call at a time, "
                        "and the same problems as one bitnet_gemv_fused_grouped call; cublas_bf16 is "
                        "the same layer as a dense bf16 torch.mm (speedup = its time / ours)",
            "l2": "weights rotated over copies totalling more than 2x L2",
            "peak_hbm_gbs": hbm, "cases": cases}


def eager_calls(bn, dev, reps=200):
    """Per-call cost of eager (not graph-captured) calls through the C ABI:
    `issue_us` is the host time per call of `reps` back-to-back calls (the
    library's own host work, plus a ctypes call from Python), and
    `latency_us` the wall clock of one call followed by a stream
    synchronisation (median)."""
    import ctypes
    L = bn.lib()
    P = ctypes.c_void_p
    st = P(torch.cuda.current_stream(dev).cuda_stream)
    res = {}
    K, N = 4096, 4096
    w = synth.ternary(synth.key(W.W_LLAMA_GEMV, 1, synth.T_WEIGHT, 0), N, K)
    wp = bn.bitnet_pack_weights(torch.from_numpy(w).to(dev))
    sw = torch.full((1,), 0.05, dtype=torch.float32, device=dev)
    cases = []
    for M in (1, 15):
        x = torch.randn((M, K), generator=torch.Generator().manual_seed(M)).to(dev, torch.bfloat16)
        out = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
        args = (P(out.data_ptr()), P(x.data_ptr()), 0, P(wp.data_ptr()), P(sw.data_ptr()), 1, M,
                N, K, st)
        cases.append((f"bitnet_gemv_fused M={M} {K}->{N}", L.bitnet_gemv_fused, args))
    for M in (64,):
        xq = torch.randint(-127, 128, (M, K), dtype=torch.int8, device=dev)
        sa = torch.full((M,), 0.01, dtype=torch.bfloat16, device=dev)
        out = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
        args = (P(out.data_ptr()), P(xq.data_ptr()), P(wp.data_ptr()), P(sa.data_ptr()),
                P(sw.data_ptr()), 1, M, N, K, st)
        cases.append((f"bitnet_gemm M={M} {K}->{N}", L.bitnet_gemm, args))
    for name, fn, args in cases:
        for _ in range(10):
            assert fn(*args) == 0
        torch.cuda.synchronize(dev)
        t0 = time.perf_counter()
        for _ in range(reps):
            fn(*args)
        t1 = time.perf_counter()
        torch.cuda.synchronize(dev)
        lat = []
        for _ in range(50):
            t2 = time.perf_counter()
            fn(*args)
            torch.cuda.current_stream(dev).synchronize()
            lat.append(time.perf_counter() - t2)
        res[name] = {"issue_us": (t1 - t0) / reps * 1e6,
                     "latency_us": statistics.median(lat) * 1e6}
    bn.bitnet_device_status()
    return res


def midbatch(bn, dev, pk):
    """M in {32, 64, 128, 256}, K=4096, N in {4096, 11008} through bitnet_gemm
    on pre-quantised activations; each case against the roof that applies
    (HBM bytes or tensor ops, whichever takes longer)."""
    hbm = pk["hbm_gbs"]
    tops_peak = pk["bf16_tflops"] * INT8_OVER_BF16
    cases = []
    for K, N in W.MIDBATCH_SHAPES:
        w = synth.ternary(synth.key(W.W_MIDBATCH, 0, synth.T_WEIGHT, N), N, K)
        wd = torch.from_numpy(w).to(dev)
        copies = weight_rotation(bn.bitnet_pack_weights(wd))
        wb_copies = bf16_rotation(wd)
        del w, wd
        swd = torch.from_numpy(synth.scale_wt(synth.key(W.W_MIDBATCH, 0, synth.T_SCALE_WT, N))).to(dev)
        for M in W.MIDBATCH_M:
            x = synth.act_bf16(synth.key(W.W_MIDBATCH, M, synth.T_ACT, N), M, K, outliers=False)
            xd = torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).to(dev)
            xq, sa = bn.bitnet_quantize_act(xd)
            out = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
            ms = time_rotation([lambda c=c: bn.bitnet_gemm(xq, c, sa, swd, out=out)
                                for c in copies])
            ops = 2.0 * M * N * K
            byts = N * K // 4 + M * K + 2 * M + 2 * M * N + 4
            t_hbm, t_tc = byts / hbm / 1e6, ops / tops_peak / 1e9
            cases.append({"M": M, "K": K, "N": N, "ms": ms, "tops": ops / ms / 1e9,
                          "gbs": byts / ms / 1e6,
                          "bound": "hbm" if t_hbm >= t_tc else "tensor",
                          "frac": max(t_hbm, t_tc) / ms,
                          "cublas_bf16": cublas_bf16(ms, xd, wb_copies, N)})
        del copies, wb_copies
    bn.bitnet_device_status()
    return {"workload": "M in {32, 64, 128, 256} x K=4096 x N in {4096, 11008} through "
                        "bitnet_gemm (pre-quantised int8 + bf16 scales); cublas_bf16 is the "
                        "same layer as a dense bf16 torch.mm (speedup = its time / ours)",
            "l2": "weights rotated over copies totalling more than 2x L2",
            "peak_hbm_gbs": hbm, "peak_tops": tops_peak, "cases": cases}


def extra_rows(bn, dev, pk):
    """The rows beyond the layer itself: absmean ternarisation of a dense
    float32 matrix (11008 x 4096, per row and per tensor; 180 MB read, 45 MB
    written, plus the per-tensor form's second read), the layer on float32
    activations (decode GEMV at M = 1, bitnet_linear at M = 2048), the
    fused bias epilogue (bitnet_linear with and without bias at M = 2048),
    and RMSNorm before the quantiser (alone at M = 2048; bitnet_linear_rmsnorm
    at M = 2048 and M = 1, each beside the same call without the norm)."""
    hbm = pk["hbm_gbs"]
    tops_peak = pk["bf16_tflops"] * INT8_OVER_BF16
    flush = L2Flush(dev)

    def timed(fn, graph=True):
        return time_flushed(fn, flush, 5, graph)

    out = {}
    N, K = 11008, 4096
    g = torch.Generator(device=dev)
    g.manual_seed(7)
    w = torch.randn((N, K), device=dev, generator=g) * 0.02
    wt = torch.empty((N, K), dtype=torch.int8, device=dev)
    for per_row, name in ((True, "ternarize_per_row"), (False, "ternarize_per_tensor")):
        sc = torch.empty((N if per_row else 1,), dtype=torch.float32, device=dev)
        ms = timed(lambda: bn.bitnet_ternarize_absmean(w, per_row=per_row, w_t=wt, scale_wt=sc),
                   graph=False)  # the call synchronises for its value check
        byts = N * K * 4 * (1 if per_row else 2) + N * K + 4 * sc.numel()
        out[name] = {"N": N, "K": K, "ms": ms, "gbs": byts / ms / 1e6,
                     "frac_hbm": byts / ms / 1e6 / hbm,
                     "note": "includes the call's synchronisation for the value check"}
    del w, wt
    wp = bn.bitnet_pack_weights(torch.ones((N, K), dtype=torch.int8, device=dev))
    copies = weight_rotation(wp)
    sw = torch.tensor([0.05], dtype=torch.float32, device=dev)
    x1 = torch.randn((1, K), device=dev, generator=g)
    o1 = torch.empty((1, N), dtype=torch.bfloat16, device=dev)
    ms = time_rotation([lambda c=c: bn.bitnet_gemv_fused(x1, c, sw, out=o1) for c in copies])
    byts = N * K // 4 + 4 * K + 2 * N + 4
    out["gemv_f32_m1"] = {"M": 1, "K": K, "N": N, "ms": ms, "gbs": byts / ms / 1e6,
                          "frac_hbm": byts / ms / 1e6 / hbm}
    del copies
    M = 2048
    xl = torch.randn((M, K), device=dev, generator=g)
    ol = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    ws = torch.empty((bn.bitnet_linear_workspace_bytes(M, K),), dtype=torch.uint8, device=dev)
    ms = timed(lambda: bn.bitnet_linear(xl, wp, sw, out=ol, workspace=ws))
    ops = 2.0 * M * N * K
    out["linear_f32_m2048"] = {"M": M, "K": K, "N": N, "ms": ms, "tops": ops / ms / 1e9,
                               "frac": ops / ms / 1e9 / tops_peak}
    # the fused bias epilogue, against the same bf16 call without it
    bias = (torch.randn((N,), device=dev, generator=g) * 0.1).to(torch.bfloat16)
    xb = xl.to(torch.bfloat16)
    ms_plain = timed(lambda: bn.bitnet_linear(xb, wp, sw, out=ol, workspace=ws))
    ms_bias = timed(lambda: bn.bitnet_linear(xb, wp, sw, out=ol, workspace=ws, bias=bias))
    out["linear_bias_m2048"] = {"M": M, "K": K, "N": N, "ms": ms_bias, "ms_without_bias": ms_plain,
                                "tops": ops / ms_bias / 1e9, "frac": ops / ms_bias / 1e9 / tops_peak}
    # RMSNorm before the quantiser: alone (x read, codes written), in front
    # of the prefill GEMM, and in front of the decode GEMV
    gn = (1.0 + 0.1 * torch.randn((K,), device=dev, generator=g)).to(torch.bfloat16)
    xq = torch.empty((M, K), dtype=torch.int8, device=dev)
    sa = torch.empty((M,), dtype=torch.bfloat16, device=dev)
    ms = timed(lambda: bn.bitnet_rmsnorm_quantize_act(xb, gn, 1e-6, x_q=xq, scale_act=sa))
    byts = 2 * M * K + 2 * K + M * K + 2 * M
    out["rmsnorm_quant_m2048"] = {"M": M, "K": K, "ms": ms, "gbs": byts / ms / 1e6,
                                  "frac_hbm": byts / ms / 1e6 / hbm}
    wsn = torch.empty((bn.bitnet_linear_rmsnorm_workspace_bytes(M, K),), dtype=torch.uint8,
                      device=dev)
    ms = timed(lambda: bn.bitnet_linear_rmsnorm(xb, gn, 1e-6, wp, sw, out=ol, workspace=wsn))
    out["linear_rmsnorm_m2048"] = {"M": M, "K": K, "N": N, "ms": ms, "ms_without_norm": ms_plain,
                                   "tops": ops / ms / 1e9, "frac": ops / ms / 1e9 / tops_peak}
    del xl, ol, xq
    copies = weight_rotation(wp)
    xd = torch.randn((1, K), device=dev, generator=g).to(torch.bfloat16)
    ws1 = torch.empty((bn.bitnet_linear_rmsnorm_workspace_bytes(1, K),), dtype=torch.uint8,
                      device=dev)
    ms_norm = time_rotation([lambda c=c: bn.bitnet_linear_rmsnorm(xd, gn, 1e-6, c, sw, out=o1,
                                                                  workspace=ws1) for c in copies])
    ms_plain1 = time_rotation([lambda c=c: bn.bitnet_gemv_fused(xd, c, sw, out=o1) for c in copies])
    byts = N * K // 4 + 2 * K + 2 * N + 4
    out["linear_rmsnorm_m1"] = {"M": 1, "K": K, "N": N, "ms": ms_norm, "ms_without_norm": ms_plain1,
                                "gbs": byts / ms_norm / 1e6, "frac_hbm": byts / ms_norm / 1e6 / hbm}
    del copies
    bn.bitnet_device_status()
    return out


# ----------------------------------------------------------- CPU oracle

def cpu_baseline(seconds):
    """The scalar oracle on the host cores: layer 0's seven decode calls,
    repeated for about `seconds` s, in GB/s of the same algorithmic bytes."""
    import oracle
    threads = os.cpu_count() or 1
    calls = [c for c in sweep_calls() if c[0] == 0]
    prepared = []
    for layer, variant, K, N in calls:
        w = synth.ternary(synth.key(W.W_DECODE_2B, layer, synth.T_WEIGHT, variant), N, K)
        p = oracle.pack(w)
        sw = synth.scale_wt(synth.key(W.W_DECODE_2B, layer, synth.T_SCALE_WT, variant))
        x = synth.act_bf16(synth.key(W.W_DECODE_2B, layer, synth.T_ACT, variant), 1, K)
        prepared.append((x, p, sw, call_bytes(1, K, N)))
    t0 = time.perf_counter()
    nbytes = 0
    reps = 0
    while True:
        for x, p, sw, b in prepared:
            oracle.linear_cols_threads(x, p, sw, threads)
            nbytes += b
        reps += 1
        if time.perf_counter() - t0 >= seconds:
            break
    dt = time.perf_counter() - t0
    return {"value": nbytes / dt / 1e9, "unit": UNIT, "cores": threads, "kind": "oracle",
            "sample": f"decode layer 0 (7 BitLinears, {nbytes // reps / 1e6:.1f} MB packed) x {reps}, "
                      f"M=1, columns split over {threads} threads, {dt:.1f} s"}


# --------------------------------------------------------- profiling aid

def run_case(bn, dev, case, reps=3):
    """Small, self-contained invocations for ncu captures (one kernel kind,
    a few launches, inputs larger than L2, well under a few GB)."""
    if case == "decode_once":
        d = build_decode(bn, dev, 0)
        make_sweep(bn, d, "grouped")()
    elif case in ("midbatch", "gemv_m15"):
        # one few-row GEMM (M = 64, 4096 -> 11008, pre-quantised) or one fused
        # tensor-core GEMV (M = 15, 11008 -> 4096), weights larger than L2
        # across the repetitions' copies
        M, K, N = (64, 4096, 11008) if case == "midbatch" else (15, 11008, 4096)
        w = synth.ternary(synth.key(W.W_MIDBATCH, M, synth.T_WEIGHT, N), N, K)
        wp = bn.bitnet_pack_weights(torch.from_numpy(w).to(dev))
        copies = weight_rotation(wp)
        x = synth.act_bf16(synth.key(W.W_MIDBATCH, M, synth.T_ACT, N), M, K)
        xd = torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).to(dev)
        sw = torch.tensor([0.05], dtype=torch.float32, device=dev)
        out = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
        if case == "midbatch":
            xq, sa = bn.bitnet_quantize_act(xd)
            for r in range(reps):
                bn.bitnet_gemm(xq, copies[r % len(copies)], sa, sw, out=out)
        else:
            for r in range(reps):
                bn.bitnet_gemv_fused(xd, copies[r % len(copies)], sw, out=out)
    elif case == "rmsnorm":
        # RMSNorm + quantiser over M = 2048 rows of K = 4096 (16.8 MB in)
        M, K = 2048, 4096
        x = synth.act_bf16(synth.key(W.W_PREFILL, M, synth.T_ACT, K), M, K)
        xd = torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).to(dev)
        g = torch.ones((K,), dtype=torch.bfloat16, device=dev)
        xq = torch.empty((M, K), dtype=torch.int8, device=dev)
        sa = torch.empty((M,), dtype=torch.bfloat16, device=dev)
        for _ in range(reps):
            bn.bitnet_rmsnorm_quantize_act(xd, g, 1e-6, x_q=xq, scale_act=sa)
    elif case == "lm_head":
        _, K, N = W.DECODE_2B_LM_HEAD
        w = synth.ternary(synth.key(W.W_DECODE_2B, W.DECODE_2B_LAYERS, synth.T_WEIGHT, 7), N, K)
        wp = bn.bitnet_pack_weights(torch.from_numpy(w).to(dev))
        x = synth.act_bf16(synth.key(W.W_DECODE_2B, W.DECODE_2B_LAYERS, synth.T_ACT, 7), 1, K)
        xd = torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).to(dev)
        sw = torch.tensor([0.05], dtype=torch.float32, device=dev)
        for _ in range(reps):
            bn.bitnet_gemv_fused(xd, wp, sw)
    else:
        M, (K, N) = max(W.PREFILL_M), W.PREFILL_SHAPES[0]
        x = synth.act_bf16(synth.key(W.W_PREFILL, M, synth.T_ACT, K), M, K)
        w = synth.ternary(synth.key(W.W_PREFILL, M, synth.T_WEIGHT, K), N, K)
        xd = torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).to(dev)
        wp = bn.bitnet_pack_weights(torch.from_numpy(w).to(dev))
        sw = torch.tensor([0.05], dtype=torch.float32, device=dev)
        for _ in range(reps):
            bn.bitnet_linear(xd, wp, sw)
    torch.cuda.synchronize()
    bn.bitnet_device_status()


# ----------------------------------------------------------------- main

def main():
    args = parse()
    rank, world, local = dist_env()
    config = {"workload": "bitnet-b1.58-2B decode sweep, M=1: 30 layers x 7 BitLinears "
                          "(2560->2560, 2560->640 x2, 2560->2560, 2560->6912 x2, 6912->2560) "
                          "+ LM head 2560->128256",
              "calls_per_step": len(W.decode_2b_sweep()),
              "packed_weight_bytes_per_step": W.decode_2b_packed_bytes(),
              "l2": "inputs larger than L2 (603 MB of packed weights streamed per step)",
              "issue_order": "the 211 independent problems (each has its own activation "
                             "row) as one bitnet_gemv_fused_grouped call; 'issue_orders' "
                             f"reports them as separate calls on {args.branches} graph "
                             "branches, in transformer-layer dependency order, and on a "
                             "single stream",
              "parallelism": f"replicas x{world}" if world > 1 else "single GPU"}

    if args.impl == "reference":
        if rank != 0:
            return 0
        cb = cpu_baseline(max(1.0, args.cpu_seconds / 2))
        per_step_s = W.decode_2b_packed_bytes() / (cb["value"] * 1e9)
        line = {"impl": "reference", "metric": METRIC, "value": cb["value"], "unit": UNIT,
                "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
                "ms_per_step": per_step_s * 1e3, "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "int8",
                "data": "synthetic (seeded, shaped like the pages' workloads)",
                "config": config, "cpu_baseline": cb,
                "e2e": {"value": cb["value"], "unit": UNIT, "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}}
        print(json.dumps(line))
        return 0

    import bit_gemm_bitnet_b200 as bn
    bn.lib()
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    if args.case:
        run_case(bn, dev, args.case)
        return 0

    pg = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)
        pg = dist

    def barrier():
        if pg is not None:
            pg.barrier()

    pk = peaks()
    d = build_decode(bn, dev, rank)
    d2 = second_buffers(d, dev)
    stream = torch.cuda.Stream(device=dev)
    graphs = {}
    with torch.cuda.stream(stream):
        sweep2 = make_sweep(bn, d2, "grouped")
        sweep2()
        g2 = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g2, stream=stream):
            sweep2()
        torch.cuda.synchronize()
        for order in ("grouped", "layer_grouped", "independent", "layer", "stream"):
            sweep = make_sweep(bn, d, order, branches=args.branches)
            sweep()
            torch.cuda.synchronize()
            bn.bitnet_device_status()
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                sweep()
            torch.cuda.synchronize()
            graphs[order] = g
        with ClockSampler(local) as clk:
            total_ms, per = time_graph(graphs["grouped"], args.steps, args.warmup, barrier)
        e2e_ms = time_e2e([graphs["grouped"], g2], [d, d2], args.steps, args.warmup, barrier)
        other = {}
        for order in ORDERS:
            t_ms, _ = time_graph(graphs[order], args.steps, args.warmup, barrier)
            other[order] = t_ms
    bn.bitnet_device_status()

    if pg is not None:
        vals = max_over_ranks([total_ms, e2e_ms] + [other[o] for o in ORDERS], dev)
        total_ms, e2e_ms = vals[0], vals[1]
        other = dict(zip(ORDERS, vals[2:]))

    ms_step = total_ms / args.steps
    value = whole_job_gbs(d["bytes"], world, args.steps, total_ms)
    e2e_val = whole_job_gbs(d["bytes"], world, args.steps, e2e_ms)
    per_rank_gbs = d["bytes"] / (ms_step / 1e3) / 1e9
    clocks = clk.summary()
    lm = lm_head_alone(bn, d, dev)
    pre = None if args.no_prefill else prefill(bn, dev, pk)
    gemv_mb = None if args.no_secondary else llama_gemv(bn, dev, pk)
    mid = None if args.no_secondary else midbatch(bn, dev, pk)
    extra = None if args.no_secondary else extra_rows(bn, dev, pk)
    eager = None if args.no_secondary else eager_calls(bn, dev)

    if rank != 0:
        if pg is not None:
            pg.destroy_process_group()
        return 0
    cb = None if args.no_cpu_baseline or world > 1 else cpu_baseline(args.cpu_seconds)
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "int8", "data": "synthetic (seeded; shapes and distributions of the pages' workloads)",
        "config": config,
        "roofline": {"bound": "hbm", "achieved": per_rank_gbs, "peak": pk["hbm_gbs"],
                     "unit": "GB/s", "frac": per_rank_gbs / pk["hbm_gbs"],
                     "peak_source": f"{pk['source']} hbm_gbs",
                     "kernel": "gemv_grouped_kernel (one launch per step)",
                     "traffic": recorded_traffic("gemv_grouped_kernel"),
                     "traffic_per": "one step, as achieved"},
        "cpu_baseline": cb,
        "e2e": {"value": e2e_val, "unit": UNIT,
                "h2d_bytes_per_step": int(d["x_host"].numel() * 2),
                "d2h_bytes_per_step": int(d["out_host"].numel() * 2)},
        "gpu_launches": args.steps,  # one grouped launch per step
        "clocks": clocks,
        "step_ms_min_median": [min(per), statistics.median(per)],
        "decode_layer_order": {
            "what": "the same 211 problems in a transformer layer's dependency order on one "
                    "stream: Q|K|V grouped, O, gate|up grouped, down; layers in sequence, LM "
                    "head last (121 launches per step, chained by programmatic dependent launch)",
            "ms_per_step": other["layer_grouped"] / args.steps,
            "gbs": whole_job_gbs(d["bytes"], world, args.steps, other["layer_grouped"]),
            "frac_hbm": whole_job_gbs(d["bytes"], 1, args.steps, other["layer_grouped"])
            / pk["hbm_gbs"]},
        "issue_orders": {
            o: {"ms_per_step": other[o] / args.steps,
                "gbs": whole_job_gbs(d["bytes"], world, args.steps, other[o])}
            for o in ORDERS},
        "lm_head_alone": {**lm, "frac": lm["gbs"] / pk["hbm_gbs"]},
        "prefill": pre,
        "llama_gemv": gemv_mb,
        "midbatch": mid,
        "extra_rows": extra,
        "eager_calls": eager,
    }
    print(json.dumps(line))
    if pg is not None:
        pg.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
