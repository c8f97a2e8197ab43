#!/usr/bin/env python
"""LC-VQ 2-bit hot-path benchmark (one JSON line on rank 0).

Headline workload: decode-GEMV, d_in = d_out = 4096, d = 8, M in {1, 4, 16}
bf16 tokens.  One step = one lcvq_gemm call per token count (the X-transform
prologue plus the decode-GEMV kernel each), every call on the next of R
rotated copies of the packed weights (R x 4 MiB > 4 x L2, so each call streams
its codes from HBM).  value = packed-weight bytes of all calls on all ranks /
max-over-ranks device time.

The other hot-path rows (assign/pack, decode, prefill GEMM in both forms, the
QAT step, the 7B-shaped stack) are measured after the headline and reported
under "rows", each with its own metric and roofline.

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                       [--rows all|none|name,...]
Multi-GPU: launched by torch.distributed.run, one process per GPU; ranks run
independent replicas (no collective in the data path) -> "scaling": "weak".
"""

from __future__ import annotations

import argparse
import json
import math
import os
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from bit_weight_only_lcvq_b200 import lcvq, synth  # noqa: E402
from bit_weight_only_lcvq_b200.replicas import Replicas as Dist  # noqa: E402

METRIC = "LC-VQ 2-bit GEMM: packed-weight GB/s (M≤16), TFLOP/s (prefill), % roofline"
MIB = 1 << 20
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# ----------------------------------------------------------------------------- setup
def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=20000)
    p.add_argument("--warmup", type=int, default=50)
    p.add_argument("--impl", choices=("ours", "reference"), default="ours")
    p.add_argument("--rows", default="all")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--stack-layers", type=int, default=32,
                   help="decoder layers of the stack row (32 = the 7B-shaped workload)")
    p.add_argument("--stack-ms", default="1,8,32", help="token counts of the stack row")
    return p.parse_args()


# DRAM bytes (dram__bytes_read.sum + dram__bytes_write.sum) of one decode-GEMV
# call (its X-transform and its GEMV) per token count, from one ncu capture of
# this benchmark's step, valid only for the kernel sources that were captured:
# keyed by the SHA-1 of each source file.
NCU_TRAFFIC = {
    "sources": {  # source file -> sha1 of the file when captured
        "bit_weight_only_lcvq_b200/csrc/gemv.cu": "6074f6c9d5883e9919885a90763e905cf566ca8b",
        "bit_weight_only_lcvq_b200/csrc/xform.cu": "33924e415c51beeb9df1fbfdc54cc3e3444c2cb2",
    },
    # token count -> bytes per call (X-transform + GEMV), mean over the captured calls
    "per_call": {1: 4292085, 4: 4341372, 16: 4513084},
}


def traffic_for(key):
    import hashlib
    if not NCU_TRAFFIC["sources"]:
        return None
    for src_rel, sha in NCU_TRAFFIC["sources"].items():
        try:
            h = hashlib.sha1(open(os.path.join(ROOT, src_rel), "rb").read()).hexdigest()
        except OSError:
            return None
        if h != sha:
            return None  # a kernel changed since the counters were taken
    return NCU_TRAFFIC["per_call"].get(key)


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled during a timed region."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        # nvidia-smi numbers GPUs physically; address ours by UUID so a
        # CUDA_VISIBLE_DEVICES remap cannot point the sampler at another GPU
        try:
            self.idx = "GPU-" + str(torch.cuda.get_device_properties(gpu_index).uuid)
        except Exception:
            vis = os.environ.get("CUDA_VISIBLE_DEVICES", "")
            self.idx = vis.split(",")[gpu_index] if vis else str(gpu_index)
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.idx}", f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                 "-lms", "50"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.3)

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.1)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        with open(self.path) as f:
            for ln in f:
                parts = [x.strip() for x in ln.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"], "samples": 0}
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        reasons = set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for r in rows:
            for nm, v in zip(names, r[5:9]):
                if v.lower() == "active":
                    reasons.add(nm)
        return {"sm_mhz": float(np.median(sm)) if sm else None,
                "sm_max_mhz": max(mx) if mx else None,
                "reasons": sorted(reasons), "samples": len(rows)}


def ev_time(fn, n, stream=None):
    """Average device time (ms) of fn() over n calls, CUDA events on the stream."""
    s = stream or torch.cuda.current_stream()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    e0.record(s)
    for _ in range(n):
        fn()
    e1.record(s)
    e1.synchronize()
    return e0.elapsed_time(e1) / n


def graph_time(fn, n, reps=3):
    """Device time (ms) per call of fn(), from a CUDA graph of n back-to-back
    calls replayed `reps` times: no host overhead between the kernels (a
    Python-level call costs tens of microseconds, more than a short kernel)."""
    g = capture(lambda: [fn() for _ in range(n)])
    g.replay()
    torch.cuda.synchronize()
    ms = ev_time(g.replay, reps)
    del g
    return ms / n


def capture(fn):
    """CUDA graph of fn() (the library launches on torch's current stream, which
    is the capture stream inside the context)."""
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        fn()
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fn()
    torch.cuda.synchronize()
    return g


class StepGraphs:
    """K steps as graph replays: one graph holds `chunk` consecutive steps and a
    second one the remainder, so exactly K steps run.  `step()` launches one
    step and returns the number of library kernels it launched."""

    def __init__(self, step, chunk: int, k: int):
        self.step = step
        self.chunk = max(1, min(chunk, k))
        self.q, self.rem = divmod(k, self.chunk)
        self.g_full, self.n_full = self._capture(self.chunk)
        self.g_rem, self.n_rem = self._capture(self.rem) if self.rem else (None, 0)

    def _capture(self, n):
        box = [0]

        def run():
            box[0] = 0
            for _ in range(n):
                box[0] += self.step()
        g = capture(run)
        return g, box[0]

    def replay(self) -> int:
        for _ in range(self.q):
            self.g_full.replay()
        if self.g_rem is not None:
            self.g_rem.replay()
        return self.q * self.n_full + self.n_rem

    def prime(self):
        """Launch each captured graph once, untimed: a graph's first launch
        uploads it to the device, which must not fall inside a timed region."""
        self.g_full.replay()
        if self.g_rem is not None:
            self.g_rem.replay()
        torch.cuda.synchronize()


def timed_graphs(D, sg: StepGraphs, sampler=None):
    """Barrier + sync on both sides; returns (max-over-ranks ms, launches, clocks).
    The graphs are primed (launched once) before the timed region."""
    sg.prime()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    if sampler:
        sampler.start()
    D.barrier()
    torch.cuda.synchronize()
    e0.record()
    launches = sg.replay()
    e1.record()
    torch.cuda.synchronize()
    D.barrier()
    ck = sampler.stop() if sampler else None
    return D.max(e0.elapsed_time(e1)), launches, ck


# ----------------------------------------------------------------------------- oracle legs
def _oracle():
    """The C++ fp64 oracle (plain loops, one thread per output row range)."""
    from oracle import cpp as C
    C.lib()
    return C


def _timed_loop(fn, seconds):
    """Calls fn() until `seconds` have passed (at least once); (calls, seconds)."""
    t0 = time.perf_counter()
    n = 0
    while True:
        fn()
        n += 1
        dt = time.perf_counter() - t0
        if dt >= seconds:
            return n, dt


def oracle_gemv_sample(Ms, seconds=10.0, threads=1):
    """The C++ oracle on the decode-GEMV workload (4096 x 4096, d = 8): Y and
    its normaliser for the three token counts, single-threaded, over as many
    full passes as fit in ~`seconds`."""
    C = _oracle()
    w = synth.workload(2, M=max(Ms), with_dy=False)
    from oracle import lcvq_oracle as O
    packed = O.pack_codes(O.assign(w["Wp"])[0])
    X = w["X"].astype(np.float64)

    def step():
        for M in Ms:
            C.forward_packed(X[:M], packed, 4096, w["A"], w["B"], threads=threads)
    passes, dt = _timed_loop(step, seconds)
    packed_bytes = passes * len(Ms) * (4096 * 4096 // 4)
    return dict(value=packed_bytes / dt / 1e9, unit="GB/s", cores=threads, kind="oracle",
                sample=f"{passes} full passes of d_in=d_out=4096, d=8 at M={list(Ms)} by the C++ "
                       f"fp64 oracle (decode, Y and its normaliser) on {threads} thread(s), "
                       f"{dt:.1f} s")


def oracle_reference_arm(Ms, steps, warmup, budget_s=60.0):
    """The reference arm: the C++ fp64 oracle itself, timed as steps on all host
    cores.  A step is one pass over the three token counts on the decode-GEMV
    workload, on all 4096 output rows when K + W such passes fit in ~budget_s,
    otherwise on the first `rows` rows (a bounded sample; the metric counts the
    packed bytes of the rows computed).  W untimed steps, then K timed ones."""
    C = _oracle()
    from oracle import lcvq_oracle as O
    threads = C.default_threads()
    w = synth.workload(2, M=max(Ms), with_dy=False)
    packed = O.pack_codes(O.assign(w["Wp"])[0])
    X = w["X"].astype(np.float64)
    t0 = time.perf_counter()
    for M in Ms:
        C.forward_packed(X[:M], packed, 4096, w["A"], w["B"], threads=threads)
    full_s = max(time.perf_counter() - t0, 1e-3)
    rows = 4096
    if (steps + warmup) * full_s > budget_s:
        rows = max(16, int(4096 * budget_s / ((steps + warmup) * full_s)) // 16 * 16)
    ps = np.ascontiguousarray(packed[:rows])

    def step():
        for M in Ms:
            C.forward_packed(X[:M], ps, 4096, w["A"], w["B"], threads=threads)

    for _ in range(warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(steps):
        step()
    dt = time.perf_counter() - t0
    packed_bytes = steps * len(Ms) * (rows * 4096 // 4)
    return dict(value=packed_bytes / dt / 1e9, unit="GB/s", cores=threads, kind="oracle",
                ms_per_step=dt / max(steps, 1) * 1e3,
                sample=f"{steps} timed steps after {warmup} untimed, each the {rows} x 4096 rows of "
                       f"d=8 codes at M={list(Ms)} (C++ fp64 oracle: decode, Y and its normaliser; "
                       f"{threads} threads), {dt:.1f} s")


# ----------------------------------------------------------------------------- headline
def _sum_or_none(xs):
    return None if any(x is None for x in xs) else float(sum(xs))


def headline(args, D: Dist, pk):
    K = N = 4096
    d = 8
    Ms = (1, 4, 16)
    dev = D.dev
    w = synth.workload(2, M=max(Ms), with_dy=False)
    Wp = torch.from_numpy(w["Wp"]).to(dev)
    packed0, _ = lcvq.assign_pack(Wp, d, with_mask=False)
    del Wp
    L2 = torch.cuda.get_device_properties(dev).L2_cache_size
    R = max(8, math.ceil(4 * L2 / (N * K // 4)))
    copies = [packed0.clone() for _ in range(R)]
    A = torch.from_numpy(w["A"]).to(dev)
    B = torch.from_numpy(w["B"]).to(dev)
    X = {M: torch.from_numpy(w["X"][:M].copy()).to(torch.bfloat16).to(dev) for M in Ms}
    Y = {M: torch.empty((M, N), dtype=torch.bfloat16, device=dev) for M in Ms}
    ws = {M: lcvq.new_workspace(lcvq.workspace_size(lcvq.OP_GEMM, torch.bfloat16, M, N, K, d), dev)
          for M in Ms}

    ctr = [0]

    def step():
        n = 0
        for M in Ms:
            r = ctr[0] % R
            ctr[0] += 1
            lcvq.gemm(X[M], copies[r], K, A, B, d, out=Y[M], workspace=ws[M])
            n += lcvq.last_launch_count()
        return n

    chunk = R  # one graph = R steps (every copy is visited 3 times)
    warm = StepGraphs(step, chunk, max(args.warmup, 3))
    warm.replay()
    sg = StepGraphs(step, chunk, args.steps)
    ms_total, launches, ck = timed_graphs(D, sg, ClockSampler(dev.index))
    per_step_bytes = len(Ms) * (N * K // 4)
    value = D.world * args.steps * per_step_bytes / (ms_total * 1e-3) / 1e9

    # the decode-GEMV call per token count, back to back (its X-transform and
    # its GEMV overlap under programmatic dependent launch, so the call, not
    # one of its two kernels, is what a CUDA event can time)
    per_m = {}
    for M in Ms:
        kc = [0]

        def kstep(M=M, kc=kc):
            lcvq.gemm(X[M], copies[kc[0] % R], K, A, B, d, out=Y[M], workspace=ws[M])
            kc[0] += 1
            return lcvq.last_launch_count()
        n = 4 * R
        g = StepGraphs(kstep, R, n)
        g.replay()
        t, _, _ = timed_graphs(D, g)
        per_m[M] = t / n
    kern_ms = sum(per_m.values())
    achieved = per_step_bytes / (kern_ms * 1e-3) / 1e9
    hbm = pk["hbm_gbs"]

    # context: the bf16 GEMV kernel alone (lcvq_gemm_xformed on a pre-transformed
    # X'', back to back; launched on its own it waits before it loads codes)
    xpp, corr = {}, {}
    for M in Ms:
        xpp[M], corr[M] = lcvq.xform(X[M], A, B, d)
    alone = {}
    for M in Ms:
        kc = [0]

        def astep(M=M, kc=kc):
            lcvq.gemm_xformed(xpp[M], corr[M], copies[kc[0] % R], out=Y[M])
            kc[0] += 1
            return lcvq.last_launch_count()
        n = 4 * R
        g = StepGraphs(astep, R, n)
        g.replay()
        t, _, _ = timed_graphs(D, g)
        alone[M] = t / n
    alone_gbs = per_step_bytes / (sum(alone.values()) * 1e-3) / 1e9

    # end to end through the public API with pinned host buffers.  Each step's
    # inputs (all token counts) go in with one host-to-device copy and its
    # outputs come back with one device-to-host copy, pipelined like a serving
    # loop: step i+1's input copy (h2d stream) and step i-1's output copy (d2h
    # stream) overlap step i's kernels; inputs and outputs are double buffered.
    rows = sum(Ms)
    offs, o = {}, 0
    for M in Ms:
        offs[M] = o
        o += M
    Xh = torch.cat([X[M].cpu() for M in Ms]).pin_memory()
    Xd = [torch.empty((rows, K), dtype=torch.bfloat16, device=dev) for _ in range(2)]
    Yd = [torch.empty((rows, N), dtype=torch.bfloat16, device=dev) for _ in range(2)]
    Yh = [torch.empty((rows, N), dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    h2d_s = torch.cuda.Stream(device=dev)
    d2h_s = torch.cuda.Stream(device=dev)
    e2e_chunk = R
    e2e_steps = max(2 * e2e_chunk, min(args.steps, 4 * R)) // e2e_chunk * e2e_chunk

    def e2e_chunk_fn():
        """e2e_chunk pipelined steps; every forked stream joins back at the end."""
        main = torch.cuda.current_stream()
        n = 0
        d2h_done = [None, None]
        h2d_s.wait_stream(main)
        with torch.cuda.stream(h2d_s):
            Xd[0].copy_(Xh, non_blocking=True)
        for i in range(e2e_chunk):
            b = i % 2
            main.wait_stream(h2d_s)                    # X of step i has arrived
            if i + 1 < e2e_chunk:
                h2d_s.wait_stream(main)                # step i-1 no longer reads Xd[1-b]
                with torch.cuda.stream(h2d_s):
                    Xd[1 - b].copy_(Xh, non_blocking=True)
            if d2h_done[b] is not None:
                main.wait_event(d2h_done[b])           # Yd[b] of step i-2 has left
            for M in Ms:
                r = ctr[0] % R
                ctr[0] += 1
                lcvq.gemm(Xd[b][offs[M]:offs[M] + M], copies[r], K, A, B, d,
                          out=Yd[b][offs[M]:offs[M] + M], workspace=ws[M])
                n += lcvq.last_launch_count()
            d2h_s.wait_stream(main)
            with torch.cuda.stream(d2h_s):
                Yh[b].copy_(Yd[b], non_blocking=True)
                ev = torch.cuda.Event()
                ev.record(d2h_s)
            d2h_done[b] = ev
        main.wait_stream(h2d_s)
        main.wait_stream(d2h_s)
        return n

    ge = StepGraphs(e2e_chunk_fn, 1, e2e_steps // e2e_chunk)
    ge.replay()
    e2e_ms, _, _ = timed_graphs(D, ge)
    e2e = dict(value=D.world * e2e_steps * per_step_bytes / (e2e_ms * 1e-3) / 1e9, unit="GB/s",
               h2d_bytes_per_step=int(sum(M * K * 2 for M in Ms)),
               d2h_bytes_per_step=int(sum(M * N * 2 for M in Ms)),
               note="each step copies its X (all token counts) in from pinned host memory in one "
                    "copy and its Y back in one copy, inside the timed graph; the copies of "
                    "neighbouring steps overlap a step's kernels on two copy streams")

    res = dict(
        metric=METRIC, value=value, unit="GB/s", n_gpus=D.world, steps=args.steps,
        warmup=args.warmup, ms_per_step=ms_total / args.steps, higher_is_better=True,
        scaling="weak", vs_baseline=None, dtype="bf16",
        data="synthetic (seeded: W_p ~ U[-0.5,3.5] -> uniform codes; X ~ N(0,1), 1% channels x20)",
        config={"workload": "decode_gemv d_in=4096 d_out=4096 d=8 M={1,4,16} bf16",
                "l2": f"inputs larger than L2: {R} rotated packed-weight copies ({R * 4} MiB)",
                "parallelism": f"replicas x{D.world}" if D.world > 1 else "single GPU"},
        roofline=dict(bound="hbm", achieved=achieved, peak=hbm, unit="GB/s", frac=achieved / hbm,
                      traffic=_sum_or_none([traffic_for(M) for M in Ms]),
                      traffic_unit="bytes per step (3 calls, each an X-transform and a GEMV)",
                      kernel="decode-GEMV call: X-transform + gemv_group_kernel (int8 path "
                             "at M = 1, 4; bf16 at M = 16), M = 1, 4, 16 summed",
                      launch="lcvq_gemm back to back per token count, graph replay, rotated "
                             "weights",
                      per_m_us={str(M): per_m[M] * 1e3 for M in Ms},
                      bf16_gemv_alone=dict(per_m_us={str(M): alone[M] * 1e3 for M in Ms},
                                           achieved=alone_gbs, frac=alone_gbs / hbm,
                                           note="context: lcvq_gemm_xformed's bf16 GEMV kernel "
                                                "alone, without its X-transform"),
                      peak_source=f"{PEAK_SRC} hbm_gbs"),
        e2e=e2e, clocks=ck, gpu_launches=int(launches),
    )
    return res


# ----------------------------------------------------------------------------- other rows
def _roof(bound, achieved, peak, unit, **kw):
    return dict(bound=bound, achieved=achieved, peak=peak, unit=unit, frac=achieved / peak, **kw)


# fp32 FMA peak: 148 SMs x 128 fp32 lanes x 2 flops x 1965 MHz (the maximum SM clock)
FP32_ALU_TFLOPS = 148 * 128 * 2 * 1965e6 / 1e12
FP32_SRC = "derived: 148 SMs x 128 fp32 FMA/clk x 2 x 1965 MHz"


def row_single_layer(D, pk, cpu=True):
    """Single linear layer, fp32 (d_in = d_out = 512, d = 4, M = 16): the
    forward Y = X W~ and the straight-through backward (dX, dA, dB, dWp), on the
    CUDA cores (fp32 activations).  Work: 3 x 2 M N K flops."""
    dev = D.dev
    M, K, N, d = 16, 512, 512, 4
    w = synth.workload(1)
    Wp = torch.from_numpy(w["Wp"]).to(dev)
    packed, mask = lcvq.assign_pack(Wp, d)
    A = torch.from_numpy(w["A"]).to(dev)
    B = torch.from_numpy(w["B"]).to(dev)
    X = torch.from_numpy(w["X"]).to(dev)
    dY = torch.from_numpy(w["dY"]).to(dev)
    Y = torch.empty((M, N), device=dev)
    wsf = lcvq.new_workspace(lcvq.workspace_size(lcvq.OP_GEMM, torch.float32, M, N, K, d), dev)
    wsb = lcvq.new_workspace(lcvq.workspace_size(lcvq.OP_GEMM_BACKWARD, torch.float32, M, N, K, d), dev)
    outs = dict(dX=torch.empty((M, K), device=dev), dWp=torch.empty((N, K), device=dev),
                dA=torch.empty((d, d), device=dev), dB=torch.empty((d,), device=dev))

    def step():
        lcvq.gemm(X, packed, K, A, B, d, out=Y, workspace=wsf)
        lcvq.gemm_backward(X, dY, packed, mask, K, A, B, d, outs=outs, workspace=wsb)
    ms = graph_time(step, 50)
    flops = 3 * 2.0 * M * N * K
    tf = flops / (ms * 1e-3) / 1e12
    out = dict(metric="single-layer fp32 forward + STE backward TFLOP/s (3 x 2MNK / time)",
               value=tf, unit="TFLOP/s", us=ms * 1e3,
               roofline=_roof("alu", tf, FP32_ALU_TFLOPS, "TFLOP/s", peak_source=FP32_SRC))
    if cpu:
        C = _oracle()
        from oracle import lcvq_oracle as O
        z, m = O.assign(w["Wp"])

        def ostep():
            C.forward(w["X"], z, w["A"], w["B"], threads=1)
            C.backward(w["X"], w["dY"], z, m, w["A"], w["B"], threads=1)
        n, dt = _timed_loop(ostep, 2.0)
        out["cpu_baseline"] = dict(value=n * flops / dt / 1e12, unit="TFLOP/s", cores=1,
                                   kind="oracle", sample=f"{n} full forward + backward passes of the "
                                   f"layer by the C++ fp64 oracle on 1 thread, {dt:.1f} s")
    return out


def row_assign_pack(D, pk):
    """Assign + pack (+ mask) on the QAT-step weights: 4096 x 14336 fp32."""
    dev = D.dev
    N, K = 4096, 14336
    w = synth.workload(4, M=1, with_dy=False)
    Wp = torch.from_numpy(w["Wp"]).to(dev)
    packed = torch.empty((N, K // 4), dtype=torch.uint8, device=dev)
    mask = torch.empty((N, K // 8), dtype=torch.uint8, device=dev)
    ms = graph_time(lambda: lcvq.assign_pack(Wp, 8, packed=packed, mask=mask), 20)
    nbytes = N * K * (4 + 0.25 + 0.125)
    gbs = nbytes / (ms * 1e-3) / 1e9
    return dict(metric="assign+pack GB/s (fp32 in, codes+mask out)", value=gbs, unit="GB/s",
                us=ms * 1e3,
                roofline=dict(bound="hbm", achieved=gbs, peak=pk["hbm_gbs"], unit="GB/s",
                              frac=gbs / pk["hbm_gbs"]))


def row_decode(D, pk):
    dev = D.dev
    N, K = 4096, 14336
    w = synth.workload(4, M=1, with_dy=False)
    packed, _ = lcvq.assign_pack(torch.from_numpy(w["Wp"]).to(dev), 8, with_mask=False)
    A = torch.from_numpy(w["A"]).to(dev)
    B = torch.from_numpy(w["B"]).to(dev)
    W = torch.empty((N, K), dtype=torch.bfloat16, device=dev)
    ms = graph_time(lambda: lcvq.decode(packed, K, A, B, 8, out=W), 20)
    nbytes = N * K * (0.25 + 2)
    gbs = nbytes / (ms * 1e-3) / 1e9
    return dict(metric="decode GB/s (codes in, bf16 W~ out)", value=gbs, unit="GB/s", us=ms * 1e3,
                roofline=dict(bound="hbm", achieved=gbs, peak=pk["hbm_gbs"], unit="GB/s",
                              frac=gbs / pk["hbm_gbs"]))


def row_prefill(D, pk, cpu=True):
    """Prefill GEMM, d_in=4096 -> d_out=11008, M=2048, both forward forms."""
    dev = D.dev
    M, K, N, d = 2048, 4096, 11008, 8
    w = synth.workload(3, M=M, with_dy=False)
    packed, _ = lcvq.assign_pack(torch.from_numpy(w["Wp"]).to(dev), d, with_mask=False)
    A = torch.from_numpy(w["A"]).to(dev)
    B = torch.from_numpy(w["B"]).to(dev)
    X = torch.from_numpy(w["X"]).to(torch.bfloat16).to(dev)
    Y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    ws = lcvq.new_workspace(lcvq.workspace_size(lcvq.OP_GEMM, torch.bfloat16, M, N, K, d), dev)
    out = {}
    flops = 2.0 * M * N * K
    for form in ("algebraic", "decode"):
        call = lambda: lcvq.gemm(X, packed, K, A, B, d, form=form, out=Y, workspace=ws)
        for _ in range(2):  # warm-up: first-launch costs stay out of the timing
            call()
        ms = ev_time(call, 5)
        tf = flops / (ms * 1e-3) / 1e12
        out[form] = dict(value=tf, unit="TFLOP/s", us=ms * 1e3,
                         roofline=_roof("tensor", tf, pk["bf16_tflops"], "TFLOP/s"))
    res = dict(metric="prefill GEMM TFLOP/s (2MNK / time)", forms=out)
    if cpu:  # the oracle on the first `rows` output rows, all host cores
        C = _oracle()
        from oracle import lcvq_oracle as O
        rows = 128
        pkd = O.pack_codes(O.assign(w["Wp"][:rows])[0])
        Xd = w["X"].astype(np.float64)
        n, dt = _timed_loop(lambda: C.forward_packed(Xd, pkd, K, w["A"], w["B"]), 3.0)
        res["cpu_baseline"] = dict(value=n * 2.0 * M * rows * K / dt / 1e12, unit="TFLOP/s",
                                   cores=C.default_threads(), kind="oracle",
                                   sample=f"{n} passes of the first {rows} of {N} output rows "
                                          f"(M={M}, K={K}) by the C++ fp64 oracle (Y and its "
                                          f"normaliser), {dt:.1f} s")
    return res


def row_qat(D, pk, cpu=True):
    """QAT step on d_in=14336, d_out=4096, M=8192: assign/pack, forward, backward."""
    dev = D.dev
    M, K, N, d = 8192, 14336, 4096, 8
    w = synth.workload(4, M=M)
    Wp = torch.from_numpy(w["Wp"]).to(dev)
    A = torch.from_numpy(w["A"]).to(dev)
    B = torch.from_numpy(w["B"]).to(dev)
    X = torch.from_numpy(w["X"]).to(torch.bfloat16).to(dev)
    dY = torch.from_numpy(w["dY"]).to(torch.bfloat16).to(dev)
    packed = torch.empty((N, K // 4), dtype=torch.uint8, device=dev)
    mask = torch.empty((N, K // 8), dtype=torch.uint8, device=dev)
    Y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    wsf = lcvq.new_workspace(lcvq.workspace_size(lcvq.OP_GEMM, torch.bfloat16, M, N, K, d), dev)
    wsb = lcvq.new_workspace(lcvq.workspace_size(lcvq.OP_GEMM_BACKWARD, torch.bfloat16, M, N, K, d), dev)
    outs = dict(dX=torch.empty((M, K), dtype=torch.bfloat16, device=dev),
                dWp=torch.empty((N, K), dtype=torch.float32, device=dev),
                dA=torch.empty((d, d), dtype=torch.float32, device=dev),
                dB=torch.empty((d,), dtype=torch.float32, device=dev))
    ap = lambda: lcvq.assign_pack(Wp, d, packed=packed, mask=mask)
    fw = lambda: lcvq.gemm(X, packed, K, A, B, d, out=Y, workspace=wsf)
    bw = lambda: lcvq.gemm_backward(X, dY, packed, mask, K, A, B, d, outs=outs, workspace=wsb)
    for f in (ap, fw, bw):  # warm-up: first-launch costs stay out of the timing
        f()
    # burst: each stage timed alone over a few calls (about 1 ms each)
    t_ap = ev_time(ap, 3)
    t_fw = ev_time(fw, 3)
    t_bw = ev_time(bw, 3)
    gemm_flops = 2.0 * M * N * K
    total = t_ap + t_fw + t_bw
    tf = 3 * gemm_flops / (total * 1e-3) / 1e12

    # sustained: whole steps back to back for about 3 s
    def step():
        ap()
        fw()
        bw()
    n_sus = max(3, int(math.ceil(3000.0 / total)))
    t_sus = ev_time(step, n_sus)
    tf_sus = 3 * gemm_flops / (t_sus * 1e-3) / 1e12
    res = dict(metric="QAT step TFLOP/s (3 x 2MNK / step time)", value=tf, unit="TFLOP/s",
               step_us=total * 1e3, assign_pack_us=t_ap * 1e3, forward_us=t_fw * 1e3,
               backward_us=t_bw * 1e3,
               roofline=_roof("tensor", tf, pk["bf16_tflops"], "TFLOP/s",
                              timing="burst: each stage over 3 calls after a warm-up call"),
               sustained=dict(value=tf_sus, unit="TFLOP/s", step_us=t_sus * 1e3, steps=n_sus,
                              roofline=_roof("tensor", tf_sus, pk["bf16_tflops_sustained"],
                                             "TFLOP/s", timing=f"{n_sus} whole steps back to back")))
    if cpu:  # the oracle's forward + backward on the first `rows` output rows, all host cores
        C = _oracle()
        from oracle import lcvq_oracle as O
        rows = 16
        z, m = O.assign(w["Wp"][:rows])
        Xd, dYd = w["X"].astype(np.float64), np.ascontiguousarray(w["dY"][:, :rows], np.float64)

        def ostep():
            C.forward(Xd, z, w["A"], w["B"])
            C.backward(Xd, dYd, z, m, w["A"], w["B"])
        n, dt = _timed_loop(ostep, 3.0)
        res["cpu_baseline"] = dict(value=n * 3 * 2.0 * M * rows * K / dt / 1e12, unit="TFLOP/s",
                                   cores=C.default_threads(), kind="oracle",
                                   sample=f"{n} forward + backward passes of the first {rows} of "
                                          f"{N} output rows (M={M}, K={K}) by the C++ fp64 "
                                          f"oracle (with normalisers), {dt:.1f} s")
    return res


def row_stack(D, pk, layers=32, ms=(1, 8, 32), cpu=True):
    """7B-shaped stack: 224 matrices, M in {1, 8, 32}; packed GB/s over the stack
    (fewer layers or token counts only for a profiler capture)."""
    dev = D.dev
    mats = []
    for layer in range(layers):
        for p in range(len(synth.STACK_PROJS)):
            m = synth.stack_matrix(layer, p, max(ms), with_x=(layer == 0))
            mats.append(m)
    total_bytes = sum(m["packed"].nbytes for m in mats)
    dmats = []
    xs = {}
    for m in mats:
        key = (m["proj"], m["d_in"])
        if m["layer"] == 0:
            xs[m["proj"]] = torch.from_numpy(m["X"]).to(torch.bfloat16).to(dev)
        dmats.append(dict(packed=torch.from_numpy(m["packed"]).to(dev), A=torch.from_numpy(m["A"]).to(dev),
                          B=torch.from_numpy(m["B"]).to(dev), proj=m["proj"], d_in=m["d_in"],
                          d_out=m["d_out"]))
    # decoder-layer phases: matrices of one phase read the same input and are
    # independent (q, k, v | o | gate, up | down)
    phases = (("q", "k", "v"), ("o",), ("gate", "up"), ("down",))
    out = {}
    for M in ms:
        ys = {p: torch.empty((M, do), dtype=torch.bfloat16, device=dev) for p, _, do in synth.STACK_PROJS}
        wss = {p: lcvq.new_workspace(lcvq.workspace_size(lcvq.OP_GEMM, torch.bfloat16, M, do, di, 8), dev)
               for p, di, do in synth.STACK_PROJS}

        def run_seq(M=M, ys=ys, wss=wss):
            n = 0
            for m in dmats:
                lcvq.gemm(xs[m["proj"]][:M], m["packed"], m["d_in"], m["A"], m["B"], 8,
                          out=ys[m["proj"]], workspace=wss[m["proj"]])
                n += lcvq.last_launch_count()
            return n

        # one grouped call per phase (4 per layer)
        by_layer = [dmats[i:i + len(synth.STACK_PROJS)] for i in range(0, len(dmats), len(synth.STACK_PROJS))]
        phase_jobs = []
        for layer in by_layer:
            named = {m["proj"]: m for m in layer}
            for ph in phases:
                phase_jobs.append([(xs[p][:M], named[p]["packed"], named[p]["A"], named[p]["B"],
                                    named[p]["d_in"]) for p in ph])
        ph_outs = [[ys[p] for p in ph] for ph in phases] * len(by_layer)
        ph_ws = lcvq.new_workspace(max(lcvq.workspace_size_grouped(j, M, 8) for j in phase_jobs), dev)

        def run_phase(phase_jobs=phase_jobs, ph_outs=ph_outs, ph_ws=ph_ws):
            n = 0
            for jobs, outs in zip(phase_jobs, ph_outs):
                lcvq.gemm_grouped(jobs, 8, workspace=ph_ws, outs=outs)
                n += lcvq.last_launch_count()
            return n

        # the whole stack as one grouped call (independent inputs per matrix)
        all_jobs = [(xs[m["proj"]][:M], m["packed"], m["A"], m["B"], m["d_in"]) for m in dmats]
        all_outs = [torch.empty((M, m["d_out"]), dtype=torch.bfloat16, device=dev) for m in dmats]
        all_ws = lcvq.new_workspace(lcvq.workspace_size_grouped(all_jobs, M, 8), dev)

        def run_all(all_jobs=all_jobs, all_outs=all_outs, all_ws=all_ws):
            lcvq.gemm_grouped(all_jobs, 8, workspace=all_ws, outs=all_outs)
            return lcvq.last_launch_count()

        res_m = {}
        for name, fn in (("sequential", run_seq), ("grouped_by_phase", run_phase),
                         ("grouped_all", run_all)):
            sg = StepGraphs(fn, 1, 5)
            sg.replay()
            t, launches, _ = timed_graphs(D, sg)
            ms_pass = t / 5
            gbs = total_bytes / (ms_pass * 1e-3) / 1e9
            res_m[name] = dict(value=gbs, unit="GB/s", us=ms_pass * 1e3, launches_per_pass=launches // 5,
                               roofline=dict(bound="hbm", achieved=gbs, peak=pk["hbm_gbs"], unit="GB/s",
                                             frac=gbs / pk["hbm_gbs"]))
            del sg
        # parity of the grouped paths against the sequential one, bitwise, on the last layer
        torch.cuda.synchronize()
        run_seq()
        torch.cuda.synchronize()
        seq_last = {p: ys[p].clone() for p, _, _ in synth.STACK_PROJS}
        run_all()
        torch.cuda.synchronize()
        pairs_ = [(all_outs[len(dmats) - len(synth.STACK_PROJS) + i], seq_last[p])
                  for i, (p, _, _) in enumerate(synth.STACK_PROJS)]
        res_m["grouped_vs_sequential"] = dict(
            bitwise_equal=all(torch.equal(a, b) for a, b in pairs_),
            max_rel_diff=max(float((a.float() - b.float()).abs().max() / b.float().abs().max())
                             for a, b in pairs_))
        out[str(M)] = res_m
        del all_ws, all_outs, ph_ws
        torch.cuda.empty_cache()
    res = dict(metric=f"stack packed-weight GB/s ({len(dmats)} matrices, "
                      f"{total_bytes / 1e9:.2f} GB of codes)",
               note="sequential: 224 lcvq_gemm calls; grouped_by_phase: one lcvq_gemm_grouped per "
                    "decoder-layer phase (q,k,v | o | gate,up | down), 128 calls; grouped_all: the "
                    "224 independent matrices in one lcvq_gemm_grouped call",
               per_m=out, packed_bytes=total_bytes)
    if cpu:  # the oracle on one decoder layer (7 matrices) per token count, all host cores
        C = _oracle()
        layer = [m for m in mats if m["layer"] == 0]
        lbytes = sum(m["packed"].nbytes for m in layer)
        cb = {}
        for M in ms:
            def ostep(M=M):
                for m in layer:
                    C.forward_packed(m["X"][:M].astype(np.float64), m["packed"], m["d_in"],
                                     m["A"], m["B"])
            n, dt = _timed_loop(ostep, 1.0)
            cb[str(M)] = n * lbytes / dt / 1e9
        res["cpu_baseline"] = dict(value=cb, unit="GB/s", cores=C.default_threads(), kind="oracle",
                                   sample="one decoder layer (q,k,v,o,gate,up,down: "
                                          f"{lbytes / 1e6:.0f} MB of codes) per token count by the "
                                          "C++ fp64 oracle (decode, Y and its normaliser), ~1 s each")
    return res


def row_fit(D, pk, cpu=True):
    """Least-squares (A, B) refit on the QAT-step matrix (4096 x 14336, d = 8):
    W0 = the workload's proxy weights, codes = their assignment; unweighted and
    with per-channel weights h."""
    dev = D.dev
    N, K, d = 4096, 14336, 8
    w = synth.workload(4, M=1, with_dy=False)
    W0 = torch.from_numpy(w["Wp"]).to(dev)
    packed, _ = lcvq.assign_pack(W0, d, with_mask=False)
    h = torch.rand(K, device=dev, generator=torch.Generator(device=dev).manual_seed(3)) + 0.5
    ws = lcvq.new_workspace(lcvq.workspace_size(lcvq.OP_FIT_AFFINE, torch.float32, 0, N, K, d), dev)
    A = torch.empty((d, d), device=dev)
    B = torch.empty(d, device=dev)
    nbytes = N * K * (4 + 0.25)
    out = {}
    for name, hh in (("unweighted", None), ("weighted", h)):
        ms = graph_time(lambda: lcvq.fit_affine(W0, packed, d, h=hh, workspace=ws, A=A, B=B), 10)
        gbs = nbytes / (ms * 1e-3) / 1e9
        out[name] = dict(value=gbs, unit="GB/s", us=ms * 1e3,
                         roofline=dict(bound="hbm", achieved=gbs, peak=pk["hbm_gbs"], unit="GB/s",
                                       frac=gbs / pk["hbm_gbs"]))
    res = dict(metric="(A, B) refit GB/s (W0 fp32 + codes read)", forms=out)
    if cpu:  # the numpy oracle's normal equations and solve on the first `rows` rows
        from oracle import lcvq_oracle as O
        rows = 256
        W0s = w["Wp"][:rows].astype(np.float64)
        zs = O.assign(w["Wp"][:rows])[0]
        n, dt = _timed_loop(lambda: O.fit_affine(W0s, zs, d), 2.0)
        res["cpu_baseline"] = dict(value=n * rows * K * 4.25 / dt / 1e9, unit="GB/s",
                                   cores=_blas_threads(), kind="oracle",
                                   sample=f"{n} unweighted refits of the first {rows} of {N} rows "
                                          f"by the numpy fp64 oracle, {dt:.1f} s")
    return res


def row_fit_h(D, pk, cpu=True):
    """Least-squares (A, B) refit under the full input Hessian on a 4096 x 4096
    matrix (d = 8) with an 8192-row calibration Hessian (outlier recipe, 1%
    ridge) formed on the device before timing.  The call's work is dominated by
    one tensor-core contraction of 2 (K + 64)(3 K + 64) N flops (the code Gram
    and the targets times the codes); value = those flops / the whole call."""
    dev = D.dev
    N = K = 4096
    d = 8
    g = np.random.Generator(np.random.PCG64(2500))
    z = g.integers(0, 4, size=(N, K), dtype=np.uint8)
    A0, B0 = synth.affine_diag_dominant(d, g)
    zt = torch.from_numpy(z).to(dev)
    W0 = (torch.from_numpy(A0).to(dev) @ zt.view(N, K // d, d).float().transpose(1, 2)).transpose(1, 2)
    W0 = (W0 + torch.from_numpy(B0).to(dev)).reshape(N, K).contiguous()
    W0 += 0.005 * torch.randn((N, K), device=dev, generator=torch.Generator(device=dev).manual_seed(1))
    packed, _ = lcvq.assign_pack(zt.float(), d, with_mask=False)
    w = synth.ldlq_workload(N, K, d, n_cal=8192)
    X = torch.from_numpy(w["Xcal"]).to(dev, torch.float64)
    H64 = X.T @ X / X.shape[0]
    H64 += 0.01 * H64.diagonal().mean() * torch.eye(K, dtype=torch.float64, device=dev)
    H = H64.float().contiguous()
    del X, H64
    ws = lcvq.new_workspace(lcvq.workspace_size(lcvq.OP_FIT_AFFINE_H, torch.float32, 0, N, K, d), dev)
    A = torch.empty((d, d), device=dev)
    B = torch.empty(d, device=dev)
    ms = graph_time(lambda: lcvq.fit_affine_h(W0, packed, d, H, workspace=ws, A=A, B=B), 5)
    flops = 2.0 * (K + 64) * (3 * K + 64) * N
    tf = flops / (ms * 1e-3) / 1e12
    res = dict(metric="(A, B) refit under the full Hessian TFLOP/s (2 (K+64)(3K+64) N / call time)",
               value=tf, unit="TFLOP/s", us=ms * 1e3,
               roofline=_roof("tensor", tf, pk["bf16_tflops"], "TFLOP/s",
                              note="whole call (operand pass, Gram GEMM, fp64 contraction, solve)"))
    if cpu:  # the numpy oracle's normal equations and solve on the first `rows` rows
        from oracle import lcvq_oracle as O
        rows = 256
        W0h = W0[:rows].cpu().numpy().astype(np.float64)
        Hh = H.cpu().numpy().astype(np.float64)
        n, dt = _timed_loop(lambda: O.fit_affine_h(W0h, z[:rows], d, Hh), 3.0)
        res["cpu_baseline"] = dict(value=n * 2.0 * (K + 64) * (3 * K + 64) * rows / dt / 1e12,
                                   unit="TFLOP/s", cores=_blas_threads(), kind="oracle",
                                   sample=f"{n} refits of the first {rows} of {N} rows by the numpy "
                                          f"fp64 oracle, {dt:.1f} s")
    return res


def row_ldlq(D, pk, cpu=True):
    """H-aware sequential code assignment on a 4096 x 4096 matrix (d = 8): the
    code-space factor of a calibration Hessian (8192 activation rows, outlier
    recipe, 1% damping) is formed on the device in fp64 before timing."""
    dev = D.dev
    N = K = 4096
    d = 8
    w = synth.ldlq_workload(N, K, d)
    X = torch.from_numpy(w["Xcal"]).to(dev, torch.float64)
    H = X.T @ X / X.shape[0]
    H += 0.01 * H.diagonal().mean() * torch.eye(K, dtype=torch.float64, device=dev)
    Abar = torch.kron(torch.eye(K // d, dtype=torch.float64, device=dev),
                      torch.from_numpy(w["A"]).to(dev, torch.float64))
    Q = Abar.T @ H @ Abar
    V = torch.linalg.cholesky(Q.flip(0, 1)).flip(0, 1)  # Q = V V^T, V upper triangular
    U = (V / V.diagonal()[None, :]).triu(1).float().contiguous()
    del X, H, Abar, Q, V
    P = torch.from_numpy(w["P"]).to(dev)
    packed = torch.empty((N, K // 4), dtype=torch.uint8, device=dev)
    ws = lcvq.new_workspace(lcvq.workspace_size(lcvq.OP_ASSIGN_LDLQ, torch.float32, 0, N, K, d), dev)
    lcvq.assign_ldlq(P, U, d, workspace=ws, packed=packed)
    ms = ev_time(lambda: lcvq.assign_ldlq(P, U, d, workspace=ws, packed=packed), 10)
    tf = N * K * (K - 1) / (ms * 1e-3) / 1e12
    res = dict(metric="H-aware assignment TFLOP/s (N K (K-1) / time: fp32 FMA, 2 flops each)",
               value=tf, unit="TFLOP/s", us=ms * 1e3,
               roofline=_roof("alu", tf, FP32_ALU_TFLOPS, "TFLOP/s", peak_source=FP32_SRC))
    if cpu:  # the numpy oracle's sequential rule on the first `rows` rows
        from oracle import lcvq_oracle as O
        rows = 8
        Ph = w["P"][:rows]
        Uh = U.cpu().numpy()
        n, dt = _timed_loop(lambda: O.ldlq_assign(Ph, Uh), 2.0)
        res["cpu_baseline"] = dict(value=n * rows * K * (K - 1) / dt / 1e12, unit="TFLOP/s",
                                   cores=_blas_threads(), kind="oracle",
                                   sample=f"{n} runs on the first {rows} of {N} rows by the numpy "
                                          f"fp64 oracle, {dt:.1f} s")
    return res


def _blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        return max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    except Exception:  # pragma: no cover
        return os.cpu_count() or 1


ROWS = {"single_layer": row_single_layer, "assign_pack": row_assign_pack, "decode": row_decode,
        "prefill": row_prefill, "qat": row_qat, "stack": row_stack, "fit": row_fit,
        "fit_h": row_fit_h, "ldlq": row_ldlq}
CPU_ROWS = ("single_layer", "prefill", "qat", "stack", "fit", "fit_h", "ldlq")


def row_summary(name, r) -> str:
    """One short line per row (printed to stderr next to the JSON line)."""
    def fr(x):
        rf = x.get("roofline") or {}
        return f"{x['value']:.4g} {x['unit']} ({100 * rf.get('frac', float('nan')):.1f}% of {rf.get('peak')})"
    if "error" in r:
        return f"row {name}: ERROR {r['error']}"
    parts = []
    if "forms" in r:
        parts += [f"{k}: {fr(v)}" for k, v in r["forms"].items()]
    elif "per_m" in r:
        for M, arr in r["per_m"].items():
            parts += [f"M={M} {a}: {fr(v)}" for a, v in arr.items() if "value" in v]
    else:
        parts.append(fr(r))
    if "sustained" in r:
        parts.append(f"sustained: {fr(r['sustained'])}")
    cb = r.get("cpu_baseline")
    if cb:
        parts.append(f"oracle: {cb['value'] if isinstance(cb['value'], dict) else round(cb['value'], 6)} "
                     f"{cb['unit']} on {cb['cores']} core(s)")
    return f"row {name}: " + "; ".join(parts)


# ----------------------------------------------------------------------------- main
def main():
    global PEAK_SRC
    args = parse()
    pk, PEAK_SRC = peaks()
    if args.impl == "reference":
        D_rank = int(os.environ.get("RANK", "0"))
        if D_rank != 0:
            return 0
        cb = oracle_reference_arm((1, 4, 16), args.steps, args.warmup)
        ms_step = cb.pop("ms_per_step")
        line = dict(impl="reference", metric=METRIC, value=cb["value"], unit="GB/s",
                    n_gpus=int(os.environ.get("WORLD_SIZE", "1")), steps=args.steps,
                    warmup=args.warmup, ms_per_step=ms_step, higher_is_better=True,
                    scaling="weak", vs_baseline=None,
                    dtype="f64", data="synthetic",
                    config={"workload": "decode_gemv d_in=4096 d_out=4096 d=8 M={1,4,16} bf16"},
                    cpu_baseline=cb,
                    e2e=dict(value=cb["value"], unit="GB/s", h2d_bytes_per_step=0, d2h_bytes_per_step=0))
        print(json.dumps(line))
        return 0

    if not torch.cuda.is_available():  # the product path has no CPU fallback
        print("bench.py: no CUDA device; the library's kernels need a B200 "
              "(--impl reference times the CPU oracle)", file=sys.stderr)
        return 2
    D = Dist()
    res = headline(args, D, pk)
    if D.rank == 0 and D.world == 1 and not args.no_cpu_baseline:
        res["cpu_baseline"] = oracle_gemv_sample((1, 4, 16), seconds=10.0)
    rows = {}
    want = list(ROWS) if args.rows == "all" else ([] if args.rows == "none" else args.rows.split(","))
    if D.rank == 0:
        cpu = D.world == 1 and not args.no_cpu_baseline
        for name in want:
            try:
                if name == "stack":
                    rows[name] = row_stack(D, pk, args.stack_layers,
                                           tuple(int(m) for m in args.stack_ms.split(",")), cpu=cpu)
                elif name in CPU_ROWS:
                    rows[name] = ROWS[name](D, pk, cpu=cpu)
                else:
                    rows[name] = ROWS[name](D, pk)
            except Exception as ex:  # report, do not hide
                rows[name] = {"error": f"{type(ex).__name__}: {ex}"}
            torch.cuda.empty_cache()
            print(row_summary(name, rows[name]), file=sys.stderr, flush=True)
    res["rows"] = rows
    if D.rank == 0:
        print(json.dumps(res))
    D.close()
    return 0


PEAK_SRC = "measured"

if __name__ == "__main__":
    sys.exit(main())
