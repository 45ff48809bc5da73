"""Benchmark of the GGUF block-quantized matmul path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl kq|reference]
                    [--workload NAME] [--no-rows]

Default workload (the headline line): decode qmv, M=1, N=14336, K=4096, one
q8_0 and one q6_K weight matrix per step (the Llama-3-8B FFN up-projection
shape).  A step runs both products on one batch of synthetic input already
resident in HBM; `value` is effective weight GB/s (packed weight bytes read
per step / step time), summed over ranks.  Steps cycle over enough distinct
weight copies that the bytes touched between reuses exceed the L2 cache.

The JSON line also carries:
  roofline      the dominant kernel's algorithmic bytes / its CUDA-event time
  e2e           the same metric through the C ABI with host buffers: pinned
                host -> device copy of the step's weights and activations,
                the kernels, device -> host copy of the result, all timed
  cpu_baseline  the CPU oracle on a bounded sample of the workload (rank 0)
  rows          every other row of the hot path (the encoder, dequantize, qmv at M up to
                16, tcgen05 qmm, MoE sort + tile map + gather, the unsort +
                score mix, the decode MoE gather_qmv and gate/up GLU) on its
                own workload:
                kernel time, GB/s or TFLOP/s, roofline fraction
  clocks        SM clock median and throttle reasons sampled while timing

With --gpus N under torchrun every rank runs an independent replica of the
workload (the path has no exchange step); times are the max over ranks.
`--impl reference` times the CPU oracle as the reference arm.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

METRIC = "qmv effective weight GB/s (% of HBM peak); qmm/gather_qmm TFLOP/s (% bf16 peak)"
Q8_0, Q4_K, Q6_K = synth.Q8_0, synth.Q4_K, synth.Q6_K
Q5_K, Q4_0 = synth.Q5_K, synth.Q4_0
L2_BYTES = 126 * 2**20


# --------------------------------------------------------------------- helpers
def peaks() -> dict:
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained", d["bf16_tflops"]), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


# source files that define the device code of the kernel behind each roofline
# tag (its translation unit and the shared device header; host-only launch
# declarations do not change what the kernel does)
KERNEL_SOURCES = {
    "qmv_q8_0_m1_14336x4096": ("kq_qmv_stream.cu", "kq_device.cuh"),
    "qmv_q6_K_m1_14336x4096": ("kq_qmv_stream.cu", "kq_device.cuh"),
}


def _code_only(text: str) -> str:
    """C/CUDA source without its comments and with whitespace collapsed, so that
    an edit of comments alone keeps a kernel's hash (string literals are kept)."""
    out, i, n = [], 0, len(text)
    while i < n:
        c = text[i]
        if c == '"':
            j = i + 1
            while j < n and text[j] != '"':
                j += 2 if text[j] == "\\" else 1
            out.append(text[i:j + 1])
            i = j + 1
        elif text.startswith("//", i):
            j = text.find("\n", i)
            i = n if j < 0 else j
        elif text.startswith("/*", i):
            j = text.find("*/", i + 2)
            i = n if j < 0 else j + 2
        else:
            out.append(c)
            i += 1
    return " ".join("".join(out).split())


def kernel_source_hash(tag: str | None = None) -> str:
    """Hash of the kernel sources' code (of one roofline tag's kernel, or of all)."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "gguf_quant_dequant_q4_b200", "csrc")
    files = KERNEL_SOURCES.get(tag) if tag else None
    for f in sorted(files or os.listdir(csrc)):
        h.update(_code_only(open(os.path.join(csrc, f), encoding="utf-8", errors="replace").read()).encode())
    return h.hexdigest()[:16]


def profiled_traffic(kernel_tag: str):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on
    the current sources of that kernel (profiles/*.txt lines 'traffic <tag> <bytes> <hash>')."""
    d = os.path.join(ROOT, "profiles")
    if not os.path.isdir(d):
        return None
    cur = kernel_source_hash(kernel_tag)
    for f in sorted(os.listdir(d)):
        if not f.endswith((".txt", ".md")):
            continue
        for line in open(os.path.join(d, f)):
            m = re.match(r"\s*traffic\s+(\S+)\s+(\d+)\s+([0-9a-f]+)", line)
            if m and m.group(1) == kernel_tag and m.group(3) == cur:
                return int(m.group(2))
    return None


class Clocks:
    """nvidia-smi sampler running while the timed region runs."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index, self.proc, self.lines = index, None, []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.Q}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *a):
        if self.proc:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self) -> dict:
        mhz, maxes, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for l in self.lines:
            f = [x.strip() for x in l.split(",")]
            if len(f) < 9:
                continue
            try:
                mhz.append(float(f[1]))
                maxes.append(float(f[2]))
            except ValueError:
                continue
            for nm, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(nm)
        if not mhz:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(mhz), "sm_max_mhz": max(maxes), "reasons": sorted(reasons),
                "samples": len(mhz)}


# ------------------------------------------------------------- distributed
class Dist:
    def __init__(self):
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.rank = int(os.environ.get("RANK", "0"))
        self.local = int(os.environ.get("LOCAL_RANK", "0"))
        self.pg = None

    def init(self, backend: str):
        if self.world > 1:
            import datetime
            import torch.distributed as dist
            dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
            self.pg = dist

    def barrier(self):
        if self.pg:
            self.pg.barrier()

    def max(self, v: float, device=None) -> float:
        if not self.pg:
            return v
        import torch
        t = torch.tensor([v], dtype=torch.float64, device=device)
        self.pg.all_reduce(t, op=self.pg.ReduceOp.MAX)
        return float(t.item())

    def close(self):
        if self.pg:
            self.pg.destroy_process_group()


def replica_value(units_per_rank: float, world: int, max_seconds: float) -> float:
    """Whole-job throughput: every rank processes units_per_rank in max_seconds."""
    return units_per_rank * world / max_seconds


# ----------------------------------------------------------------- GPU arm
def run_kq(args, dist: Dist) -> dict | None:
    import torch
    import gguf_quant_dequant_q4_b200 as kq

    torch.cuda.set_device(dist.local)
    dev = torch.device("cuda", dist.local)
    pk = peaks()

    def u8(a):
        return torch.from_numpy(np.ascontiguousarray(a)).to(dev)

    def bf(bits):
        return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).to(dev).view(torch.bfloat16)

    # ---- headline workload: c1 q8_0 + q6_K qmv, M=1, N=14336, K=4096
    n, k = 14336, 4096
    w8 = synth.weights(Q8_0, n, k)
    w6 = synth.weights(Q6_K, n, k)
    x = synth.activations(1, k)
    bytes_step = w8.nbytes + w6.nbytes
    copies = max(2, -(-3 * L2_BYTES // bytes_step))
    W8 = [u8(w8) for _ in range(copies)]
    W6 = [u8(w6) for _ in range(copies)]
    X = bf(x)
    Y8 = torch.empty(1, n, device=dev)
    Y6 = torch.empty(1, n, device=dev)
    steps, warm = args.steps, args.warmup
    s = torch.cuda.Stream(device=dev)

    def step(i):
        c = i % copies
        kq.qmv(X, W8[c], Q8_0, out=Y8)
        kq.qmv(X, W6[c], Q6_K, out=Y6)

    with torch.cuda.stream(s):
        for i in range(warm):
            step(i)
    s.synchronize()
    # the timed graph holds the K steps back to back (consecutive kernels stay
    # adjacent, so programmatic dependent launch overlaps them) between two
    # events on the launching stream
    t0, t1 = torch.cuda.Event(enable_timing=True, external=True), torch.cuda.Event(enable_timing=True, external=True)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        t0.record()
        for i in range(steps):
            step(i)
        t1.record()
    g.replay()                      # one untimed replay
    torch.cuda.synchronize()
    dist.barrier()
    torch.cuda.synchronize()
    with Clocks(dist.local) as clk:
        g.replay()
        torch.cuda.synchronize()
    dist.barrier()
    torch.cuda.synchronize()
    total_ms = t0.elapsed_time(t1)
    # per-kernel launch duration: the same launches, one kernel at a time, in
    # graphs of K back-to-back launches on the same rotating copies
    k8 = time_graph(torch, lambda i: kq.qmv(X, W8[i % copies], Q8_0, out=Y8), steps, s)
    k6 = time_graph(torch, lambda i: kq.qmv(X, W6[i % copies], Q6_K, out=Y6), steps, s)
    max_s = dist.max(total_ms / 1e3, dev)
    value = replica_value(bytes_step * steps / 1e9, dist.world, max_s)
    ms_per_step = max_s * 1e3 / steps
    dom = ("qmv_q8_0_m1_14336x4096", w8.nbytes, k8) if k8 >= k6 else ("qmv_q6_K_m1_14336x4096", w6.nbytes, k6)
    ach = dom[1] / (dom[2] / 1e3) / 1e9
    roofline = {"bound": "hbm", "kernel": dom[0], "achieved": round(ach, 1), "peak": pk["hbm_gbs"], "unit": "GB/s",
                "frac": round(ach / pk["hbm_gbs"], 4), "traffic": profiled_traffic(dom[0]),
                "bytes_per_launch": dom[1], "kernel_us": round(dom[2] * 1e3, 2),
                "peak_source": pk["source"] + " (hbm_gbs: STREAM-style copy, burst)",
                "other_kernel": {"name": ("qmv_q6_K_m1_14336x4096" if dom[0].startswith("qmv_q8") else
                                          "qmv_q8_0_m1_14336x4096"),
                                 "kernel_us": round(min(k8, k6) * 1e3, 2),
                                 "achieved_gbs": round((w6.nbytes if k8 >= k6 else w8.nbytes) / (min(k8, k6) / 1e3) / 1e9, 1)}}
    launches = 2 * steps   # in the timed region

    # ---- e2e: host buffers through the C ABI, copies inside the timed region
    hw8 = torch.from_numpy(w8).pin_memory()
    hw6 = torch.from_numpy(w6).pin_memory()
    hx = torch.from_numpy(x.view(np.int16)).pin_memory()
    hy8 = torch.empty(1, n).pin_memory()
    hy6 = torch.empty(1, n).pin_memory()
    dw8, dw6 = torch.empty_like(W8[0]), torch.empty_like(W6[0])
    dx = torch.empty(1, k, dtype=torch.int16, device=dev)
    e_steps = max(3, min(steps, 10))

    def e2e_step():
        dw8.copy_(hw8, non_blocking=True)
        dw6.copy_(hw6, non_blocking=True)
        dx.copy_(hx, non_blocking=True)
        kq.qmv(dx.view(torch.bfloat16), dw8, Q8_0, out=Y8)
        kq.qmv(dx.view(torch.bfloat16), dw6, Q6_K, out=Y6)
        hy8.copy_(Y8, non_blocking=True)
        hy6.copy_(Y6, non_blocking=True)

    with torch.cuda.stream(s):
        for _ in range(2):
            e2e_step()
        s.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        dist.barrier()
        a.record()
        for _ in range(e_steps):
            e2e_step()
        b.record()
    torch.cuda.synchronize()
    e_max = dist.max(a.elapsed_time(b) / 1e3, dev)
    e2e = {"value": round(replica_value(bytes_step * e_steps / 1e9, dist.world, e_max), 2), "unit": "GB/s",
           "h2d_bytes_per_step": int(w8.nbytes + w6.nbytes + x.nbytes), "d2h_bytes_per_step": int(2 * n * 4),
           "steps": e_steps}
    launches_e2e = 2 * e_steps
    del W8, W6, dw8, dw6

    out = {"metric": METRIC, "value": round(value, 1), "unit": "GB/s", "n_gpus": dist.world, "steps": steps,
           "warmup": warm, "ms_per_step": round(ms_per_step, 5), "higher_is_better": True, "scaling": "weak",
           "vs_baseline": None, "dtype": "f16xf16->f32 (exact integer codes)", "data": "synthetic (seeded PCG64)",
           "config": {"workload": "c1_q8_0_q6K_qmv_m1_n14336_k4096", "model": None, "global_batch": dist.world,
                      "seq_len": 1, "parallelism": f"replicas x{dist.world}",
                      "l2": f"rotating {copies} weight copies ({copies * bytes_step / 2**20:.0f} MiB > L2)",
                      "timing": "CUDA graph of the timed steps, CUDA events on the launching stream around "
                                "them; per-kernel times from graphs of K launches of one kernel"},
           "roofline": roofline, "e2e": e2e, "gpu_launches": launches, "clocks": clk.summary()}
    if not args.no_rows:
        out["rows"] = measure_rows(kq, torch, dev, pk, args)
        out["gpu_launches_rows"] = out["rows"].pop("_launches")
    out["gpu_launches_e2e"] = launches_e2e
    return out


def time_graph(torch, fn, reps: int, stream):
    """Average ms per call of fn() over a CUDA graph of `reps` calls."""
    with torch.cuda.stream(stream):
        for i in range(3):
            fn(i)
    stream.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for i in range(reps):
            fn(i)
    g.replay()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        a.record()
        g.replay()
        b.record()
    torch.cuda.synchronize()
    return a.elapsed_time(b) / reps


def measure_rows(kq, torch, dev, pk, args) -> dict:
    """Each remaining row of the hot path on its own workload (kernel-only)."""
    s = torch.cuda.Stream(device=dev)
    rows, launches = {}, 0
    reps = 20

    def u8(a):
        return torch.from_numpy(np.ascontiguousarray(a)).to(dev)

    def bf(bits):
        return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).to(dev).view(torch.bfloat16)

    def ncopies(nbytes):
        return max(2, -(-3 * L2_BYTES // nbytes))

    # c0: q4_K qmv M=1 4096x4096 and its full dequantize
    w = synth.weights(Q4_K, 4096, 4096)
    cp = ncopies(w.nbytes)
    Ws = [u8(w) for _ in range(cp)]
    x = bf(synth.activations(1, 4096))
    y = torch.empty(1, 4096, device=dev)
    t = time_graph(torch, lambda i: kq.qmv(x, Ws[i % cp], Q4_K, out=y), reps, s)
    launches += reps + 3
    gbs = w.nbytes / (t / 1e3) / 1e9
    rows["c0_qmv_q4K_m1_4096x4096"] = {"kernel_us": round(t * 1e3, 2), "GB/s": round(gbs, 1),
                                       "frac_hbm": round(gbs / pk["hbm_gbs"], 4), "bytes": w.nbytes}
    out = torch.empty(4096, 4096, device=dev)
    t = time_graph(torch, lambda i: kq.dequantize(Ws[i % cp], Q4_K, 4096, out=out), reps, s)
    launches += reps + 3
    db = w.nbytes + 4096 * 4096 * 4
    rows["c0_dequantize_q4K_4096x4096_fp32"] = {"kernel_us": round(t * 1e3, 2), "GB/s": round(db / (t / 1e3) / 1e9, 1),
                                                "frac_hbm": round(db / (t / 1e3) / 1e9 / pk["hbm_gbs"], 4),
                                                "bytes": db}
    del Ws, out
    # the encoder on the c0 shape: fp32 4096 x 4096 -> wire bytes of each codec
    # (rotating fp32 copies larger than L2 between launches)
    wf = [torch.randn(4096, 4096, device=dev) * 0.02 for _ in range(ncopies(4096 * 4096 * 4))]
    for qt, nm in ((Q4_K, "q4K"), (Q6_K, "q6K"), (Q8_0, "q8_0")):
        qo = torch.empty(4096, synth.row_bytes(qt, 4096), dtype=torch.uint8, device=dev)
        t = time_graph(torch, lambda i: kq.quantize(wf[i % len(wf)], qt, out=qo), reps, s)
        launches += reps + 3
        qb = 4096 * 4096 * 4 + qo.numel()
        rows[f"quantize_{nm}_4096x4096_from_fp32"] = {"kernel_us": round(t * 1e3, 2),
                                                     "GB/s": round(qb / (t / 1e3) / 1e9, 1),
                                                     "frac_hbm": round(qb / (t / 1e3) / 1e9 / pk["hbm_gbs"], 4),
                                                     "bytes": qb}
    del wf
    # q5_K and q4_0: dequantize 4096 x 4096; qmv M = 1, 2 on the c1 shape (the
    # staged decode kernel); gather_qmv, one token routed top-2 over a bank of
    # 4 such experts; qmm on the c3 shape
    for qt, nm in ((Q5_K, "q5K"), (Q4_0, "q4_0")):
        w = synth.weights(qt, 4096, 4096)
        cp = ncopies(w.nbytes)
        Ws = [u8(w) for _ in range(cp)]
        out = torch.empty(4096, 4096, device=dev)
        t = time_graph(torch, lambda i: kq.dequantize(Ws[i % cp], qt, 4096, out=out), reps, s)
        launches += reps + 3
        db = w.nbytes + 4096 * 4096 * 4
        rows[f"dequantize_{nm}_4096x4096_fp32"] = {"kernel_us": round(t * 1e3, 2), "GB/s": round(db / (t / 1e3) / 1e9, 1),
                                                  "frac_hbm": round(db / (t / 1e3) / 1e9 / pk["hbm_gbs"], 4), "bytes": db}
        del Ws, out
        w = synth.weights(qt, 14336, 4096)
        cp = ncopies(w.nbytes)
        Ws = [u8(w) for _ in range(cp)]
        for m in (1, 2):
            xm = bf(synth.activations(m, 4096))
            ym = torch.empty(m, 14336, device=dev)
            t = time_graph(torch, lambda i: kq.qmv(xm, Ws[i % cp], qt, out=ym), reps, s)
            launches += reps + 3
            gbs = w.nbytes / (t / 1e3) / 1e9
            rows[f"qmv_{nm}_m{m}_14336x4096"] = {"kernel_us": round(t * 1e3, 2), "GB/s": round(gbs, 1),
                                                 "frac_hbm": round(gbs / pk["hbm_gbs"], 4), "bytes": w.nbytes}
        bank0 = torch.stack([Ws[i % cp] for i in range(4)])
        qbanks = [bank0] + [bank0.clone() for _ in range(ncopies(2 * w.nbytes) - 1)]
        rid = torch.from_numpy(synth.routing(1, 4, 2, seed=9)).to(dev)
        distinct = int(torch.unique(rid).numel())
        xg = bf(synth.activations(1, 4096, seed=10))
        yg = torch.empty(2, 14336, device=dev)
        t = time_graph(torch, lambda i: kq.gather_qmv(xg, qbanks[i % len(qbanks)], qt, rid, x_per_token=True,
                                                      out=yg), reps, s)
        launches += reps + 3
        gbs = distinct * w.nbytes / (t / 1e3) / 1e9
        rows[f"decode_moe_gather_qmv_{nm}_4x14336x4096_t1_top2"] = {
            "kernel_us": round(t * 1e3, 2), "GB/s": round(gbs, 1), "frac_hbm": round(gbs / pk["hbm_gbs"], 4),
            "bytes": distinct * w.nbytes, "experts_read": distinct}
        del qbanks, bank0
        xq = bf(synth.activations(2048, 4096))
        yq = torch.empty(2048, 14336, device=dev)
        t = time_graph(torch, lambda i: kq.qmm(xq, Ws[i % cp], qt, out=yq), 8, s)
        launches += 8 + 3
        tf = 2 * 2048 * 14336 * 4096 / (t / 1e3) / 1e12
        rows[f"qmm_{nm}_2048x14336x4096"] = {"kernel_us": round(t * 1e3, 2), "TFLOP/s": round(tf, 1),
                                             "frac_bf16": round(tf / pk["bf16_tflops"], 4)}
        del Ws, xq, yq
    # c2: q4_K qmv 4096x14336, M in {1, 4, 8, 16}
    w = synth.weights(Q4_K, 4096, 14336)
    cp = ncopies(w.nbytes)
    Ws = [u8(w) for _ in range(cp)]
    xa = synth.activations(16, 14336)
    for m in (1, 4, 8, 16):
        x = bf(xa[:m])
        y = torch.empty(m, 4096, device=dev)
        t = time_graph(torch, lambda i: kq.qmv(x, Ws[i % cp], Q4_K, out=y), reps, s)
        launches += reps + 3
        gbs = w.nbytes / (t / 1e3) / 1e9
        rows[f"c2_qmv_q4K_m{m}_4096x14336"] = {"kernel_us": round(t * 1e3, 2), "GB/s": round(gbs, 1),
                                               "frac_hbm": round(gbs / pk["hbm_gbs"], 4), "bytes": w.nbytes}
    del Ws
    # c3: tcgen05 qmm M=2048, N=14336, K=4096 for q4_K and q6_K
    m, n, k = 2048, 14336, 4096
    xq = bf(synth.activations(m, k))
    y = torch.empty(m, n, device=dev)
    flops = 2 * m * n * k
    for qt, nm in ((Q4_K, "q4K"), (Q6_K, "q6K")):
        w = synth.weights(qt, n, k)
        cp = ncopies(w.nbytes + m * k * 2)
        Ws = [u8(w) for _ in range(cp)]
        t = time_graph(torch, lambda i: kq.qmm(xq, Ws[i % cp], qt, out=y), 8, s)
        launches += 8 + 3
        tf = flops / (t / 1e3) / 1e12
        rows[f"c3_qmm_{nm}_2048x14336x4096"] = {"kernel_us": round(t * 1e3, 2), "TFLOP/s": round(tf, 1),
                                               "frac_bf16": round(tf / pk["bf16_tflops"], 4),
                                               "frac_bf16_sustained": round(tf / pk["bf16_tflops_sustained"], 4)}
        del Ws
    del y, xq
    # q6_K qmm with rows that are not a 16-byte multiple (K = 11008: 9030-byte
    # rows, the flat view of the weights), M = 2048, N = 14336
    k6 = 11008
    xq = bf(synth.activations(m, k6))
    y = torch.empty(m, n, device=dev)
    w = synth.weights(Q6_K, n, k6)
    cp = ncopies(w.nbytes + m * k6 * 2)
    Ws = [u8(w) for _ in range(cp)]
    t = time_graph(torch, lambda i: kq.qmm(xq, Ws[i % cp], Q6_K, out=y), 8, s)
    launches += 8 + 3
    tf = 2 * m * n * k6 / (t / 1e3) / 1e12
    rows["qmm_q6K_2048x14336x11008_unaligned_rows"] = {"kernel_us": round(t * 1e3, 2), "TFLOP/s": round(tf, 1),
                                                       "frac_bf16": round(tf / pk["bf16_tflops"], 4)}
    del Ws, y, xq
    # c4: MoE sort + tile map + gather, 8 experts x 14336 x 4096 q4_K, 512 tokens top-2
    e, n, k, tok, topk = 8, 14336, 4096, 512, 2
    wb = u8(synth.weights(Q4_K, n, k, experts=e))
    xt = bf(synth.activations(tok, k))
    ids = torch.from_numpy(synth.routing(tok, e, topk)).to(dev)
    sids, pair, xs = kq.moe_sort(ids, e, xt)
    tmap, cnt = kq.expert_tile_map(sids, e)
    y = torch.empty(tok * topk, n, device=dev)
    t = time_graph(torch, lambda i: kq.gather_qmm(xs, wb, Q4_K, tmap, cnt, out=y), 8, s)
    launches += 8 + 3
    tf = 2 * tok * topk * n * k / (t / 1e3) / 1e12
    rows["c4_gather_qmm_q4K_8x14336x4096_t512_top2"] = {"kernel_us": round(t * 1e3, 2), "TFLOP/s": round(tf, 1),
                                                        "frac_bf16": round(tf / pk["bf16_tflops"], 4)}

    def route(i):
        kq.moe_sort(ids, e, xt)
        kq.expert_tile_map(sids, e)
    t = time_graph(torch, route, 8, s)
    launches += 3 * (8 + 3)
    rows["c4_moe_sort_and_tile_map"] = {"us": round(t * 1e3, 2), "launches_per_call": 3}
    # c4 epilogue: unsort + score mix of the 1024 expert-sorted output rows
    _, _, _, inv = kq.moe_sort(ids, e, with_inverse=True)
    sc = torch.rand(tok, topk, device=dev)
    mixo = torch.empty(tok, n, device=dev)
    ys = [y] + [torch.randn_like(y) for _ in range(ncopies(y.numel() * 4 + mixo.numel() * 4) - 1)]
    t = time_graph(torch, lambda i: kq.gather_mix(ys[i % len(ys)], inv, sc, out=mixo), reps, s)
    launches += reps + 3
    mb = (tok * topk + tok) * n * 4
    rows["c4_gather_mix_t512_top2_n14336"] = {"kernel_us": round(t * 1e3, 2), "GB/s": round(mb / (t / 1e3) / 1e9, 1),
                                             "frac_hbm": round(mb / (t / 1e3) / 1e9 / pk["hbm_gbs"], 4), "bytes": mb}
    del ys, mixo, y
    # decode MoE: gather_qmv on the same q4_K bank, 1 and 4 tokens routed
    # top-2, one activation row per token (the gate/up product); the weight
    # bytes are those of the distinct experts routed.  Rotating copies of the
    # whole bank keep the experts' bytes out of L2 between launches.
    ebytes = synth.row_bytes(Q4_K, k) * n
    banks = [wb] + [wb.clone() for _ in range(ncopies(2 * ebytes) - 1)]
    for tk in (1, 4):
        rid = torch.from_numpy(synth.routing(tk, e, topk, seed=9)).to(dev)
        distinct = int(torch.unique(rid).numel())
        xd = bf(synth.activations(tk, k, seed=10))
        yd = torch.empty(tk * topk, n, device=dev)
        t = time_graph(torch, lambda i: kq.gather_qmv(xd, banks[i % len(banks)], Q4_K, rid, x_per_token=True,
                                                      out=yd), reps, s)
        launches += reps + 3
        gbs = distinct * ebytes / (t / 1e3) / 1e9
        rows[f"decode_moe_gather_qmv_q4K_8x14336x4096_t{tk}_top2"] = {
            "kernel_us": round(t * 1e3, 2), "GB/s": round(gbs, 1), "frac_hbm": round(gbs / pk["hbm_gbs"], 4),
            "bytes": distinct * ebytes, "experts_read": distinct}
        # the fused gate/up GLU on the same routing: two banks (gate = the
        # rotating copies, up = the next copy), each routed expert read once
        yg = torch.empty(tk * topk, n, device=dev)
        t = time_graph(torch, lambda i: kq.moe_glu_gather(xd, banks[i % len(banks)], banks[(i + 1) % len(banks)],
                                                          Q4_K, rid, out=yg), reps, s)
        launches += reps + 3
        gbs = 2 * distinct * ebytes / (t / 1e3) / 1e9
        rows[f"decode_moe_glu_gather_q4K_2x8x14336x4096_t{tk}_top2"] = {
            "kernel_us": round(t * 1e3, 2), "GB/s": round(gbs, 1), "frac_hbm": round(gbs / pk["hbm_gbs"], 4),
            "bytes": 2 * distinct * ebytes, "experts_read": distinct}
    del banks
    rows["_launches"] = launches
    return rows


# ------------------------------------------------------------ CPU oracle arm
def cpu_sample(seconds: float = 10.0) -> dict:
    """The oracle (fp32 variant, as it stands) on the c1 workload, repeated for
    about `seconds` of wall time on the host cores."""
    import oracle
    n, k = 14336, 4096
    w8 = synth.weights(Q8_0, n, k)
    w6 = synth.weights(Q6_K, n, k)
    x = synth.activations(1, k)
    oracle.matmul_f32(Q8_0, w8[:64], k, x)   # build + warm
    done, t0 = 0, time.perf_counter()
    while True:
        oracle.matmul_f32(Q8_0, w8, k, x)
        oracle.matmul_f32(Q6_K, w6, k, x)
        done += 1
        el = time.perf_counter() - t0
        if el >= seconds:
            break
    gbs = (w8.nbytes + w6.nbytes) * done / el / 1e9
    return {"value": round(gbs, 3), "unit": "GB/s", "cores": oracle.threads(), "kind": "oracle",
            "sample": f"{done} full passes of c1 (q8_0 + q6_K qmv, 14336x4096, M=1) in {el:.1f} s",
            "cpu": _cpu_model()}


def cpu_baseline_configs(min_seconds: float = 0.3) -> dict:
    """The oracle's fp32 product (as it stands) on every configuration, once on
    one host thread and once on all host cores; c0-c2 in full, c3 / c4 on a
    fixed subset of activation rows with the per-call time extrapolated by
    the row ratio (labelled).  About 15 s of CPU work."""
    import oracle
    out = {}

    def timed(fn):
        n, t0 = 0, time.perf_counter()
        while True:
            fn()
            n += 1
            el = time.perf_counter() - t0
            if el >= min_seconds:
                return el / n

    def both(fn):
        res = {}
        for label, t in (("1_thread", 1), ("all_cores", 0)):
            oracle.set_threads(t)
            res[label] = (timed(fn), oracle.threads())
        oracle.set_threads(0)
        return res

    def gbs_entry(nbytes, fn, note=None):
        r = both(fn)
        e = {f"{lab}_GB/s": round(nbytes / t / 1e9, 3) for lab, (t, _) in r.items()}
        e["cores"] = r["all_cores"][1]
        if note:
            e["sample"] = note
        return e

    # c0: q4_K qmv 4096 x 4096, M = 1, and its full dequantize to fp32
    w = synth.weights(Q4_K, 4096, 4096)
    x = synth.activations(1, 4096)
    out["c0_qmv_q4K_m1_4096x4096"] = gbs_entry(w.nbytes, lambda: oracle.matmul_f32(Q4_K, w, 4096, x))
    out["c0_dequantize_q4K_4096x4096_fp32"] = gbs_entry(w.nbytes + 4096 * 4096 * 4,
                                                        lambda: oracle.dequantize(Q4_K, w, 4096))
    # c1: q8_0 + q6_K qmv 14336 x 4096, M = 1
    w8, w6 = synth.weights(Q8_0, 14336, 4096), synth.weights(Q6_K, 14336, 4096)
    x = synth.activations(1, 4096)
    out["c1_qmv_q8_0_q6K_m1_14336x4096"] = gbs_entry(
        w8.nbytes + w6.nbytes, lambda: (oracle.matmul_f32(Q8_0, w8, 4096, x), oracle.matmul_f32(Q6_K, w6, 4096, x)))
    del w8, w6
    # c2: q4_K qmv 4096 x 14336, M in {1, 4, 8, 16}
    w = synth.weights(Q4_K, 4096, 14336)
    xa = synth.activations(16, 14336)
    for m in (1, 4, 8, 16):
        xm = xa[:m]
        out[f"c2_qmv_q4K_m{m}_4096x14336"] = gbs_entry(w.nbytes, lambda: oracle.matmul_f32(Q4_K, w, 14336, xm))
    # c3: qmm 2048 x 14336 x 4096 (q4_K, q6_K): 32 of the 2048 activation rows
    sub = 32
    xs = synth.activations(2048, 4096)[:sub]
    for qt, nm in ((Q4_K, "q4K"), (Q6_K, "q6K")):
        w = synth.weights(qt, 14336, 4096)
        r = both(lambda: oracle.matmul_f32(qt, w, 4096, xs))
        e = {}
        for lab, (t, _) in r.items():
            full = t * 2048 / sub
            e[f"{lab}_TFLOP/s"] = round(2 * 2048 * 14336 * 4096 / full / 1e12, 6)
            e[f"{lab}_extrapolated_ms_per_call"] = round(full * 1e3, 1)
        e["cores"] = r["all_cores"][1]
        e["sample"] = f"{sub} of 2048 activation rows, per-call time extrapolated x{2048 // sub}"
        out[f"c3_qmm_{nm}_2048x14336x4096"] = e
    del w
    # c4: gather q4_K, 8 experts x 14336 x 4096, 512 tokens top-2 (1024 rows):
    # every expert's first 4 sorted rows (32 of 1024)
    e_, tok, topk = 8, 512, 2
    wb = synth.weights(Q4_K, 14336, 4096, experts=e_)
    ids = synth.routing(tok, e_, topk)
    srt, pair = oracle.moe_sort(ids, e_)
    xt = synth.activations(tok, 4096)
    per = 4
    groups = [(ex, xt[pair[srt == ex][:per] // topk]) for ex in range(e_) if np.any(srt == ex)]
    rows = sum(g[1].shape[0] for g in groups)
    r = both(lambda: [oracle.matmul_f32(Q4_K, wb[ex], 4096, xg) for ex, xg in groups])
    e = {}
    for lab, (t, _) in r.items():
        full = t * (tok * topk) / rows
        e[f"{lab}_TFLOP/s"] = round(2 * tok * topk * 14336 * 4096 / full / 1e12, 6)
        e[f"{lab}_extrapolated_ms_per_call"] = round(full * 1e3, 1)
    e["cores"] = r["all_cores"][1]
    e["sample"] = f"{rows} of {tok * topk} sorted rows ({per} per expert), per-call time extrapolated"
    out["c4_gather_qmm_q4K_8x14336x4096_t512_top2"] = e
    return out


def _cpu_model() -> str:
    try:
        for line in open("/proc/cpuinfo"):
            if line.startswith("model name"):
                return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def run_reference(args, dist: Dist) -> dict | None:
    if dist.rank != 0:
        return None
    per = max(1.0, 60.0 / max(1, args.steps + args.warmup))
    for _ in range(args.warmup):
        cpu_sample(seconds=0.0)
    vals, descr = [], None
    t0 = time.perf_counter()
    for _ in range(args.steps):
        r = cpu_sample(seconds=per)
        vals.append(r["value"])
        descr = r
    el = time.perf_counter() - t0
    v = statistics.mean(vals)
    return {"impl": "reference", "metric": METRIC, "value": round(v, 3), "unit": "GB/s", "n_gpus": dist.world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(el * 1e3 / max(1, args.steps), 1),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
            "data": "synthetic (seeded PCG64)",
            "config": {"workload": "c1_q8_0_q6K_qmv_m1_n14336_k4096", "model": None, "global_batch": 1,
                       "seq_len": 1, "parallelism": "cpu"},
            "cpu_baseline": {"value": round(v, 3), "unit": "GB/s", "cores": descr["cores"], "kind": "oracle",
                             "sample": descr["sample"], "cpu": descr["cpu"]},
            "e2e": {"value": round(v, 3), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


# ------------------------------------------------------------ profile cases
CASES = ("qmv_q8_0", "qmv_q6_K", "qmv_q4_K_m1", "qmv_q4_K_m16", "dequant_q4_K", "qmm_q4_K", "qmm_q6_K",
         "gather_q4_K", "gather_qmv_q4_K", "gather_mix", "quantize_q4_K", "quantize_q6_K", "quantize_q8_0",
         "glu_q4_K", "qmv_q5_K", "qmv_q4_0", "dequant_q5_K")


def run_case(name: str, iters: int) -> None:
    """Run one kernel of the path `iters` times on its full-size workload,
    untimed (for ncu captures: `ncu ... python bench.py --case NAME`)."""
    import torch
    import gguf_quant_dequant_q4_b200 as kq

    dev = torch.device("cuda", 0)

    def u8(a):
        return torch.from_numpy(np.ascontiguousarray(a)).to(dev)

    def bf(bits):
        return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).to(dev).view(torch.bfloat16)

    if name in ("qmv_q8_0", "qmv_q6_K"):
        qt = Q8_0 if name == "qmv_q8_0" else Q6_K
        w, x = u8(synth.weights(qt, 14336, 4096)), bf(synth.activations(1, 4096))
        fn = lambda: kq.qmv(x, w, qt)
    elif name.startswith("qmv_q4_K"):
        m = 1 if name.endswith("m1") else 16
        n, k = (4096, 4096) if m == 1 else (4096, 14336)
        w, x = u8(synth.weights(Q4_K, n, k)), bf(synth.activations(m, k))
        fn = lambda: kq.qmv(x, w, Q4_K)
    elif name == "dequant_q4_K":
        w = u8(synth.weights(Q4_K, 4096, 4096))
        fn = lambda: kq.dequantize(w, Q4_K, 4096)
    elif name.startswith("qmm"):
        qt = Q4_K if name == "qmm_q4_K" else Q6_K
        w, x = u8(synth.weights(qt, 14336, 4096)), bf(synth.activations(2048, 4096))
        fn = lambda: kq.qmm(x, w, qt)
    elif name == "gather_q4_K":
        wb = u8(synth.weights(Q4_K, 14336, 4096, experts=8))
        xt = bf(synth.activations(512, 4096))
        sids, pair, xs = kq.moe_sort(torch.from_numpy(synth.routing(512, 8, 2)).to(dev), 8, xt)
        tmap, cnt = kq.expert_tile_map(sids, 8)
        fn = lambda: kq.gather_qmm(xs, wb, Q4_K, tmap, cnt)
    elif name == "gather_qmv_q4_K":
        wb = u8(synth.weights(Q4_K, 14336, 4096, experts=8))
        xd = bf(synth.activations(4, 4096, seed=10))
        rid = torch.from_numpy(synth.routing(4, 8, 2, seed=9)).to(dev)
        fn = lambda: kq.gather_qmv(xd, wb, Q4_K, rid, x_per_token=True)
    elif name.startswith("quantize_"):
        qt = {"quantize_q4_K": Q4_K, "quantize_q6_K": Q6_K, "quantize_q8_0": Q8_0}[name]
        wf = torch.randn(4096, 4096, device=dev) * 0.02
        fn = lambda: kq.quantize(wf, qt)
    elif name == "glu_q4_K":
        wg = u8(synth.weights(Q4_K, 14336, 4096, experts=8))
        wu = u8(synth.weights(Q4_K, 14336, 4096, experts=8, seed=1))
        xd = bf(synth.activations(4, 4096, seed=10))
        rid = torch.from_numpy(synth.routing(4, 8, 2, seed=9)).to(dev)
        fn = lambda: kq.moe_glu_gather(xd, wg, wu, Q4_K, rid)
    elif name in ("qmv_q5_K", "qmv_q4_0"):
        qt = Q5_K if name == "qmv_q5_K" else Q4_0
        w, x = u8(synth.weights(qt, 14336, 4096)), bf(synth.activations(1, 4096))
        fn = lambda: kq.qmv(x, w, qt)
    elif name == "dequant_q5_K":
        w = u8(synth.weights(Q5_K, 4096, 4096))
        fn = lambda: kq.dequantize(w, Q5_K, 4096)
    elif name == "gather_mix":
        ids = torch.from_numpy(synth.routing(512, 8, 2)).to(dev)
        _, _, _, inv = kq.moe_sort(ids, 8, with_inverse=True)
        yy = torch.randn(1024, 14336, device=dev)
        sc = torch.rand(512, 2, device=dev)
        fn = lambda: kq.gather_mix(yy, inv, sc)
    else:
        raise SystemExit(f"unknown case {name}; one of {CASES}")
    for _ in range(iters):
        fn()
    torch.cuda.synchronize()
    print(json.dumps({"case": name, "iters": iters, "status": "ok"}))


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="kq", choices=["kq", "reference"])
    ap.add_argument("--no-rows", action="store_true", help="skip the per-row measurements")
    ap.add_argument("--no-cpu", action="store_true", help="skip the CPU oracle baseline")
    ap.add_argument("--case", choices=CASES, help="run one kernel untimed (profiling)")
    ap.add_argument("--iters", type=int, default=3)
    args = ap.parse_args(argv)
    if args.case:
        run_case(args.case, args.iters)
        return
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    dist = Dist()
    if args.impl == "reference":
        res = run_reference(args, dist)     # rank 0 only, no process group needed
    else:
        dist.init("nccl")
        res = run_kq(args, dist)
        if res is not None and dist.rank == 0 and not args.no_cpu:
            res["cpu_baseline"] = cpu_sample(5.0)
            res["cpu_baseline"]["configs"] = cpu_baseline_configs()
    if dist.rank == 0 and res is not None:
        print(json.dumps(res), flush=True)
    dist.close()


if __name__ == "__main__":
    main()
