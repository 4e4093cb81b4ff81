#!/usr/bin/env python
"""Benchmark of the CSA / HCA compressed-attention hot path on B200.

Headline (the `value` of the JSON line): CSA decode queries/s at 128K context --
32 sequences x 1 new query each, 32768 compressed entries per sequence, top-k 1024,
window 128, 64 heads of dim 512, MXFP4 indexer with 64 heads of dim 128.  One step
= MXFP4 encoding of the indexer queries, indexer scores over every entry, top-k
selection, sparse MQA over the selected entries plus the window.  The cache is
resident in HBM; 4 independent input replicas rotate between steps so that every
step reads inputs that are not in the 126 MB L2.

Also reported in the same line: CSA prefill T=8192 tokens/s and HCA prefill
T=65536 tokens/s, each with the roofline of its dominant kernel; end-to-end decode
through the public API with host buffers; the CPU oracle on a bounded sample.

    python bench.py [--gpus N --steps K --warmup W] [--impl reference]

For N > 1 launch one process per GPU (torchrun); every rank runs its own 32
sequences (weak scaling, no collective on the data path); time = max over ranks.
"""
from __future__ import annotations

import argparse
import datetime
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "CSA decode queries/s at 128K ctx; prefill tok/s; % of HBM / tensor roofline"
UNIT = "queries/s"


def load_peaks() -> dict:
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained", d["bf16_tflops"]), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


# ----------------------------------------------------------------------------- tensor peaks
FP4_DATASHEET_TFLOPS = 9000.0  # NVIDIA B200 dense FP4 (the 18 PFLOP/s figure is with 2:4 sparsity)


def measure_tensor_peaks(dev, reps: int = 3) -> dict:
    """Dense tcgen05 rates of this GPU from the library's throughput probe (one CTA per SM,
    M = 128, N = 256, operands resident in shared memory): kind::mxf4 block-scaled FP4,
    the denominator of the FP4 indexer, and kind::f16 bf16 for comparison with the
    library GEMM's measured bf16 rate.  Best of `reps` launches of a few ms each."""
    import ctypes
    import torch
    from compressed_sparse_long_02_b200 import binding as B
    L = B.lib()
    L.csa_mma_peak_probe.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                     ctypes.POINTER(ctypes.c_double), ctypes.c_void_p]
    L.csa_mma_peak_probe.restype = ctypes.c_int
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    stream = ctypes.c_void_p(torch.cuda.current_stream(dev).cuda_stream)
    out = {}
    for name, mxf4, iters in (("mxf4", 1, 20000), ("bf16", 0, 40000)):
        best = 0.0
        for r in range(reps + 1):
            s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            flops = ctypes.c_double(0.0)
            s.record()
            st = L.csa_mma_peak_probe(mxf4, 256, iters, sms, ctypes.byref(flops), stream)
            e.record()
            torch.cuda.synchronize()
            assert st == 0, f"csa_mma_peak_probe: status {st}"
            if r > 0:  # the first launch warms up
                best = max(best, flops.value / (s.elapsed_time(e) / 1e3) / 1e12)
        out[name] = round(best, 1)
    assert B.csa_get_device_error() == 0
    return {"mxf4_tflops": out["mxf4"], "bf16_tflops_probe": out["bf16"], "ctas": sms,
            "how": "tcgen05 M=128 N=256, operands in shared memory, one CTA per SM, best of 3",
            "mxf4_datasheet_tflops": FP4_DATASHEET_TFLOPS}


# ----------------------------------------------------------------------------- ncu traffic
# DRAM bytes (read + write) per launch from one `ncu --set full` capture of the 128K
# decode step (profiles/*_decode_128k.md), keyed by the sha1 of the kernel's source file
# at capture time: a kernel changed since its capture reports traffic null.
NCU_TRAFFIC = {
    "attention": {"bytes": 40066048 + 717312, "src": "compressed_sparse_long_02_b200/csrc/attn.cu",
                  "sha1": "4559cbf1e5cbfa46e50cc43a5a7a30025fa7a6fa"},
    "index_score": {"bytes": 71483904 + 1665792, "src": "compressed_sparse_long_02_b200/csrc/index.cu",
                    "sha1": "b271de5f29ab6b90adcc34a460af7ad5b475c231"},
    "topk_select": {"bytes": 4253184, "src": "compressed_sparse_long_02_b200/csrc/topk.cu",
                    "sha1": "7fc5928a6f3c6ac7669c341815142304cacfdf34"},
}


def ncu_traffic(kernel: str):
    import hashlib
    e = NCU_TRAFFIC.get(kernel)
    if e is None:
        return None
    try:
        with open(os.path.join(ROOT, e["src"]), "rb") as f:
            h = hashlib.sha1(f.read()).hexdigest()
    except OSError:
        return None
    return e["bytes"] if h == e["sha1"] else None


# ----------------------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled every 200 ms while running."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
         "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
         "clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.f = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        self.p = None

    def start(self):
        try:
            self.p = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                                       "-i", str(self.gpu), "-lms", "200"], stdout=self.f, stderr=subprocess.DEVNULL)
        except OSError:
            self.p = None
        time.sleep(0.3)

    def stop(self) -> dict:
        if self.p is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.p.terminate()
        self.p.wait()
        self.f.flush()
        self.f.seek(0)
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.f.read().splitlines():
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx.append(float(parts[2]))
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        os.unlink(self.f.name)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        top = max(sm)
        loaded = [x for x in sm if x >= 0.5 * top] or sm
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


# ----------------------------------------------------------------------------- distributed
class Dist:
    def __init__(self):
        import torch
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.rank = int(os.environ.get("RANK", "0"))
        self.local_rank = int(os.environ.get("LOCAL_RANK", "0"))
        self.pg = None
        if torch.cuda.is_available():
            torch.cuda.set_device(self.local_rank)
        if self.world > 1:
            import torch.distributed as dist
            backend = "nccl" if torch.cuda.is_available() else "gloo"
            dist.init_process_group(backend, timeout=datetime.timedelta(seconds=180))
            self.pg = dist

    def barrier(self):
        if self.pg is not None:
            self.pg.barrier()

    def max(self, x: float) -> float:
        if self.pg is None:
            return x
        import torch
        dev = torch.device("cuda", self.local_rank) if torch.cuda.is_available() else torch.device("cpu")
        t = torch.tensor([x], dtype=torch.float64, device=dev)
        self.pg.all_reduce(t, op=self.pg.ReduceOp.MAX)
        return float(t.item())

    def close(self):
        if self.pg is not None:
            self.pg.destroy_process_group()


# ----------------------------------------------------------------------------- decode 128K
def decode_bytes_per_query(wl) -> dict:
    """Algorithmic bytes of one decode query (compulsory traffic, no scratch)."""
    E, k, W, D, H, Hi, Di = wl.E, wl.k, wl.W, wl.D, wl.H, wl.Hi, wl.Di
    keys = E * (Di // 2 + Di // 32)
    qi = Hi * (Di * 4) + Hi * 4           # raw fp32 indexer query + head weights
    gathered = k * D * 2
    window = W * D * 2
    q_o = 2 * H * D * 2
    idx = k * 4
    score_out = E * 4
    return {"step": keys + qi + gathered + window + q_o + idx,
            "index_score": keys + Hi * (Di // 2 + Di // 32) + Hi * 4 + score_out,
            "index_topk": keys + Hi * (Di // 2 + Di // 32) + Hi * 4 + idx + 4,
            "attention": gathered + window + q_o + idx,
            "keys": keys}


def setup_decode(wl, dev, replicas: int):
    import torch
    from compressed_sparse_long_02_b200 import binding as B
    from compressed_sparse_long_02_b200 import synth
    caches, steps = [], []
    for r in range(replicas):
        d = synth.decode_inputs_torch(wl, dev, replica=r)
        k_fp4, k_sc = B.csa_quantize_mxfp4(d["ki"])
        del d["ki"]
        Bn = d["q"].shape[0]
        caches.append({"entries": d["entries"], "k_fp4": k_fp4, "k_scale": k_sc, "window": d["window"],
                       "window_base": (d["pos"] - wl.W + 1).to(torch.int32),
                       "n_entries": torch.full((Bn,), wl.E, dtype=torch.int32, device=dev)})
        steps.append({"q": d["q"], "qi": d["qi"], "w": d["w"], "pos": d["pos"]})
    torch.cuda.synchronize()
    Bn = wl.B
    ws = {
        "index_ws": torch.empty(B.csa_index_topk_workspace(Bn, wl.E, wl.k), dtype=torch.uint8, device=dev),
        "idx": torch.empty((Bn, wl.k), dtype=torch.int32, device=dev),
        "cnt": torch.empty((Bn,), dtype=torch.int32, device=dev),
        "seq": torch.arange(Bn, dtype=torch.int32, device=dev),
        "attn_ws": torch.empty(B.csa_sparse_attn_workspace(Bn, wl.H, wl.D, wl.k, wl.W), dtype=torch.uint8,
                               device=dev),
        "out": torch.empty((Bn, wl.H, wl.D), dtype=torch.bfloat16, device=dev),
        "q_fp4": torch.empty((Bn, wl.Hi, wl.Di // 2), dtype=torch.uint8, device=dev),
        "q_scale": torch.empty((Bn, wl.Hi, wl.Di // 32), dtype=torch.uint8, device=dev),
    }
    return caches, steps, ws


DECODE_CALLS = ["quantize", "index_topk", "attention"]
# buffer sets of the pipelined end-to-end decode, i.e. steps in flight at once; the host
# waits for step i - E2E_BUFFERS's download before it issues step i.  Measured (32-query
# 128K decode, 71 us device step, 3.15 MB up and 2 MB down per step at ~50 GB/s each
# way): 2 sets 300K, 3 sets 393K, 4 sets 440K queries/s against 459K on the device alone
E2E_BUFFERS = 4
# steps of the end-to-end measurement (host wall clock around the pipelined steps): at
# ~70 us a step, the default 20 would time ~1.4 ms, where one host hiccup moves the figure
E2E_MIN_STEPS = 400


def decode_step(wl, cache, step, ws, ev=None):
    """One decode step as three C-ABI calls (query encoding, indexer + top-k, attention);
    `ev` (optional) gets CUDA events between calls.  csa_index_topk runs the scoring and
    the top-k kernels (its fused form, scores kept on chip, is off by default: slower at
    this shape).  (csa_index_score_q would encode the queries inside the indexer instead,
    but with nine indexer CTAs per query that repeats the encoding: 77 vs 71 us a step.)"""
    from compressed_sparse_long_02_b200 import binding as B
    if ev is not None:
        ev[0].record()
    B.csa_quantize_mxfp4(step["qi"], ws["q_fp4"], ws["q_scale"])
    if ev is not None:
        ev[1].record()
    B.csa_index_topk(ws["q_fp4"], ws["q_scale"], step["w"], step["pos"], ws["seq"], cache["k_fp4"], cache["k_scale"],
                     cache["n_entries"], k=wl.k, m=wl.m, workspace=ws["index_ws"], idx=ws["idx"], cnt=ws["cnt"])
    if ev is not None:
        ev[2].record()
    B.csa_sparse_attn(step["q"], step["pos"], ws["seq"], cache["entries"], ws["idx"], ws["cnt"], cache["window"],
                      cache["window_base"], W=wl.W, out=ws["out"], workspace=ws["attn_ws"])
    if ev is not None:
        ev[3].record()


def capture_step(fn):
    """Capture `fn` (a sequence of C-ABI calls on the current stream) into a CUDA graph."""
    import torch
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        fn()
    torch.cuda.current_stream().wait_stream(side)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fn()
    return g


def bench_decode(args, dist, peaks, name: str = "csa_decode_128k", e2e: bool = True, steps: int | None = None):
    import torch
    from compressed_sparse_long_02_b200 import binding as B
    from compressed_sparse_long_02_b200 import synth
    wl = synth.WORKLOADS[name]
    steps = args.steps if steps is None else steps
    dev = torch.device("cuda", dist.local_rank)
    R = args.replicas
    caches, step_inputs, ws = setup_decode(wl, dev, R)
    for i in range(R):  # eager pass: sets kernel attributes before capture
        decode_step(wl, caches[i], step_inputs[i], ws)
    torch.cuda.synchronize()
    graphs = [capture_step(lambda i=i: decode_step(wl, caches[i], step_inputs[i], ws)) for i in range(R)]
    for i in range(args.warmup):
        graphs[i % R].replay()
    torch.cuda.synchronize()
    assert B.csa_get_device_error() == 0, "device error during warm-up"

    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(dist.local_rank)
    clocks.start()
    dist.barrier()
    torch.cuda.synchronize()
    start.record()
    for i in range(steps):
        graphs[i % R].replay()
    end.record()
    torch.cuda.synchronize()
    dist.barrier()
    clk = clocks.stop()
    ms_local = start.elapsed_time(end)
    ms = dist.max(ms_local)
    assert B.csa_get_device_error() == 0, "device error in the timed region"

    # per-call device time: the same steps run eagerly behind a GPU sleep, so that the
    # calls queue up and execute back to back between the events
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(len(DECODE_CALLS) + 1)] for _ in range(steps)]
    for i in range(steps):
        torch.cuda._sleep(2_000_000)
        decode_step(wl, caches[i % R], step_inputs[i % R], ws, evs[i])
    torch.cuda.synchronize()
    per = {n: statistics.mean(e[j].elapsed_time(e[j + 1]) for e in evs) for j, n in enumerate(DECODE_CALLS)}
    nb = decode_bytes_per_query(wl)
    queries_per_step = wl.B * dist.world
    value = queries_per_step * steps / (ms / 1e3)
    ms_step = ms / steps
    dom = max(per, key=per.get)
    dom_bytes = {"index_topk": nb["index_topk"], "attention": nb["attention"],
                 "quantize": wl.Hi * wl.Di * 4}[dom] * wl.B
    achieved = dom_bytes / (per[dom] / 1e3) / 1e9
    step_gbs = nb["step"] * wl.B / (ms_local / steps / 1e3) / 1e9
    res = {
        "value": value, "ms_per_step": ms_step,
        "roofline": {"bound": "hbm", "kernel": dom, "achieved": round(achieved, 1), "peak": peaks["hbm_gbs"],
                     "unit": "GB/s", "frac": round(achieved / peaks["hbm_gbs"], 4), "traffic": ncu_traffic(dom),
                     "algorithmic_bytes_per_launch": dom_bytes, "peak_source": peaks["source"]},
        "step_roofline": {"bound": "hbm", "algorithmic_bytes": nb["step"] * wl.B, "achieved_gbs": round(step_gbs, 1),
                          "frac": round(step_gbs / peaks["hbm_gbs"], 4)},
        "per_call_us": {k: round(v * 1e3, 2) for k, v in per.items()},
        "clocks": clk,
        # query encoding, indexer + top-k (one fused kernel or two), attention (split merge inside)
        "gpu_launches": steps * (2 + B.csa_index_topk_launches(wl.B, wl.Hi, wl.Di, wl.E, wl.k)),
        "graph": "one CUDA graph per input replica, replayed back to back",
    }
    if e2e:
        res["e2e"] = bench_decode_e2e(args, wl, caches, step_inputs, ws, dist)
    del graphs, caches, step_inputs, ws
    torch.cuda.empty_cache()
    return wl, res


def bench_decode_mq(args, dist, peaks, name: str = "csa_decode_128k", steps: int = 20):
    """Multi-query decode at the 128K shape: every sequence advances by two tokens per
    step (a new token and one draft, at positions L-2 and L-1 of the resident cache), so a
    step has 2 x B queries.  The indexer runs grouped (csa_index_topk_grouped: the two
    queries of a sequence read its key cache once) and, for comparison, ungrouped on the
    same inputs; attention is per query either way.  Graph replays, input replicas
    rotating as in the headline line."""
    import torch
    from compressed_sparse_long_02_b200 import binding as B
    from compressed_sparse_long_02_b200 import synth
    wl = synth.WORKLOADS[name]
    dev = torch.device("cuda", dist.local_rank)
    R = args.replicas
    caches, _, _ = setup_decode(wl, dev, R)
    Bn, nq = wl.B, 2 * wl.B
    g = torch.Generator(device=dev)
    g.manual_seed(wl.seed * 104729)
    L = wl.E * wl.m
    steps_in = []
    for _ in range(R):
        steps_in.append({
            "q": torch.randn((nq, wl.H, wl.D), generator=g, device=dev).to(torch.bfloat16),
            "qi": torch.randn((nq, wl.Hi, wl.Di), generator=g, device=dev),
            "w": torch.rand((nq, wl.Hi), generator=g, device=dev),
            "pos": torch.tensor([L - 2, L - 1] * Bn, dtype=torch.int32, device=dev)})
    ws = {
        "index_ws": torch.empty(B.csa_index_topk_workspace(nq, wl.E, wl.k), dtype=torch.uint8, device=dev),
        "idx": torch.empty((nq, wl.k), dtype=torch.int32, device=dev),
        "cnt": torch.empty((nq,), dtype=torch.int32, device=dev),
        "seq": torch.arange(Bn, dtype=torch.int32, device=dev).repeat_interleave(2),
        "attn_ws": torch.empty(B.csa_sparse_attn_workspace(nq, wl.H, wl.D, wl.k, wl.W), dtype=torch.uint8,
                               device=dev),
        "out": torch.empty((nq, wl.H, wl.D), dtype=torch.bfloat16, device=dev),
        "q_fp4": torch.empty((nq, wl.Hi, wl.Di // 2), dtype=torch.uint8, device=dev),
        "q_scale": torch.empty((nq, wl.Hi, wl.Di // 32), dtype=torch.uint8, device=dev)}

    def step(i, q_group, ev=None):
        c, st = caches[i % R], steps_in[i % R]
        if ev is not None:
            ev[0].record()
        B.csa_quantize_mxfp4(st["qi"], ws["q_fp4"], ws["q_scale"])
        if ev is not None:
            ev[1].record()
        B.csa_index_topk(ws["q_fp4"], ws["q_scale"], st["w"], st["pos"], ws["seq"], c["k_fp4"], c["k_scale"],
                         c["n_entries"], k=wl.k, m=wl.m, workspace=ws["index_ws"], idx=ws["idx"], cnt=ws["cnt"],
                         q_group=q_group)
        if ev is not None:
            ev[2].record()
        B.csa_sparse_attn(st["q"], st["pos"], ws["seq"], c["entries"], ws["idx"], ws["cnt"], c["window"],
                          c["window_base"], W=wl.W, out=ws["out"], workspace=ws["attn_ws"])
        if ev is not None:
            ev[3].record()

    out = {"workload": name + "_2tok", "sequences": Bn, "queries_per_step": nq, "unit": UNIT}
    for q_group in (2, 1):
        for i in range(R):
            step(i, q_group)
        torch.cuda.synchronize()
        graphs = [capture_step(lambda i=i: step(i, q_group)) for i in range(R)]
        for i in range(args.warmup):
            graphs[i % R].replay()
        torch.cuda.synchronize()
        s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        dist.barrier()
        s0.record()
        for i in range(steps):
            graphs[i % R].replay()
        s1.record()
        torch.cuda.synchronize()
        ms = dist.max(s0.elapsed_time(s1)) / steps
        assert B.csa_get_device_error() == 0
        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(steps)]
        for i in range(steps):
            torch.cuda._sleep(2_000_000)
            step(i, q_group, evs[i])
        torch.cuda.synchronize()
        per = {n: round(1e3 * statistics.mean(e[j].elapsed_time(e[j + 1]) for e in evs), 2)
               for j, n in enumerate(DECODE_CALLS)}
        key = "grouped" if q_group == 2 else "ungrouped"
        out[key] = {"value": nq * dist.world / (ms / 1e3), "ms_per_step": ms, "per_call_us": per}
        del graphs
    # the grouped indexer reads each sequence's keys once: its HBM roofline
    keys = wl.E * (wl.Di // 2 + wl.Di // 32) * Bn
    us = out["grouped"]["per_call_us"]["index_topk"]
    out["index_topk_roofline"] = {"bound": "hbm", "algorithmic_bytes": keys, "achieved": round(keys / us / 1e3, 1),
                                  "unit": "GB/s", "frac": round(keys / us / 1e3 / peaks["hbm_gbs"], 4)}
    out["value"] = out["grouped"]["value"]
    del caches, steps_in, ws
    torch.cuda.empty_cache()
    return out


def bench_decode_e2e(args, wl, caches, steps, ws, dist):
    """Decode through the public API with host buffers: every step copies its inputs (q,
    indexer query, head weights, positions; one packed block, one copy) from pinned host
    memory and its output back.
    Steps are independent batches (the input replicas rotate), so they are pipelined
    over three streams: the upload of step i+1 and the download of step i-1 overlap the
    layer call of step i (two buffer sets, ordered by events).  As a serving loop would,
    each stage is a CUDA graph captured once per buffer set and replica (the upload's
    memcpy nodes, the layer's four C-ABI calls, the download's memcpy node) and replayed
    every step, so the host issues three graph launches per step."""
    import torch
    from compressed_sparse_long_02_b200 import layer
    R = len(caches)
    dev = ws["out"].device
    # The step's inputs (q, indexer query, head weights, positions) travel as one block:
    # packed at 256-byte offsets into one pinned host buffer per replica, copied with a
    # single memcpy into one device buffer, whose views the layer call reads.
    names = list(steps[0].keys())
    offs, off = {}, 0
    for k in names:
        offs[k] = off
        off += (steps[0][k].numel() * steps[0][k].element_size() + 255) // 256 * 256
    total = off

    def views(buf):
        return {k: buf[offs[k]:offs[k] + steps[0][k].numel() * steps[0][k].element_size()]
                .view(steps[0][k].dtype).view(steps[0][k].shape) for k in names}

    host = []
    for r in range(R):
        hb = torch.zeros(total, dtype=torch.uint8).pin_memory()
        hv = views(hb)
        for k in names:
            hv[k].copy_(steps[r][k].cpu())
        host.append(hb)
    NB = E2E_BUFFERS
    dev_buf = [torch.empty(total, dtype=torch.uint8, device=dev) for _ in range(NB)]
    dev_in = [views(b) for b in dev_buf]
    dev_out = [torch.empty((wl.B, wl.H, wl.D), dtype=torch.bfloat16, device=dev) for _ in range(NB)]
    out_host = [torch.empty((wl.B, wl.H, wl.D), dtype=torch.bfloat16).pin_memory() for _ in range(NB)]
    h2d = sum(steps[0][k].numel() * steps[0][k].element_size() for k in names)
    d2h = out_host[0].numel() * out_host[0].element_size()
    lws = {"q_fp4": ws["q_fp4"], "q_scale": ws["q_scale"], "index_ws": ws["index_ws"], "idx": ws["idx"], "cnt": ws["cnt"],
           "seq": ws["seq"], "attn_ws": ws["attn_ws"]}

    def upload(b, r):
        dev_buf[b].copy_(host[r], non_blocking=True)  # one host-to-device copy per step

    def compute(b, r):
        layer.csa_decode(wl, caches[r], dev_in[b], lws, out=dev_out[b])

    def download(b):
        out_host[b].copy_(dev_out[b], non_blocking=True)

    for b in range(NB):  # eager once per buffer set before capture
        upload(b, 0)
        compute(b, 0)
        download(b)
    torch.cuda.synchronize()
    g_up = [[capture_step(lambda b=b, r=r: upload(b, r)) for r in range(R)] for b in range(NB)]
    g_comp = [[capture_step(lambda b=b, r=r: compute(b, r)) for r in range(R)] for b in range(NB)]
    g_down = [capture_step(lambda b=b: download(b)) for b in range(NB)]
    torch.cuda.synchronize()
    s_up, s_comp, s_down = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    ev_up = [torch.cuda.Event() for _ in range(NB)]
    ev_comp = [torch.cuda.Event() for _ in range(NB)]
    ev_down = [torch.cuda.Event() for _ in range(NB)]

    def run(n0, n):
        for i in range(n0, n0 + n):
            b = i % NB
            if i - n0 >= NB:
                ev_down[b].synchronize()  # out_host[b] and dev_out[b] of step i - NB are free
            with torch.cuda.stream(s_up):
                s_up.wait_event(ev_comp[b])  # dev_in[b] no longer read by step i - NB
                g_up[b][i % R].replay()
                ev_up[b].record(s_up)
            with torch.cuda.stream(s_comp):
                s_comp.wait_event(ev_up[b])
                s_comp.wait_event(ev_down[b])  # dev_out[b] downloaded
                g_comp[b][i % R].replay()
                ev_comp[b].record(s_comp)
            with torch.cuda.stream(s_down):
                s_down.wait_event(ev_comp[b])
                g_down[b].replay()
                ev_down[b].record(s_down)
        for b in range(NB):
            ev_down[b].synchronize()

    torch.cuda.synchronize()
    run(0, max(args.warmup, NB))
    torch.cuda.synchronize()
    dist.barrier()
    t0 = time.perf_counter()
    n_steps = max(args.steps, E2E_MIN_STEPS)  # wall-clock timing: long enough that host jitter averages out
    run(0, n_steps)
    t = dist.max(time.perf_counter() - t0)
    del g_up, g_comp, g_down
    return {"value": wl.B * dist.world * n_steps / t, "unit": UNIT, "steps": n_steps, "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h,
            "pipelined": "upload of step i+1 and download of step i-1 overlap step i; each stage a CUDA graph replay"}


# ----------------------------------------------------------------------------- prefill
def _dev_inputs(inp, dev):
    import numpy as np
    import torch
    out = {}
    for k, v in inp.items():
        if v.dtype == np.uint16:
            out[k] = torch.from_numpy(v.view(np.int16)).view(torch.bfloat16).to(dev)
        else:
            out[k] = torch.from_numpy(np.ascontiguousarray(v)).to(dev)
    return out


def prefill_calls(wl, t, dev):
    """The prefill layer's C-ABI calls in the order the layer issues them, as (name, fn)
    pairs (the indexer's scoring and top-k as the two calls csa_index_topk is made of, so
    each is timed on its own)."""
    import torch
    from compressed_sparse_long_02_b200 import binding as B
    T, E = wl.T, wl.E
    pos = torch.arange(T, dtype=torch.int32, device=dev)
    seq = torch.zeros(T, dtype=torch.int32, device=dev)
    zero = torch.zeros(1, dtype=torch.int32, device=dev)
    ne = torch.tensor([E], dtype=torch.int32, device=dev)
    st = {}
    kw = dict(m=wl.m, overlap=wl.overlap, norm=wl.norm, eps=wl.eps, rope_dims=wl.rope_dims, theta=wl.theta)
    calls = [("compress_kv", lambda: st.__setitem__("pool", B.csa_compress(t["kv"], t["z"], t["bias"], want_window=True,
                                                                            **kw)))]
    if wl.kind == "csa_prefill":
        E_pad = max(8, (E + 7) // 8 * 8)
        calls += [
            ("compress_ki", lambda: st.__setitem__("keys", B.csa_compress(
                t["ki"], t["zi"], t["bias_i"], m=wl.m, overlap=wl.overlap, norm=False, want_entries=False,
                want_fp4=True, E_max=E_pad))),
            ("quantize_qi", lambda: st.__setitem__("qq", B.csa_quantize_mxfp4(t["qi"][0]))),
        ]
    q = t["q"][0]  # raw queries: the attention call applies their RMSNorm + RoPE as it loads them
    prep = dict(norm=wl.norm, eps=wl.eps, rope_dims=wl.rope_dims, theta=wl.theta)
    if wl.kind == "csa_prefill":
        w = t["w"][0].contiguous()
        scores = torch.empty((T, max(8, (E + 7) // 8 * 8)), dtype=torch.float32, device=dev)  # no fill inside the timing
        calls += [
            ("index_score", lambda: st.__setitem__("scores", B.csa_index_score(
                st["qq"][0], st["qq"][1], w, pos, seq, st["keys"]["fp4"], st["keys"]["fp4_scale"], ne, m=wl.m,
                scores=scores))),
            ("topk_select", lambda: st.__setitem__("sel", B.csa_topk_select(
                st["scores"], pos, seq, ne, k=wl.k, m=wl.m, E_max=st["keys"]["fp4"].shape[1]))),
            ("attention", lambda: st.__setitem__("out", B.csa_sparse_attn(
                q, pos, seq, st["pool"]["entries"], st["sel"][0], st["sel"][1], st["pool"]["window"], zero,
                W=wl.W, prep=prep)[0])),
        ]
    else:
        calls.append(("attention", lambda: st.__setitem__("out", B.hca_attn(
            q, pos, seq, st["pool"]["entries"], ne, st["pool"]["window"], zero, mprime=wl.m, W=wl.W, prep=prep)[0])))
    return calls


def prefill_work(wl) -> dict:
    """Algorithmic work of each prefill call: (bound, amount, unit) with bytes for the
    HBM-bound calls (compulsory traffic: inputs read once, outputs written once) and
    dense FLOPs for the contractions."""
    T, C, E, s = wl.T, wl.C, wl.E, (2 if wl.dtype == "bf16" else 4)
    w = {"compress_kv": ("hbm", 2 * T * C * s + E * C * 2 + T * C * 2)}  # kv, z in; entries, window rows out
    if wl.kind == "csa_prefill":
        Hi, Di = wl.Hi, wl.Di
        vis = sum(min((t + 1) // wl.m, E) for t in range(T))
        w["compress_ki"] = ("hbm", 2 * T * Di * s + E * (Di // 2 + Di // 32))
        w["quantize_qi"] = ("hbm", T * Hi * Di * s + T * Hi * (Di // 2 + Di // 32))
        w["index_score"] = ("tensor_fp4", indexer_flops(wl))
        w["topk_select"] = ("hbm", vis * 4 + T * wl.k * 4 + T * 4)
    w["attention"] = ("tensor_bf16", attention_flops(wl))
    return w


def bench_prefill(name, steps, warmup, dist, peaks, tensor_peaks):
    """One prefill workload: the whole layer per step (tok/s), then every call timed on
    its own (the calls queued behind a GPU sleep so that they run back to back between
    events), each against its roofline: HBM for the memory-bound calls, the measured
    bf16 library-GEMM burst peak for attention, the measured tcgen05 mxf4 rate for the
    FP4 indexer (burst figures: each call is timed alone)."""
    import torch
    from compressed_sparse_long_02_b200 import binding as B
    from compressed_sparse_long_02_b200 import layer, synth
    wl = synth.WORKLOADS[name]
    dev = torch.device("cuda", dist.local_rank)
    t = synth.prefill_inputs_torch(wl, dev)
    run = layer.csa_prefill if wl.kind == "csa_prefill" else layer.hca_prefill
    for _ in range(warmup):
        run(wl, t)
    torch.cuda.synchronize()
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    dist.barrier()
    s.record()
    for _ in range(steps):
        run(wl, t)
    e.record()
    torch.cuda.synchronize()
    ms = dist.max(s.elapsed_time(e)) / steps
    assert B.csa_get_device_error() == 0
    calls = prefill_calls(wl, t, dev)
    for _, fn in calls:  # warm the call sequence once
        fn()
    torch.cuda.synchronize()
    reps = max(2, steps)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(len(calls) + 1)] for _ in range(reps)]
    for r in range(reps):
        torch.cuda._sleep(20_000_000)
        evs[r][0].record()
        for j, (_, fn) in enumerate(calls):
            fn()
            evs[r][j + 1].record()
    torch.cuda.synchronize()
    assert B.csa_get_device_error() == 0
    per_us = {n: statistics.median(1e3 * ev[j].elapsed_time(ev[j + 1]) for ev in evs) for j, (n, _) in
              enumerate(calls)}
    work = prefill_work(wl)
    per_call = {}
    for n, us in per_us.items():
        bound, amount = work[n]
        if bound == "hbm":
            ach = amount / (us / 1e6) / 1e9
            per_call[n] = {"us": round(us, 2), "bound": "hbm", "algorithmic_bytes": amount, "achieved": round(ach, 1),
                           "unit": "GB/s", "frac": round(ach / peaks["hbm_gbs"], 4)}
        else:
            pk = tensor_peaks["mxf4_tflops"] if bound == "tensor_fp4" else peaks["bf16_tflops"]
            ach = amount / (us / 1e6) / 1e12
            per_call[n] = {"us": round(us, 2), "bound": "tensor", "algorithmic_flops": amount,
                           "achieved": round(ach, 1), "unit": "TFLOP/s", "frac": round(ach / pk, 4),
                           "peak": pk}
    att = per_call["attention"]
    out = {"workload": name, "tokens": wl.T, "tok_per_s": wl.T * dist.world / (ms / 1e3), "ms_per_step": ms,
           "roofline": {"bound": "tensor", "kernel": "attention", "achieved": att["achieved"],
                        "peak": peaks["bf16_tflops"], "unit": "TFLOP/s", "frac": att["frac"],
                        "attention_ms": round(att["us"] / 1e3, 4), "algorithmic_flops": att["algorithmic_flops"],
                        "peak_source": "measured bf16 library GEMM, burst (the call is timed alone)"},
           "per_call": per_call,
           "per_call_sum_us": round(sum(per_us.values()), 1)}
    if wl.kind == "csa_prefill":
        ix = per_call["index_score"]
        out["indexer"] = {"bound": "tensor", "kernel": "index_score", "achieved": ix["achieved"],
                          "peak": tensor_peaks["mxf4_tflops"], "unit": "TFLOP/s", "frac": ix["frac"],
                          "frac_of_datasheet": round(ix["achieved"] / tensor_peaks["mxf4_datasheet_tflops"], 4),
                          "index_ms": round(ix["us"] / 1e3, 4), "algorithmic_flops": ix["algorithmic_flops"],
                          "peak_source": "measured: tcgen05 kind::mxf4 probe (csa_mma_peak_probe)"}
    del t, calls
    torch.cuda.empty_cache()
    return out


def bench_out_proj(dist, peaks, reps: int = 5) -> dict:
    """The grouped output projection at the 8K prefill's size (8192 tokens, 64 heads of
    512 in 8 groups, R = 1024, hidden 4096): both tcgen05 GEMM stages of one call, timed
    alone with events, against the measured bf16 library-GEMM burst peak."""
    import torch
    from compressed_sparse_long_02_b200 import binding as B
    from compressed_sparse_long_02_b200 import synth
    ps = synth.PROJ["csa_prefill_8k"]
    dev = torch.device("cuda", dist.local_rank)
    d = synth.proj_inputs_torch(ps, dev)
    z = torch.empty((ps.T, ps.G * ps.R), dtype=torch.bfloat16, device=dev)
    y = torch.empty((ps.T, ps.d_model), dtype=torch.bfloat16, device=dev)
    for _ in range(2):
        B.csa_grouped_out_proj(d["o"], d["A"], d["Bm"], z=z, y=y)
    torch.cuda.synchronize()
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record()
    for _ in range(reps):
        B.csa_grouped_out_proj(d["o"], d["A"], d["Bm"], z=z, y=y)
    e.record()
    torch.cuda.synchronize()
    assert B.csa_get_device_error() == 0
    ms = s.elapsed_time(e) / reps
    flops = out_proj_flops(ps)
    tf = flops / (ms / 1e3) / 1e12
    del d, z, y
    torch.cuda.empty_cache()
    return {"workload": "grouped_out_proj_8k", "tokens": ps.T, "heads": ps.H, "head_dim": ps.D, "groups": ps.G,
            "group_rank": ps.R, "d_model": ps.d_model, "ms": round(ms, 4), "tok_per_s": ps.T / (ms / 1e3),
            "roofline": {"bound": "tensor", "kernel": "gemm_bf16 (two stages)", "achieved": round(tf, 1),
                         "peak": peaks["bf16_tflops"], "unit": "TFLOP/s", "frac": round(tf / peaks["bf16_tflops"], 4),
                         "algorithmic_flops": flops,
                         "peak_source": "measured bf16 library GEMM, burst (the call is timed alone)"}}


def out_proj_flops(ps) -> float:
    """2 x T x (H D R   (each group: (H/G) D inputs x R outputs, G groups)  +  G R d_model)."""
    return 2.0 * ps.T * (ps.H * ps.D * ps.R + ps.G * ps.R * ps.d_model)


def indexer_flops(wl) -> float:
    """2 x Hi x Di over every visible (query, entry) pair the indexer scores."""
    tot = sum(min((t + 1) // wl.m, wl.E) for t in range(wl.T))
    return 2.0 * wl.Hi * wl.Di * tot


def attention_flops(wl) -> float:
    """2 x (QK + PV) x H x D over every (query, key) pair the layer attends to."""
    tot = 0
    for t in range(wl.T):
        nv = (t + 1) // wl.m
        sel = min(wl.k, nv) if wl.kind == "csa_prefill" else min(nv, wl.E)
        tot += sel + min(wl.W, t + 1)
    return 4.0 * wl.H * wl.D * tot


# ----------------------------------------------------------------------------- CPU oracle
def cpu_oracle_decode(wl, n_seq: int, budget_s: float = 12.0, seed_replica: int = 0):
    """The oracle on a bounded sample of decode queries (full 32768-entry caches): rounds
    over `n_seq` sequences, one query per core at a time, until ~`budget_s` of CPU work."""
    import numpy as np
    import oracle
    from compressed_sparse_long_02_b200 import synth
    d = synth.decode_inputs(wl, B=n_seq, seed_offset=seed_replica)
    kp, ks = oracle.mxfp4_quantize(d["ki"])
    done, t_used = 0, 0.0
    cores = os.cpu_count() or 1
    chunk = max(1, min(n_seq, cores))
    start = 0
    while t_used < budget_s:
        seqs = np.arange(start, min(n_seq, start + chunk))
        start = 0 if start + chunk >= n_seq else start + chunk
        t0 = time.perf_counter()
        qp, qs = oracle.mxfp4_quantize(d["qi"])
        oracle.csa_decode(wl, d["entries"], kp, ks, d["q"], qp, qs, d["w"], d["window"], d["pos"], seqs=seqs)
        t_used += time.perf_counter() - t0
        done += len(seqs)
    threads = int(os.environ.get("OMP_NUM_THREADS", cores))
    return {"value": done / t_used, "unit": UNIT, "cores": threads, "kind": "oracle",
            "sample": f"{done} decode queries over {n_seq} sequences (full {wl.E}-entry caches, k={wl.k}, "
                      f"W={wl.W}), {chunk} in parallel, {t_used:.1f} s"}


def cpu_oracle_single_thread(wl, n_query: int = 4, timeout_s: float = 240.0) -> dict:
    """The same oracle decode on one thread: a child process with OMP_NUM_THREADS=1 (the
    oracle's OpenMP pool is sized when the library loads, so this process cannot shrink
    its own) runs `n_query` decode queries of full caches and reports queries/s."""
    code = ("import json, sys, time; sys.path.insert(0, %r)\n"
            "import oracle\nfrom compressed_sparse_long_02_b200 import synth\n"
            "wl = synth.WORKLOADS['csa_decode_128k']\n"
            "d = synth.decode_inputs(wl, B=%d)\n"
            "kp, ks = oracle.mxfp4_quantize(d['ki'])\n"
            "t0 = time.perf_counter()\n"
            "qp, qs = oracle.mxfp4_quantize(d['qi'])\n"
            "oracle.csa_decode(wl, d['entries'], kp, ks, d['q'], qp, qs, d['w'], d['window'], d['pos'])\n"
            "print(json.dumps({'s': time.perf_counter() - t0}))\n") % (ROOT, n_query)
    env = dict(os.environ, OMP_NUM_THREADS="1", CUDA_VISIBLE_DEVICES="")
    try:
        r = subprocess.run([sys.executable, "-c", code], env=env, cwd=ROOT, capture_output=True, text=True,
                           timeout=timeout_s)
        t = json.loads(r.stdout.strip().splitlines()[-1])["s"]
    except Exception as e:  # a baseline figure, never a reason to fail the benchmark
        return {"value": None, "unit": UNIT, "cores": 1, "error": str(e)[:200]}
    return {"value": n_query / t, "unit": UNIT, "cores": 1, "kind": "oracle",
            "sample": f"{n_query} decode queries (full {wl.E}-entry caches), OMP_NUM_THREADS=1, {t:.1f} s"}


def run_reference(args, dist):
    """The reference arm: the CPU oracle, as it stands, on bounded decode samples."""
    if dist.rank != 0:
        return None
    from compressed_sparse_long_02_b200 import synth
    wl = synth.WORKLOADS["csa_decode_128k"]
    cores = os.cpu_count() or 1
    per_step = max(1, min(wl.B, cores))
    import numpy as np
    import oracle
    d = synth.decode_inputs(wl, B=per_step)
    kp, ks = oracle.mxfp4_quantize(d["ki"])
    times = []
    for i in range(args.warmup + args.steps):
        t0 = time.perf_counter()
        qp, qs = oracle.mxfp4_quantize(d["qi"])
        oracle.csa_decode(wl, d["entries"], kp, ks, d["q"], qp, qs, d["w"], d["window"], d["pos"])
        if i >= args.warmup:
            times.append(time.perf_counter() - t0)
    tot = sum(times)
    value = per_step * len(times) / tot
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * tot / len(times),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": decode_config(wl, args),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": int(os.environ.get("OMP_NUM_THREADS", cores)),
                             "kind": "oracle",
                             "sample": f"{per_step} decode queries per step (full {wl.E}-entry caches)"},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    return line


def decode_config(wl, args):
    return {"workload": "csa_decode_128k", "sequences_per_gpu": wl.B, "context": wl.L, "entries": wl.E,
            "top_k": wl.k, "window": wl.W, "heads": wl.H, "head_dim": wl.D, "indexer_heads": wl.Hi,
            "indexer_dim": wl.Di, "indexer_format": "MXFP4 (E2M1, UE8M0 per 32)", "parallelism": f"dp{args.gpus}",
            "l2": f"inputs larger than L2: {args.replicas} rotating input replicas (~1.1 GB each); a replica is "
                  f"re-read only after {args.replicas - 1} other steps"}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="csa", choices=["csa", "reference"])
    ap.add_argument("--replicas", type=int, default=4)
    ap.add_argument("--no-secondary", action="store_true", help="skip the prefill lines")
    ap.add_argument("--no-cpu", action="store_true", help="skip the CPU oracle baseline")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)
    dist = Dist()
    try:
        if args.impl == "reference":
            line = run_reference(args, dist)
            if line is not None:
                print(json.dumps(line), flush=True)
            return
        import torch
        from compressed_sparse_long_02_b200 import binding
        binding.lib()
        peaks = load_peaks()
        wl, res = bench_decode(args, dist, peaks)
        line = {"metric": METRIC, "value": res["value"], "unit": UNIT, "n_gpus": dist.world, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": res["ms_per_step"], "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "bf16+mxfp4 (fp32 accumulate)",
                "data": "synthetic (seeded; N(0,1) caches and queries, U(0,1) head weights)",
                "config": decode_config(wl, args), "roofline": res["roofline"],
                "step_roofline": res["step_roofline"], "per_call_us": res["per_call_us"], "e2e": res["e2e"],
                "clocks": res["clocks"], "gpu_launches": res["gpu_launches"], "launch": res["graph"]}
        if not args.no_secondary:
            dev = torch.device("cuda", dist.local_rank)
            tp = measure_tensor_peaks(dev)
            line["tensor_peaks"] = tp
            wl1, r1 = bench_decode(args, dist, peaks, name="csa_decode_1m", e2e=False, steps=min(args.steps, 20))
            line["decode_1m"] = {"workload": "csa_decode_1m", "sequences_per_gpu": wl1.B, "context": wl1.L,
                                 "entries": wl1.E, "value": r1["value"], "unit": UNIT, "ms_per_step": r1["ms_per_step"],
                                 "step_roofline": r1["step_roofline"], "roofline": r1["roofline"],
                                 "per_call_us": r1["per_call_us"], "clocks": r1["clocks"]}
            line["gpu_launches_decode_1m"] = r1["gpu_launches"]
            line["decode_2tok"] = bench_decode_mq(args, dist, peaks)
            line["prefill"] = bench_prefill("csa_prefill_8k", 5, 2, dist, peaks, tp)
            line["hca_prefill"] = bench_prefill("hca_prefill_64k", 3, 1, dist, peaks, tp)
            line["out_proj"] = bench_out_proj(dist, peaks)
        if dist.rank == 0 and dist.world == 1 and not args.no_cpu:
            cb = cpu_oracle_decode(wl, n_seq=min(wl.B, max(4, os.cpu_count() or 4)))
            cb["single_thread"] = cpu_oracle_single_thread(wl)
            line["cpu_baseline"] = cb
        if dist.rank == 0:
            print(json.dumps(line), flush=True)
    finally:
        dist.close()


if __name__ == "__main__":
    main()
