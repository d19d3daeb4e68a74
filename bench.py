#!/usr/bin/env python
"""Benchmark of the packed binary-g128 decode GEMV (and the other hot-path kernels) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl {bq,reference}] [--quick]

Headline workload: binary-g128 decode GEMV at K = 5120, N in {5120, 20480}, M in {1, 4, 8},
x bf16 ~ N(0,1), sign bits Bernoulli(0.5), scales fp16 |N(0, 0.02)| + 1e-3, y fp32. One
step is the six GEMVs. The metric is algorithmic GB/s: (packed words + scales + x) bytes
per step / device time per step. The weights of each step are one of several copies that
together exceed twice the L2 size, so every step streams its weights from HBM.

Prints ONE JSON line (rank 0). With --gpus N > 1 (under torchrun) every rank runs the same
workload on its own GPU (independent replicas, no data-path collective); the value is the
bytes of all ranks over the slowest rank's time ("scaling": "weak").

--impl reference times the CPU oracle (fp64, plain C) on the host cores on bounded samples
of the same workload, in the same metric.
"""

from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import synth  # noqa: E402

K_HEAD = 5120
GEMV_SHAPES = [(5120, 1), (5120, 4), (5120, 8), (20480, 1), (20480, 4), (20480, 8)]   # (N, M)
METRIC = "packed-weight GEMV HBM GB/s & % of 8 TB/s roofline at K=5120; prefill TFLOP/s"
NOMINAL_HBM_GBS = 8000.0


def gemv_bytes(N, K, M, fmt_bits=1):
    """Algorithmic bytes of one GEMV: packed weights + fp16 scales + bf16 activations."""
    return N * K * fmt_bits // 8 + N * (K // 128) * 2 + M * K * 2


def read_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained"), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "source": "fallback"}


# --------------------------------------------------------------------------------------
# distributed plumbing (one process per GPU; replicas)
# --------------------------------------------------------------------------------------

def dist_init():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if world <= 1:
        return 0, 1, None
    import torch.distributed as dist
    import datetime
    backend = "nccl" if torch.cuda.is_available() else "gloo"
    dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return dist.get_rank(), dist.get_world_size(), dist


def reduce_max(value: float, dist, device) -> float:
    if dist is None:
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(dist, device):
    if dist is not None:
        if device.type == "cuda":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


# --------------------------------------------------------------------------------------
# clocks during the timed region
# --------------------------------------------------------------------------------------

class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.proc = None
        self.lines = []
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(device_index), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except (OSError, FileNotFoundError):
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.t.join(timeout=2)
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                mx.append(float(parts[1]))
            except ValueError:
                continue
            for n, v in zip(names, parts[4:8]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "samples": len(sm),
                "reasons": sorted(reasons)}


# --------------------------------------------------------------------------------------
# GPU workloads
# --------------------------------------------------------------------------------------

def l2_bytes(device) -> int:
    return torch.cuda.get_device_properties(device).L2_cache_size


def make_gemv_sets(bq, device, copies: int):
    """`copies` independent weight sets for the six headline GEMVs (seed = copy index)."""
    sets = []
    for c in range(copies):
        layer = []
        for (N, M) in GEMV_SHAPES:
            words = synth.binary_words(c, N, K_HEAD, device=device)
            s = synth.scales(c, N, K_HEAD // 128).to(device)
            w = bq.BQWeight(bq.BINARY_G128, N, K_HEAD, words, s)
            x = synth.activations(c, M, K_HEAD, dtype=torch.bfloat16).to(device)
            y = torch.empty((M, N), dtype=torch.float32, device=device)
            layer.append((w, x, y))
        sets.append(layer)
    return sets


def capture_step_graphs(bq, sets, stream):
    """One CUDA graph per weight copy; each replays the six GEMVs of a step."""
    graphs, launches = [], []
    for layer in sets:
        for (w, x, y) in layer:                     # eager warm-up outside capture
            bq.gemv(x, w, out=y)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        before = bq.kernel_launches()
        with torch.cuda.graph(g, stream=stream):
            for (w, x, y) in layer:
                bq.gemv(x, w, out=y)
        launches.append(bq.kernel_launches() - before)
        graphs.append(g)
    return graphs, launches


def time_graphs(graphs, steps, warmup, stream, dist, device):
    """Device ms of exactly `steps` steps after `warmup` untimed ones, bracketed by a barrier and
    a synchronize on both sides."""
    for i in range(warmup):
        graphs[i % len(graphs)].replay()
    torch.cuda.synchronize()
    barrier(dist, device)
    torch.cuda.synchronize()
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        start.record(stream)
        for i in range(steps):
            graphs[i % len(graphs)].replay()
        end.record(stream)
    end.synchronize()
    torch.cuda.synchronize()
    barrier(dist, device)
    return start.elapsed_time(end)


def time_regions(graphs, steps, warmup, stream, dist, device, min_seconds=1.0, max_regions=2000):
    """The timed region (exactly `steps` steps) repeated R times, so that a clock sampler running
    alongside sees the GPU under load; R is the same on every rank. Returns (the median region's
    ms, every region's ms)."""
    first = time_graphs(graphs, steps, warmup, stream, dist, device)
    R = max(1, min(max_regions, math.ceil(min_seconds * 1e3 / max(first, 1e-3))))
    R = int(reduce_max(float(R), dist, device))
    times = [time_graphs(graphs, steps, 0, stream, dist, device) for _ in range(R)]
    return statistics.median(times), times


def time_single(fn, reps, warmup, stream):
    """Average device time (ms) of one call of fn() over reps back-to-back calls."""
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(reps):
        fn()
    b.record(stream)
    b.synchronize()
    return a.elapsed_time(b) / reps


def per_config_breakdown(bq, sets, stream):
    """GB/s of each headline GEMV alone, rotating over the weight copies (L2-cold)."""
    out = []
    for j, (N, M) in enumerate(GEMV_SHAPES):
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=stream):
            for layer in sets:
                w, x, y = layer[j]
                bq.gemv(x, w, out=y)
        ms = time_single(graph.replay, 20, 3, stream) / len(sets)
        gb = gemv_bytes(N, K_HEAD, M) / 1e9
        out.append({"N": N, "K": K_HEAD, "M": M, "us": round(ms * 1e3, 3),
                    "GBps": round(gb / (ms / 1e3), 1)})
        del graph
    return out


# --------------------------------------------------------------------------------------
# every configuration of the benchmark: device time, roofline fraction, the CPU oracle's time
# on the host cores beside it, and a sampled oracle check of the same outputs
# --------------------------------------------------------------------------------------

class OracleBench:
    """The CPU oracle (plain C, fp64) timed on the host cores on bounded samples of a workload,
    and used to check sampled outputs of the GPU runs (outside every timed region)."""

    def __init__(self, budget_s: float = 1.5):
        import oracle
        self.o = oracle
        self.orc = oracle.default()
        self.cores = os.cpu_count() or 1
        self.budget = budget_s

    def time_items(self, work, n_items: int, threads: int):
        """Seconds for n items of `work(lo, hi)` (item indices taken modulo n_items) on `threads`
        threads, with n sized to about the budget (one item is timed first). Returns (seconds, n)."""
        import concurrent.futures as cf
        t0 = time.perf_counter()
        work(0, 1)
        one = max(time.perf_counter() - t0, 1e-6)
        n = max(threads, int(self.budget * threads / one))
        chunks = []
        for i in range(threads):                       # each thread's share, in passes over the items
            lo, hi = n * i // threads, n * (i + 1) // threads
            while hi > lo:
                a = lo % n_items
                b = min(n_items, a + (hi - lo))
                chunks.append((a, b))
                lo += b - a
        t0 = time.perf_counter()
        with cf.ThreadPoolExecutor(max_workers=threads) as ex:
            list(ex.map(lambda c: work(*c), chunks))
        return time.perf_counter() - t0, n

    def gemv_timing(self, fmt, x, xt, words, scales, K, bytes_per_row, x_bytes, one_core: bool):
        """Oracle GB/s on the rows of `words` (host arrays), all cores (and one core)."""
        def work(lo, hi):
            self.orc.gemv(fmt, x, xt, words[lo:hi], scales[lo:hi], K)
        res = {}
        for label, th in (("all_cores", self.cores), ("one_core", 1)) if one_core else (("all_cores", self.cores),):
            dt, n = self.time_items(work, len(words), th)
            res[label] = {"GBps": round((n * bytes_per_row + x_bytes) / 1e9 / dt, 4), "cores": th,
                          "sample": f"{n} rows x all K (passes over {len(words)} distinct rows), {dt:.3f} s"}
        return res

    def max_ratio(self, fmt, x, xt, words, scales, K, y_rows):
        """max |y - y_ref| / (2e-3 sum |x s|) over the given rows (y_rows [M, R] from the GPU)."""
        y_ref, bound = self.orc.gemv(fmt, x, xt, words, scales, K)
        import numpy as np
        err = np.abs(y_rows.astype(np.float64) - y_ref)
        return float(np.max(err / np.maximum(bound, 1e-300)))


def _host_binary(seed, rows, K, row0=0):
    return (synth.binary_words(seed, rows, K, row0=row0).numpy(),
            synth.scales(seed, rows, K // 128, row0=row0).numpy())


def _host_ternary(ob, seed, rows, K, row0=0):
    q = synth.random_ternary(seed, synth.TID_TERNARY, (rows, K), row0=row0)
    s = synth.scales(seed, rows, K // 128, row0=row0)
    st, words, s_out = ob.orc.pack(ob.o.TERNARY, q.numpy(), s.numpy())
    assert st == ob.o.OK
    return words, s_out


def _host_ternary_b3(ob, seed, rows, K, row0=0):
    q = synth.random_ternary(seed, synth.TID_TERNARY, (rows, K), row0=row0)
    s = synth.scales(seed, rows, K // 128, row0=row0)
    st, packed, s_out = ob.orc.pack(ob.o.TERNARY_B3, q.numpy(), s.numpy())
    assert st == ob.o.OK
    return packed, s_out


def _gemv_entry(name, N, K, M, fmt_bits, ms, peaks, extra=None):
    gb = gemv_bytes(N, K, M, fmt_bits) / 1e9
    gbs = gb / (ms / 1e3)
    e = {"workload": name, "N": N, "K": K, "M": M, "us": round(ms * 1e3, 2), "GBps": round(gbs, 1),
         "bound": "hbm", "frac": round(gbs / peaks["hbm_gbs"], 4), "peak": peaks["hbm_gbs"]}
    if extra:
        e.update(extra)
    return e


def lm_head_topk_entry(bq, device, stream, peaks, ob, w, x, xd, oracle_timing):
    """The LM head fused with top-k 20 and a draw (temperature 0.7, top-p 0.95), M = 1: one call
    computes the 248 320 logits, keeps the 20 largest and draws a token; the logits are never
    written. Timed like the plain LM head; checked against the oracle on the full row."""
    import numpy as np
    o = ob.o
    N, K, k = w.N, w.K, 20
    u = torch.tensor([0.37], dtype=torch.float32, device=device)
    ws = torch.empty(bq.gemv_topk_workspace_bytes(1, w, k), dtype=torch.uint8, device=device)
    vals = torch.empty((1, k), dtype=torch.float32, device=device)
    idx = torch.empty((1, k), dtype=torch.int32, device=device)
    tok = torch.empty((1,), dtype=torch.int32, device=device)
    call = lambda: bq.gemv_topk(xd, w, k=k, u=u, temperature=0.7, top_p=0.95, workspace=ws, out=(vals, idx, tok))
    call()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for _ in range(20):
            call()
    ms = time_single(g.replay, 10, 3, stream) / 20
    del g
    call()
    torch.cuda.synchronize()
    # parity: the oracle's logits of the full row (all 248320), its top 20, and its draw
    words, sc = _host_binary(0, N, K)
    y_ref, bound = ob.orc.gemv(o.BINARY, x, o.X_BF16, words, sc, K)
    oi, ov = ob.orc.topk(y_ref, k)
    gi, gv = idx.cpu().numpy()[0], vals.cpu().numpy()[0].astype(np.float64)
    same_set = set(gi.tolist()) == set(oi[0].tolist())
    ratio = float(np.max(np.abs(gv - y_ref[0, gi]) / bound[0, gi]))
    draw_ref = ob.orc.sample_topk(gv, gi, 0.7, 0.95, 0.37)
    ent = _gemv_entry(f"LM head fused with top-k {k} and a draw (temperature 0.7, top-p 0.95), binary g128, "
                      f"M=1, K=5120, N=248320", N, K, 1, 1, ms, peaks,
                      {"timing": "graph of 20 back-to-back calls (179 MB of weights per call, above L2)",
                       "parity": {"max_err_over_bound": round(ratio, 5), "same_set_as_oracle": same_set,
                                  "token": int(tok.item()), "oracle_draw_on_same_candidates": draw_ref,
                                  "rows": N}})
    ent["oracle"] = oracle_timing
    return ent


def mlp_entry(bq, device, stream, peaks, ob):
    """The SwiGLU MLP of one block at M = 1: gate and up 20480 x 5120 and down 5120 x 20480, binary
    (the two MLP GEMVs of the full-depth step), as one fused call and as three GEMVs with SwiGLU
    in torch between them. Weights of 8 blocks rotate (together above L2)."""
    import numpy as np
    o = ob.o
    K, F, N, M = K_HEAD, 20480, K_HEAD, 1
    copies = 8
    blocks = []
    for c in range(copies):
        mk = lambda rows, cols, tid: bq.BQWeight(bq.BINARY_G128, rows, cols,
                                                 synth.binary_words(100 * c + tid, rows, cols, device=device),
                                                 synth.scales(100 * c + tid, rows, cols // 128, device=device))
        blocks.append((mk(F, K, 1), mk(F, K, 2), mk(N, F, 3)))
    x = synth.activations(0, M, K)
    xd = x.to(device)
    y = torch.empty((M, N), dtype=torch.float32, device=device)
    ws = torch.empty(bq.mlp_swiglu_workspace_bytes(M, *blocks[0]), dtype=torch.uint8, device=device)
    g = torch.cuda.CUDAGraph()
    for b in blocks:
        bq.mlp_swiglu(xd, *b, out=y, workspace=ws)
    torch.cuda.synchronize()
    with torch.cuda.graph(g, stream=stream):
        for i in range(2 * copies):
            bq.mlp_swiglu(xd, *blocks[i % copies], out=y, workspace=ws)
    ms = time_single(g.replay, 10, 3, stream) / (2 * copies)
    del g
    # separate: gate, up, SwiGLU (torch), down
    gy = torch.empty((M, F), dtype=torch.float32, device=device)
    uy = torch.empty((M, F), dtype=torch.float32, device=device)
    act = torch.empty((M, F), dtype=torch.float32, device=device)
    g2 = torch.cuda.CUDAGraph()
    def sep(b):
        bq.gemv(xd, b[0], out=gy)
        bq.gemv(xd, b[1], out=uy)
        torch.mul(torch.nn.functional.silu(gy), uy, out=act)
        bq.gemv(act, b[2], out=y)
    for b in blocks:
        sep(b)
    torch.cuda.synchronize()
    with torch.cuda.graph(g2, stream=stream):
        for i in range(2 * copies):
            sep(blocks[i % copies])
    ms_sep = time_single(g2.replay, 10, 3, stream) / (2 * copies)
    del g2
    bq.mlp_swiglu(xd, *blocks[0], out=y, workspace=ws)
    torch.cuda.synchronize()
    # parity: sampled rows of the first block against the oracle
    b0 = blocks[0]
    host = lambda w: (w.words.cpu().numpy().view(np.uint32), w.scales.cpu().numpy())
    rows = np.arange(0, N, 40)
    _, y_ref, bound = ob.orc.mlp_swiglu(x, o.X_BF16, o.BINARY, host(b0[0]), host(b0[1]), o.BINARY, host(b0[2]))
    ratio = float(np.max(np.abs(y.cpu().numpy()[:, rows] - y_ref[:, rows]) / bound[:, rows]))
    nbytes = 2 * gemv_bytes(F, K, M, 1) + gemv_bytes(N, F, M, 1)
    gbs = nbytes / 1e9 / (ms / 1e3)
    del blocks, ws
    return {"workload": "SwiGLU MLP of one block, binary g128, M=1: gate and up 20480x5120 (one GEMV with the "
                        "SwiGLU epilogue), down 5120x20480 on the fp32 activations",
            "us": round(ms * 1e3, 2), "GBps": round(gbs, 1), "bound": "hbm",
            "frac": round(gbs / peaks["hbm_gbs"], 4), "peak": peaks["hbm_gbs"],
            "separate_calls_us": round(ms_sep * 1e3, 2),
            "timing": f"graphs of back-to-back calls rotating {copies} blocks ({copies * nbytes / 1e6:.0f} MB)",
            "parity": {"max_err_over_bound": round(ratio, 5), "rows": int(len(rows))}}


def quantize_entry(bq, device, stream, peaks, ob, fmt_name):
    """Dense bf16 weights (N=20480, K=5120, 210 MB, above L2) to the packed format by the
    least-squares fit of every group of 128; algorithmic bytes = dense read + packed and scales
    written."""
    import numpy as np
    o = ob.o
    N, K = 20480, K_HEAD
    fmt = {"binary": bq.BINARY_G128, "ternary": bq.TERNARY_G128, "ternary_b3": bq.TERNARY_B3_G128}[fmt_name]
    ofmt = {"binary": o.BINARY, "ternary": o.TERNARY, "ternary_b3": o.TERNARY_B3}[fmt_name]
    wd = (synth.activations(5, N, K, dtype=torch.float32) * 0.02).to(torch.bfloat16).to(device)
    pw = bq.quantize_g128(wd, fmt)
    out_bytes = pw.words.numel() * pw.words.element_size() + pw.scales.numel() * 2
    nbytes = N * K * 2 + out_bytes
    ms = time_single(lambda: bq.quantize_g128(wd, fmt), 10, 3, stream)
    gbs = nbytes / 1e9 / (ms / 1e3)
    # parity: the first 64 rows against the oracle's fit, bit for bit (codes and scales)
    rows = 64
    w_host = wd[:rows].float().cpu().numpy()
    q_ref, s_ref = ob.orc.quantize(o.TERNARY if ofmt == o.TERNARY_B3 else ofmt, w_host)
    st, packed_ref, _ = ob.orc.pack(ofmt, q_ref, s_ref.view(np.float16))
    got = pw.words[:rows].cpu().numpy()
    if ofmt != o.TERNARY_B3:
        got = got.view(np.uint32)
    exact = bool(np.array_equal(got, packed_ref) and
                 np.array_equal(pw.scales[:rows].cpu().view(torch.int16).numpy().view(np.uint16), s_ref))

    def work(lo, hi):
        ob.orc.quantize(o.TERNARY if ofmt == o.TERNARY_B3 else ofmt, w_host[lo:hi])
    dt, n = ob.time_items(work, rows, ob.cores)
    del wd, pw
    return {"workload": f"dense bf16 -> {fmt_name} g128 quantiser (least-squares fit per group), N=20480, K=5120",
            "us": round(ms * 1e3, 1), "GBps": round(gbs, 1), "bound": "hbm",
            "frac": round(gbs / peaks["hbm_gbs"], 4), "peak": peaks["hbm_gbs"],
            "timing": "back-to-back calls on one 210 MB dense matrix (above L2)",
            "parity": {"bit_exact_rows": rows, "bit_exact": exact},
            "oracle": {"all_cores": {"GBps": round(n * (K * 2 + out_bytes / N) / 1e9 / dt, 4), "cores": ob.cores,
                                     "sample": f"{n} rows of the 64-row slice, {dt:.3f} s"}}}


def _rotating_gemv_ms(bq, mats, x, y, ws, stream, reps=20):
    """Device ms of one call over a CUDA graph of back-to-back calls that rotate through `mats`
    (weight copies together larger than L2)."""
    g = torch.cuda.CUDAGraph()
    for w in mats:
        bq.gemv(x, w, out=y, workspace=ws)
    torch.cuda.synchronize()
    with torch.cuda.graph(g, stream=stream):
        for i in range(reps):
            bq.gemv(x, mats[i % len(mats)], out=y, workspace=ws)
    ms = time_single(g.replay, 10, 3, stream) / reps
    del g
    return ms


def config_reports(bq, device, stream, peaks, ob: "OracleBench", breakdown):
    """One entry per workload: the 1024 x 1024 GEMV, the headline GEMVs, the LM head and the gather,
    the ternary GEMV and prefill, the binary prefill and the full-depth step, with the native
    ternary, top-k, MLP and quantiser entries beside them."""
    import numpy as np
    l2 = l2_bytes(device)
    out = []
    o = ob.o

    # ---- binary GEMV, M=1, K=N=1024, x fp16, seed 0 (L2-resident: reported in us)
    N, K = 1024, 1024
    w = bq.BQWeight(bq.BINARY_G128, N, K, synth.binary_words(0, N, K, device=device),
                    synth.scales(0, N, K // 128, device=device))
    x = synth.activations(0, 1, K, dtype=torch.float16)
    xd = x.to(device)
    y = torch.empty((1, N), dtype=torch.float32, device=device)
    ws = torch.empty(max(bq.gemv_workspace_bytes(1, w), 16), dtype=torch.uint8, device=device)
    ms = _rotating_gemv_ms(bq, [w], xd, y, ws, stream, reps=50)
    bq.gemv(xd, w, out=y, workspace=ws)
    words, sc = _host_binary(0, N, K)
    ratio = ob.max_ratio(o.BINARY, x, o.X_F16, words, sc, K, y.cpu().numpy())
    e = _gemv_entry("binary g128 GEMV, M=1, K=N=1024, x fp16, seed 0 (all 1024 outputs checked)",
                    N, K, 1, 1, ms, peaks,
                    {"timing": "graph of 50 back-to-back calls on the same weights (147 KB: L2-resident)",
                     "parity": {"max_err_over_bound": round(ratio, 5), "outputs": N}})
    e["oracle"] = ob.gemv_timing(o.BINARY, x, o.X_F16, words, sc, K, K // 8 + K // 64, 2 * K, True)
    out.append(e)
    del w, y, ws

    # ---- the headline GEMVs (K=5120, N in {5120, 20480}, M in {1, 4, 8}); the
    # device times are the breakdown's (rotating weight copies); parity on copy 0
    shapes = []
    for j, (N, M) in enumerate(GEMV_SHAPES):
        K = K_HEAD
        bd = breakdown[j] if breakdown else None
        w = bq.BQWeight(bq.BINARY_G128, N, K, synth.binary_words(0, N, K, device=device),
                        synth.scales(0, N, K // 128, device=device))
        x = synth.activations(0, M, K)
        y = bq.gemv(x.to(device), w)
        rows = 256
        words, sc = _host_binary(0, rows, K)
        ratio = ob.max_ratio(o.BINARY, x, o.X_BF16, words, sc, K, y[:, :rows].cpu().numpy())
        ent = {"N": N, "M": M, "parity": {"max_err_over_bound": round(ratio, 5), "rows": rows}}
        if bd:
            ent.update({"us": bd["us"], "GBps": bd["GBps"], "frac": round(bd["GBps"] / peaks["hbm_gbs"], 4)})
        ent["oracle"] = ob.gemv_timing(o.BINARY, x, o.X_BF16, *_host_binary(0, 4096, K), K,
                                       K // 8 + K // 64, 2 * M * K, N <= 5120)
        shapes.append(ent)
        del w, y
    out.append({"workload": "binary g128 decode GEMV, K=5120, N in {5120, 20480}, M in {1, 4, 8} "
                            "(the headline step; one entry per GEMV, each timed alone over rotating copies)",
                "bound": "hbm", "peak": peaks["hbm_gbs"], "gemvs": shapes})

    # ---- LM head (M=1, K=5120, N=248320) and the embedding gather of 4096 ids
    N, K = 248320, K_HEAD
    w = bq.BQWeight(bq.BINARY_G128, N, K, synth.binary_words(0, N, K, device=device),
                    synth.scales(0, N, K // 128, device=device))
    x = synth.activations(0, 1, K)
    xd = x.to(device)
    y = torch.empty((1, N), dtype=torch.float32, device=device)
    ws = torch.empty(max(bq.gemv_workspace_bytes(1, w), 16), dtype=torch.uint8, device=device)
    ms = _rotating_gemv_ms(bq, [w], xd, y, ws, stream, reps=20)
    rows = 512
    words, sc = _host_binary(0, rows, K, row0=N - rows)
    ratio = ob.max_ratio(o.BINARY, x, o.X_BF16, words, sc, K, y[:, N - rows:].cpu().numpy())
    e = _gemv_entry("LM-head GEMV, binary g128, M=1, K=5120, N=248320", N, K, 1, 1, ms, peaks,
                    {"timing": "graph of 20 back-to-back calls (179 MB of weights per call, above L2)",
                     "parity": {"max_err_over_bound": round(ratio, 5), "rows": rows}})
    e["oracle"] = ob.gemv_timing(o.BINARY, x, o.X_BF16, *_host_binary(0, 4096, K), K, K // 8 + K // 64,
                                 2 * K, False)
    out.append(e)
    out.append(lm_head_topk_entry(bq, device, stream, peaks, ob, w, x, xd, e["oracle"]))
    # embedding gather: output buffers rotate (together above L2), so the writes reach HBM
    T = 4096
    ids = synth.random_ids(0, synth.TID_IDS, T, N)
    idd = ids.to(device)
    nbuf = max(2, math.ceil(2.5 * l2 / (T * K * 2)))
    outs = [torch.empty((T, K), dtype=torch.bfloat16, device=device) for _ in range(nbuf)]
    for o_ in outs:
        bq.embed_gather(idd, w, out=o_)
    torch.cuda.synchronize()
    # a graph of back-to-back calls, as for the GEMVs: eager launches from Python take longer than
    # one gather and would time the host instead
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for i in range(2 * nbuf):
            bq.embed_gather(idd, w, out=outs[i % nbuf])
    ms = time_single(g.replay, 10, 3, stream) / (2 * nbuf)
    del g
    eb = T * (K // 8 + K // 64 + K * 2) + T * 4
    # bit-exact check of the ids that fall in the first 4096 rows (host words of those rows only)
    R = 4096
    words, sc = _host_binary(0, R, K)
    sel = (ids < R).nonzero().flatten()
    ref, bad = ob.orc.embed(o.BINARY, ids[sel].numpy(), words, sc, K)
    got = outs[0][sel.to(device)].view(torch.int16).cpu().numpy().view(np.uint16)
    exact = bool(np.array_equal(got, ob.orc.to_bf16_bits(ref))) and bad == 0

    def ework(lo, hi):
        ob.orc.embed(o.BINARY, (ids[lo:hi] % R).numpy(), words, sc, K)
    dt, n = ob.time_items(ework, T, ob.cores)
    gbs = eb / 1e9 / (ms / 1e3)
    out.append({"workload": "embedding gather, 4096 ids uniform in [0, 248320), K=5120, bf16 out",
                "us": round(ms * 1e3, 2), "GBps": round(gbs, 1), "bound": "hbm",
                "frac": round(gbs / peaks["hbm_gbs"], 4), "peak": peaks["hbm_gbs"],
                "timing": f"graph of {2 * nbuf} back-to-back calls, {nbuf} output buffers rotated ({nbuf * T * K * 2 / 1e6:.0f} MB vs {l2 / 1e6:.0f} MB L2)",
                "parity": {"bit_exact": exact, "ids_checked": int(len(sel))},
                "oracle": {"all_cores": {"GBps": round(n / T * eb / 1e9 / dt, 4), "cores": ob.cores,
                                         "sample": f"{n} ids (rows of a 4096-row slice), {dt:.3f} s"}}})
    del w, y, ws, outs

    # ---- ternary GEMV (N=20480, K=5120, M=1) and ternary prefill (M=512)
    N, K = 20480, K_HEAD
    copies = max(2, math.ceil(2.5 * l2 / gemv_bytes(N, K, 1, 2)))
    tmats = []
    for c in range(copies):
        q = synth.random_ternary(c, synth.TID_TERNARY, (N, K), device=device)
        tmats.append(bq.pack_ternary_g128(q, synth.scales(c, N, K // 128, device=device)))
        del q
    x = synth.activations(0, 1, K)
    xd = x.to(device)
    y = torch.empty((1, N), dtype=torch.float32, device=device)
    ws = torch.empty(max(bq.gemv_workspace_bytes(1, tmats[0]), 16), dtype=torch.uint8, device=device)
    ms = _rotating_gemv_ms(bq, tmats, xd, y, ws, stream, reps=2 * copies)
    bq.gemv(xd, tmats[0], out=y, workspace=ws)
    rows = 256
    words, sc = _host_ternary(ob, 0, rows, K)
    ratio = ob.max_ratio(o.TERNARY, x, o.X_BF16, words, sc, K, y[:, :rows].cpu().numpy())
    e = _gemv_entry("ternary g128 GEMV, M=1, K=5120, N=20480", N, K, 1, 2, ms, peaks,
                    {"timing": f"graph of back-to-back calls rotating {copies} weight copies (above L2)",
                     "parity": {"max_err_over_bound": round(ratio, 5), "rows": rows}})
    e["oracle"] = ob.gemv_timing(o.TERNARY, x, o.X_BF16, *_host_ternary(ob, 0, 2048, K), K,
                                 K // 4 + K // 64, 2 * K, False)
    out.append(e)
    del tmats

    # ---- the same ternary matrix in base-3 storage (26 bytes per group: 1.625 bits per weight
    # of codes, 1.75 with the scale), decoded inside the GEMV
    b3_bits = 26 * 8 / 128
    copies = max(2, math.ceil(2.5 * l2 / gemv_bytes(N, K, 1, b3_bits)))
    bmats = []
    for c in range(copies):
        q = synth.random_ternary(c, synth.TID_TERNARY, (N, K), device=device)
        bmats.append(bq.pack_ternary_b3_g128(q, synth.scales(c, N, K // 128, device=device)))
        del q
    ms = _rotating_gemv_ms(bq, bmats, xd, y, ws, stream, reps=2 * copies)
    bq.gemv(xd, bmats[0], out=y, workspace=ws)
    packed, sc = _host_ternary_b3(ob, 0, rows, K)
    ratio = ob.max_ratio(o.TERNARY_B3, x, o.X_BF16, packed, sc, K, y[:, :rows].cpu().numpy())
    e = _gemv_entry("ternary g128 in base-3 storage (1.75 bits/weight) GEMV, M=1, K=5120, N=20480",
                    N, K, 1, b3_bits, ms, peaks,
                    {"timing": f"graph of back-to-back calls rotating {copies} weight copies (above L2)",
                     "parity": {"max_err_over_bound": round(ratio, 5), "rows": rows},
                     "bytes_vs_2bit": round(gemv_bytes(N, K, 1, b3_bits) / gemv_bytes(N, K, 1, 2), 4)})
    e["oracle"] = ob.gemv_timing(o.TERNARY_B3, x, o.X_BF16, *_host_ternary_b3(ob, 0, 2048, K), K,
                                 26 * K // 128 + K // 64, 2 * K, False)
    out.append(e)
    del bmats, y, ws
    out.append(prefill_report(bq, device, stream, peaks, ob, "ternary", l2))
    out.append(prefill_report(bq, device, stream, peaks, ob, "ternary_b3", l2))

    # ---- binary prefill (M=512) and the full-depth decode step
    out.append(prefill_report(bq, device, stream, peaks, ob, "binary", l2))
    out.append(full_depth_step(bq, device, stream, peaks, ob))
    out.append(mlp_entry(bq, device, stream, peaks, ob))
    for fmt_name in ("binary", "ternary", "ternary_b3"):
        out.append(quantize_entry(bq, device, stream, peaks, ob, fmt_name))
    torch.cuda.empty_cache()
    return out


def prefill_report(bq, device, stream, peaks, ob, fmt_name, l2):
    """M=512, K=5120, N=20480 prefill GEMM, bf16 x and out; sets of (weights, x, y) rotate so
    that they are together larger than L2."""
    M, N, K = 512, 20480, K_HEAD
    o = ob.o
    bits = {"binary": 1, "ternary": 2, "ternary_b3": 26 * 8 / 128}[fmt_name]
    per_set = gemv_bytes(N, K, 0, bits) + M * K * 2 + M * N * 2
    nset = max(2, math.ceil(1.5 * l2 / per_set))
    sets = []
    for c in range(nset):
        if fmt_name == "binary":
            pw = bq.BQWeight(bq.BINARY_G128, N, K, synth.binary_words(c, N, K, device=device),
                             synth.scales(c, N, K // 128, device=device))
        else:
            q = synth.random_ternary(c, synth.TID_TERNARY, (N, K), device=device)
            pack = bq.pack_ternary_g128 if fmt_name == "ternary" else bq.pack_ternary_b3_g128
            pw = pack(q, synth.scales(c, N, K // 128, device=device))
            del q
        sets.append((pw, synth.activations(c, M, K).to(device),
                     torch.empty((M, N), dtype=torch.bfloat16, device=device)))
    ws = torch.empty(max(bq.prefill_workspace_bytes(M, sets[0][0]), 16), dtype=torch.uint8, device=device)
    it = [0]

    def call():
        pw, X, Y = sets[it[0] % nset]
        bq.gemm_prefill(X, pw, out=Y, workspace=ws)
        it[0] += 1
    ms = time_single(call, 4 * nset, nset, stream)
    tf = 2 * M * N * K / (ms / 1e3) / 1e12
    # parity: rows 0..63 of set 0 against the oracle, all 512 tokens
    pw, X, Y = sets[0]
    bq.gemm_prefill(X, pw, out=Y, workspace=ws)
    x = synth.activations(0, M, K)
    rows = 64
    fmt = {"binary": o.BINARY, "ternary": o.TERNARY, "ternary_b3": o.TERNARY_B3}[fmt_name]
    words, sc = {"binary": lambda: _host_binary(0, rows, K), "ternary": lambda: _host_ternary(ob, 0, rows, K),
                 "ternary_b3": lambda: _host_ternary_b3(ob, 0, rows, K)}[fmt_name]()
    ratio = ob.max_ratio(fmt, x, o.X_BF16, words, sc, K, Y[:, :rows].float().cpu().numpy())

    def work(lo, hi):
        ob.orc.gemv(fmt, x, o.X_BF16, words[lo:hi], sc[lo:hi], K)
    dt, n = ob.time_items(work, rows, ob.cores)
    del sets, ws
    name = {"binary": "binary g128", "ternary": "ternary g128",
            "ternary_b3": "ternary g128 in base-3 storage (1.75 bits/weight)"}[fmt_name]
    return {"workload": f"{name} prefill GEMM, M=512, K=5120, N=20480, x and y bf16",
            "us": round(ms * 1e3, 1), "TFLOPs": round(tf, 1), "bound": "tensor",
            "frac": round(tf / peaks["bf16_tflops"], 4), "peak": peaks["bf16_tflops"],
            "timing": f"back-to-back calls rotating {nset} sets of weights, x and y "
                      f"({nset * per_set / 1e6:.0f} MB vs {l2 / 1e6:.0f} MB L2)",
            "parity": {"max_err_over_bound": round(ratio, 5), "rows": rows, "tokens": M},
            "oracle": {"all_cores": {"GFLOPs": round(2 * M * n * K / dt / 1e9, 3), "cores": ob.cores,
                                     "sample": f"{n} weight rows x 512 tokens x K, {dt:.3f} s"}}}


# the 64 blocks of the full-depth decode step: (N, K) of each block's four binary GEMVs
FULL_DEPTH_BLOCK = [(9120, 5120), (5120, 5120), (40960, 5120), (5120, 20480)]
FULL_DEPTH_BLOCKS = 64


def full_depth_step(bq, device, stream, peaks, ob=None):
    """One decode token through all 64 blocks: 256 binary GEMVs at M = 1 (24.8e9 weights,
    3.49 GB, every block's weights distinct), replayed as one CUDA graph. Each call is ordered
    after the previous one on the stream, as the layers of a decode step are."""
    mats = []
    for b in range(FULL_DEPTH_BLOCKS):
        for j, (N, K) in enumerate(FULL_DEPTH_BLOCK):
            seed = 1000 + 4 * b + j
            mats.append(bq.BQWeight(bq.BINARY_G128, N, K, synth.binary_words(seed, N, K, device=device),
                                    synth.scales(seed, N, K // 128, device=device)))
    xh = {K: synth.activations(0, 1, K) for K in (5120, 20480)}
    xs = {K: v.to(device) for K, v in xh.items()}
    ys = {(N, K): torch.empty((1, N), dtype=torch.float32, device=device) for (N, K) in FULL_DEPTH_BLOCK}
    ws_bytes = max(bq.gemv_workspace_bytes(1, w) for w in mats[:4])
    ws = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device=device)
    total = sum(gemv_bytes(w.N, w.K, 1) for w in mats)
    with torch.cuda.stream(stream):
        for w in mats[:4]:
            bq.gemv(xs[w.K], w, out=ys[(w.N, w.K)], workspace=ws)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for w in mats:
                bq.gemv(xs[w.K], w, out=ys[(w.N, w.K)], workspace=ws)
        ms = time_single(g.replay, 20, 3, stream)
    gbs = total / 1e9 / (ms / 1e3)
    res = {"workload": "full-depth decode step, 64 blocks x {9120x5120, 5120x5120, 40960x5120, "
                       "5120x20480} binary GEMVs at M=1 (24.8e9 weights)",
           "blocks": FULL_DEPTH_BLOCKS, "gemvs": 4 * FULL_DEPTH_BLOCKS, "bytes": total,
           "us": round(ms * 1e3, 1), "tokens_per_s": round(1e3 / ms, 1), "GBps": round(gbs, 1),
           "bound": "hbm", "frac": round(gbs / peaks["hbm_gbs"], 4), "peak": peaks["hbm_gbs"],
           "timing": "one CUDA graph of the 256 calls, 3.49 GB of distinct weights per step"}
    if ob is not None:
        # the last block's four outputs (held in ys after the graph) against the oracle
        o = ob.o
        ratios = []
        g.replay()
        torch.cuda.synchronize()
        for j, (N, K) in enumerate(FULL_DEPTH_BLOCK):
            seed = 1000 + 4 * (FULL_DEPTH_BLOCKS - 1) + j
            words, sc = _host_binary(seed, 64, K)
            ratios.append(ob.max_ratio(o.BINARY, xh[K], o.X_BF16, words, sc, K, ys[(N, K)][:, :64].cpu().numpy()))
        res["parity"] = {"max_err_over_bound": round(max(ratios), 5), "rows": "64 of each of the last block's 4 GEMVs"}
        timing = {}
        for (N, K) in FULL_DEPTH_BLOCK:
            words, sc = _host_binary(1000, 1024, K)
            t = ob.gemv_timing(o.BINARY, xh[K], o.X_BF16, words, sc, K, K // 8 + K // 64, 2 * K, False)
            timing[f"{N}x{K}"] = t["all_cores"]["GBps"]
        gb_o = sum(timing.values()) / len(timing)
        res["oracle"] = {"all_cores": {"GBps": round(gb_o, 4), "cores": ob.cores,
                                       "tokens_per_s": round(gb_o * 1e9 / total, 6),
                                       "sample": "up to 1024 rows of each block shape, mean GB/s of the four"}}
    del g, mats
    torch.cuda.empty_cache()
    return res


def stage_step_io(layer, device, pin):
    """One device buffer for the six x of a step and one for the six y, with the GEMV operands
    as views into them, plus host twins made by `pin` (pinned host memory in the bench), so a step
    moves its inputs and its results with one copy each way. Returns (x_dev, y_dev, x_host,
    y_host, [(w, x_view, y_view)]). Every view starts at a multiple of 16 bytes."""
    nx = [x.numel() for (_, x, _) in layer]
    ny = [y.numel() for (_, _, y) in layer]
    x_dev = torch.empty(sum(nx), dtype=layer[0][1].dtype, device=device)
    y_dev = torch.empty(sum(ny), dtype=layer[0][2].dtype, device=device)
    ops, ox, oy = [], 0, 0
    for (w, x, y), a, b in zip(layer, nx, ny):
        assert (ox * x_dev.element_size()) % 16 == 0 and (oy * y_dev.element_size()) % 16 == 0
        xv = x_dev[ox:ox + a].view(x.shape)
        xv.copy_(x)
        yv = y_dev[oy:oy + b].view(y.shape)
        ops.append((w, xv, yv))
        ox += a
        oy += b
    x_host = pin(x_dev.cpu())
    y_host = pin(torch.empty(y_dev.shape, dtype=y_dev.dtype))
    return x_dev, y_dev, x_host, y_host, ops


def e2e_gemv(bq, device, steps, warmup, stream):
    """The headline step through the public API with host buffers: per step, one copy of the
    six x from pinned host memory, the six GEMVs (one workspace, shared in stream order), one
    copy of the six y back to pinned memory."""
    sets = make_gemv_sets(bq, device, 6)
    staged = [stage_step_io(layer, device, lambda t: t.pin_memory()) for layer in sets]
    ws_bytes = max(bq.gemv_workspace_bytes(M, w) for (w, _, _) in sets[0] for M in (1, 4, 8))
    ws = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device=device)
    h2d = staged[0][2].numel() * staged[0][2].element_size()
    d2h = staged[0][3].numel() * staged[0][3].element_size()

    def step(i):
        x_dev, y_dev, x_host, y_host, ops = staged[i % len(staged)]
        x_dev.copy_(x_host, non_blocking=True)
        for (w, x, y) in ops:
            bq.gemv(x, w, out=y, workspace=ws)
        y_host.copy_(y_dev, non_blocking=True)
    for i in range(warmup):
        step(i)
    torch.cuda.synchronize()
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for i in range(steps):
        step(i)
    b.record(stream)
    b.synchronize()
    ms = a.elapsed_time(b) / steps
    step_bytes = sum(gemv_bytes(N, K_HEAD, M) for (N, M) in GEMV_SHAPES)
    del sets, staged
    return {"value": round(step_bytes / 1e9 / (ms / 1e3), 1), "unit": "GB/s",
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": round(ms, 5)}


GEMV_SOURCES = ("gemv_rows.cu", "gemv_mma.cuh")


def gemv_source_sha() -> str:
    """Hash of the GEMV kernel sources the bench step runs (mma.sync and tcgen05 kernels)."""
    h = hashlib.sha256()
    for name in GEMV_SOURCES:
        with open(os.path.join(ROOT, "ternary_g128_weight_bq_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def traffic_record():
    """ncu DRAM bytes (read + write) of one bench step's launches, if taken on the current
    kernel sources (profiles/gemv_traffic.json records the source hash and the command)."""
    p = os.path.join(ROOT, "profiles", "gemv_traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        rec = json.load(f)
    h = gemv_source_sha()
    if rec.get("source_sha") != h:
        return None
    return rec


# --------------------------------------------------------------------------------------
# CPU oracle timing (cpu_baseline leg and --impl reference)
# --------------------------------------------------------------------------------------

class OracleSample:
    """The CPU oracle on bounded samples of the six headline GEMVs: the first R rows of
    each (all K), run on every host core through a thread pool (ctypes releases the GIL)."""

    def __init__(self, max_rows: int = 512):
        import oracle
        self.oracle = oracle
        self.orc = oracle.default()
        self.cores = os.cpu_count() or 1
        self.inputs = []
        for (N, M) in GEMV_SHAPES:
            self.inputs.append((synth.activations(0, M, K_HEAD), synth.binary_words(0, max_rows, K_HEAD),
                                synth.scales(0, max_rows, K_HEAD // 128), M))
        self.max_rows = max_rows
        # calibration: seconds per row of all six shapes on one core
        t0 = time.perf_counter()
        for (x, w, s, M) in self.inputs:
            self.orc.gemv(oracle.BINARY, x, oracle.X_BF16, w[:1], s[:1], K_HEAD)
        self.row_seconds = max(time.perf_counter() - t0, 1e-6)

    def rows_for(self, budget_s: float) -> int:
        return max(1, min(self.max_rows, int(budget_s * self.cores / self.row_seconds)))

    def run(self, rows: int):
        """Returns (GB/s, seconds) for one pass over `rows` rows of each shape."""
        import concurrent.futures as cf
        o = self.oracle
        chunks = max(1, min(self.cores, rows))
        jobs = []
        for (x, w, s, M) in self.inputs:
            b = [rows * i // chunks for i in range(chunks + 1)]
            jobs += [(x, w, s, b[i], b[i + 1]) for i in range(chunks) if b[i + 1] > b[i]]

        def work(a):
            x, w, s, lo, hi = a
            return self.orc.gemv(o.BINARY, x, o.X_BF16, w[lo:hi], s[lo:hi], K_HEAD)
        t0 = time.perf_counter()
        with cf.ThreadPoolExecutor(max_workers=self.cores) as ex:
            list(ex.map(work, jobs))
        dt = time.perf_counter() - t0
        nbytes = sum(gemv_bytes(rows, K_HEAD, M) for (_, _, _, M) in self.inputs)
        return nbytes / 1e9 / dt, dt

    def describe(self, rows: int, dt: float) -> str:
        macs = sum(rows * K_HEAD * M for (_, M) in GEMV_SHAPES)
        return (f"first {rows} rows of each of the six GEMVs (K=5120, M in 1,4,8; "
                f"{macs / 1e6:.1f}M fp64 multiply-adds) in {dt:.3f} s")


def oracle_gemv_sample(budget_s: float):
    """One bounded oracle run of about budget_s seconds: (GB/s, cores, description)."""
    o = OracleSample(max_rows=4096)
    rows = o.rows_for(budget_s)
    v, dt = o.run(rows)
    return v, o.cores, o.describe(rows, dt)


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    o = OracleSample(max_rows=512)
    budget = args.ref_seconds / max(1, args.steps + args.warmup)
    rows = o.rows_for(budget)
    for _ in range(args.warmup):
        o.run(rows)
    vals, dts = [], []
    t0 = time.perf_counter()
    for _ in range(args.steps):
        v, dt = o.run(rows)
        vals.append(v)
        dts.append(dt)
    wall = time.perf_counter() - t0
    value = statistics.median(vals)
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "GB/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(wall / max(1, args.steps) * 1e3, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": "binary g128 decode GEMV, K=5120, N in {5120, 20480}, "
                               "M in {1, 4, 8}, x bf16; CPU oracle on a row sample per step"},
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": o.cores,
                         "kind": "oracle", "sample": o.describe(rows, statistics.median(dts))},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# --------------------------------------------------------------------------------------
# main GPU arm
# --------------------------------------------------------------------------------------

def run_gpu(args):
    rank, world, dist = dist_init()
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    import ternary_g128_weight_bq_b200 as bq
    from ternary_g128_weight_bq_b200 import build as bqbuild
    bqbuild.build()
    peaks = read_peaks()
    stream = torch.cuda.Stream(device)

    step_bytes = sum(gemv_bytes(N, K_HEAD, M) for (N, M) in GEMV_SHAPES)
    l2 = l2_bytes(device)
    copies = max(2, math.ceil(2.5 * l2 / step_bytes))
    with torch.cuda.stream(stream):
        sets = make_gemv_sets(bq, device, copies)
        graphs, launches = capture_step_graphs(bq, sets, stream)
        torch.cuda.synchronize()
        clocks = ClockSampler(local) if rank == 0 else None
        ms_total, region_ms = time_regions(graphs, args.steps, args.warmup, stream, dist, device)
        clk = clocks.stop() if clocks else None
    ms_step = reduce_max(ms_total / args.steps, dist, device)
    value = world * step_bytes / 1e9 / (ms_step / 1e3)
    launches_timed = sum(launches[i % len(graphs)] for i in range(args.steps))

    extras = None
    breakdown = None
    e2e = None
    if rank == 0 and not args.quick:
        with torch.cuda.stream(stream):
            breakdown = per_config_breakdown(bq, sets, stream)
    del graphs, sets
    torch.cuda.empty_cache()
    if not args.quick:
        with torch.cuda.stream(stream):
            try:
                e2e = e2e_gemv(bq, device, min(args.steps, 2000), args.warmup, stream)
            except Exception as ex:   # keep the kernel-timed line; say why e2e is missing
                e2e = {"error": str(ex).splitlines()[0][:200]}
            if rank == 0:
                try:
                    extras = config_reports(bq, device, stream, peaks, OracleBench(), breakdown)
                except Exception as ex:   # keep the headline line; say why the configs are missing
                    extras = {"error": str(ex).splitlines()[0][:300]}
        if e2e is not None and "ms_per_step" in e2e:
            e2e_ms = reduce_max(e2e["ms_per_step"], dist, device)
            e2e["value"] = round(world * step_bytes / 1e9 / (e2e_ms / 1e3), 1)

    if rank == 0:
        tr = traffic_record()
        achieved = step_bytes / 1e9 / (ms_total / args.steps / 1e3)
        cpu = None
        if not args.quick:
            v, cores, desc = oracle_gemv_sample(args.cpu_seconds)
            cpu = {"value": round(v, 4), "unit": "GB/s", "cores": cores, "kind": "oracle",
                   "sample": desc}
        line = {
            "metric": METRIC, "value": round(value, 1), "unit": "GB/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_step, 5),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f32", "data": "synthetic",
            "config": {
                "workload": "binary g128 decode GEMV, K=5120, N in {5120, 20480}, M in {1, 4, 8} "
                            "(six GEMVs per step), x bf16 ~N(0,1), bits Bernoulli(0.5), "
                            "scales fp16 |N(0,0.02)|+1e-3, y fp32",
                "l2": f"inputs larger than L2: {copies} weight copies rotated "
                      f"({copies * step_bytes / 1e6:.0f} MB vs {l2 / 1e6:.0f} MB L2)",
                "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
                "bytes_per_step": step_bytes,
                "timing": f"CUDA graph per step (six GEMV calls, each ordered after the previous), CUDA "
                          f"events on the launch stream; value from the median of {len(region_ms)} timed "
                          f"regions of {args.steps} steps (min {min(region_ms) / args.steps:.5f}, max "
                          f"{max(region_ms) / args.steps:.5f} ms per step)",
            },
            "pct_of_8TBs": round(100 * value / world / NOMINAL_HBM_GBS, 1),
            "roofline": {
                "bound": "hbm", "achieved": round(achieved, 1), "peak": peaks["hbm_gbs"],
                "unit": "GB/s", "frac": round(achieved / peaks["hbm_gbs"], 4),
                "traffic": tr["dram_bytes_per_step"] if tr else None,
                "traffic_unit": "DRAM bytes per step (the twelve launches of six GEMV calls), one ncu capture",
                "bytes_per_step": step_bytes,
                "peak_source": f"{peaks['source']} (HBM copy, burst)",
                "kernel": "bq gemv: gemv_rows_prep_kernel (x digits) + gemv_rows_kernel (mma.sync s8, whole "
                          "output rows per CTA) per GEMV call, six calls per step; achieved = algorithmic "
                          "bytes per step / device time per step",
            },
            "cpu_baseline": cpu,
            "e2e": e2e,
            "gpu_launches": launches_timed,
            "clocks": clk,
            "configs": extras,
        }
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.destroy_process_group()
    return 0


def run_case(args):
    """One workload alone, --steps calls after --warmup, for profiling (ncu -k / -c) and
    spot timing; prints one JSON line with the average device time per call."""
    import ternary_g128_weight_bq_b200 as bq
    from ternary_g128_weight_bq_b200 import build as bqbuild
    bqbuild.build()
    device = torch.device("cuda", 0)
    stream = torch.cuda.Stream(device)
    N, M, K = args.N, args.M, args.K
    with torch.cuda.stream(stream):
        if args.case in ("gemv", "prefill", "topk"):
            if args.fmt == "binary":
                w = bq.BQWeight(bq.BINARY_G128, N, K, synth.binary_words(0, N, K, device=device),
                                synth.scales(0, N, K // 128, device=device))
            else:
                q = synth.random_ternary(0, synth.TID_TERNARY, (N, K), device=device)
                pack = bq.pack_ternary_g128 if args.fmt == "ternary" else bq.pack_ternary_b3_g128
                w = pack(q, synth.scales(0, N, K // 128, device=device))
                del q
            x = synth.activations(0, M, K).to(device)
            if args.case == "topk":
                ws = torch.empty(bq.gemv_topk_workspace_bytes(M, w, 20), dtype=torch.uint8, device=device)
                u = torch.full((M,), 0.37, dtype=torch.float32, device=device)
                outs = (torch.empty((M, 20), dtype=torch.float32, device=device),
                        torch.empty((M, 20), dtype=torch.int32, device=device),
                        torch.empty((M,), dtype=torch.int32, device=device))
                fn = lambda: bq.gemv_topk(x, w, k=20, u=u, workspace=ws, out=outs)
                bits = {"binary": 1, "ternary": 2, "ternary_b3": 26 * 8 / 128}[args.fmt]
                work = {"GBps": gemv_bytes(N, K, M, bits) / 1e9}
            elif args.case == "gemv":
                y = torch.empty((M, N), dtype=torch.float32, device=device)
                ws = torch.empty(max(bq.gemv_workspace_bytes(M, w), 16), dtype=torch.uint8, device=device)
                fn = lambda: bq.gemv(x, w, out=y, workspace=ws)
                bits = {"binary": 1, "ternary": 2, "ternary_b3": 26 * 8 / 128}[args.fmt]
                work = {"GBps": gemv_bytes(N, K, M, bits) / 1e9}
            else:
                y = torch.empty((M, N), dtype=torch.bfloat16, device=device)
                fn = lambda: bq.gemm_prefill(x, w, out=y)
                work = {"TFLOPs": 2 * M * N * K / 1e12}
        elif args.case == "quantize":
            fmt = {"binary": bq.BINARY_G128, "ternary": bq.TERNARY_G128, "ternary_b3": bq.TERNARY_B3_G128}[args.fmt]
            wd = (synth.activations(5, N, K, dtype=torch.float32) * 0.02).to(torch.bfloat16).to(device)
            pw = bq.quantize_g128(wd, fmt)
            fn = lambda: bq.quantize_g128(wd, fmt)
            work = {"GBps": (N * K * 2 + pw.words.numel() * pw.words.element_size() + pw.scales.numel() * 2) / 1e9}
        elif args.case == "mlp":
            mk = lambda rows, cols, tid: bq.BQWeight(bq.BINARY_G128, rows, cols,
                                                     synth.binary_words(tid, rows, cols, device=device),
                                                     synth.scales(tid, rows, cols // 128, device=device))
            gate, up, down = mk(N, K, 1), mk(N, K, 2), mk(K, N, 3)
            x = synth.activations(0, M, K).to(device)
            y = torch.empty((M, K), dtype=torch.float32, device=device)
            ws = torch.empty(bq.mlp_swiglu_workspace_bytes(M, gate, up, down), dtype=torch.uint8, device=device)
            fn = lambda: bq.mlp_swiglu(x, gate, up, down, out=y, workspace=ws)
            work = {"GBps": (2 * gemv_bytes(N, K, M, 1) + gemv_bytes(K, N, M, 1)) / 1e9}
        elif args.case == "embed":
            w = bq.BQWeight(bq.BINARY_G128, N, K, synth.binary_words(0, N, K, device=device),
                            synth.scales(0, N, K // 128, device=device))
            ids = synth.random_ids(0, synth.TID_IDS, M, N).to(device)
            out = torch.empty((M, K), dtype=torch.bfloat16, device=device)
            fn = lambda: bq.embed_gather(ids, w, out=out)
            work = {"GBps": M * (K // 8 + K // 64 + K * 2 + 4) / 1e9}
        ms = time_single(fn, args.steps, args.warmup, stream)
    line = {"case": args.case, "fmt": args.fmt, "N": N, "M": M, "K": K, "steps": args.steps,
            "us_per_call": round(ms * 1e3, 3)}
    for k, v in work.items():
        line[k] = round(v / (ms / 1e3), 1)
    print(json.dumps(line), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20000)
    ap.add_argument("--warmup", type=int, default=50)
    ap.add_argument("--impl", choices=["bq", "reference"], default="bq")
    ap.add_argument("--quick", action="store_true", help="headline number only")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--ref-seconds", type=float, default=150.0,
                    help="total CPU time budget of --impl reference (split over warm-up and steps)")
    ap.add_argument("--case", choices=["gemv", "prefill", "embed", "topk", "quantize", "mlp"],
                    help="time one workload alone (for profiling) instead of the benchmark")
    ap.add_argument("--fmt", choices=["binary", "ternary", "ternary_b3"], default="binary")
    ap.add_argument("--N", type=int, default=248320)
    ap.add_argument("--M", type=int, default=1)
    ap.add_argument("--K", type=int, default=K_HEAD)
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    if args.impl == "reference":
        return run_reference(args)
    if not torch.cuda.is_available():
        print(json.dumps({"error": "no CUDA device"}))
        return 1
    if args.case:
        return run_case(args)
    return run_gpu(args)


if __name__ == "__main__":
    sys.exit(main())
