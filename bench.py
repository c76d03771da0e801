"""Benchmark: quantized GEMV HBM GB/s and decoder-layer us/token on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Workload (one step): batch-1 decode of a 36-layer Qwen3-8B-like stack
(hidden 4096, 32 q heads and 8 kv heads of dim 128, MLP 12288), seven
projections per layer with per-matrix grids mixed 75.1% ternary / 6.0%
2-bit / 18.8% 3-bit by parameter count (q at 3 bits, k and v at 2 bits).
Each layer is ONE grouped launch (tb_layer_gemv) over its seven matrices.
Weights are seeded N(0, 0.02) draws quantized on the GPU by the library
(absmax scales, round-half-even), 2.01 GB packed, resident in HBM; the
working set is 16x the L2, so no L2 flush is needed.  The other hot-path
rows (scales + pack, unpack, small-batch GEMM) are timed in the same run
and reported under "rows".

Multi-GPU: the path does not shard (single-GPU method); N ranks run N
independent replicas, one per GPU, and `value` is the sum of their bytes
over the slowest rank's time.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from decode_gemv_tb_b200 import build as tbbuild  # noqa: E402
from decode_gemv_tb_b200 import synth, tb  # noqa: E402

METRIC = "quantized GEMV achieved HBM GB/s (% of B200 peak); decoder-layer µs/token"
SPEC_HBM_GBS = 8000.0


def input_role(m):
    """The projection's name within its layer (q, k, v, o, gate, up, down)."""
    return m.name.rsplit(".", 1)[1]


SHARING = ("k", "v", "up")  # projections that read the input of q (k, v) or of gate (up)


def algo_bytes(N, K, grid, M=1, ybytes=4):
    """packed codes + bf16 scales + activations + outputs of one product."""
    if grid == tb.TERNARY_B3:  # 26 bytes per 128-group, rows padded to 16 bytes
        codes = N * 16 * ((26 * (K // 128) + 15) // 16)
    else:
        codes = N * K * (3 if grid == synth.INT3 else 2) // 8
    return codes + N * (K // 128) * 2 + M * K * 2 + M * N * ybytes


def layer_algo_bytes(mats):
    """Algorithmic bytes of one decoder layer's projections: each product's
    own, with an input that q/k/v (gate/up) share counted once."""
    return sum(algo_bytes(m.N, m.K, m.grid) - (2 * m.K if input_role(m) in SHARING else 0) for m in mats)


TRAFFIC_RECORD = os.path.join("profiles", "k_gemv8_traffic.json")


def traffic_per_launch(algorithmic_bytes):
    """DRAM bytes per k_gemv8 launch from the committed ncu capture: its
    measured traffic / algorithmic ratio times this launch's algorithmic
    bytes; None when there is no capture or the kernel's sources changed
    after it."""
    import hashlib
    p = os.path.join(ROOT, TRAFFIC_RECORD)
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    h = hashlib.sha256()
    for s in d["kernel_sources"]:
        with open(os.path.join(ROOT, s), "rb") as f:
            h.update(f.read())
    if h.hexdigest() != d["kernel_sources_sha256"]:
        return None
    return algorithmic_bytes * d["traffic_over_algorithmic"]


def workload_config(stack, world):
    """The `config` object of the JSON line (both arms): the decode stack's
    shape, grid mix and bytes."""
    packed = sum(m.N * m.K * (3 if m.grid == synth.INT3 else 2) // 8 for mats in stack for m in mats)
    step_bytes = sum(layer_algo_bytes(mats) for mats in stack)
    return {"workload": f"qwen3_8b_like_decode_stack_{len(stack)}L_mixed_grids", "batch": 1, "layers": len(stack),
            "hidden": 4096, "mlp": 12288, "kv_dim": 1024,
            "grid_mix": {synth.GRID_NAMES[g]: round(v, 4) for g, v in synth.grid_fractions(stack).items()},
            "packed_GB": packed / 1e9, "step_algorithmic_bytes": step_bytes,
            "l2": "working set larger than L2 (no flush)", "parallelism": f"replicas{world}", "prewarm_s": PREWARM_S}


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), float(d["bf16_tflops_sustained"]), "measured"
    return 6650.0, 1590.0, 1400.0, "fallback"


class Clocks:
    """SM clock and throttle reasons during the timed region: NVML polled
    back to back (about every 0.1 ms) from a thread between begin() and
    end(), plus an nvidia-smi log (100 ms) over the whole context for the
    record."""

    NAMES = {"hw_slowdown": 0x8, "hw_thermal_slowdown": 0x40, "sw_thermal_slowdown": 0x20, "sw_power_cap": 0x4}

    def __init__(self, gpu: int, log_path: str | None = None):
        import tempfile
        self.gpu = gpu
        self.proc = None
        self.path = log_path or os.path.join(tempfile.gettempdir(), f"tb_bench_clocks_gpu{gpu}.csv")
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self.nvml, self.thread, self.active = None, None, False

    def __enter__(self):
        os.makedirs(os.path.dirname(os.path.abspath(self.path)), exist_ok=True)
        q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={q}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=self.f, stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        try:
            import pynvml
            pynvml.nvmlInit()
            idx = self.gpu
            vis = os.environ.get("CUDA_VISIBLE_DEVICES")
            if vis and vis.split(",")[0].strip().isdigit():
                idx = int(vis.split(",")[self.gpu])
            self.nvml = (pynvml, pynvml.nvmlDeviceGetHandleByIndex(idx))
            self.max_mhz = float(pynvml.nvmlDeviceGetMaxClockInfo(self.nvml[1], pynvml.NVML_CLOCK_SM))
        except Exception:
            self.nvml = None
        return self

    def _poll(self):
        import threading
        nv, h = self.nvml
        while self.active:
            try:
                self.samples.append(float(nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)))
                r = nv.nvmlDeviceGetCurrentClocksEventReasons(h)
                for nm, bit in self.NAMES.items():
                    if r & bit:
                        self.reasons.add(nm)
            except Exception:
                pass

    def begin(self):
        if self.nvml:
            import threading
            self.active = True
            self.thread = threading.Thread(target=self._poll, daemon=True)
            self.thread.start()

    def end(self):
        if self.thread:
            self.active = False
            self.thread.join()
            self.thread = None

    def __exit__(self, *a):
        self.end()
        if self.proc:
            self.proc.terminate()
            self.proc.wait()
            self.f.close()

    def summary(self):
        if self.samples:
            return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                    "reasons": sorted(self.reasons), "samples": len(self.samples), "source": "nvml, back to back"}
        if not self.proc or not os.path.exists(self.path):
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no clock source"]}
        sm, mx, reasons = [], None, set()
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for nm, v in zip(list(self.NAMES), parts[5:9]):
                if v.lower() == "active":
                    reasons.add(nm)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm), "source": "nvidia-smi 100 ms"}


# ---------------------------------------------------------------- workload

class DecodeStack:
    """Packed, resident 36-layer stack.  The inputs are those of a decoder
    layer: q, k and v read one x (the normed hidden state), gate and up one
    x, o and down one each, so a layer has four input vectors; every
    projection has its own output.  x vectors and y outputs live in single
    flat buffers so the end-to-end variant moves them with one copy each way
    per step."""

    def __init__(self, dev, layers=None):
        self.dev = dev
        stack = synth.config3_stack()
        if layers is not None:
            stack = stack[:layers]
        self.stack = stack
        self.layers = []
        self.bytes_per_layer = []
        xs, ys = 0, 0
        for mats in stack:
            for m in mats:
                xs += m.K if input_role(m) not in SHARING else 0
                ys += m.N
        self.x_all = torch.empty(xs, dtype=torch.bfloat16, device=dev)
        self.y_all = torch.empty(ys, dtype=torch.float32, device=dev)
        xo, yo = 0, 0
        self.packed_bytes = 0
        ws_bytes = 0
        self.y_spans = []  # [y_begin, y_end) of each layer's outputs in y_all
        for li, mats in enumerate(stack):
            items, b = [], 0
            y_begin = yo
            shared = {}
            for m in mats:
                W = synth.gaussian_weights(m.N, m.K, seed=m.seed, device=dev, dtype=torch.bfloat16)
                s = tb.tb_scales_absmax(W, m.grid)
                p = tb.tb_pack(W, m.grid, s)
                del W
                role = input_role(m)
                if role in SHARING:  # the input of q (gate)
                    x = shared["q" if role != "up" else "gate"]
                else:
                    x = self.x_all[xo:xo + m.K]
                    x.copy_(synth.activations(m.K, seed=m.seed, device=dev))
                    xo += m.K
                    shared[role] = x
                y = self.y_all[yo:yo + m.N]
                yo += m.N
                items.append((p, m.grid, s, x, y, m.N, m.K))
                b += algo_bytes(m.N, m.K, m.grid) - (2 * m.K if role in SHARING else 0)
                self.packed_bytes += p.numel()
            arr = tb.linear_items(items)
            self.y_spans.append((y_begin, yo))
            ws_bytes = max(ws_bytes, tb.layer_workspace_bytes(arr))
            self.layers.append((items, arr))
            self.bytes_per_layer.append(b)
        # one workspace for all layers: the calls are ordered on one stream
        self.ws = tb.workspace(ws_bytes, dev)
        torch.cuda.synchronize(dev)
        self.step_bytes = sum(self.bytes_per_layer)

    def step(self, flags=0):
        stream = torch.cuda.current_stream().cuda_stream
        for _, arr in self.layers:
            tb.tb_layer_gemv(arr, self.ws, flags, stream)


def capture(fn):
    """CUDA graph of fn() (launch overhead off the device timeline)."""
    fn()  # warm (sets kernel attributes outside the capture)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fn()
    torch.cuda.synchronize()
    return g


PREWARM_S = 0.2


def time_region(fn, steps, warmup, stream, dist=None, clocks=None):
    # untimed: about PREWARM_S of replays (clock and memory-state ramp,
    # graph upload), then the W warm-up steps
    t0 = time.perf_counter()
    while time.perf_counter() - t0 < PREWARM_S:
        for _ in range(10):
            fn()
        torch.cuda.synchronize()
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if clocks:
        clocks.begin()
    e0.record(stream)
    for _ in range(steps):
        fn()
    e1.record(stream)
    torch.cuda.synchronize()
    if clocks:
        clocks.end()
    ms = max_over_ranks(e0.elapsed_time(e1), dist)
    if dist:
        dist.barrier()
    return ms


def max_over_ranks(ms, dist=None):
    """The slowest rank's time (every rank calls this at the same step)."""
    if not dist:
        return ms
    t = torch.tensor([ms], dtype=torch.float64, device="cuda" if dist.get_backend() == "nccl" else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(world, step_bytes, ms_per_step):
    """Whole-job GB/s: each of the `world` replicas processes one step's
    bytes in the slowest rank's step time."""
    return world * step_bytes / (ms_per_step * 1e-3) / 1e9


def rows_section(dev, stream):
    """Time the other hot-path rows (graph-captured, 10 calls per replay,
    median of 5 replays after warm-up)."""
    out = {}

    def med(fn, reps=5, inner=10):
        g = capture(lambda: [fn() for _ in range(inner)])
        for _ in range(2):
            g.replay()
        ts = []
        for _ in range(reps):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            g.replay()
            b.record(stream)
            torch.cuda.synchronize()
            ts.append(a.elapsed_time(b) / inner)
        del g
        return statistics.median(ts)

    # scales + pack of one Qwen3-14B-like layer, outlier weights (config-5 recipe)
    mats = synth.config5_stack()[0]
    Ws = [(synth.outlier_weights(m.N, m.K, seed=m.seed, device=dev), m) for m in mats]
    bufs = []
    for W, m in Ws:
        s = torch.empty((m.N, m.K // 128), dtype=torch.bfloat16, device=dev)
        p = torch.empty(tb.packed_bytes(m.grid, m.N, m.K), dtype=torch.uint8, device=dev)
        bufs.append((W, m, s, p))

    def pack_layer():
        for W, m, s, p in bufs:
            tb.tb_scales_absmax(W, m.grid, s)
            tb.tb_pack(W, m.grid, s, p)

    ms = med(pack_layer)
    rw = sum(2 * m.N * m.K * 2 + 2 * m.N * (m.K // 128) * 2 + tb.packed_bytes(m.grid, m.N, m.K) for _, m, _, _ in bufs)
    out["scales_pack_14b_layer"] = {"ms": ms, "GB_s": rw / ms / 1e6, "weights": sum(m.N * m.K for _, m, _, _ in bufs),
                                    "bytes_read_written": rw}

    # unpack of the 3-bit q projection
    W, m, s, p = bufs[0]
    codes = torch.empty((m.N, m.K), dtype=torch.int8, device=dev)
    ms = med(lambda: tb.tb_unpack(p, m.grid, m.N, m.K, codes))
    ub = tb.packed_bytes(m.grid, m.N, m.K) + m.N * m.K
    out["unpack_q_5120x5120_int3"] = {"ms": ms, "GB_s": ub / ms / 1e6}

    # small-batch GEMM, Qwen3-14B-like gate (17408 x 5120), int2 and int3
    gate = [(W, m, s, p) for W, m, s, p in bufs if m.name.endswith("gate")][0]
    W = gate[0]
    g = {}
    for grid in (synth.INT2, synth.INT3):
        s = tb.tb_scales_absmax(W, grid)
        p = tb.tb_pack(W, grid, s)
        for M in synth.CONFIG4_M:
            X = synth.activations(W.shape[1], seed=4000 + M, device=dev, M=M)
            Y = torch.empty((M, W.shape[0]), dtype=torch.float32, device=dev)
            ws = tb.workspace(tb.workspace_bytes(M, W.shape[0], W.shape[1]), dev)
            ms = med(lambda: tb.tb_gemm(p, grid, s, X, W.shape[0], W.shape[1], Y, ws=ws))
            fl = 2.0 * M * W.shape[0] * W.shape[1]
            by = algo_bytes(W.shape[0], W.shape[1], grid, M=M)
            g[f"{synth.GRID_NAMES[grid]}_M{M}"] = {"us": ms * 1e3, "TFLOP_s": fl / ms / 1e9, "GB_s": by / ms / 1e6}
    # prefill: 256 and 1024 batch rows in one tb_gemm launch (blocks of 128 batch rows), both grids
    for grid in (synth.INT2, synth.INT3):
        try:
            s = tb.tb_scales_absmax(W, grid)
            p = tb.tb_pack(W, grid, s)
            for M in (256, 1024):
                X = synth.activations(W.shape[1], seed=4000 + M, device=dev, M=M)
                Y = torch.empty((M, W.shape[0]), dtype=torch.float32, device=dev)
                ws = tb.workspace(tb.workspace_bytes(M, W.shape[0], W.shape[1]), dev)
                ms = med(lambda: tb.tb_gemm(p, grid, s, X, W.shape[0], W.shape[1], Y, ws=ws), inner=3)
                fl = 2.0 * M * W.shape[0] * W.shape[1]
                g[f"{synth.GRID_NAMES[grid]}_M{M}_prefill"] = {"us": ms * 1e3, "TFLOP_s": fl / ms / 1e9}
        except tb.TBError as e:  # reported in the row; the line still prints
            g[f"{synth.GRID_NAMES[grid]}_prefill"] = {"error": str(e)[:200]}
    out["gemm_gate_17408x5120"] = g
    del bufs, Ws
    torch.cuda.empty_cache()

    # hot L2 (repeated calls on the same buffers) and cold L2 (a 256 MB write
    # before every call, its own time subtracted)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    t_flush = med(lambda: flush.fill_(1))

    def hot_cold(fn):
        hot = med(fn)
        cold = med(lambda: (flush.fill_(1), fn())) - t_flush
        return hot, max(cold, 1e-6)

    def gemv_row(N, K, grid, p, s, x):
        y = torch.empty(N, dtype=torch.float32, device=dev)
        ws = tb.workspace(tb.workspace_bytes(1, N, K), dev)
        hot, cold = hot_cold(lambda: tb.tb_gemv(p, grid, s, x, N, K, y=y, ws=ws))
        by = algo_bytes(N, K, grid)
        return {"hot_us": hot * 1e3, "hot_GB_s": by / hot / 1e6, "cold_us": cold * 1e3, "cold_GB_s": by / cold / 1e6}

    # config 1: 256 x 1024 2-bit, W = c s exactly
    c1 = synth.CONFIG1
    codes = synth.uniform_codes(c1["N"], c1["K"], -2, 1, seed=c1["seed"])
    s1 = synth.config1_scales(c1["N"], c1["K"], seed=c1["seed"])
    W1 = (codes.float() * s1.float().repeat_interleave(128, dim=1)).to(dev)
    s1 = s1.to(dev)
    p1 = tb.tb_pack(W1, synth.INT2, s1)
    out["gemv_config1_256x1024_int2"] = gemv_row(c1["N"], c1["K"], synth.INT2, p1, s1,
                                                 synth.activations(c1["K"], seed=c1["seed"], device=dev))
    # config 2: Qwen3-1.7B-like shapes over the three grids
    c2 = {}
    for m in synth.config2_cases():
        W = synth.gaussian_weights(m.N, m.K, seed=m.seed, device=dev)
        s2 = tb.tb_scales_absmax(W, m.grid)
        p2 = tb.tb_pack(W, m.grid, s2)
        c2[m.name] = gemv_row(m.N, m.K, m.grid, p2, s2, synth.activations(m.K, seed=m.seed, device=dev))
        del W
    out["gemv_config2"] = c2
    # the same ternary cases in the optional 5-trits-per-byte layout
    c2b = {}
    for m in synth.config2_cases():
        if m.grid != synth.TERNARY:
            continue
        W = synth.gaussian_weights(m.N, m.K, seed=m.seed, device=dev)
        s2 = tb.tb_scales_absmax(W, tb.TERNARY_B3)
        p2 = tb.tb_pack(W, tb.TERNARY_B3, s2)
        c2b[m.name] = gemv_row(m.N, m.K, tb.TERNARY_B3, p2, s2, synth.activations(m.K, seed=m.seed, device=dev))
        del W
    out["gemv_config2_ternary_5trit"] = c2b

    # one isolated 8B-like layer (q, o 3-bit; k, v 2-bit; MLP ternary), one tb_layer_gemv per launch
    items = []
    for m in synth.isolated_layer():
        W = synth.gaussian_weights(m.N, m.K, seed=m.seed, device=dev, dtype=torch.bfloat16)
        si = tb.tb_scales_absmax(W, m.grid)
        items.append((tb.tb_pack(W, m.grid, si), m.grid, si, synth.activations(m.K, seed=m.seed, device=dev),
                      torch.empty(m.N, dtype=torch.float32, device=dev), m.N, m.K))
        del W
    arr = tb.linear_items(items)
    wsl = tb.workspace(tb.layer_workspace_bytes(arr), dev)
    hot, cold = hot_cold(lambda: tb.tb_layer_gemv(arr, wsl, 0))
    by = sum(algo_bytes(n, k, gr) for _, gr, _, _, _, n, k in items)
    out["isolated_layer_8b_q3_k2_v2_o3_mlp_ternary"] = {"hot_us_per_launch": hot * 1e3, "cold_us_per_launch": cold * 1e3,
                                                        "cold_GB_s": by / cold / 1e6, "algorithmic_bytes": by}
    del items, arr, wsl, flush
    torch.cuda.empty_cache()

    # decode order: per layer q/k/v in one call on one shared x, o, gate/up with
    # h = bf16(silu(gate) * up) in one call, down on h -- four dependent calls
    # per layer (TB_FLAG_OVERLAP_PREVIOUS), 8 layers of the 8B-like stack
    dl, dby = [], 0
    for li, mats in enumerate(synth.config3_stack()[:8]):
        P = {}
        for m in mats:
            W = synth.gaussian_weights(m.N, m.K, seed=m.seed, device=dev, dtype=torch.bfloat16)
            sd = tb.tb_scales_absmax(W, m.grid)
            P[m.name.split(".")[1]] = (tb.tb_pack(W, m.grid, sd), m.grid, sd, m.N, m.K)
            dby += algo_bytes(m.N, m.K, m.grid)
            del W
        xa = synth.activations(4096, seed=9000 + li, device=dev)
        xo = synth.activations(4096, seed=9100 + li, device=dev)
        xm = synth.activations(4096, seed=9200 + li, device=dev)
        y = {k: torch.empty(v[3], dtype=torch.float32, device=dev) for k, v in P.items()}
        h = torch.empty(P["gate"][3], dtype=torch.bfloat16, device=dev)
        it = lambda name, x: (P[name][0], P[name][1], P[name][2], x, y[name], P[name][3], P[name][4])
        qkv = tb.linear_items([it("q", xa), it("k", xa), it("v", xa)])
        o = tb.linear_items([it("o", xo)])
        gu = (it("gate", xm), it("up", xm))
        down = tb.linear_items([it("down", h)])
        dl.append((qkv, o, gu, h, down))
    # one workspace for every call (sized for the largest: calls of different shapes may share it)
    wsd = tb.workspace(max(max(tb.layer_workspace_bytes(a), tb.layer_workspace_bytes(o), tb.layer_workspace_bytes(d),
                               tb.gate_up_workspace_bytes(gu[0], gu[1])) for a, o, gu, _, d in dl), dev)

    def decode_pass():
        for qkv, o, gu, h, down in dl:
            tb.tb_layer_gemv(qkv, wsd, tb.FLAG_OVERLAP_PREVIOUS)
            tb.tb_layer_gemv(o, wsd, tb.FLAG_OVERLAP_PREVIOUS)
            tb.tb_gate_up_silu(gu[0], gu[1], h, ws=wsd, flags=tb.FLAG_OVERLAP_PREVIOUS)
            tb.tb_layer_gemv(down, wsd, tb.FLAG_OVERLAP_PREVIOUS)

    msd = med(decode_pass, reps=5, inner=1)
    out["decode_order_layer_8b"] = {"us_per_layer": msd * 1e3 / len(dl), "GB_s": dby / msd / 1e6, "layers": len(dl),
                                    "calls_per_layer": 4, "algorithmic_bytes_per_layer": dby // len(dl)}
    del dl, wsd
    torch.cuda.empty_cache()

    # config 5: batch-1 GEMV over all 280 matrices of a 40-layer 14B-like stack
    # (outlier weights, mixed grids), packed by the library; one pass = 40 layer calls
    layers, packed5, by5 = [], 0, 0
    for mats in synth.config5_stack():
        its = []
        for m in mats:
            W = synth.outlier_weights(m.N, m.K, seed=m.seed, device=dev)
            s5 = tb.tb_scales_absmax(W, m.grid)
            p5 = tb.tb_pack(W, m.grid, s5)
            del W
            its.append((p5, m.grid, s5, synth.activations(m.K, seed=m.seed, device=dev),
                        torch.empty(m.N, dtype=torch.float32, device=dev), m.N, m.K))
            packed5 += p5.numel()
            by5 += algo_bytes(m.N, m.K, m.grid)
        layers.append((its, tb.linear_items(its)))
    ws5 = tb.workspace(max(tb.layer_workspace_bytes(a) for _, a in layers), dev)
    ms5 = med(lambda: [tb.tb_layer_gemv(a, ws5, 0) for _, a in layers], reps=5, inner=1)
    out["config5_stack_14b_40L_gemv"] = {"ms_per_pass": ms5, "GB_s": by5 / ms5 / 1e6, "packed_GB": packed5 / 1e9,
                                         "algorithmic_GB": by5 / 1e9, "matrices": 280}
    del layers, ws5
    torch.cuda.empty_cache()
    return out


def host_description():
    """nproc, the CPU model and the oracle's compiler flags (the CPU
    baseline's context)."""
    model = None
    try:
        for line in open("/proc/cpuinfo"):
            if line.startswith("model name"):
                model = line.split(":", 1)[1].strip()
                break
    except OSError:
        pass
    from oracle import tb_oracle as oracle
    return {"nproc": os.cpu_count(), "cpu_model": model, "oracle_cflags": " ".join(oracle.CFLAGS),
            "threads_used": 1}


def cpu_baseline(seconds_budget=20.0):
    """The oracle as it stands, single-threaded fp64, on a bounded sample of
    the same workload: GEMV of the stack's layer-0 projections (as many as
    fit the time budget), GB/s on the same algorithmic bytes."""
    sys.path.insert(0, ROOT)
    from oracle import tb_oracle as oracle

    oracle.build()
    mats = synth.config3_stack()[0]
    done_bytes, t_total, names = 0, 0.0, []
    for m in mats:
        W = synth.gaussian_weights(m.N, m.K, seed=m.seed, dtype=torch.bfloat16)
        wb = W.view(torch.int16).numpy().view("uint16")
        s = oracle.scales_absmax(wb, m.grid)
        p, _ = oracle.pack(wb, m.grid, s)
        x = synth.activations(m.K, seed=m.seed).view(torch.int16).numpy().view("uint16")
        t0 = time.perf_counter()
        oracle.gemv64(p, m.grid, s, x, m.N, m.K)
        t_total += time.perf_counter() - t0
        done_bytes += algo_bytes(m.N, m.K, m.grid)
        names.append(m.name)
        if t_total > seconds_budget:
            break
    return {"value": done_bytes / t_total / 1e9, "unit": "GB/s", "cores": 1, "kind": "oracle",
            "sample": f"fp64 oracle GEMV over {'+'.join(names)} of the 36-layer stack "
                      f"({done_bytes / 1e6:.1f} MB algorithmic), {t_total:.1f} s",
            "host": host_description()}


def run_reference(args):
    """Reference arm: the CPU oracle, timed as it stands, per step a bounded
    sample of the workload (layer-0 k, v projections)."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    from oracle import tb_oracle as oracle

    oracle.build()
    mats = [m for m in synth.config3_stack()[0] if m.name.endswith((".k", ".v"))]
    prob = []
    for m in mats:
        W = synth.gaussian_weights(m.N, m.K, seed=m.seed, dtype=torch.bfloat16)
        wb = W.view(torch.int16).numpy().view("uint16")
        s = oracle.scales_absmax(wb, m.grid)
        p, _ = oracle.pack(wb, m.grid, s)
        x = synth.activations(m.K, seed=m.seed).view(torch.int16).numpy().view("uint16")
        prob.append((p, m, s, x))
    step_bytes = sum(algo_bytes(m.N, m.K, m.grid) for _, m, _, _ in prob)

    def step():
        for p, m, s, x in prob:
            oracle.gemv64(p, m.grid, s, x, m.N, m.K)

    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    dt = time.perf_counter() - t0
    value = step_bytes * args.steps / dt / 1e9
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": workload_config(synth.config3_stack(), 1),
            "cpu_baseline": {"value": value, "unit": "GB/s", "cores": 1, "kind": "oracle",
                             "sample": "each step: fp64 single-threaded oracle GEMV of layer-0 k and v (1024x4096, "
                                       "2-bit) of this workload; value = their algorithmic bytes / time",
                             "host": host_description()},
            "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--layers", type=int, default=None, help="fewer layers (debug only)")
    ap.add_argument("--no-rows", action="store_true")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--clocks-log", default=None,
                    help="nvidia-smi clock log (CSV) of the run (rank r of N > 1 writes PATH.r); "
                         "default: a file in the temp directory")
    args = ap.parse_args()
    if args.impl == "reference":
        run_reference(args)
        return

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    dist = None
    if world > 1:
        import datetime

        import torch.distributed as tdist

        tdist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
        dist = tdist
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    tbbuild.build()
    tb.load()
    stream = torch.cuda.current_stream(dev).cuda_stream

    S = DecodeStack(dev, layers=args.layers)
    n_layers = len(S.layers)
    hbm_peak, bf16_peak, bf16_sus, peak_src = measured_peaks()
    cur = torch.cuda.current_stream(dev)

    # --- device-resident timing (the headline `value`): graph of one step,
    # every layer called with TB_FLAG_OVERLAP_PREVIOUS (resident weights: a
    # call streams its weights while the previous one finishes; activations,
    # outputs and workspace still wait for it)
    FLAGS = tb.FLAG_OVERLAP_PREVIOUS
    g_step = capture(lambda: S.step(FLAGS))
    log = args.clocks_log if (args.clocks_log is None or world == 1) else f"{args.clocks_log}.{rank}"
    with Clocks(local, log) as clk:
        ms = time_region(g_step.replay, args.steps, args.warmup, cur, dist, clk)
    clocks = clk.summary()
    ms_step = ms / args.steps
    value = job_throughput(world, S.step_bytes, ms_step)
    us_layer = ms_step * 1e3 / n_layers
    # dominant kernel: the batch-1 GEMV (k_gemv8), the one kernel of each
    # tb_layer_gemv call; its duration is the call's, averaged over the timed region
    avg_layer_bytes = S.step_bytes / n_layers
    achieved = avg_layer_bytes / (us_layer * 1e-6) / 1e9

    # ablation: the same step without the overlap flag (each call starts after the previous one ends)
    g_plain = capture(lambda: S.step(0))
    ms_plain = time_region(g_plain.replay, args.steps, args.warmup, cur, dist) / args.steps
    del g_plain

    # --- end to end through the public API: each step copies every layer's x
    # from pinned host memory, makes the 36 tb_layer_gemv calls (ctypes, argument
    # checks and tensor-map encoding on the host, every step), and copies every y
    # back; eager (the headline) and captured in a CUDA graph (host work off the
    # timeline, for comparison).  The outputs go back six layers at a time on a
    # copy stream while the next layers run; the step ends when the last of
    # them is on the host.
    x_host = torch.empty_like(S.x_all, device="cpu").pin_memory()
    x_host.copy_(S.x_all.cpu())
    y_host = torch.empty_like(S.y_all, device="cpu").pin_memory()
    copy_out = torch.cuda.Stream(local)
    OUT_EVERY = 6
    out_events = [torch.cuda.Event() for _ in range(n_layers)]

    def e2e_step():
        main = torch.cuda.current_stream(local)
        S.x_all.copy_(x_host, non_blocking=True)
        y0 = 0
        for li, (_, arr) in enumerate(S.layers):
            tb.tb_layer_gemv(arr, S.ws, FLAGS, main.cuda_stream)
            if (li + 1) % OUT_EVERY == 0 or li + 1 == n_layers:
                y1 = S.y_spans[li][1]
                out_events[li].record(main)
                copy_out.wait_event(out_events[li])
                with torch.cuda.stream(copy_out):
                    y_host[y0:y1].copy_(S.y_all[y0:y1], non_blocking=True)
                y0 = y1
        main.wait_stream(copy_out)

    ms_e2e = time_region(e2e_step, args.steps, args.warmup, cur, dist)
    e2e_value = job_throughput(world, S.step_bytes, ms_e2e / args.steps)
    g_e2e = capture(e2e_step)
    ms_e2e_graph = time_region(g_e2e.replay, args.steps, args.warmup, cur, dist)
    e2e_graph_value = job_throughput(world, S.step_bytes, ms_e2e_graph / args.steps)
    del g_e2e, g_step

    rows = None if args.no_rows else rows_section(dev, torch.cuda.current_stream(dev))
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu:
        cpu = cpu_baseline()

    if rank == 0:
        profile_traffic = traffic_per_launch(avg_layer_bytes)
        line = {
            "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": workload_config(S.stack, world),
            "decoder_layer_us_per_token": us_layer,
            "flags": "TB_FLAG_OVERLAP_PREVIOUS",
            "decoder_layer_us_per_token_no_overlap_flag": ms_plain * 1e3 / n_layers,
            "tokens_per_s_equivalent": 1e6 / (us_layer * n_layers),
            "frac_of_spec_8TBs": value / world / SPEC_HBM_GBS,
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": hbm_peak, "unit": "GB/s",
                         "frac": achieved / hbm_peak, "traffic": profile_traffic,
                         "peak_source": f"{peak_src} (MEASURED_PEAKS.json hbm_gbs)" if peak_src == "measured"
                         else "fallback 6.65 TB/s", "kernel": "k_gemv8 (with its record kernel, one pair per tb_layer_gemv call)"},
            "e2e": {"value": e2e_value, "unit": "GB/s",
                    "h2d_bytes_per_step": S.x_all.numel() * 2, "d2h_bytes_per_step": S.y_all.numel() * 4,
                    "ms_per_step": ms_e2e / args.steps, "calls": "eager: 36 tb_layer_gemv C-ABI calls per step",
                    "graph_value": e2e_graph_value, "graph_ms_per_step": ms_e2e_graph / args.steps},
            "gpu_launches": 2 * n_layers * args.steps,  # per call: the record kernel and k_gemv8
            "clocks": clocks,
            "us_x_median_sm_ghz_per_layer": (us_layer * clocks["sm_mhz"] / 1e3) if clocks.get("sm_mhz") else None,
            "rows": rows,
        }
        if cpu:
            line["cpu_baseline"] = cpu
        print(json.dumps(line), flush=True)
    if dist:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
