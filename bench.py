"""Benchmark of the BitLinear W1.58A8 matmul on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Workload (one step): one decode token through the up (2560 -> 6912) and the
down (6912 -> 2560) BitLinear projections of the 2B decoder, each with its own
bf16 token (x ~ N(0,1), 1% outlier channels x50) and absmean-ternarised
N(0, 0.02) latents packed 2 bits per weight. The packed weights rotate over
32 device copies (283 MB, more than twice the 126 MB L2), so every step
streams its weights from HBM. The headline is the GEMV's HBM throughput on
packed-weight bytes. The same line carries the prefill GEMM (M = 2048 tokens,
int8 tensor cores) in ``prefill_gemm``, the 30-layer decoder set at decode
batches 1, 8 and 64 in ``layer_set`` and the large-model shapes in
``large_sweep``.

With ``--gpus N`` (launched by torchrun, one process per GPU) every rank runs
the same independent workload (weak scaling: the path has no data-path
collective); the time is the max over ranks and ``value`` counts all ranks'
bytes.

``--impl reference`` times the CPU oracle (test infrastructure, plain C,
one thread) on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads  # noqa: E402

METRIC = "BitLinear GEMV HBM GB/s (% of peak); prefill GEMM int8 TOPS (% of peak)"
UNIT = "GB/s"
ROTATE = 32                # packed weight copies per matrix (> 2 x L2 in total)
GRAPH_CHUNK = 1024         # most decode steps captured in one CUDA graph (a multiple of ROTATE)
PREFILL_COPIES = 8
MEASURED_PEAKS = os.path.join(ROOT, "MEASURED_PEAKS.json")
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
INT8_PER_BF16 = 2.0        # nominal dense int8 / bf16 tensor ratio (4.5 / 2.25 P)

# DRAM traffic per launch of the dominant kernels, from an ncu capture
# (dram__bytes_read.sum + dram__bytes_write.sum), keyed by the sha256 of the
# kernel source it was taken on; reported only while that source is unchanged.
TRAFFIC = {
    # grouped decode launch (up 2560->6912 + down 6912->2560, M=1): 8,847,360
    # algorithmic bytes; dram__bytes_read.sum + dram__bytes_write.sum of one
    # ncu capture (profiles/gemv_grouped_decode_2b_m1.md), keyed by the hash
    # of the kernel sources it was taken on.
    "gemv": {"src": "979a28baa44430f6", "bytes_per_launch": 8901376},
}


GEMV_SOURCES = ("gemv.cuh", "common.cuh")


def kernel_source_hash(*names: str) -> str:
    """First 16 hex digits of the SHA-256 of the named csrc files, in order."""
    h = hashlib.sha256()
    for name in names:
        with open(os.path.join(ROOT, "ternary_weight_w1_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def load_peaks():
    try:
        with open(MEASURED_PEAKS) as f:
            d = json.load(f)
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                "source": "measured"}
    except (OSError, KeyError, ValueError):
        return {"hbm_gbs": FALLBACK_HBM_GBS, "bf16_tflops": FALLBACK_BF16_TFLOPS,
                "bf16_tflops_sustained": 1400.0, "source": "fallback"}


# ------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons in the background."""

    FIELDS = ("timestamp,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str, interval_ms: int = 50):
        self.gpu_id = gpu_id
        self.interval_ms = interval_ms
        self.proc = None
        self.lines = []
        self.t0 = self.t1 = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-i", self.gpu_id, "-lms", str(self.interval_ms)],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return
        self.reader = threading.Thread(target=self._read, daemon=True)
        self.reader.start()
        time.sleep(0.3)

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.time(), line.strip()))

    def mark(self, start: bool):
        if start:
            self.t0 = time.time()
        else:
            self.t1 = time.time()

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.2)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        for t, line in self.lines:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                rows.append((t, float(parts[1]), float(parts[2]), parts[4:9]))
            except ValueError:
                continue
        inside = [r for r in rows if self.t0 is not None and self.t0 - 0.06 <= r[0] <= (self.t1 or r[0]) + 0.06]
        use = inside if inside else rows
        if not use:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        names = ["active_mask", "hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown",
                 "sw_power_cap"]
        reasons = set()
        for r in use:
            for n, v in zip(names[1:], r[3][1:]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(r[1] for r in use),
                "sm_max_mhz": max(r[2] for r in use),
                "reasons": sorted(reasons), "samples": len(use),
                "samples_in_timed_region": len(inside)}


def smi_gpu_id(local_rank: int) -> str:
    vis = os.environ.get("CUDA_VISIBLE_DEVICES")
    if vis:
        ids = [v.strip() for v in vis.split(",") if v.strip()]
        if local_rank < len(ids):
            return ids[local_rank]
    return str(local_rank)


# ----------------------------------------------------------- distributed

class Dist:
    def __init__(self):
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.rank = int(os.environ.get("RANK", "0"))
        self.local_rank = int(os.environ.get("LOCAL_RANK", "0"))
        self.pg = None

    def init(self, backend: str):
        if self.world > 1:
            import datetime
            import torch.distributed as dist
            dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
            self.pg = dist

    def barrier(self):
        if self.pg is not None:
            self.pg.barrier()

    def max(self, v: float) -> float:
        if self.pg is None:
            return v
        import torch
        t = torch.tensor([v], dtype=torch.float64,
                         device="cuda" if torch.cuda.is_available() else "cpu")
        self.pg.all_reduce(t, op=self.pg.ReduceOp.MAX)
        return float(t.item())

    def close(self):
        if self.pg is not None:
            self.pg.destroy_process_group()


# ------------------------------------------------------------ our arm

def bf16_tensor(bits, device):
    import torch
    return torch.from_numpy(bits.view(np.int16).copy()).view(torch.bfloat16).to(device)


class DecodeWorkload:
    """Device-resident inputs of the decode step with ROTATE weight copies."""

    def __init__(self, bl, device):
        import torch
        self.bl = bl
        probs = workloads.decode_gemv_2b(1).problems
        self.mats = []
        for p in probs:
            packed, gamma = bl.bitlinear_pack_weights(p.weights())
            dev_packed = torch.from_numpy(packed).to(device)
            copies = [dev_packed] + [dev_packed.clone() for _ in range(ROTATE - 1)]
            xs = [bf16_tensor(workloads.activations_bf16(1, p.K, p.x_seed + 7919 * i), device)
                  for i in range(ROTATE)]
            ys = [torch.empty((1, p.N), dtype=torch.bfloat16, device=device)
                  for _ in range(ROTATE)]
            self.mats.append({"p": p, "gamma": gamma, "packed": copies, "x": xs, "y": ys})
        self.packed_bytes_per_step = sum(m["p"].N * m["p"].K // 4 for m in self.mats)
        self.io_bytes_per_step = sum(2 * m["p"].K + 2 * m["p"].N for m in self.mats)
        self.launches_per_step = 1

    def step(self, i: int):
        """Both projections of one token in one grouped launch."""
        j = i % ROTATE
        self.bl.bitlinear_forward_grouped(
            [(m["x"][j], m["packed"][j], m["gamma"], m["p"].N, m["y"][j]) for m in self.mats])

    def step_separate(self, i: int):
        """Both projections of one token, one bitlinear_forward call each."""
        j = i % ROTATE
        for m in self.mats:
            self.bl.bitlinear_forward(m["x"][j], m["packed"][j], m["gamma"], m["p"].N,
                                      y=m["y"][j])

    def run_steps(self, start: int, count: int, separate: bool = False):
        for i in range(start, start + count):
            (self.step_separate if separate else self.step)(i)


def capture_graph(fn):
    import torch
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fn()
    return g


class L2Flush:
    """A device buffer larger than L2 (126 MB on B200); writing it evicts
    whatever the warm-up left in L2."""

    BYTES = 256 << 20

    def __init__(self, device):
        import torch
        self.buf = torch.empty((self.BYTES,), dtype=torch.uint8, device=device)

    def __call__(self):
        self.buf.fill_(0x5A)


def lead_in():
    """Keeps the GPU busy for ~50 us (torch's spin kernel) so that the timed
    region's first event and the graph replays behind it are already queued
    when the device reaches them: host launch latency stays outside the
    device-timed region."""
    import torch
    torch.cuda._sleep(100_000)


def time_graph_steps(dist, wl, steps: int, clocks: ClockSampler | None, separate=False,
                     warm_replays: int = 3, flush: L2Flush | None = None):
    """Time exactly `steps` decode steps replayed from CUDA graphs.

    The steps are captured as one graph of `steps` steps (or, for more than
    GRAPH_CHUNK steps, a GRAPH_CHUNK-step graph replayed several times and a
    graph of the remaining steps). Every captured graph is replayed
    `warm_replays` times before the timed region, so the timed replays pay
    no first-launch cost; L2 is then flushed, and a spin kernel holds the
    device while the replays are queued behind the start event."""
    import torch
    chunk = min(steps, GRAPH_CHUNK)
    full = capture_graph(lambda: wl.run_steps(0, chunk, separate))
    n_full = steps // chunk
    rem = steps - n_full * chunk
    tail = capture_graph(lambda: wl.run_steps(0, rem, separate)) if rem else None
    for _ in range(max(1, warm_replays)):
        full.replay()
        if tail is not None:
            tail.replay()
    torch.cuda.synchronize()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    dist.barrier()
    torch.cuda.synchronize()
    if flush is not None:
        flush()
    lead_in()
    if clocks:
        clocks.mark(True)
    torch.cuda.nvtx.range_push("decode_timed")
    start.record()
    for _ in range(n_full):
        full.replay()
    if tail is not None:
        tail.replay()
    end.record()
    torch.cuda.nvtx.range_pop()
    torch.cuda.synchronize()
    if clocks:
        clocks.mark(False)
    dist.barrier()
    ms = start.elapsed_time(end)
    del full, tail
    return dist.max(ms)


def time_e2e(dist, wl, steps: int):
    """Same steps through the library's host-buffer call
    (bitlinear_forward_grouped_host): each step's tokens are copied from
    pinned host memory, the grouped launch runs, and its outputs are copied
    back to pinned host memory, all inside one library call per step. Both
    tokens of a step sit in one pinned buffer and one device staging buffer
    (one host-to-device copy); both outputs land in one device buffer and one
    pinned buffer (one device-to-host copy)."""
    import torch
    xk = [m["p"].K for m in wl.mats]
    yn = [m["p"].N for m in wl.mats]
    host_x = [torch.cat([m["x"][j].reshape(-1) for m in wl.mats]).cpu().pin_memory()
              for j in range(ROTATE)]
    host_y = torch.empty(sum(yn), dtype=torch.bfloat16).pin_memory()
    dev_x = torch.empty(sum(xk), dtype=torch.bfloat16, device=wl.mats[0]["x"][0].device)
    dev_y = torch.empty(sum(yn), dtype=torch.bfloat16, device=dev_x.device)
    xs = list(torch.split(dev_x, xk))
    ys = list(torch.split(dev_y, yn))
    calls = [wl.bl.GroupedHostCall(
                 [(xs[k].view(1, -1), m["packed"][j], m["gamma"], m["p"].N, ys[k].view(1, -1))
                  for k, m in enumerate(wl.mats)])
             for j in range(ROTATE)]

    def one(i):
        j = i % ROTATE
        calls[j](host_x[j], host_y)

    for i in range(5):
        one(i)
    torch.cuda.synchronize()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    dist.barrier()
    torch.cuda.synchronize()
    start.record()
    for i in range(steps):
        one(i)
    end.record()
    torch.cuda.synchronize()
    dist.barrier()
    return dist.max(start.elapsed_time(end))


def bench_prefill(bl, device, reps: int = 20, norm: bool = False):
    """Prefill step (M = 2048: up and down, quantisation kernel + tcgen05
    GEMM each), inputs rotating over copies larger than L2; with `norm` the
    tokens are RMS-normalised in the quantisation kernel
    (bitlinear_forward_rmsnorm). Returns (ms per step, int8 ops per step)."""
    import torch
    probs = workloads.prefill_2b(2048).problems
    mats = []
    for p in probs:
        packed, gamma = bl.bitlinear_pack_weights(p.weights())
        dp = torch.from_numpy(packed).to(device)
        x = bf16_tensor(p.x_input(), device)
        ws_bytes = bl.bitlinear_workspace_bytes(p.M, p.N, p.K)
        mats.append({"p": p, "gamma": gamma,
                     "packed": [dp] + [dp.clone() for _ in range(PREFILL_COPIES - 1)],
                     "x": [x] + [x.clone() for _ in range(PREFILL_COPIES - 1)],
                     "y": torch.empty((p.M, p.N), dtype=torch.bfloat16, device=device),
                     "ws": torch.empty((ws_bytes,), dtype=torch.uint8, device=device),
                     "g": torch.from_numpy(workloads.norm_gains(p.K, p.w_seed + 50)).to(device)})

    def step(i):
        j = i % PREFILL_COPIES
        for m in mats:
            if norm:
                bl.bitlinear_forward_rmsnorm(m["x"][j], m["packed"][j], m["gamma"], m["p"].N,
                                             m["g"], y=m["y"], workspace=m["ws"])
            else:
                bl.bitlinear_forward(m["x"][j], m["packed"][j], m["gamma"], m["p"].N,
                                     y=m["y"], workspace=m["ws"])

    for i in range(3):
        step(i)
    g = capture_graph(lambda: [step(i) for i in range(PREFILL_COPIES)])
    g.replay()
    torch.cuda.synchronize()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.nvtx.range_push("rmsnorm_prefill_timed" if norm else "prefill_timed")
    start.record()
    for _ in range(reps):
        g.replay()
    end.record()
    torch.cuda.nvtx.range_pop()
    torch.cuda.synchronize()
    ms = start.elapsed_time(end) / (reps * PREFILL_COPIES)
    ops = sum(2 * m["p"].M * m["p"].N * m["p"].K for m in mats)
    return ms, ops


def time_graph(fn, reps: int, nvtx: str | None = None) -> float:
    """Mean ms of `fn` (captured once in a CUDA graph) over `reps` replays,
    after three warm-up replays; the timed replays sit in NVTX range `nvtx`."""
    import torch
    g = capture_graph(fn)
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if nvtx:
        torch.cuda.nvtx.range_push(nvtx)
    start.record()
    for _ in range(reps):
        g.replay()
    end.record()
    if nvtx:
        torch.cuda.nvtx.range_pop()
    torch.cuda.synchronize()
    del g
    return start.elapsed_time(end) / reps


def bench_rmsnorm_decode(bl, wl, reps: int = 200) -> float:
    """The decode step's two projections (M = 1) with the tokens
    RMS-normalised in the GEMV prologue, one bitlinear_forward_rmsnorm launch
    per projection, over the same rotating weight copies as the headline
    step. Returns ms per step."""
    import torch
    gains = [torch.from_numpy(workloads.norm_gains(m["p"].K, m["p"].w_seed + 50)).to(
        m["x"][0].device) for m in wl.mats]

    def steps():
        for j in range(ROTATE):
            for m, g in zip(wl.mats, gains):
                bl.bitlinear_forward_rmsnorm(m["x"][j], m["packed"][j], m["gamma"], m["p"].N,
                                             g, y=m["y"][j])
    steps()
    torch.cuda.synchronize()
    return time_graph(steps, reps, nvtx="rmsnorm_decode_timed") / ROTATE


def bench_b3_decode(bl, wl, reps: int = 200):
    """The decode step's two projections (M = 1) on base-3 packed weights
    (bitlinear_forward_grouped_b3, one launch per step, as the 2-bit step)
    over ROTATE copies, the footprint option: µs per step, GB/s of base-3
    bytes, and the bytes per step against the 2-bit layout's."""
    import torch
    mats = []
    for m in wl.mats:
        p = m["p"]
        pk, gamma = bl.bitlinear_pack_weights_b3(p.weights())
        dp = torch.from_numpy(pk).to(m["x"][0].device)
        mats.append((m, [dp] + [dp.clone() for _ in range(ROTATE - 1)], gamma))
    b3_bytes = sum(d[0].numel() for _, d, _ in mats)

    def steps():
        for j in range(ROTATE):
            bl.bitlinear_forward_grouped_b3(
                [(m["x"][j], d[j], g, m["p"].N, m["y"][j]) for m, d, g in mats])
    steps()
    torch.cuda.synchronize()
    ms = time_graph(steps, reps, nvtx="b3_decode_timed") / ROTATE
    return {"us_per_step": round(ms * 1e3, 3),
            "GBps_b3_bytes": round(b3_bytes / (ms * 1e-3) / 1e9, 1),
            "b3_bytes_per_step": b3_bytes,
            "two_bit_bytes_per_step": wl.packed_bytes_per_step,
            "launches_per_step": 1}


def bench_ffn(bl, device, batches=(1, 8), copies: int = 16, reps: int = 20):
    """The 2B decoder's feed-forward block (gate and up 2560 -> 6912, the
    gated ReLU^2, down 6912 -> 2560) for B decode tokens through
    bitlinear_ffn_forward: at B <= 6 one GEMV launch for gate and up with h
    written from its epilogue and one launch for down; at larger B a grouped
    quantisation + GEMM pair for gate and up, the h kernel, and a
    quantisation + GEMM pair for down. The three matrices (13.3 MB packed)
    rotate over `copies` device copies (212 MB > L2). Per B: microseconds per
    block and GB/s of packed weights."""
    import torch
    K, F = 2560, 6912
    mats = []
    for seed, (n, k) in zip((7001, 7002, 7003), ((F, K), (F, K), (K, F))):
        pk, gamma = bl.bitlinear_pack_weights(workloads.latent_weights(n, k, seed))
        dp = torch.from_numpy(pk).to(device)
        mats.append(([dp] + [dp.clone() for _ in range(copies - 1)], gamma))
    wbytes = 3 * F * K // 4
    out = {}
    for B in batches:
        x = bf16_tensor(workloads.activations_bf16(B, K, 7004), device)
        h = torch.empty((B, F), dtype=torch.float32, device=device)
        y = torch.empty((B, K), dtype=torch.bfloat16, device=device)
        need = bl.bitlinear_workspace_bytes_ffn(B, K, F)
        ws = torch.empty((max(need, 1),), dtype=torch.uint8, device=device)

        def steps():
            for c in range(copies):
                bl.bitlinear_ffn_forward(x, *[(m[0][c], m[1]) for m in mats], h=h, y=y,
                                         workspace=ws)
        steps()
        torch.cuda.synchronize()
        ms = time_graph(steps, reps, nvtx=f"ffn_b{B}_timed") / copies
        out[f"B={B}"] = {"us_per_block": round(ms * 1e3, 2),
                         "GBps_packed": round(wbytes / (ms * 1e-3) / 1e9, 1),
                         "launches_per_block": 2 if need == 0 else (3 if B <= 6 else 5)}
    return out


def bench_layer_set(bl, device, batches=(1, 8, 64), reps: int = 10):
    """The seven projections of the 2B decoder layer for 30 layers (521 MB of
    packed weights, more than four times L2) at decode batch B, one grouped
    call per layer: one GEMV launch at B = 1, one quantisation launch and one
    tensor-core GEMM launch over the seven problems at B > 6. The 30 layers
    hold distinct device copies of one seeded layer's packed weights (the
    parity tests use independent seeds per layer)."""
    import torch
    layer = workloads.layer_set_2b(1, layers=1).problems
    packed = []
    for p in layer:
        pk, gamma = bl.bitlinear_pack_weights(p.weights())
        packed.append((p, torch.from_numpy(pk).to(device), gamma))
    layers = workloads.NUM_LAYERS
    copies = [[(p, dp if li == 0 else dp.clone(), g) for p, dp, g in packed]
              for li in range(layers)]
    wbytes = layers * sum(p.N * p.K // 4 for p, _, _ in packed)
    out = {}
    for B in batches:
        xs = [bf16_tensor(workloads.activations_bf16(B, p.K, p.x_seed), device) for p, _, _ in packed]
        ys = [torch.empty((B, p.N), dtype=torch.bfloat16, device=device) for p, _, _ in packed]
        groups = [[(xs[k], dp, g, p.N, ys[k]) for k, (p, dp, g) in enumerate(copies[li])]
                  for li in range(layers)]
        ws_bytes = bl.bitlinear_workspace_bytes_grouped(groups[0])
        ws = torch.empty((max(ws_bytes, 1),), dtype=torch.uint8, device=device)

        def step():
            for li in range(layers):
                bl.bitlinear_forward_grouped(groups[li], workspace=ws)
        launches = layers * (1 if ws_bytes == 0 else 2)
        step()
        torch.cuda.synchronize()
        ms = time_graph(step, reps, nvtx=f"layer_set_b{B}_timed")
        out[f"B={B}"] = {"us_per_layer": round(ms * 1e3 / layers, 2),
                         "GBps_packed": round(wbytes / (ms * 1e-3) / 1e9, 1),
                         "TOPS": round(2 * B * wbytes * 4 / (ms * 1e-3) / 1e12, 2),
                         "launches_per_step": launches}
    return out


def bench_large_sweep(bl, device, ms_list=(1, 16, 256, 4096), reps: int = 5):
    """K=8192->N=28672 and K=28672->N=8192 (58.7 MB of packed weights each)
    at M tokens, automatic dispatch, weights rotating over 3 copies per matrix
    (352 MB in total). Per M: microseconds per matrix pair, GB/s of packed
    weights and int8 TOPS."""
    import torch
    out = {}
    mats = []
    for p in workloads.large_sweep(1).problems:
        pk, gamma = bl.bitlinear_pack_weights(p.weights())
        dp = torch.from_numpy(pk).to(device)
        mats.append((p, [dp, dp.clone(), dp.clone()], gamma))
    wbytes = sum(p.N * p.K // 4 for p, _, _ in mats)
    for M in ms_list:
        xs = [bf16_tensor(workloads.activations_bf16(M, p.K, p.x_seed), device) for p, _, _ in mats]
        ys = [torch.empty((M, p.N), dtype=torch.bfloat16, device=device) for p, _, _ in mats]
        ws_bytes = max(bl.bitlinear_workspace_bytes(M, p.N, p.K) for p, _, _ in mats)
        ws = torch.empty((max(ws_bytes, 1),), dtype=torch.uint8, device=device)

        def step():
            for c in range(3):
                for k, (p, dps, g) in enumerate(mats):
                    bl.bitlinear_forward(xs[k], dps[c], g, p.N, y=ys[k], workspace=ws)
        step()
        torch.cuda.synchronize()
        ms = time_graph(step, reps, nvtx=f"large_m{M}_timed") / 3
        out[f"M={M}"] = {"us_per_pair": round(ms * 1e3, 2),
                         "GBps_packed": round(wbytes / (ms * 1e-3) / 1e9, 1),
                         "TOPS": round(2 * M * wbytes * 4 / (ms * 1e-3) / 1e12, 1)}
        del xs, ys, ws
    return out


def cpu_info():
    """(CPU model name, logical cores available to this process)."""
    model = "unknown"
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    try:
        cores = len(os.sched_getaffinity(0))
    except (AttributeError, OSError):
        cores = os.cpu_count() or 1
    return model, cores


def _oracle_decode_rate(orc, mats, seconds):
    """Full decode steps (quantise, integer product, rescale of both
    projections) of one oracle build for about `seconds`: (steps, seconds)."""
    t0 = time.perf_counter()
    steps = 0
    while True:
        for p, Wq, g, xf in mats:
            xq, beta = orc.quant_act(xf)
            acc = orc.matmul_i32(xq, Wq)
            orc.rescale_bf16(acc, beta, g)
        steps += 1
        el = time.perf_counter() - t0
        if el >= seconds:
            return steps, el


def _oracle_forward_us(orc, problems):
    """Microseconds of one oracle forward over each prepared problem, summed.
    A problem prepared on a sample of its tokens or weight rows is scaled to
    its full M and N (an extrapolation; the time is linear in both)."""
    total = 0.0
    for p, Wq, g, xf in problems:
        t0 = time.perf_counter()
        xq, beta = orc.quant_act(xf)
        acc = orc.matmul_i32(xq, Wq)
        orc.rescale_bf16(acc, beta, g)
        el = time.perf_counter() - t0
        total += el * (p.M / xf.shape[0]) * (p.N / Wq.shape[0])
    return total * 1e6


def cpu_baseline_oracle(seconds: float = 10.0):
    """The oracle (plain C) on the host cores: the headline is the
    single-threaded build on full decode steps (both projections, M = 1) for
    about `seconds`; the same steps run on the OpenMP build over all cores
    for half as long; and one forward per workload with each build (the
    prefill and M = 4096 times extrapolated from a token sample, as labelled).
    Returns the cpu_baseline dict."""
    import oracle
    one = oracle.default()
    omp = oracle.Oracle(oracle.load_omp())
    model, cores = cpu_info()

    def prep(problems, tokens=None, row_div=1):
        """Oracle inputs of each problem: every weight row, or the first
        N / row_div of them (seeded latents of that many rows), and every
        token or the first `tokens`."""
        out = []
        for p in problems:
            W = workloads.latent_weights(p.N // row_div, p.K, p.w_seed)
            g = one.absmean_gamma(W)
            xf = one.bf16_to_f32(workloads.to_bf16_bits(
                workloads.activations_f32(tokens or p.M, p.K, p.x_seed)))
            out.append((p, one.ternarize(W, g), g, xf))
        return out

    dec = prep(workloads.decode_gemv_2b(1).problems)
    nbytes = sum(p.N * p.K // 4 for p, *_ in dec)
    steps1, el1 = _oracle_decode_rate(one, dec, seconds)
    stepsn, eln = _oracle_decode_rate(omp, dec, seconds / 2)
    layer = prep(workloads.layer_set_2b(1, layers=1).problems)
    pre = prep(workloads.prefill_2b(2048).problems, tokens=16)
    big1 = prep(workloads.large_sweep(1).problems, row_div=8)
    per_config = {}
    for name, probs, label in (
            ("decode_2b_m1_us_per_step", dec, "measured"),
            ("layer_2b_b1_us_per_layer", layer, "measured"),
            ("prefill_2b_m2048_us_per_step", pre, "extrapolated from 16 of the 2048 tokens"),
            ("large_m1_us_per_pair", big1, "extrapolated from 1/8 of the weight rows")):
        per_config[name] = {"one_thread": round(_oracle_forward_us(one, probs), 1),
                            "all_cores": round(_oracle_forward_us(omp, probs), 1),
                            "how": label}
    v1 = nbytes * steps1 / el1 / 1e9
    vn = nbytes * stepsn / eln / 1e9
    return {"value": round(v1, 4), "unit": UNIT, "cores": 1, "kind": "oracle",
            "sample": f"{steps1} full decode steps (up+down, M=1) of the single-threaded "
                      f"C oracle in {el1:.1f} s",
            "cpu_model": model, "nproc": cores,
            "all_cores": {"value": round(vn, 4), "unit": UNIT, "cores": cores,
                          "kind": "oracle-omp",
                          "sample": f"{stepsn} full decode steps of the same oracle built with "
                                    f"-fopenmp (integer products over all {cores} cores) in "
                                    f"{eln:.1f} s"},
            "per_config": per_config}


def run_ours(args, dist):
    import torch
    import ternary_weight_w1_b200 as bl
    torch.cuda.set_device(dist.local_rank)
    device = torch.device("cuda", dist.local_rank)
    bl.lib()
    peaks = load_peaks()
    wl = DecodeWorkload(bl, device)
    for i in range(args.warmup):
        wl.step(i)
    torch.cuda.synchronize()

    flush = L2Flush(device)
    clocks = ClockSampler(smi_gpu_id(dist.local_rank))
    clocks.start()
    ms = time_graph_steps(dist, wl, args.steps, clocks, flush=flush)
    clk = clocks.stop()
    ms_sep = time_graph_steps(dist, wl, args.steps, None, separate=True, flush=flush)

    bytes_all = wl.packed_bytes_per_step * args.steps * dist.world
    value = bytes_all / (ms * 1e-3) / 1e9
    launches = wl.launches_per_step * args.steps
    per_launch_bytes = wl.packed_bytes_per_step / wl.launches_per_step
    avg_launch_ms = ms / launches
    achieved = per_launch_bytes / (avg_launch_ms * 1e-3) / 1e9
    traffic = None
    t = TRAFFIC.get("gemv")
    if t is not None and t.get("src") == kernel_source_hash(*GEMV_SOURCES):
        traffic = t["bytes_per_launch"]

    e2e_steps = min(args.steps, args.e2e_steps)
    ms_e2e = time_e2e(dist, wl, e2e_steps)
    e2e_value = wl.packed_bytes_per_step * e2e_steps * dist.world / (ms_e2e * 1e-3) / 1e9

    if args.layer_set_only:
        return {"layer_set": bench_layer_set(bl, device)}
    if args.large_only:
        return {"large_sweep": bench_large_sweep(bl, device, ms_list=(1,))}
    if args.decode_only:
        return {"decode_only": {"value": round(value, 2), "unit": UNIT,
                                "ms_per_step": ms / args.steps, "steps": args.steps,
                                "separate_ms_per_step": ms_sep / args.steps,
                                "e2e": round(e2e_value, 2), "clocks": clk}}
    pre_ms, pre_ops = bench_prefill(bl, device)
    pre_tops = pre_ops / (pre_ms * 1e-3) / 1e12
    int8_peak = peaks["bf16_tflops"] * INT8_PER_BF16
    norm_dec_ms = bench_rmsnorm_decode(bl, wl)
    norm_pre_ms, _ = bench_prefill(bl, device, norm=True)
    norm_pre_tops = pre_ops / (norm_pre_ms * 1e-3) / 1e12

    out = {
        "metric": METRIC,
        "value": round(value, 2),
        "unit": UNIT,
        "n_gpus": dist.world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": ms / args.steps,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "int8xternary->int32 (bf16 in/out)",
        "data": "synthetic (seeded N(0,0.02) latents, N(0,1) bf16 tokens with 1% x50 outlier channels)",
        "config": {"workload": "decode GEMV, 2B shape, M=1: up 2560->6912 and down 6912->2560 "
                               "(independent tokens) per step in one grouped launch, packed "
                               f"weights rotating over {ROTATE} device copies "
                               f"({ROTATE * wl.packed_bytes_per_step / 1e6:.0f} MB > L2), "
                               "CUDA-graph replay",
                   "l2": "L2 flushed (256 MB write) before the timed region; inputs larger "
                         "than L2 inside it (rotating weight copies)",
                   "parallelism": f"replicas x{dist.world}"},
        "roofline": {"bound": "hbm", "achieved": round(achieved, 1),
                     "peak": peaks["hbm_gbs"], "unit": "GB/s",
                     "frac": round(achieved / peaks["hbm_gbs"], 4), "traffic": traffic,
                     "kernel": "gemv_kernel<1,bf16> (grouped: up + down)",
                     "algorithmic_bytes_per_launch": per_launch_bytes,
                     "peak_source": peaks["source"]},
        "e2e": {"value": round(e2e_value, 2), "unit": UNIT,
                "h2d_bytes_per_step": sum(2 * m["p"].K for m in wl.mats),
                "d2h_bytes_per_step": sum(2 * m["p"].N for m in wl.mats),
                "steps": e2e_steps},
        "gpu_launches": launches,
        "decode_separate_launches": {
            "value": round(wl.packed_bytes_per_step * args.steps * dist.world
                           / (ms_sep * 1e-3) / 1e9, 2),
            "unit": UNIT, "ms_per_step": ms_sep / args.steps,
            "note": "same step with one bitlinear_forward launch per projection"},
        "clocks": clk,
        "prefill_gemm": {"workload": "M=2048 tokens: up 2560->6912 and down 6912->2560, "
                                     "quantisation kernel + tcgen05 kind::i8 GEMM each",
                         "value": round(pre_tops, 1), "unit": "TOPS (int8)",
                         "ms_per_step": pre_ms,
                         "peak": int8_peak, "peak_note": "measured bf16 burst x 2 (nominal int8/bf16)",
                         "frac": round(pre_tops / int8_peak, 4)},
        "rmsnorm_forward": {
            "workload": "the same decode and prefill steps with every token RMS-normalised "
                        "(gains [K]) inside the quantisation pass (bitlinear_forward_rmsnorm, "
                        "one launch per projection at decode)",
            "decode_m1": {"value": round(wl.packed_bytes_per_step * dist.world
                                         / (norm_dec_ms * 1e-3) / 1e9, 2),
                          "unit": UNIT, "ms_per_step": norm_dec_ms,
                          "plain_ms_per_step": ms_sep / args.steps},
            "prefill_m2048": {"value": round(norm_pre_tops, 1), "unit": "TOPS (int8)",
                              "ms_per_step": norm_pre_ms, "plain_ms_per_step": pre_ms,
                              "frac": round(norm_pre_tops / int8_peak, 4)}},
    }
    if not args.no_extra:
        out["b3_decode"] = {
            "workload": "the decode step (up 2560->6912, down 6912->2560, M=1) on base-3 packed "
                        "weights (5 codes per byte, K padded to a multiple of 160), one grouped "
                        "launch per step; compare the headline value",
            **bench_b3_decode(bl, wl)}
        out["ffn_chain"] = {
            "workload": "2B feed-forward block: gate and up 2560->6912 (B<=6: one GEMV "
                        "launch, h = max(gate,0)^2 * up written from its epilogue; larger B: "
                        "grouped tensor-core launches and an h kernel), down 6912->2560 on h; "
                        "13.3 MB of packed weights per block",
            **bench_ffn(bl, device)}
        out["layer_set"] = {
            "workload": "2B decoder layer (q 2560->2560, k/v 2560->640, o 2560->2560, gate/up "
                        "2560->6912, down 6912->2560) x 30 layers, 521 MB of packed weights",
            **bench_layer_set(bl, device)}
        out["large_sweep"] = {
            "workload": "K=8192->N=28672 and K=28672->N=8192 per step, 117 MB of packed weights",
            **bench_large_sweep(bl, device)}
    if dist.rank == 0 and dist.world == 1 and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline_oracle(args.cpu_seconds)
    return out


# ------------------------------------------------------ reference arm

def run_reference(args, dist):
    """The oracle on the host cores: each step a bounded sample of the decode
    step (1/64 of the output rows of both projections)."""
    import oracle
    orc = oracle.default()
    sample = 64
    mats = []
    for p in workloads.decode_gemv_2b(1).problems:
        W = p.weights()
        g = orc.absmean_gamma(W)
        rows = p.N // sample
        Wq = orc.ternarize(W[:rows], g)
        mats.append((p, Wq, g, orc.bf16_to_f32(p.x_input())))
    nbytes = sum(Wq.shape[0] * p.K // 4 for p, Wq, *_ in mats)

    def step():
        for p, Wq, g, xf in mats:
            xq, beta = orc.quant_act(xf)
            acc = orc.matmul_i32(xq, Wq)
            orc.rescale_bf16(acc, beta, g)

    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    el = time.perf_counter() - t0
    v = nbytes * args.steps / el / 1e9
    return {"metric": METRIC, "value": round(v, 4), "unit": UNIT, "n_gpus": dist.world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": el * 1e3 / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "int8xternary->int32 (bf16 in/out)", "data": "synthetic",
            "impl": "reference",
            "config": {"workload": "decode GEMV, 2B shape, M=1: up 2560->6912 then down "
                                   "6912->2560 per step (oracle on 1/64 of the output rows)",
                       "parallelism": "host cores, 1 thread"},
            "cpu_baseline": {"value": round(v, 4), "unit": UNIT, "cores": 1, "kind": "oracle",
                             "sample": f"1/{sample} of the output rows of each projection per step"},
            "e2e": {"value": round(v, 4), "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50000)
    ap.add_argument("--warmup", type=int, default=64)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--e2e-steps", type=int, default=20000)
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extra", action="store_true",
                    help="skip the layer-set and large-shape measurements")
    ap.add_argument("--large-only", action="store_true",
                    help="only the large-shape M = 1 measurement after the decode step "
                         "(for profiling)")
    ap.add_argument("--decode-only", action="store_true",
                    help="only the decode step (headline) measurements (for profiling)")
    ap.add_argument("--layer-set-only", action="store_true",
                    help="only the layer-set measurement after the decode step (for profiling)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    dist = Dist()
    if args.impl == "reference":
        if dist.rank != 0:
            return 0
        print(json.dumps(run_reference(args, dist)), flush=True)
        return 0
    dist.init("nccl")
    try:
        out = run_ours(args, dist)
        if dist.rank == 0:
            print(json.dumps(out), flush=True)
    finally:
        dist.close()
    return 0


if __name__ == "__main__":
    sys.exit(main())
