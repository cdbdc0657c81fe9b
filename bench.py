"""Benchmark: mixer tokens/s of exact online long convolution on B200.

One step = one closed-loop generation of the whole sequence (fi_reset, then
fi_generate over L positions) for the 18-layer x 864-channel, L = 32768, B = 4
fp32 workload; tokens per step = B * L. Inputs (filters, first token, noise)
are resident in HBM before timing; the state the step streams through (8.6 GB)
is far larger than L2, so no flush is needed between steps.

Also reported: the dominant kernel's roofline (from CUDA events recorded around
every launch during the timed steps), the whole-run roofline of the schedule's
algorithmic bytes and flops, end-to-end throughput through fi_generate_host
(host buffers, copies inside the timed region), the quadratic Lazy baseline on
the GPU (extrapolated from a measured prefix), and the float64 oracle on the
host cores (a bounded sample, extrapolated).

python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference] [--workload NAME]
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import math
import multiprocessing as mp
import os
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import synth  # noqa: E402

METRIC = "mixer tokens/s at 18\u00d7864, L=32K on 1 B200; % of roofline; speedup vs O(L\u00b2)"


def metric_name(w: synth.Workload, api: str = "generate", block: str = "tanh") -> str:
    """The headline metric's name for the headline workload, the same form for the others."""
    if w.name == synth.HEADLINE and api == "generate" and block == "tanh":
        return METRIC
    kind = "mixer tokens/s" if api == "generate" else "mixer tokens/s through fi_step (one call per position)"
    if block == "mlp":
        kind += " with MLP + GELU blocks"
    return (f"{kind} at {w.layers}\u00d7{w.channels}, L={w.length}, B={w.batch} {w.dtype} on 1 B200; "
            "% of roofline; speedup vs O(L\u00b2)")
UNIT = "tokens/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0}
NOMINAL_HBM_GBS = 8000.0            # the HBM figure the roofline target is quoted against
FP32_LANES_PER_SM = 128
NUM_SMS = 148
L2_BYTES = 126 * 1024 * 1024


# ----------------------------------------------------------------------------- cost model
def schedule_levels(L: int):
    """(U, count): blocks of side U = 2^q occur 2^(P-1-q) times per layer and stream."""
    P = int(math.log2(L))
    return [(1 << q, 1 << (P - 1 - q)) for q in range(P)]


def fft_flops(U: int) -> float:
    """Model flops of one FFT block per stream: two real FFTs of length 2U plus the product."""
    return 2 * 2.5 * (2 * U) * math.log2(2 * U) + 7 * U


def cost_model(w: synth.Workload, chunk: int, fft_from: int, fft_max: int = 1 << 14, tc_max: int = 0):
    """Algorithmic bytes and flops of one full generation, split by kernel class.

    Bytes (compulsory HBM traffic of the schedule): per block of side U and (layer,
    channel) the taps (2U-1)*s_h (direct) or the spectrum (U+1)*8 (FFT); per (layer,
    sequence, channel) the U sources (s_x each) and the accumulator read-modify-write
    (2U*4); per position and (layer, sequence, channel) the accumulator row (4) and
    the activation write (s_x); per position and (sequence, channel) token, noise and
    output (s_x + 4 + 4). Flops: direct block 2U^2, FFT block fft_flops(U), red cell 3.
    Tensor-core blocks (sides 64..tc_max) count like direct ones: taps, sources,
    accumulators, 2U^2 flops per row (the Toeplitz product, not the padded MMA work).
    Blocks wider than fft_max are partitioned FFT blocks (fft class).
    """
    M, D, L, B = w.layers, w.channels, w.length, w.batch
    s = 2 if w.dtype == "bf16" else 4
    out = {k: {"bytes": 0.0, "flops": 0.0, "blocks": 0} for k in ("chunk", "direct", "fft", "tc")}
    for U, n in schedule_levels(L):
        if U < chunk:
            cls = "chunk"
        elif 64 <= U <= tc_max:
            cls = "tc"
        elif fft_from and fft_from <= U:
            cls = "fft"
        else:
            cls = "direct"
        m = U // fft_max if (cls == "fft" and U > fft_max) else 0
        if m:
            # partitioned: m sub-blocks of side fft_max; 2m-1 segment spectra per
            # (layer, channel); per row m forward and m inverse transforms and m^2
            # spectrum products of fft_max + 1 points (8 flops each)
            per_ld = (2 * m - 1) * (fft_max + 1) * 8
            row_flops = m * fft_flops(fft_max) + 8.0 * m * m * (fft_max + 1)
        else:
            per_ld = (U + 1) * 8 if cls == "fft" else (2 * U - 1) * s
            row_flops = fft_flops(U) if cls == "fft" else 2.0 * U * U
        per_lbd = U * s + 2 * U * 4
        out[cls]["bytes"] += n * (M * D * per_ld + M * B * D * per_lbd)
        if cls == "chunk":
            out[cls]["block_bytes"] = out[cls].get("block_bytes", 0.0) + n * (M * D * per_ld + M * B * D * per_lbd)
        out[cls]["flops"] += n * M * B * D * row_flops
        out[cls]["blocks"] += n
    out["chunk"]["bytes"] += L * (M * B * D * (4 + s) + B * D * (s + 8))
    out["chunk"]["flops"] += L * M * B * D * 3.0
    tot = {"bytes": sum(v["bytes"] for v in out.values()), "flops": sum(v["flops"] for v in out.values())}
    return out, tot


# Widest block the per-position launches add themselves (fi_step's red-cell
# kernel for stacks of up to 32 layers, the channel-mixing block's small-block
# launch always); wider ones are launches of their own.
TOKEN_BLOCK_MAX, TOKEN_MAX_LAYERS, MLP_BLOCK_MAX = 8, 32, 8


def per_position_model(w: synth.Workload, fft_from: int, tc_max: int, mlp_hidden: int = 0):
    """cost_model for the position-by-position paths (fi_step, the channel-mixing
    block): the per-position bytes and flops, and the blocks the per-position
    launches add themselves, belong to "token"; wider blocks keep their classes
    (direct, FFT, tensor cores). The channel-mixing block adds its weights (read
    once per position) and 2 * 2 * D * Dh flops per (layer, sequence)."""
    fused = MLP_BLOCK_MAX if mlp_hidden else (TOKEN_BLOCK_MAX if w.layers <= TOKEN_MAX_LAYERS else 0)
    model, tot = cost_model(w, 2 * fused if fused else 1, fft_from, tc_max=tc_max)
    model["token"] = dict(model["chunk"])
    model["chunk"] = {"bytes": 0.0, "flops": 0.0, "blocks": 0}
    if mlp_hidden:
        extra_b = w.length * w.layers * (2.0 * w.channels * mlp_hidden + mlp_hidden + w.channels) * 4
        extra_f = w.length * w.layers * w.batch * 4.0 * w.channels * mlp_hidden
        model["token"]["bytes"] += extra_b
        model["token"]["flops"] += extra_f
        tot = {"bytes": tot["bytes"] + extra_b, "flops": tot["flops"] + extra_f}
    return model, tot


def closed_form_block_bytes(w: synth.Workload) -> float:
    """The schedule's block bytes in closed form, M*D*(L/2)*log2(L)*(8 + B(s_x+8))."""
    s = 2 if w.dtype == "bf16" else 4
    return w.layers * w.channels * (w.length / 2) * math.log2(w.length) * (8 + w.batch * (s + 8))


def lazy_bytes(w: synth.Workload) -> float:
    """HBM bytes of the Lazy method: every position re-reads its whole history and taps."""
    s = 2 if w.dtype == "bf16" else 4
    pairs = w.length * (w.length - 1) / 2
    return pairs * w.layers * w.channels * (w.batch * s + s)


# ----------------------------------------------------------------------------- peaks and clocks
def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": float(p["hbm_gbs"]), "bf16_tflops": float(p["bf16_tflops"]),
                "sm_max_mhz": float(p.get("sm_max_mhz", 1965.0)), "source": "measured"}
    except Exception:
        return dict(FALLBACK_PEAKS, sm_max_mhz=1965.0, source="fallback")


def fp32_peak_tflops(mhz: float) -> float:
    return NUM_SMS * FP32_LANES_PER_SM * 2 * mhz * 1e6 / 1e12


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 200 ms while running."""

    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.path = None

    def __enter__(self):
        try:
            import tempfile
            fd, self.path = tempfile.mkstemp(prefix="clocks", suffix=".csv")
            os.close(fd)
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.QUERY}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=self.fh, stderr=subprocess.DEVNULL)
            self._wait_lines(1, 5.0)      # the sampler is live before the region starts
        except Exception:
            self.proc = None
        return self

    def _lines(self) -> int:
        self.fh.flush()
        with open(self.path) as f:
            return sum(1 for _ in f)

    def _wait_lines(self, n: int, limit_s: float):
        t0 = time.perf_counter()
        while self._lines() < n and time.perf_counter() - t0 < limit_s:
            time.sleep(0.02)

    def __exit__(self, *exc):
        if self.proc is not None:
            # one more sample after the region, so that a region shorter than the
            # sampling period still has one taken while or right after it ran
            self._wait_lines(self._lines() + 1, 1.0)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
            self.fh.close()

    def summary(self):
        if self.proc is None or not self.path:
            return None
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    rows.append((float(parts[1]), float(parts[2]), float(parts[3]), parts[5:9]))
                except ValueError:
                    continue
        os.unlink(self.path)
        if not rows:
            return None
        sm = [r[0] for r in rows]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[k] for r in rows for k, v in enumerate(r[3]) if v.lower() == "active"})
        return {"sm_mhz": float(np.median(sm)), "sm_max_mhz": max(r[1] for r in rows),
                "power_w_max": max(r[2] for r in rows), "samples": len(rows), "reasons": reasons}


# ----------------------------------------------------------------------------- distributed plumbing
def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", str(rank)))
    return world, rank, local


def dist_init(world: int, backend: str):
    if world <= 1:
        return False
    import torch.distributed as dist
    os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
    dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=120))
    return True


def rank_seed(seed: int, rank: int) -> int:
    """Each rank draws an independent batch of the same workload (weak scaling)."""
    return seed + 1000003 * rank


def reduce_max(value: float, device=None) -> float:
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(device=None):
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        if device is not None:
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


# ----------------------------------------------------------------------------- oracle on the host
def _oracle_job(args):
    """Run the float64 oracle on a stream subset for the first n positions (test infra)."""
    name, seed, streams, n = args
    import oracle
    w = synth.WORKLOADS[name]
    lam = synth.decay_rates(w, seed)
    chans = sorted({d for (_, d) in streams})
    h = np.empty((w.layers, len(streams), w.length))
    for l in range(w.layers):
        hl = synth.filter_layer(w, seed, l, lam, np.array(chans))
        for j, (_, d) in enumerate(streams):
            hl64 = hl[chans.index(d)].astype(np.float64)
            h[l, j] = oracle.bf16_round(hl64) if w.dtype == "bf16" else hl64
    x0 = synth.first_token(w, seed)
    eps = synth.noise(w, seed, n)
    x0s = np.array([x0[b, d] for (b, d) in streams], dtype=np.float64)
    epss = np.stack([eps[:, b, d] for (b, d) in streams], axis=1)
    t0 = time.perf_counter()
    oracle.online_lcsm(h, x0s, epss, 0.1, w.dtype == "bf16", n=n)
    return time.perf_counter() - t0


def oracle_baseline(w: synth.Workload, seed: int, n_pos: int, streams_per_core: int, cores: int | None = None):
    """Time the oracle on `cores` processes x streams_per_core streams over two prefixes
    (n_pos/4 and n_pos positions), fit time = a*n + b*n^2 (per-position overhead plus the
    O(n^2) sums), and extrapolate to all L positions and all streams (streams are
    independent, so the work scales with their number)."""
    cores = cores or os.cpu_count() or 1
    rng = np.random.default_rng(seed + 17)
    streams = [[(int(rng.integers(w.batch)), int(rng.integers(w.channels))) for _ in range(streams_per_core)]
               for _ in range(cores)]
    ctx = mp.get_context("spawn")
    n2 = min(n_pos, w.length)
    n1 = max(n2 // 4, 1)
    times = []
    t0 = time.perf_counter()
    with ctx.Pool(cores) as pool:
        for n in (n1, n2):
            times.append(max(pool.map(_oracle_job, [(w.name, seed, st, n) for st in streams])))
    wall = time.perf_counter() - t0
    A = np.array([[n1, n1 * n1], [n2, n2 * n2]], dtype=np.float64)
    a_, b_ = np.linalg.solve(A, np.array(times))
    if a_ < 0 or b_ < 0:                       # noisy fit: fall back to the pure n^2 law
        a_, b_ = 0.0, times[1] / (n2 * n2)
    sample_streams = cores * streams_per_core
    t_full = (a_ * w.length + b_ * w.length ** 2) * w.streams / sample_streams
    return {
        "value": w.batch * w.length / t_full,
        "unit": UNIT,
        "cores": cores,
        "kind": "oracle",
        "sample": (f"float64 oracle, all {w.layers} layers, {sample_streams} (sequence, channel) streams x first "
                   f"{n1} and {n2} positions ({cores} spawned processes, {times[0]:.1f} + {times[1]:.1f} s compute, "
                   f"{wall:.1f} s wall); time fitted as a*n + b*n^2 and extrapolated to {w.streams} streams x "
                   f"{w.length} positions"),
        "extrapolated": True,
        "seconds_sample": float(sum(times)),
        "fit": {"a_s_per_position": float(a_), "b_s_per_position2": float(b_)},
    }


# ----------------------------------------------------------------------------- GPU arm
def source_sha(paths):
    h = hashlib.sha256()
    for p in paths:
        with open(os.path.join(ROOT, p), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


KERNEL_SOURCES = {
    "chunk": ["long_convolution_sequence_online_b200/csrc/k_chunk.cu"],
    "fft": ["long_convolution_sequence_online_b200/csrc/k_fft.cu", "long_convolution_sequence_online_b200/csrc/fft.cuh"],
    "direct": ["long_convolution_sequence_online_b200/csrc/k_basic.cu"],
    "tc": ["long_convolution_sequence_online_b200/csrc/k_tile_tc.cu"],
}


def ncu_traffic(cls: str, workload: str):
    """Per-launch DRAM bytes of a kernel class from the committed ncu summary, if still current."""
    path = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f)
        e = rec[cls]
        if e.get("source_sha") != source_sha(KERNEL_SOURCES[cls]) or e.get("workload") != workload:
            return None
        return float(e["dram_bytes_per_launch"])
    except Exception:
        return None


def gpu_arm(args, world, rank, local):
    import torch
    from long_convolution_sequence_online_b200 import fi

    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    w = synth.WORKLOADS[args.workload]
    seed = rank_seed(args.seed, rank)
    h = synth.filters(w, seed)
    x0 = synth.first_token(w, seed)
    eps = synth.noise(w, seed)
    td = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    h_d = torch.from_numpy(h).to(device).to(td)
    x0_d = torch.from_numpy(x0).to(device).to(td).contiguous()
    eps_d = torch.from_numpy(eps).to(device)
    y_d = torch.empty((w.length, w.batch, w.channels), dtype=torch.float32, device=device)
    stream = torch.cuda.current_stream(device)
    t_init = time.perf_counter()
    ctx = fi.Context(h_d, w.batch, w.dtype, chunk=args.chunk, fft_from=args.fft_from, stream=stream,
                     tc_max=args.tc_max)
    t_init = time.perf_counter() - t_init
    del h_d
    chunk, fft_from, tc_max = ctx.plan()
    mlp_hidden = 0
    if args.block == "mlp":
        # channel-mixing block after every layer: random weights of the stated shape
        mlp_hidden = args.hidden or w.channels
        r = np.random.default_rng(seed + 7)
        ws = [r.standard_normal((w.layers, mlp_hidden, w.channels)) * (0.3 / np.sqrt(w.channels)),
              0.1 * r.standard_normal((w.layers, mlp_hidden)),
              r.standard_normal((w.layers, w.channels, mlp_hidden)) * (0.3 / np.sqrt(mlp_hidden)),
              0.1 * r.standard_normal((w.layers, w.channels))]
        ctx.set_mlp_block(*(torch.from_numpy(a.astype(np.float32)).to(device) for a in ws))
        del ws

    step_api = args.api == "step"
    if step_api:
        # one fi_step call per position on given tokens (the noise stands in for them),
        # each position's output written to its row of y
        tok_d = eps_d.to(td).contiguous()
        row_x = tok_d[0].numel() * tok_d.element_size()
        row_y = w.batch * w.channels * 4
        x_base, y_base = tok_d.data_ptr(), y_d.data_ptr()

    def step():
        ctx.reset()
        if step_api:
            for t in range(w.length):
                ctx.step_ptr(x_base + t * row_x, y_base + t * row_y)
        else:
            ctx.generate(w.length, x0_d, eps_d, y_d, 0.1)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(device)

    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    with ClockSampler(local) as clocks:
        barrier(device)
        torch.cuda.synchronize(device)
        for k in range(args.steps):
            ev[k][0].record(stream)
            step()
            ev[k][1].record(stream)
        torch.cuda.synchronize(device)
        barrier(device)
    # Per-kernel times: the same number of steps again with CUDA events around
    # every launch (the events themselves cost about 5 % of a step, so they stay
    # out of the region `value` is timed on).
    ctx.profile(True)
    ctx.profile_read()
    for _ in range(args.steps):
        step()
    prof, sides = ctx.profile_read_sides()
    ctx.profile(False)
    step_ms = [a.elapsed_time(b) for a, b in ev]
    total_ms = reduce_max(float(sum(step_ms)), device)
    ms_per_step = total_ms / args.steps
    tokens_per_step = w.batch * w.length
    value = world * tokens_per_step * args.steps / (total_ms / 1e3)

    # --- end to end: host buffers through the C-ABI call, copies inside the timed region
    x0_h = torch.from_numpy(x0.astype(np.float32) if w.dtype == "f32" else x0).to(td).pin_memory()
    eps_h = torch.from_numpy(eps).pin_memory()
    y_h = torch.empty((w.length, w.batch, w.channels), dtype=torch.float32).pin_memory()

    def e2e_step():
        ctx.reset()
        ctx.generate_host_ptr(w.length, x0_h.data_ptr(), eps_h.data_ptr(), y_h.data_ptr(), 0.1)

    e2e = None
    if args.e2e_steps > 0 and not step_api:
        e2e_step()
        barrier(device)
        t0 = time.perf_counter()
        for _ in range(args.e2e_steps):
            e2e_step()
        e2e_s = reduce_max(time.perf_counter() - t0, device)
        # the host-link share: the same copies alone, from and to the same pinned buffers
        eps_tmp = torch.empty_like(eps_d)
        c0, c1, c2 = (torch.cuda.Event(enable_timing=True) for _ in range(3))
        torch.cuda.synchronize(device)
        c0.record(stream)
        eps_tmp.copy_(eps_h, non_blocking=True)
        c1.record(stream)
        y_h.copy_(y_d, non_blocking=True)
        c2.record(stream)
        torch.cuda.synchronize(device)
        h2d_ms, d2h_ms = c0.elapsed_time(c1), c1.elapsed_time(c2)
        del eps_tmp
        h2d_b = int(x0_h.numel() * x0_h.element_size() + eps_h.numel() * 4)
        d2h_b = int(y_h.numel() * 4)
        e2e = {"value": world * tokens_per_step * args.e2e_steps / e2e_s, "unit": UNIT,
               "h2d_bytes_per_step": h2d_b, "d2h_bytes_per_step": d2h_b,
               "ms_per_step": 1e3 * e2e_s / args.e2e_steps,
               "copies_alone_ms": {"h2d": h2d_ms, "d2h": d2h_ms,
                                   "h2d_gbs": h2d_b / h2d_ms / 1e6, "d2h_gbs": d2h_b / d2h_ms / 1e6},
               "timing": "host wall clock around fi_generate_host (synchronous), max over ranks"}

    # --- roofline: dominant kernel class during the timed steps
    peaks = measured_peaks()
    clk = clocks.summary()
    # fi_step and the channel-mixing block run position by position: no on-chip
    # chunk; the per-position launches take the red cells and the narrowest blocks
    # ("token", per_position_model), wider blocks their own launches
    per_pos = step_api or mlp_hidden > 0
    if per_pos:
        model, tot = per_position_model(w, fft_from, tc_max, mlp_hidden)
    else:
        model, tot = cost_model(w, chunk, fft_from, tc_max=tc_max)
        model["token"] = {"bytes": 0.0, "flops": 0.0}
    classes = {}
    for cls in ("chunk", "direct", "fft", "tc", "token"):
        n, ms = prof[cls]
        if n == 0:
            continue
        secs = ms / 1e3
        byt = model[cls]["bytes"] * args.steps
        flo = model[cls]["flops"] * args.steps
        classes[cls] = {"launches": n, "ms": ms, "avg_launch_us": 1e3 * ms / n, "bytes": byt, "flops": flo,
                        "gbs": byt / secs / 1e9, "tflops": flo / secs / 1e12}
    dom = max(classes, key=lambda k: classes[k]["ms"])
    d = classes[dom]
    mhz = peaks["sm_max_mhz"]
    fp32_peak = fp32_peak_tflops(mhz)
    t_mem = d["bytes"] / (peaks["hbm_gbs"] * 1e9)
    t_alu = d["flops"] / (fp32_peak * 1e12)
    per_launch_bytes = d["bytes"] / d["launches"]
    traffic = ncu_traffic(dom, w.name)
    if t_mem >= t_alu:
        roof = {"bound": "hbm", "achieved": d["gbs"], "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": d["gbs"] / peaks["hbm_gbs"]}
    else:
        roof = {"bound": "alu", "achieved": d["tflops"], "peak": fp32_peak, "unit": "TFLOP/s",
                "frac": d["tflops"] / fp32_peak}
    roof.update({"traffic": traffic, "kernel": dom, "peak_source": peaks["source"],
                 "algorithmic_bytes_per_launch": per_launch_bytes, "avg_launch_us": d["avg_launch_us"],
                 "launches": d["launches"]})
    # whole-run roofline of the schedule (bytes at HBM bandwidth vs flops at the FP32 peak)
    run_s = ms_per_step / 1e3
    t_roof_meas = max(tot["bytes"] / (peaks["hbm_gbs"] * 1e9), tot["flops"] / (fp32_peak * 1e12))
    t_roof_nom = max(tot["bytes"] / (NOMINAL_HBM_GBS * 1e9), tot["flops"] / (fp32_peak * 1e12))
    # stricter bound: blocks below the chunk side never leave the chip, so only the
    # other blocks and the per-position rows must cross HBM
    onchip_bytes = tot["bytes"] - model["chunk"].get("block_bytes", 0.0)
    t_onchip = max(onchip_bytes / (peaks["hbm_gbs"] * 1e9), tot["flops"] / (fp32_peak * 1e12))
    step_roof = {"algorithmic_bytes": tot["bytes"], "algorithmic_flops": tot["flops"],
                 "roofline_ms_measured_hbm": 1e3 * t_roof_meas, "frac_of_measured": t_roof_meas / run_s,
                 "roofline_ms_8tbs": 1e3 * t_roof_nom, "frac_of_8tbs": t_roof_nom / run_s,
                 "achieved_gbs": tot["bytes"] / run_s / 1e9, "fp32_peak_tflops": fp32_peak,
                 "onchip_small_blocks_bytes": onchip_bytes,
                 "roofline_ms_onchip_small_blocks": 1e3 * t_onchip, "frac_onchip_small_blocks": t_onchip / run_s}

    # --- quadratic Lazy baseline on the GPU: measured on two prefixes, extrapolated a*n + b*n^2/2
    # (it runs the elementwise block only)
    lazy = None
    if args.lazy_prefix > 0 and rank == 0 and not step_api and not mlp_hidden:
        n2 = min(args.lazy_prefix, w.length)
        n1 = n2 // 4
        times = []
        for n in (n1, n2):
            ctx.reset()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            ctx.generate_lazy(n, x0_d, eps_d, y_d, 0.1)
            e1.record(stream)
            torch.cuda.synchronize(device)
            times.append(e0.elapsed_time(e1) / 1e3)
        A = np.array([[n1, n1 * n1 / 2], [n2, n2 * n2 / 2]])
        a_, b_ = np.linalg.solve(A, np.array(times))
        Lf = w.length
        t_lazy = a_ * Lf + b_ * Lf * Lf / 2
        lazy = {"seconds_extrapolated": t_lazy, "measured_prefixes": [n1, n2], "measured_s": times,
                "speedup": t_lazy / run_s, "tokens_s": tokens_per_step / t_lazy,
                "lazy_bytes": lazy_bytes(w), "achieved_gbs": lazy_bytes(w) / t_lazy / 1e9}
        ctx.reset()
    ctx.close()

    launches_per_step = sum(prof[k][0] for k in prof) / args.steps
    res = {
        "metric": metric_name(w, args.api, args.block), "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32" if w.dtype == "f32" else "bf16", "data": "synthetic",
        "config": {"workload": w.name, "layers": w.layers, "channels": w.channels, "seq_len": w.length,
                   "batch": w.batch, "global_batch": w.batch * world, "tokens_per_step": tokens_per_step,
                   "parallelism": f"dp{world}" if world > 1 else "single",
                   "plan": {"chunk": chunk, "fft_from": fft_from, "fft_max": 1 << 14, "tc_max": tc_max},
                   "l2": (f"inputs larger than L2 (state {4 * (w.layers + 1) * w.streams * w.length / 1e9:.1f} GB "
                          "streamed every step)") if 4 * (w.layers + 1) * w.streams * w.length > L2_BYTES
                         else "state fits in L2 (latency-bound workload)",
                   "step": ("fi_reset + one fi_step per position over all L given tokens (host loop)" if step_api
                            else "fi_reset + fi_generate over all L positions, closed loop"),
                   "api": args.api,
                   "block": (f"MLP + GELU, hidden {mlp_hidden}, random weights" if mlp_hidden else "tanh"),
                   "init_s": t_init},
        "roofline": roof,
        "step_roofline": step_roof,
        "kernels": classes,
        "block_sides_ms_per_step": {str(k): ms / args.steps for k, (n, ms) in sorted(sides.items())},
        "kernels_timing": "CUDA events around every launch, on as many further steps as timed (same stream)",
        "e2e": e2e,
        "gpu_launches": int(round(launches_per_step * args.steps)),
        "clocks": clk,
        "speedup_vs_lazy": lazy,
        "step_ms": step_ms,
    }
    return res


# ----------------------------------------------------------------------------- main
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--workload", default=synth.HEADLINE, choices=sorted(synth.WORKLOADS))
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--chunk", type=int, default=0)
    ap.add_argument("--fft-from", dest="fft_from", type=int, default=0)
    ap.add_argument("--tc-max", dest="tc_max", type=int, default=0,
                    help="largest block side on the tensor cores (0 = automatic, -1 = none)")
    ap.add_argument("--api", default="generate", choices=["generate", "step"],
                    help="generate: closed-loop fi_generate per step; step: one fi_step call per position")
    ap.add_argument("--block", default="tanh", choices=["tanh", "mlp"],
                    help="block after every layer: elementwise tanh, or the channel-mixing MLP + GELU")
    ap.add_argument("--hidden", type=int, default=0, help="MLP hidden width (0 = channels)")
    ap.add_argument("--e2e-steps", dest="e2e_steps", type=int, default=3)
    ap.add_argument("--lazy-prefix", dest="lazy_prefix", type=int, default=4096)
    ap.add_argument("--oracle-positions", dest="oracle_positions", type=int, default=6144)
    ap.add_argument("--oracle-streams", dest="oracle_streams", type=int, default=4)
    ap.add_argument("--no-cpu-baseline", dest="cpu_baseline", action="store_false")
    args = ap.parse_args()

    world, rank, local = dist_env()
    w = synth.WORKLOADS[args.workload]

    if args.impl == "reference":
        # The reference arm is the float64 oracle on the host cores (rank 0 only).
        if rank != 0:
            return
        per = []
        for k in range(args.warmup + args.steps):
            # the same sample as the native arm's cpu_baseline (about 8 s per step on 16 cores)
            r = oracle_baseline(w, args.seed + k, args.oracle_positions, args.oracle_streams)
            if k >= args.warmup:
                per.append(r)
        value = float(np.mean([r["value"] for r in per]))
        t_step = w.batch * w.length / value
        cpu = {k: per[-1][k] for k in ("unit", "cores", "kind", "sample")}
        cpu["value"] = value
        print(json.dumps({
            "metric": metric_name(w, args.api), "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": 1e3 * t_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
            "config": {"workload": w.name, "layers": w.layers, "channels": w.channels, "seq_len": w.length,
                       "batch": w.batch, "step": "one bounded oracle sample per step, extrapolated"},
            "cpu_baseline": cpu,
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        }))
        return

    dist_on = dist_init(world, "nccl")
    try:
        res = gpu_arm(args, world, rank, local)
    finally:
        if dist_on:
            import torch.distributed as dist
            dist.destroy_process_group()
    if rank == 0:
        if args.cpu_baseline and world == 1 and args.block == "tanh":
            res["cpu_baseline"] = oracle_baseline(w, args.seed, args.oracle_positions, args.oracle_streams)
        else:
            res["cpu_baseline"] = None
        print(json.dumps(res))


if __name__ == "__main__":
    main()
