"""Benchmark of the int8-state LeapQuant GDN/KDA decode step on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload kimi_linear_kda|qwen35_9b_gdn|gdn_sweep_bB|ragged_gdn]
                    [--layers L] [--no-others]

One step = one 16-token quantization window (15 plain decode tokens and the
boundary token whose kernel also folds, compensates, smooths and requantizes)
for every (sequence, value head) tile of L independent layer states, cycled
token by token as a model's layers are.  The L states keep the working set far
above the 126 MB L2, so every step streams its state from HBM.

value = tile-steps/s (one tile-step = one decode token of one value head of
one layer) with all inputs resident in HBM, timed with CUDA events around a
CUDA-graph replay of K steps.  The default workload is the Kimi-Linear-like
KDA layer (128 sequences x 32 heads = 4,096 tiles, the batch x heads >= 4096
regime); the line also carries, as sub-objects with their own fp32-state
comparison and roofline, the Qwen3.5-9B-like GDN layer (2,048 tiles), the
largest bandwidth-sweep point (32,768 tiles) and a ragged batch whose
sequences sit in different window phases (8,192 tiles, about 1/16 of them
folding at every token).  The same line carries: the in-house fp32-state
kernel on the same workload and its speedup ratio, the roofline of the decode
kernel against the measured HBM copy bandwidth, end-to-end throughput through
the host-buffer C entry point, the CPU oracle timed on a sample, and the SM
clocks sampled during the timed region.

Multi-GPU (torchrun): every rank runs its own batch of sequences (weak
scaling, no collective on the data path); time is the max over ranks.
--impl reference times the CPU oracle (the reference arm) on host cores.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import re
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from recurrent_state_quantization_decode_b200 import workloads as wl  # noqa: E402

METRIC = ("decode tokens/s·head (int8 state) & achieved HBM GB/s vs 8 TB/s; "
          "speedup vs fp32 state")
UNIT = "tile-steps/s"
NOMINAL_HBM_GBS = 8000.0
WORKLOADS = {"qwen35_9b_gdn": wl.QWEN35_9B_GDN, "kimi_linear_kda": wl.KIMI_LINEAR_KDA,
             "ragged_gdn": wl.RAGGED,
             **{f"gdn_sweep_b{b}": wl.sweep_workload(b) for b in wl.SWEEP_BATCHES}}
DEFAULT_WORKLOAD = "kimi_linear_kda"
# the other workloads the default line reports as sub-objects, with the layer
# count each cycles (enough to keep the working set above L2)
OTHER_WORKLOADS = (("qwen35_9b_gdn", 8), ("ragged_gdn", 4))


def sweep_layers(w: wl.Workload) -> int:
    """Layers cycled at a sweep point: enough for a working set of four times
    the L2 where 16 layers suffice, else 16 (the line then says it is partly
    L2-resident)."""
    per_layer = working_set_bytes(w, 1)
    return int(min(16, max(2, math.ceil(4 * L2_BYTES / per_layer))))


def sweep_steps(w: wl.Workload) -> int:
    """Timed steps at a sweep point: fewer for larger batches, so that every
    point takes a similar time."""
    return int(min(200, max(10, round(200 * 2048 / w.tiles))))
PROFILE_DIR = os.path.join(ROOT, "profiles")
KERNEL_SOURCES = [os.path.join(ROOT, "recurrent_state_quantization_decode_b200", "csrc", f)
                  for f in ("lq_decode.cu", "lq_internal.h")]


# ---------------------------------------------------------------------------
# Algorithmic bytes (what the method must move, not what a kernel happens to)
# ---------------------------------------------------------------------------

def algorithmic_bytes_per_tile_step(w: wl.Workload, out_bytes: int = 4) -> dict:
    """Average bytes one tile-step must move over a full window (token slots
    n = 0..W-1).  Keys are shared by the Hv/Hk value heads of a key head, so
    their bytes are divided among them."""
    d, W, K = w.d, w.window, w.n_comp
    inb = 2 if w.io_bf16 else 4
    g = w.num_v_heads // w.num_k_heads
    ga = d if w.gate == wl.GATE_DIAG else 1
    record = d * d + 8 * d + 4 * K * d + 4 * K
    record = (record + 15) // 16 * 16
    entry = 4 * d + 4 * ga + inb * d / g          # d_i, alpha_i, k_i (shared)
    mean_n = (W - 1) / 2.0
    parts = {
        "record_read": record,
        "buffer_read": mean_n * entry,
        "buffer_append": entry,
        "fold_record_write": record / W,
        "inputs": 2 * inb * d / g + inb * d + 4 * ga + 4,   # q, k (shared), v, alpha, beta
        "output": out_bytes * d,
        "phase_counter": 8,
    }
    parts["total"] = sum(parts.values())
    return parts


def fp32_bytes_per_tile_step(w: wl.Workload, out_bytes: int = 4) -> float:
    d = w.d
    inb = 2 if w.io_bf16 else 4
    g = w.num_v_heads // w.num_k_heads
    ga = d if w.gate == wl.GATE_DIAG else 1
    return 2 * 4 * d * d + 2 * inb * d / g + inb * d + 4 * ga + 4 + out_bytes * d


_COMMENTS = re.compile(rb"/\*.*?\*/|//[^\n]*", re.S)


def kernel_source_sha() -> str:
    """Hash of the decode kernel's source with its comments left out and its
    whitespace collapsed, so that a change of wording or layout alone keeps a
    profile summary tied to the kernel that it measured."""
    h = hashlib.sha256()
    for f in KERNEL_SOURCES:
        code = _COMMENTS.sub(b" ", open(f, "rb").read())
        h.update(re.sub(rb"\s+", b" ", code).strip())
    return h.hexdigest()[:16]


def profile_summary_path(key: str) -> str:
    """The committed ncu summary of the decode kernel on workload `key`."""
    return os.path.join(PROFILE_DIR, f"decode_kernel_{key}.md")


def kernel_label(w: wl.Workload) -> str:
    return (f"decode_kernel<{w.d},{'bf16' if w.io_bf16 else 'f32'},"
            f"{'KDA' if w.gate == wl.GATE_DIAG else 'GDN'}> (int8 state)")


def profiled_traffic(tiles: int, key: str = "qwen35_9b_gdn"):
    """DRAM bytes per launch of the decode kernel from the committed ncu summary
    of workload `key`, scaled to `tiles`; None if the summary is missing or the
    kernel source has changed since it was captured."""
    try:
        txt = open(profile_summary_path(key)).read()
    except OSError:
        return None
    sha = re.search(r"kernel_source_sha:\s*([0-9a-f]+)", txt)
    per_tile = re.search(r"dram_bytes_per_tile_step:\s*([0-9.]+)", txt)
    if not sha or not per_tile or sha.group(1) != kernel_source_sha():
        return None
    return float(per_tile.group(1)) * tiles


# ---------------------------------------------------------------------------
# Clocks during the timed region
# ---------------------------------------------------------------------------

class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, uuid: str | None):
        self.uuid = uuid
        self.proc = None
        self.lines: list[str] = []

    def __enter__(self):
        cmd = ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
               "-lms", "100"]
        if self.uuid:
            cmd += ["-i", self.uuid]
        try:
            self.proc = subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL,
                                         text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except OSError:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.time(), line.strip()))

    def window(self, t0: float, t1: float) -> None:
        """Keep only the samples taken between t0 and t1 (time.time())."""
        self.t0, self.t1 = t0, t1

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.thread.join(timeout=2)

    def summary(self) -> dict:
        sm, mx, reasons = [], [], set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        t0, t1 = getattr(self, "t0", 0.0), getattr(self, "t1", float("inf"))
        for ts, ln in self.lines:
            if ts < t0 or ts > t1:
                continue
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 8:
                continue
            try:
                sm.append(float(f[0]))
                mx.append(float(f[1]))
            except ValueError:
                continue
            for n, val in zip(names, f[4:8]):
                if val.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx),
                "reasons": sorted(reasons), "samples": len(sm)}


# ---------------------------------------------------------------------------
# CPU oracle legs
# ---------------------------------------------------------------------------

def _oracle_inputs(w: wl.Workload, tiles_b: int, T: int, seed: int):
    """Seeded inputs of `tiles_b` sequences (all heads) for T tokens, fp64."""
    rng = np.random.default_rng(seed)
    S0, _, _ = wl.initial_states(rng, tiles_b * w.num_v_heads, w.d, w.d)
    ti = wl.token_inputs(rng, w, T, batch=tiles_b)
    return S0, ti


def run_oracle_sample(w: wl.Workload, seqs: int, windows: int = 1,
                      seed: int = 1234) -> tuple[float, int, int]:
    """Time the oracle on `seqs` sequences x all heads for `windows` consecutive
    W-token windows (each incl. its fold), the state carried from one window to
    the next.  Only the oracle's decode calls are timed: the records are built
    and each window's inputs drawn outside the timed region.  Returns
    (seconds, tile_steps, threads)."""
    import oracle

    cfg = oracle.Cfg(w.d, w.d, W=w.window, K=w.n_comp, gate=w.gate, quant=1, smooth=w.smooth)
    T = w.window
    S0, _ = _oracle_inputs(w, seqs, 1, seed)
    tiles = seqs * w.num_v_heads
    recs = [oracle.quantize(cfg, S0[t].astype(np.float64)) for t in range(tiles)]
    rec = {"Q": np.stack([r.Q for r in recs]), "sig": np.stack([r.sig for r in recs]),
           "m": np.stack([r.m for r in recs]), "cv": np.stack([r.cv for r in recs]),
           "cid": np.stack([r.cid for r in recs])}
    ga = w.d if w.gate == wl.GATE_DIAG else 1
    buf = {"n": np.zeros(tiles, np.int32), "bk": np.zeros((tiles, w.window, w.d)),
           "bd": np.zeros((tiles, w.window, w.d)), "ba": np.zeros((tiles, w.window, ga))}
    threads = len(os.sched_getaffinity(0))
    dt, used = 0.0, threads
    for win in range(windows):
        ti = wl.token_inputs(np.random.default_rng(seed + 7919 * (win + 1)), w, T, batch=seqs)
        inp = {n: np.ascontiguousarray(getattr(ti, n), dtype=np.float64)
               for n in ("q", "k", "v", "alpha", "beta")}
        inp["o"] = np.zeros((T, seqs, w.num_v_heads, w.d))
        t0 = time.perf_counter()
        used = oracle.batch_run(cfg, seqs, w.num_k_heads, w.num_v_heads, T, rec, buf, inp,
                                nthreads=threads)
        dt += time.perf_counter() - t0
    return dt, tiles * T * windows, used


def oracle_sample_size(w: wl.Workload, target_s: float) -> tuple[int, int]:
    """(sequences, windows) for about `target_s` seconds of oracle work: first
    more sequences (up to the batch), then more windows."""
    dt1, _, _ = run_oracle_sample(w, 1)
    per_seq = max(dt1, 1e-4)
    seqs = int(max(1, min(w.batch, math.floor(target_s / per_seq))))
    if seqs < w.batch:
        return seqs, 1
    dtb, _, _ = run_oracle_sample(w, seqs)
    return seqs, int(max(1, math.floor(target_s / max(dtb, 1e-4))))


def cpu_baseline(w: wl.Workload, target_s: float = 15.0) -> dict:
    seqs, windows = oracle_sample_size(w, target_s)
    dt, ts, used = run_oracle_sample(w, seqs, windows)
    return {"value": ts / dt, "unit": UNIT, "cores": used, "kind": "oracle",
            "sample": (f"{seqs} of {w.batch} sequences x {w.num_v_heads} heads, {windows} "
                       f"consecutive {w.window}-token windows incl. their folds, one layer; "
                       f"fp64 C oracle, OpenMP over tiles; {dt:.1f} s of oracle time")}


REFERENCE_BUDGET_S = 150.0  # oracle seconds of the whole --impl reference run


def reference_arm(args, w: wl.Workload, rank: int, world: int) -> None:
    if rank != 0:
        return
    steps, warm = args.steps, args.warmup
    budget = REFERENCE_BUDGET_S
    seqs, windows = oracle_sample_size(w, budget / (steps + warm))
    for _ in range(warm):
        run_oracle_sample(w, seqs, windows)
    tot_t, tot_ts, used = 0.0, 0, 1
    for s in range(steps):
        dt, ts, used = run_oracle_sample(w, seqs, windows, seed=1234 + s)
        tot_t += dt
        tot_ts += ts
    value = tot_ts / tot_t
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": steps, "warmup": warm, "ms_per_step": 1e3 * tot_t / steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": workload_config(w, args.layers),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": used, "kind": "oracle",
                         "sample": (f"per step: {seqs} sequences x {w.num_v_heads} heads, "
                                    f"{windows} {w.window}-token window(s) incl. the fold")},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


L2_BYTES = 126 * 2**20  # B200 L2


def working_set_bytes(w: wl.Workload, layers: int) -> int:
    """Device bytes one timed int8 step touches: every layer's records, window
    buffers and counters, the W tokens of inputs it decodes and its output."""
    d, W, tiles = w.d, w.window, w.tiles
    inb = 2 if w.io_bf16 else 4
    ga = d if w.gate == wl.GATE_DIAG else 1
    record = (d * d + 8 * d + 4 * w.n_comp * d + 4 * w.n_comp + 15) // 16 * 16
    state = (tiles * record + w.batch * w.num_k_heads * W * d * inb + tiles * W * d * 4
             + tiles * (W * d * 4 if ga > 1 else 16 * 4) + tiles * 4)
    inputs = W * (2 * w.batch * w.num_k_heads * d * inb + tiles * d * inb
                  + tiles * ga * 4 + tiles * 4)
    return layers * (state + inputs + tiles * d * 4)


def l2_statement(ws: int) -> str:
    mb, l2 = ws / 2**20, L2_BYTES / 2**20
    if ws < L2_BYTES:
        return (f"working set {mb:.0f} MB fits in the {l2:.0f} MB L2: L2-resident, "
                "not an HBM figure")
    if ws < 2 * L2_BYTES:
        return f"working set {mb:.0f} MB, under twice the {l2:.0f} MB L2: partly L2-resident"
    return (f"inputs larger than L2: working set {mb:.0f} MB = {ws / L2_BYTES:.1f}x the "
            f"{l2:.0f} MB L2 (layer states cycled every token)")


def workload_config(w: wl.Workload, layers: int) -> dict:
    ws = working_set_bytes(w, layers)
    return {"workload": w.name, "batch": w.batch, "num_k_heads": w.num_k_heads,
            "num_v_heads": w.num_v_heads, "d_k": w.d, "d_v": w.d,
            "gate": "scalar (GDN)" if w.gate == wl.GATE_SCALAR else "diagonal (KDA)",
            "io": "bf16 q/k/v, fp32 o" if w.io_bf16 else "fp32", "window": w.window,
            "compensators": w.n_comp, "smooth": w.smooth, "layers_cycled": layers,
            "tiles_per_layer": w.tiles,
            "step": f"one {w.window}-token window x {layers} layers",
            "working_set_mb": round(ws / 2**20, 1),
            "l2": l2_statement(ws)}


# ---------------------------------------------------------------------------
# GPU arm
# ---------------------------------------------------------------------------

STATE_POOL = 512  # distinct initial states drawn per layer; larger batches repeat them


class Layer:
    """One layer's stored state, fp32 comparison state and W tokens of inputs.
    With `phases`, sequence b first decodes phases[b] tokens (active masks), so
    that the layer's tiles sit in different window phases."""

    def __init__(self, B, w: wl.Workload, seed: int, device, phases=None):
        import torch

        rng = np.random.default_rng(seed)
        pool = min(w.tiles, STATE_POOL)
        S0, _, _ = wl.initial_states(rng, pool, w.d, w.d)
        ti = wl.token_inputs(rng, w, w.window)
        dt = torch.bfloat16 if w.io_bf16 else torch.float32
        self.cfg = B.config_for(w)
        self.ds = B.DeviceState(self.cfg, device=device)
        S0_dev = torch.from_numpy(S0).to(device)
        if pool < w.tiles:
            S0_dev = S0_dev[torch.arange(w.tiles, device=device) % pool].contiguous()
        B.lq_state_init(self.cfg, S0_dev, self.ds.st)
        self.S32 = S0_dev  # the fp32-state path starts from the same states
        self.q = torch.from_numpy(ti.q).to(device=device, dtype=dt)
        self.k = torch.from_numpy(ti.k).to(device=device, dtype=dt)
        self.v = torch.from_numpy(ti.v).to(device=device, dtype=dt)
        self.alpha = torch.from_numpy(ti.alpha).to(device)
        self.beta = torch.from_numpy(ti.beta).to(device)
        self.out = torch.empty((w.batch, w.num_v_heads, w.d), dtype=torch.float32, device=device)
        # Each token's inputs are also kept in lq_decode_step_packed's per-tile
        # blocks, which the int8 step reads: one copy per tile instead of three
        # or four.  With grouped heads (Hv > Hk) the blocks repeat q and k per
        # value head, more bytes than the shared arrays, and still faster.
        self.packed = [B.pack_tile_inputs(self.cfg, self.q[t], self.k[t], self.v[t],
                                          self.alpha[t]) for t in range(w.window)]
        self.host = None
        if phases is not None:
            ph = torch.as_tensor(phases, dtype=torch.int32, device=device)
            for t in range(int(ph.max().item())):
                act = (ph > t).to(torch.int32)
                B.lq_decode_step(self.cfg, self.q[t], self.k[t], self.v[t], self.alpha[t],
                                 self.beta[t], self.ds.st, self.out, active=act)
            torch.cuda.synchronize(device)

    def pin_host_inputs(self):
        """Pinned host copies of the W tokens' inputs: per token, q, k, v,
        alpha and beta back to back in one block, which lq_decode_step_host
        moves with one copy."""
        import torch

        names = ("q", "k", "v", "alpha", "beta")
        W = self.q.shape[0]
        sizes = [getattr(self, n)[0].numel() * getattr(self, n)[0].element_size() for n in names]
        block = torch.empty((W, sum(sizes)), dtype=torch.uint8).pin_memory()
        self.host = {n: [] for n in names}
        for t in range(W):
            off = 0
            for n, sz in zip(names, sizes):
                x = getattr(self, n)[t].cpu()
                view = block[t, off:off + sz].view(x.dtype).view(x.shape)
                view.copy_(x)
                self.host[n].append(view)
                off += sz
        self.host_out = torch.empty(self.out.shape, dtype=torch.float32).pin_memory()
        self.staging = torch.empty(self.ds.layout.host_staging_bytes, dtype=torch.uint8,
                                   device=self.out.device)


def ragged_phases(w: wl.Workload, seed: int) -> np.ndarray:
    """Per-sequence window phases of the ragged workload (its recipe's phase
    offsets): sequence b has decoded phase[b] tokens of its current window."""
    _, phase = wl.ragged_lengths(np.random.default_rng(seed), w.batch)
    return phase


# ---------------------------------------------------------------------------
# Ranks: one process per GPU, each on its own sequences (weak scaling)
# ---------------------------------------------------------------------------

def layer_seed(rank: int, layer: int) -> int:
    """Seed of one rank's layer: every rank decodes its own sequences, so the
    ranks share no data and the path needs no collective."""
    return 1000 * rank + layer


def max_over_ranks(x: float, world: int, device="cpu") -> float:
    """Largest `x` over all ranks (the job takes as long as its slowest rank)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist

    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(units_per_step: int, world: int, steps: int, ms_max: float) -> float:
    """Units all ranks processed per second, over the slowest rank's time."""
    return world * units_per_step * steps / (ms_max / 1e3)


PREFILL_TOKENS = 256
PREFILL_CHUNK = 16  # tokens per chunk of the WY-form prefill
FP32_ALU_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12  # SMs x fp32 lanes x 2 flops x max clock
TF32_PER_BF16 = 1.1 / 2.25  # nominal dense tf32 / bf16 tensor rates


def prefill_tensor_flops_per_token(d: int) -> float:
    """Tensor-path flops of the chunked prefill per tile-token: S0 Kg^T and
    S0 Qg^T (2 x 2 C d^2 per chunk of C tokens) and the rank-C state update
    (2 C d^2), each run as three tf32 products (hi/lo split): 18 d^2."""
    return 3.0 * (4.0 + 2.0) * d * d


def prefill_measure(B, w: wl.Workload, ly, stream, device, world: int) -> dict:
    """lq_prefill of one layer's tiles over a PREFILL_TOKENS-token prompt
    (seeded inputs), CUDA-event timed after one warm-up run.  The roofline
    counts the tensor-path products of the chunked form against the tf32
    peak (the measured bf16 peak times the nominal tf32/bf16 ratio); the exact
    recurrence's 7 d^2 flops per tile-token are given as context."""
    import torch

    T = PREFILL_TOKENS
    ti = wl.token_inputs(np.random.default_rng(4242), w, T)
    dt = torch.bfloat16 if w.io_bf16 else torch.float32
    dev = {n: torch.from_numpy(getattr(ti, n)).to(device) for n in ("alpha", "beta")}
    for n in ("q", "k", "v"):
        dev[n] = torch.from_numpy(getattr(ti, n)).to(device=device, dtype=dt)
    out = torch.empty((T, w.batch, w.num_v_heads, w.d), dtype=torch.float32, device=device)
    ds = B.DeviceState(ly.cfg, device=device)
    runs = 3

    def run():
        B.lq_prefill(ly.cfg, dev["q"], dev["k"], dev["v"], dev["alpha"], dev["beta"], T,
                     ly.S32, ds.st, out, stream=stream.cuda_stream)

    with torch.cuda.stream(stream):
        run()
        torch.cuda.synchronize()
        start = torch.cuda.Event(enable_timing=True)
        end = torch.cuda.Event(enable_timing=True)
        start.record(stream)
        for _ in range(runs):
            run()
        end.record(stream)
    torch.cuda.synchronize()
    ms = max_over_ranks(start.elapsed_time(end) / runs, world, device)
    tile_tokens = w.tiles * T
    sec = ms / 1e3
    exact = 7.0 * w.d * w.d * tile_tokens / sec / 1e12
    tensor = prefill_tensor_flops_per_token(w.d) * tile_tokens / sec / 1e12
    try:
        bf16 = float(json.load(open(os.path.join(ROOT, "MEASURED_PEAKS.json")))["bf16_tflops"])
        src = "measured bf16 x nominal tf32/bf16 ratio (1.1 / 2.25)"
    except (OSError, ValueError, KeyError):
        bf16, src = 1590.0, "fallback bf16 x nominal tf32/bf16 ratio (1.1 / 2.25)"
    peak = bf16 * TF32_PER_BF16
    return {"tile_tokens_per_s": world * tile_tokens / sec, "ms": ms,
            "prompt_tokens": T, "tiles": w.tiles, "chunk_tokens": PREFILL_CHUNK,
            "roofline": {"bound": "tensor", "achieved": tensor, "peak": peak,
                         "unit": "TFLOP/s", "frac": tensor / peak, "peak_source": src,
                         "flops": "18 d^2 per tile-token: S0 Kg^T, S0 Qg^T and the rank-16 "
                                  "update, three tf32 products each"},
            "exact_recurrence": {"tflops": exact, "fp32_alu_peak": FP32_ALU_TFLOPS,
                                 "frac_of_fp32_alu": exact / FP32_ALU_TFLOPS,
                                 "flops": "7 d^2 per tile-token"},
            "kernel": "chunk_prefill_kernel (WY form in 16-token chunks, then quantizer)"}


def load_peaks() -> tuple[float, str]:
    try:
        peaks = json.load(open(os.path.join(ROOT, "MEASURED_PEAKS.json")))
    except (OSError, ValueError):
        peaks = {}
    if "hbm_gbs" in peaks:
        return float(peaks["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


def measure_decode(B, w: wl.Workload, key: str, L: int, steps: int, warmup: int, stream,
                   device, world: int, rank: int, sample_clocks: bool = False,
                   phases: bool = False, keep_layers: bool = False) -> dict:
    """Time `steps` steps (one W-token window for every tile of L layers) of
    the int8-state decode and steps/4 of the fp32-state kernel, each as a
    CUDA-graph replay after `warmup` replays; return the workload's figures."""
    import torch
    import torch.distributed as dist

    layers = []
    for l in range(L):
        ph = ragged_phases(w, layer_seed(rank, l)) if phases else None
        layers.append(Layer(B, w, seed=layer_seed(rank, l), device=device, phases=ph))
    W = w.window
    launches_per_step = W * L

    def step_int8(s):
        for t in range(W):
            for ly in layers:
                if ly.packed is not None:  # (always; None leaves the separate arrays)
                    kda = ly.cfg.gate == B.LQ_GATE_DIAG
                    B.lq_decode_step_packed(ly.cfg, ly.packed[t], None if kda else ly.alpha[t],
                                            ly.beta[t], ly.ds.st, ly.out, stream=s)
                else:
                    B.lq_decode_step(ly.cfg, ly.q[t], ly.k[t], ly.v[t], ly.alpha[t], ly.beta[t],
                                     ly.ds.st, ly.out, stream=s)

    def step_fp32(s):
        for t in range(W):
            for ly in layers:
                B.lq_fp32_decode_step(ly.cfg, ly.q[t], ly.k[t], ly.v[t], ly.alpha[t],
                                      ly.beta[t], ly.S32, ly.out, stream=s)

    def capture(fn):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.stream(stream):
            fn(stream.cuda_stream)          # one eager pass (also warms up)
            stream.synchronize()
            with torch.cuda.graph(g, stream=stream):
                fn(stream.cuda_stream)
        torch.cuda.synchronize()
        return g

    def barrier():
        if world > 1:
            dist.barrier()

    def timed(graph, n, sample):
        with torch.cuda.stream(stream):
            for _ in range(warmup):
                graph.replay()
        torch.cuda.synchronize()
        barrier()
        torch.cuda.synchronize()
        start = torch.cuda.Event(enable_timing=True)
        end = torch.cuda.Event(enable_timing=True)
        uuid = None
        try:
            uuid = "GPU-" + str(torch.cuda.get_device_properties(device).uuid)
        except Exception:
            pass
        sampler = ClockSampler(uuid if sample else None)
        if sample:
            sampler.__enter__()
            time.sleep(0.3)
        wall0 = time.time()
        with torch.cuda.stream(stream):
            start.record(stream)
            for _ in range(n):
                graph.replay()
            end.record(stream)
        torch.cuda.synchronize()
        wall1 = time.time()
        if sample:
            time.sleep(0.15)
            sampler.__exit__(None, None, None)
            sampler.window(wall0, wall1)
        barrier()
        torch.cuda.synchronize()
        ms = max_over_ranks(start.elapsed_time(end), world, device)
        return ms, (sampler.summary() if sample else None)

    nvtx = torch.cuda.nvtx.range
    with nvtx(f"int8-state decode ({key}): capture, warm-up, timed replay"):
        g8 = capture(step_int8)
        ms8, clocks = timed(g8, steps, sample_clocks)
    err = max(B.lq_get_last_error(ly.ds.st, stream.cuda_stream) for ly in layers)
    if err != B.LQ_OK:
        raise RuntimeError(f"device error word set: {B.lq_status_string(err)}")
    del g8
    steps32 = max(3, steps // 4)
    with nvtx(f"fp32-state decode ({key}): capture, warm-up, timed replay"):
        g32 = capture(step_fp32)
        ms32, _ = timed(g32, steps32, False)
    del g32

    units_per_step = w.tiles * W * L               # per rank
    value = whole_job_rate(units_per_step, world, steps, ms8)
    value32 = whole_job_rate(units_per_step, world, steps32, ms32)
    # roofline of the decode kernel (algorithmic bytes / graph time per launch)
    ab = algorithmic_bytes_per_tile_step(w)
    bytes_per_launch = ab["total"] * w.tiles
    launch_s = (ms8 / 1e3) / (steps * launches_per_step)
    achieved = bytes_per_launch / launch_s / 1e9
    peak, peak_src = load_peaks()
    fp32_bytes = fp32_bytes_per_tile_step(w) * w.tiles
    fp32_achieved = fp32_bytes / ((ms32 / 1e3) / (steps32 * launches_per_step)) / 1e9
    cfg = workload_config(w, L)
    if w.tiles > STATE_POOL:
        cfg["initial_states"] = f"{STATE_POOL} drawn per layer, repeated over the tiles"
    if phases:
        cfg["window_phases"] = ("per sequence, the recipe's offsets U{0..15}: about 1/16 "
                                "of the tiles fold at every token")
    res = {
        "workload": w.name, "value": value, "unit": UNIT, "steps": steps,
        "ms_per_step": ms8 / steps, "config": cfg,
        "gpu_launches": steps * launches_per_step,
        "hbm_gbs": achieved, "hbm_frac_of_8tbs": achieved / NOMINAL_HBM_GBS,
        "bytes_per_value": {"stored": ab["record_read"] / (w.d * w.d),
                            "moved_per_step": ab["total"] / (w.d * w.d)},
        "fp32_state": {"value": value32, "unit": UNIT, "ms_per_step": ms32 / steps32,
                       "hbm_gbs": fp32_achieved, "steps": steps32,
                       "kernel": f"fp32_step_kernel<{w.d}> (fp32 state)"},
        "speedup_vs_fp32_state": value / value32,
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "traffic": profiled_traffic(w.tiles, key),
                     "peak_source": peak_src, "kernel": kernel_label(w),
                     "algorithmic_bytes_per_tile_step": ab["total"],
                     "launch_time": ("graph replay time / launches (includes inter-kernel "
                                     "gaps)")},
    }
    if clocks is not None:
        res["clocks"] = clocks
    if keep_layers:
        res["_layers"] = layers
    return res


def gpu_arm(args, w: wl.Workload, rank: int, world: int, local_rank: int) -> None:
    import torch
    import torch.distributed as dist

    from recurrent_state_quantization_decode_b200 import binding as B

    device = torch.device("cuda", local_rank)
    torch.cuda.set_device(device)
    L = args.layers
    stream = torch.cuda.Stream(device=device)
    nvtx = torch.cuda.nvtx.range
    W = w.window

    def barrier():
        if world > 1:
            dist.barrier()

    main = measure_decode(B, w, args.workload, L, args.steps, args.warmup, stream, device,
                          world, rank, sample_clocks=True,
                          phases=args.workload == "ragged_gdn", keep_layers=True)
    layers = main.pop("_layers")
    units_per_step = w.tiles * W * L               # per rank

    # end to end through the host-buffer entry point (pinned host memory)
    e2e = None
    if not args.no_e2e:
        for ly in layers:
            ly.pin_host_inputs()
        h2d = sum(ly.host[n][0].numel() * ly.host[n][0].element_size()
                  for ly in layers for n in ("q", "k", "v", "alpha", "beta")) * W
        d2h = sum(ly.host_out.numel() * 4 for ly in layers) * W
        e2e_steps = max(2, min(args.steps, 20))

        # Eight streams, layer index mod 8 picks one (fewer when L is not a
        # multiple): each layer stays on its own stream (its tokens in order,
        # its own staging and output buffers), while one layer's input copy
        # and output copy overlap other layers' kernels.
        n_streams = next(n for n in (8, 4, 2, 1) if L % n == 0)
        streams = [stream] + [torch.cuda.Stream(device=device) for _ in range(n_streams - 1)]

        def step_host():
            for t in range(W):
                for li, ly in enumerate(layers):
                    hs = ly.host
                    B.lq_decode_step_host(ly.cfg, hs["q"][t], hs["k"][t], hs["v"][t],
                                          hs["alpha"][t], hs["beta"][t], ly.ds.st,
                                          ly.host_out, ly.staging,
                                          stream=streams[li % len(streams)].cuda_stream)

        for _ in range(2):
            step_host()
        torch.cuda.synchronize()
        barrier()
        start = torch.cuda.Event(enable_timing=True)
        end = torch.cuda.Event(enable_timing=True)
        start.record(stream)
        for st2 in streams[1:]:
            st2.wait_event(start)
        with nvtx("end to end through lq_decode_step_host, timed"):
            for _ in range(e2e_steps):
                step_host()
        for st2 in streams[1:]:
            done = torch.cuda.Event()
            done.record(st2)
            stream.wait_event(done)
        end.record(stream)
        torch.cuda.synchronize()
        barrier()
        ms_e2e = max_over_ranks(start.elapsed_time(end), world, device)
        e2e = {"value": whole_job_rate(units_per_step, world, e2e_steps, ms_e2e), "unit": UNIT,
               "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
               "path": ("lq_decode_step_host: each token's pinned host q, k, v, alpha, "
                        "beta back to back, moved by one cudaMemcpyAsync, o back by "
                        f"cudaMemcpyAsync; {len(streams)} streams by layer index")}

    # prefill of one layer's tiles over a prompt, ending in the quantizer
    prefill = None
    if not args.no_prefill:
        with nvtx("prefill of one layer"):
            prefill = prefill_measure(B, w, layers[0], stream, device, world)
    del layers
    torch.cuda.synchronize()
    torch.cuda.empty_cache()

    # the other workloads, each with its own fp32 comparison and roofline
    others = {}
    if not args.no_others and args.workload == DEFAULT_WORKLOAD:
        sub_steps = max(5, args.steps // 5)
        for key, lay in OTHER_WORKLOADS:
            with nvtx(f"sub-workload {key}"):
                others[key] = measure_decode(B, WORKLOADS[key], key, lay, sub_steps,
                                             args.warmup, stream, device, world, rank,
                                             phases=key == "ragged_gdn")
            torch.cuda.synchronize()
            torch.cuda.empty_cache()
        # the bandwidth sweep: int8 and fp32 states side by side, batch 8 .. 1024
        sweep = []
        for b in wl.SWEEP_BATCHES:
            sw = wl.sweep_workload(b)
            with nvtx(f"sweep point batch {b}"):
                r = measure_decode(B, sw, f"gdn_sweep_b{b}", sweep_layers(sw), sweep_steps(sw),
                                   args.warmup, stream, device, world, rank)
            sweep.append({"batch": b, "tiles": sw.tiles, "int8_state": r["value"],
                          "fp32_state": r["fp32_state"]["value"],
                          "speedup_vs_fp32_state": r["speedup_vs_fp32_state"],
                          "int8_hbm_gbs": r["hbm_gbs"], "fp32_hbm_gbs": r["fp32_state"]["hbm_gbs"],
                          "roofline_frac": r["roofline"]["frac"], "steps": r["steps"],
                          "layers_cycled": r["config"]["layers_cycled"],
                          "l2": r["config"]["l2"]})
            torch.cuda.synchronize()
            torch.cuda.empty_cache()
        others["gdn_bandwidth_sweep"] = {"unit": UNIT, "points": sweep}

    if rank != 0:
        return
    line = {
        "metric": METRIC, "value": main["value"], "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": main["ms_per_step"],
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "state_dtype": "int8", "data": "synthetic", "config": main["config"],
        "gpu_launches": main["gpu_launches"],
        "hbm_gbs": main["hbm_gbs"], "hbm_frac_of_8tbs": main["hbm_frac_of_8tbs"],
        "bytes_per_value": main["bytes_per_value"],
        "fp32_state": main["fp32_state"],
        "speedup_vs_fp32_state": main["speedup_vs_fp32_state"],
        "roofline": main["roofline"],
        "clocks": main.get("clocks"),
    }
    if e2e is not None:
        line["e2e"] = e2e
    if prefill is not None:
        line["prefill"] = prefill
    if others:
        line["other_workloads"] = others
    if world == 1 and not args.no_cpu:
        with nvtx("CPU oracle baseline"):
            line["cpu_baseline"] = cpu_baseline(w)
    print(json.dumps(line), flush=True)


def main() -> None:
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--workload", choices=sorted(WORKLOADS), default=DEFAULT_WORKLOAD)
    ap.add_argument("--layers", type=int, default=8)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--no-prefill", action="store_true")
    ap.add_argument("--no-others", action="store_true",
                    help="skip the other workloads' sub-objects of the default line")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    w = WORKLOADS[args.workload]
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        reference_arm(args, w, rank, world)
        return
    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist

        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    try:
        gpu_arm(args, w, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist

            dist.destroy_process_group()


if __name__ == "__main__":
    main()
