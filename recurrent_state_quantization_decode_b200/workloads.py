"""Seeded synthetic workloads for the int8-state GDN/KDA decode step.

This module only draws random inputs and names workload shapes.  It holds none
of the decode method's arithmetic, so both the CUDA path and the CPU oracle can
be fed from it.

The shapes and distributions follow the workloads named for this decode step:
  * tiny GDN: 1 sequence, 1 head, d = 32, fp32 I/O, 64 tokens;
  * Qwen3.5-9B-like GDN layer: 64 sequences, 16 key heads / 32 value heads
    (grouped values), d = 128, bf16 q/k/v, scalar gate;
  * Kimi-Linear-like KDA layer: 128 sequences, 32 heads, d = 128, bf16 q/k/v,
    per-key-channel gate alpha_j = exp(-softplus(N(0,1)) * 0.05), 4 value
    channels of v scaled x10;
  * bandwidth sweep: the GDN shape at 8 .. 1024 sequences;
  * ragged continuous batch: 256 sequences x 32 heads with lengths drawn from
    LogNormal(7, 1) clipped to [1, 32768] and a window phase per sequence.

Common recipe: q, k ~ N(0, 1) then L2-normalised per head; v ~ N(0, 1);
beta = sigmoid(N(0, 1)); GDN alpha ~ U(0.9, 1).  Initial state per tile:
N(0, 0.02^2) entries (0.02 read as the standard deviation) with 2 rows and
2 columns multiplied by 20 (an entry in both is multiplied once).

bf16 inputs are returned as float32 arrays holding bf16-representable values,
so every consumer sees the same numbers.
"""
from __future__ import annotations

import dataclasses
from typing import Optional

import numpy as np

GATE_SCALAR = 0  # GDN: one decay per (sequence, value head) and token
GATE_DIAG = 1  # KDA: one decay per key channel


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    num_k_heads: int
    num_v_heads: int
    d: int
    gate: int
    io_bf16: bool
    steps: int
    window: int = 16
    n_comp: int = 4
    smooth: float = 0.5
    v_outlier_channels: int = 0  # value channels of v scaled x10

    @property
    def tiles(self) -> int:
        return self.batch * self.num_v_heads


TINY_GDN = Workload("tiny_gdn_d32", 1, 1, 1, 32, GATE_SCALAR, False, 64)
QWEN35_9B_GDN = Workload("qwen35_9b_like_gdn_b64_hk16_hv32_d128", 64, 16, 32, 128,
                         GATE_SCALAR, True, 1024)
KIMI_LINEAR_KDA = Workload("kimi_linear_like_kda_b128_h32_d128", 128, 32, 32, 128,
                           GATE_DIAG, True, 2048, v_outlier_channels=4)
SWEEP_BATCHES = (8, 16, 32, 64, 128, 256, 512, 1024)


def sweep_workload(batch: int) -> Workload:
    return Workload(f"gdn_sweep_b{batch}_hk16_hv32_d128", batch, 16, 32, 128, GATE_SCALAR,
                    True, 256)


RAGGED = Workload("ragged_gdn_b256_h32_d128", 256, 32, 32, 128, GATE_SCALAR, True, 32768)

WORKLOADS = {w.name: w for w in (TINY_GDN, QWEN35_9B_GDN, KIMI_LINEAR_KDA, RAGGED)}


def to_bf16_values(x: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bf16 (ties to even); float32 result."""
    import torch

    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
    return t.to(torch.bfloat16).to(torch.float32).numpy()


def _l2_normalise(x: np.ndarray) -> np.ndarray:
    n = np.sqrt(np.sum(x.astype(np.float64) ** 2, axis=-1, keepdims=True))
    return (x / np.maximum(n, 1e-30)).astype(np.float32)


def initial_states(rng: np.random.Generator, tiles: int, d_v: int, d_k: int,
                   std: float = 0.02, planted_rows: int = 2, planted_cols: int = 2,
                   factor: float = 20.0) -> tuple[np.ndarray, np.ndarray, np.ndarray]:
    """Per-tile initial states [tiles, d_v, d_k] float32, with planted outlier
    rows and columns.  Returns (S0, rows [tiles, planted_rows],
    cols [tiles, planted_cols]).  Draw order: all state entries, then per tile
    the planted rows, then the planted columns."""
    S = (rng.standard_normal((tiles, d_v, d_k)) * std).astype(np.float32)
    rows = np.zeros((tiles, planted_rows), dtype=np.int64)
    cols = np.zeros((tiles, planted_cols), dtype=np.int64)
    for t in range(tiles):
        rows[t] = rng.choice(d_v, planted_rows, replace=False)
        cols[t] = rng.choice(d_k, planted_cols, replace=False)
        mask = np.zeros((d_v, d_k), dtype=bool)
        mask[rows[t], :] = True
        mask[:, cols[t]] = True
        S[t][mask] *= np.float32(factor)
    return S, rows, cols


@dataclasses.dataclass
class TokenInputs:
    """Inputs of T tokens, token-major, as float32 arrays.
    q, k: [T, B, Hk, d]; v: [T, B, Hv, d]; alpha: [T, B, Hv] (GDN) or
    [T, B, Hv, d] (KDA); beta: [T, B, Hv]."""
    q: np.ndarray
    k: np.ndarray
    v: np.ndarray
    alpha: np.ndarray
    beta: np.ndarray


def token_inputs(rng: np.random.Generator, w: Workload, T: int, batch: Optional[int] = None,
                 outlier_channels: Optional[np.ndarray] = None) -> TokenInputs:
    """Draw T tokens of inputs for workload w (optionally with another batch)."""
    B = w.batch if batch is None else batch
    Hk, Hv, d = w.num_k_heads, w.num_v_heads, w.d
    q = _l2_normalise(rng.standard_normal((T, B, Hk, d)).astype(np.float32))
    k = _l2_normalise(rng.standard_normal((T, B, Hk, d)).astype(np.float32))
    v = rng.standard_normal((T, B, Hv, d)).astype(np.float32)
    if w.v_outlier_channels:
        ch = outlier_channels
        if ch is None:
            ch = np.random.default_rng(12345).choice(d, w.v_outlier_channels, replace=False)
        v[..., ch] *= np.float32(10.0)
    beta = (1.0 / (1.0 + np.exp(-rng.standard_normal((T, B, Hv))))).astype(np.float32)
    if w.gate == GATE_SCALAR:
        alpha = rng.uniform(0.9, 1.0, (T, B, Hv)).astype(np.float32)
    else:
        z = rng.standard_normal((T, B, Hv, d))
        softplus = np.logaddexp(0.0, z)
        alpha = np.exp(-softplus * 0.05).astype(np.float32)
    if w.io_bf16:
        q, k, v = to_bf16_values(q), to_bf16_values(k), to_bf16_values(v)
    return TokenInputs(q, k, v, alpha, beta)


def ragged_lengths(rng: np.random.Generator, n: int, mu: float = 7.0, sigma: float = 1.0,
                   max_len: int = 32768) -> tuple[np.ndarray, np.ndarray]:
    """Decode lengths ~ round(LogNormal(mu, sigma)) clipped to [1, max_len], and a
    window phase offset phi in 0..15 per sequence: the prompt length is taken as
    phi mod 16, so the first decode window holds 16 - phi tokens and every later
    window boundary falls on an absolute position that is a multiple of 16."""
    L = np.clip(np.rint(rng.lognormal(mu, sigma, n)), 1, max_len).astype(np.int64)
    phase = rng.integers(0, 16, n).astype(np.int64)
    return L, phase


def token_inputs_device(gen, w: Workload, T: int, device, batch: Optional[int] = None) -> dict:
    """T tokens of inputs for workload w drawn on the device with a seeded
    torch.Generator, by the same recipe as token_inputs (q, k ~ N(0, 1)
    L2-normalised per head, v ~ N(0, 1), beta = sigmoid(N(0, 1)), GDN alpha ~
    U(0.9, 1), KDA alpha = exp(-softplus(N(0, 1)) 0.05), q, k, v rounded to bf16
    for bf16 workloads).  For batches too large to draw on the host every
    token; returns torch tensors q, k [T, B, Hk, d], v [T, B, Hv, d] (bf16 or
    fp32), alpha, beta fp32."""
    import torch

    B = w.batch if batch is None else batch
    Hk, Hv, d = w.num_k_heads, w.num_v_heads, w.d

    def normal(*shape):
        return torch.randn(shape, generator=gen, device=device, dtype=torch.float32)

    def unit(x):
        return x / torch.linalg.vector_norm(x.double(), dim=-1, keepdim=True).clamp_min(1e-30).float()

    q, k = unit(normal(T, B, Hk, d)), unit(normal(T, B, Hk, d))
    v = normal(T, B, Hv, d)
    if w.v_outlier_channels:
        ch = np.random.default_rng(12345).choice(d, w.v_outlier_channels, replace=False)
        v[..., torch.as_tensor(ch, device=device)] *= 10.0
    beta = torch.sigmoid(normal(T, B, Hv))
    if w.gate == GATE_SCALAR:
        alpha = 0.9 + 0.1 * torch.rand((T, B, Hv), generator=gen, device=device)
    else:
        alpha = torch.exp(-torch.nn.functional.softplus(normal(T, B, Hv, d)) * 0.05)
    dt = torch.bfloat16 if w.io_bf16 else torch.float32
    return {"q": q.to(dt), "k": k.to(dt), "v": v.to(dt), "alpha": alpha.contiguous(),
            "beta": beta.contiguous()}
