"""Ablations of the three techniques on the GPU path: output drift from the
exact fp64 recurrence for window, compensator and smoothing settings, all on
the same seeded inputs and initial states (Qwen3.5-9B-like GDN heads, bf16
inputs).

The pages credit each technique with lower quantization error (zhichai.net
summary, "Abstract (translated)" items 1-3: the windowed buffer, the
compensator lines, the smoothing).  The test checks that each of the three
lowers the median drift against the configuration without it:

- window 16 against per-token requantization (W = 1), both with K = 4 and
  smoothing 1/2;
- K = 4 compensator lines against none, both W = 16 with smoothing 1/2;
- smoothing 1/2 against none, both W = 16 and K = 4.

Longer windows keep lowering it: W = 32 (run on the per-tile kernel that
serves windows above 16 tokens) must beat W = 16, and W = 16 must beat
W = 8.

The full LeapQuant configuration must also beat naive per-token int8.  The
drift table is printed (pytest -s)."""
import numpy as np
import pytest
import torch

import oracle
from recurrent_state_quantization_decode_b200 import workloads as wl

pytestmark = pytest.mark.gpu

B_SEQ, HK, HV, D, T = 8, 16, 32, 128, 1024
SAMPLES = 16

# (name, window, compensators, smoothing exponent)
VARIANTS = [
    ("leapquant W16 K4 s1/2", 16, 4, 0.5),
    ("window W1 (K4 s1/2)", 1, 4, 0.5),
    ("window W8 (K4 s1/2)", 8, 4, 0.5),
    ("window W32 (K4 s1/2)", 32, 4, 0.5),
    ("no compensators K0", 16, 0, 0.5),
    ("K2", 16, 2, 0.5),
    ("K8", 16, 8, 0.5),
    ("no smoothing s0", 16, 4, 0.0),
    ("full smoothing s1", 16, 4, 1.0),
    ("naive int8 W1 K0 s0", 1, 0, 0.0),
]


def _binding():
    from recurrent_state_quantization_decode_b200 import build

    build.build()
    from recurrent_state_quantization_decode_b200 import binding

    return binding


def test_each_technique_lowers_drift_on_gpu():
    B = _binding()
    rng = np.random.default_rng(21)
    w = wl.Workload("ablation", B_SEQ, HK, HV, D, wl.GATE_SCALAR, True, T)
    S0, _, _ = wl.initial_states(rng, w.tiles, D, D)
    ti = wl.token_inputs(rng, w, T)
    sample = np.sort(rng.choice(w.tiles, SAMPLES, replace=False))
    S0_dev = torch.from_numpy(S0).cuda()
    dev = {n: torch.from_numpy(getattr(ti, n)).cuda() for n in ("q", "k", "v", "alpha", "beta")}
    for n in ("q", "k", "v"):
        dev[n] = dev[n].to(torch.bfloat16)
    sample_dev = torch.from_numpy(sample).cuda()

    # exact fp64 recurrence on the sampled tiles
    ex_cfg = oracle.Cfg(D, D, gate=wl.GATE_SCALAR)
    o_ex = []
    for tile in sample:
        b, h = divmod(int(tile), HV)
        hk = h // (HV // HK)
        o_ex.append(oracle.exact_run(ex_cfg, S0[tile].astype(np.float64), ti.q[:, b, hk],
                                     ti.k[:, b, hk], ti.v[:, b, h], ti.alpha[:, b, h],
                                     ti.beta[:, b, h])[1])
    o_ex = np.stack(o_ex, axis=1)                       # [T, SAMPLES, D]

    med = {}
    print(f"\nablation drift: {B_SEQ} sequences x {HV} heads, {T} tokens, "
          f"{SAMPLES} sampled tiles")
    print("variant                      median     p99        max")
    for name, W, K, sm in VARIANTS:
        cfg = B.make_config(B_SEQ, HK, HV, D, W, K, gate=B.LQ_GATE_SCALAR, in_bf16=True,
                            smooth=sm)
        ds = B.DeviceState(cfg)
        B.lq_state_init(cfg, S0_dev, ds.st)
        out = torch.empty((B_SEQ, HV, D), device="cuda")
        hist = torch.empty((T, SAMPLES, D), device="cuda")
        for t in range(T):
            B.lq_decode_step(cfg, dev["q"][t], dev["k"][t], dev["v"][t], dev["alpha"][t],
                             dev["beta"][t], ds.st, out)
            hist[t] = out.view(w.tiles, D)[sample_dev]
        assert B.lq_get_last_error(ds.st) == B.LQ_OK
        o = hist.cpu().numpy().astype(np.float64)
        drift = (np.linalg.norm(o - o_ex, axis=-1) /
                 np.maximum(np.linalg.norm(o_ex, axis=-1), 1e-30)).ravel()
        assert np.all(np.isfinite(drift)), name
        med[name] = float(np.median(drift))
        print(f"{name:28s} {med[name]:.2e}   {np.quantile(drift, 0.99):.2e}   "
              f"{drift.max():.2e}")

    full = med["leapquant W16 K4 s1/2"]
    assert med["window W32 (K4 s1/2)"] < full < med["window W8 (K4 s1/2)"]
    assert full < med["window W1 (K4 s1/2)"]
    assert full < med["no compensators K0"]
    assert full < med["no smoothing s0"]
    assert full < med["naive int8 W1 K0 s0"]
