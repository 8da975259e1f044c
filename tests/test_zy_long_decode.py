"""Long ragged continuous batch: the long-decode workload at its stated size
(256 sequences x 32 heads, GDN, d = 128, ragged lengths ~ LogNormal(7, 1),
per-sequence window phases, a checkpoint every 1,024 tokens), through the
C-ABI decode step.  The sampled tiles' inputs are drawn on the host (numpy,
seeded) and also feed the oracle; every other tile's inputs are drawn on the
device by the same recipe (torch, seeded), since the whole batch is too
large to draw on the host token by token.

It checks three things:

- Checkpoint / resume: lq_checkpoint_save at a 1,024-token boundary (news
  article, paragraph 5: one state checkpoint per 1,024 tokens for prefix
  caching), lq_checkpoint_restore into a fresh state, and replaying the same
  tokens reproduces the original outputs bit for bit.
- Drift against the exact recurrence: on sampled tiles (the longest
  sequences among them) the int8-state outputs are compared with the exact
  fp64 recurrence over the whole decode.  The drift of LeapQuant (W = 16,
  K = 4, smoothing 1/2) must stay below that of naive per-token int8
  (W = 1, K = 0, no smoothing) run on the same inputs: the pages credit
  each of the three techniques with lower quantization error (zhichai.net
  summary, "Abstract (translated)" items 1-3).
- No blow-up: LeapQuant's worst normwise drift stays below 5 %.

The maximum length is 4,096 tokens by default (LQ_LONG_DECODE_MAX_LEN raises
it, up to 32,768).  The per-bucket drift table is printed (pytest -s)."""
import os

import numpy as np
import pytest
import torch

import oracle
from recurrent_state_quantization_decode_b200 import workloads as wl

pytestmark = pytest.mark.gpu

B_SEQ, HK, HV, D = wl.RAGGED.batch, wl.RAGGED.num_k_heads, wl.RAGGED.num_v_heads, wl.RAGGED.d
CHUNK = 128                      # tokens drawn per host batch
CKPT = 1024                      # checkpoint cadence in absolute positions
MAX_LEN = int(os.environ.get("LQ_LONG_DECODE_MAX_LEN", "4096"))
DRIFT_CAP = 0.05


def _binding():
    from recurrent_state_quantization_decode_b200 import build

    build.build()
    from recurrent_state_quantization_decode_b200 import binding

    return binding


def ds_layout_record(B, cfg) -> int:
    return B.lq_state_layout(cfg).record_bytes


def _normwise(a, b):
    return np.linalg.norm(a - b, axis=-1) / np.maximum(np.linalg.norm(b, axis=-1), 1e-30)


def test_long_ragged_decode_checkpoint_resume_and_drift():
    B = _binding()
    rng = np.random.default_rng(11)
    lengths, phase = wl.ragged_lengths(rng, B_SEQ, max_len=min(MAX_LEN, 32768))
    T = int(lengths.max())
    w = wl.Workload("ragged_long", B_SEQ, HK, HV, D, wl.GATE_SCALAR, True, T)
    tiles = w.tiles
    S0, _, _ = wl.initial_states(rng, tiles, D, D)
    S0_dev = torch.from_numpy(S0).cuda()
    cfg = B.config_for(w)
    naive = B.make_config(B_SEQ, HK, HV, D, 1, 0, gate=B.LQ_GATE_SCALAR, in_bf16=True,
                          smooth=0.0)
    states = {"leapquant": B.DeviceState(cfg), "naive": B.DeviceState(naive)}
    for name, ds in states.items():
        B.lq_state_init(cfg if name == "leapquant" else naive, S0_dev, ds.st)

    # sampled tiles: both heads 0 and 1 of the four longest sequences, and eight more
    longest = np.argsort(-lengths)[:4]
    sample = sorted(set([int(b) * HV + h for b in longest for h in (0, 1)]) |
                    set(int(x) for x in rng.choice(tiles, 8, replace=False)))
    sample_dev = torch.tensor(sample, device="cuda")
    # the sequence whose first checkpoint is replayed
    rb = int(longest[0])
    ck_step = next((t for t in range(T) if (phase[rb] + t + 1) % CKPT == 0
                    and t + 1 < lengths[rb]), None)
    assert ck_step is not None, "the longest sequence must reach a checkpoint"
    rb_tiles = slice(rb * HV, (rb + 1) * HV)

    hist = {n: torch.full((T, len(sample), D), float("nan"), device="cuda") for n in states}
    rb_hist = torch.full((T, HV, D), float("nan"), device="cuda")
    # host copies of the sampled tiles' inputs only (token, sample, ...)
    smp_b = np.array([t // HV for t in sample])
    smp_h = np.array([t % HV for t in sample])
    smp_hk = smp_h // (HV // HK)
    host_inputs = {n: [] for n in ("q", "k", "v", "alpha", "beta")}
    out = torch.empty((B_SEQ, HV, D), device="cuda")
    # a one-slot checkpoint pool; sequence rb's checkpoint goes to slot 0
    pool = torch.zeros(HV * ds_layout_record(B, cfg), dtype=torch.uint8, device="cuda")
    slots = torch.full((B_SEQ,), -1, dtype=torch.int32, device="cuda")
    slots[rb] = 0
    dev_chunks = []
    gen = torch.Generator(device="cuda")
    gen.manual_seed(11)
    smp_w = wl.Workload("ragged_sampled", len(sample), 1, 1, D, wl.GATE_SCALAR, True, T)
    smp_b_dev = torch.from_numpy(smp_b).cuda()
    smp_h_dev = torch.from_numpy(smp_h).cuda()
    smp_hk_dev = torch.from_numpy(smp_hk).cuda()
    for c0 in range(0, T, CHUNK):
        n_tok = min(CHUNK, T - c0)
        dev = wl.token_inputs_device(gen, w, n_tok, "cuda")
        # the sampled tiles: host draws, written into the device inputs
        ti = wl.token_inputs(rng, smp_w, n_tok)            # [n_tok, sample, 1, D]
        host = {n: getattr(ti, n)[:, :, 0] for n in ("q", "k", "v", "alpha", "beta")}
        for n in host:
            host_inputs[n].append(host[n])
        dev["q"][:, smp_b_dev, smp_hk_dev] = torch.from_numpy(host["q"]).cuda().to(torch.bfloat16)
        dev["k"][:, smp_b_dev, smp_hk_dev] = torch.from_numpy(host["k"]).cuda().to(torch.bfloat16)
        dev["v"][:, smp_b_dev, smp_h_dev] = torch.from_numpy(host["v"]).cuda().to(torch.bfloat16)
        dev["alpha"][:, smp_b_dev, smp_h_dev] = torch.from_numpy(host["alpha"]).cuda()
        dev["beta"][:, smp_b_dev, smp_h_dev] = torch.from_numpy(host["beta"]).cuda()
        dev_chunks.append(dev)
        for tt in range(dev["q"].shape[0]):
            t = c0 + tt
            act = torch.from_numpy((t < lengths).astype(np.int32)).cuda()
            args = [dev[n][tt] for n in ("q", "k", "v", "alpha", "beta")]
            for name, ds in states.items():
                c = cfg if name == "leapquant" else naive
                out.fill_(float("nan"))
                B.lq_decode_step(c, *args, ds.st, out, active=act)
                o = out.view(tiles, D)
                hist[name][t] = o[sample_dev]
                if name == "leapquant":
                    rb_hist[t] = o[rb_tiles]
            # after 16 - phi tokens the first window closes early, so that every
            # later boundary is a multiple of 16 in absolute position
            first = (t + 1 == 16 - phase) & (phase > 0) & (t < lengths)
            if first.any():
                m = torch.from_numpy(first.astype(np.int32)).cuda()
                B.lq_window_flush(cfg, states["leapquant"].st, m)
            if t == ck_step:
                ds = states["leapquant"]
                assert int(ds.buf_n[rb * HV]) == 0          # on a window boundary
                B.lq_checkpoint_save(cfg, ds.st, slots, pool, 1)
    for ds in states.values():
        assert B.lq_get_last_error(ds.st) == B.LQ_OK

    # resume from the checkpoint in a fresh state: only sequence rb is active
    ds2 = B.DeviceState(cfg)
    B.lq_state_init(cfg, S0_dev, ds2.st)
    B.lq_checkpoint_restore(cfg, pool, 1, slots, ds2.st)
    only = torch.zeros(B_SEQ, dtype=torch.int32, device="cuda")
    only[rb] = 1
    replay = torch.full_like(rb_hist, float("nan"))
    for t in range(ck_step + 1, int(lengths[rb])):
        dev = dev_chunks[t // CHUNK]
        args = [dev[n][t % CHUNK] for n in ("q", "k", "v", "alpha", "beta")]
        out.fill_(float("nan"))
        B.lq_decode_step(cfg, *args, ds2.st, out, active=only)
        replay[t] = out.view(tiles, D)[rb_tiles]
    assert B.lq_get_last_error(ds2.st) == B.LQ_OK
    span = slice(ck_step + 1, int(lengths[rb]))
    assert torch.equal(replay[span], rb_hist[span])

    # drift against the exact fp64 recurrence on the sampled tiles
    inp = {n: np.concatenate(v, axis=0) for n, v in host_inputs.items()}
    ex_cfg = oracle.Cfg(D, D, gate=wl.GATE_SCALAR)
    drift = {n: [] for n in states}
    for j, tile in enumerate(sample):
        Lb = int(lengths[tile // HV])
        _, o_ex = oracle.exact_run(ex_cfg, S0[tile].astype(np.float64), inp["q"][:Lb, j],
                                   inp["k"][:Lb, j], inp["v"][:Lb, j], inp["alpha"][:Lb, j],
                                   inp["beta"][:Lb, j])
        for name in states:
            o_gpu = hist[name][:Lb, j].cpu().numpy().astype(np.float64)
            drift[name].append(_normwise(o_gpu, o_ex))
    print(f"\nlong decode: {B_SEQ} sequences x {HV} heads, lengths up to {T}, "
          f"{len(sample)} sampled tiles")
    print("bucket (tokens)   leapquant median / max     naive median / max")
    for lo in range(0, T, CKPT):
        lq = np.concatenate([d[lo:lo + CKPT] for d in drift["leapquant"]])
        nv = np.concatenate([d[lo:lo + CKPT] for d in drift["naive"]])
        if lq.size:
            print(f"{lo:6d}-{lo + CKPT:6d}      {np.median(lq):.2e} / {lq.max():.2e}"
                  f"        {np.median(nv):.2e} / {nv.max():.2e}")
    lq_all = np.concatenate(drift["leapquant"])
    nv_all = np.concatenate(drift["naive"])
    assert np.all(np.isfinite(lq_all))
    assert np.median(lq_all) < np.median(nv_all)
    assert lq_all.max() < DRIFT_CAP
