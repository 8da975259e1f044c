"""GPU parity: libleapquant's CUDA kernels, called through the C ABI, against
the CPU oracle on the same seeded inputs.  Needs a B200 (sm_100a)."""
import numpy as np
import pytest
import torch

import oracle
from recurrent_state_quantization_decode_b200 import workloads as wl

pytestmark = pytest.mark.gpu

B = None  # the binding, imported lazily so that collection works without a build


@pytest.fixture(scope="module", autouse=True)
def _binding():
    global B
    from recurrent_state_quantization_decode_b200 import build

    build.build()
    from recurrent_state_quantization_decode_b200 import binding

    B = binding
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    yield


import _parity as P  # noqa: E402


def _sync():
    torch.cuda.synchronize()


def _init_both(w, cfg, S0):
    ds = B.DeviceState(cfg)
    B.lq_state_init(cfg, torch.from_numpy(S0).cuda(), ds.st)
    tiles = [oracle.Tile(P.orc_cfg(w), S0[t].astype(np.float64)) for t in range(w.tiles)]
    return ds, tiles


# --------------------------------------------------------------------------
# quantize(): bit-exact given the same fp32 state
# --------------------------------------------------------------------------

def _special_states(S, d):
    S[0] = 0.0                                  # all zero
    S[1][5, :] = 0.0                            # a zero row and a zero column
    S[1][:, 7] = 0.0
    S[2] = (S[2] * np.float32(1e-39)).astype(np.float32)   # below FLT_MIN everywhere
    S[3][:, :] = np.float32(0.25)               # every line ties
    S[4][2, 3] = np.float32(1e3)                # one huge entry: its row and column tie
    S[5] = np.where(np.abs(S[5]) < 0.01, 0, S[5]).astype(np.float32)
    return S


@pytest.mark.parametrize("d,K,smooth", [(32, 4, 0.5), (64, 4, 0.5), (128, 4, 0.5),
                                        (128, 0, 0.5), (128, 8, 1.0), (128, 4, 0.0),
                                        (64, 2, 1.0)])
def test_init_bit_exact(d, K, smooth):
    rng = np.random.default_rng(100 + d + K)
    w = wl.Workload("t", 3, 2, 4, d, wl.GATE_SCALAR, False, 1, n_comp=K, smooth=smooth)
    S0, _, _ = wl.initial_states(rng, w.tiles, d, d)
    S0 = _special_states(S0, d)
    cfg = B.config_for(w)
    ds = B.DeviceState(cfg)
    B.lq_state_init(cfg, torch.from_numpy(S0).cuda(), ds.st)
    _sync()
    g = P.gpu_records(ds)
    assert np.all(ds.buf_n.cpu().numpy() == 0)
    for t in range(w.tiles):
        diag = oracle.new_diag()
        r = oracle.quantize(P.orc_cfg(w), S0[t].astype(np.float64), diag)
        if K and not np.array_equal(g["cid"][t], r.cid[:K]):
            assert diag[oracle.D_MIN_MARGIN] < P.NEAR_TIE_MARGIN, (t, g["cid"][t], r.cid)
            continue
        np.testing.assert_array_equal(g["Q"][t], r.Q, err_msg=f"tile {t}")
        np.testing.assert_array_equal(g["sig"][t], r.sig, err_msg=f"tile {t}")
        np.testing.assert_array_equal(g["m"][t], r.m, err_msg=f"tile {t}")
        if K:
            np.testing.assert_array_equal(g["cv"][t], r.cv[:K], err_msg=f"tile {t}")


# --------------------------------------------------------------------------
# decode, teacher-forced per window
# --------------------------------------------------------------------------

CASES = {
    "tiny_gdn_d32": (wl.TINY_GDN, 64),
    "gdn_gva_d128": (wl.Workload("g", 3, 16, 32, 128, wl.GATE_SCALAR, True, 40), 40),
    "kda_d128": (wl.Workload("k", 2, 32, 32, 128, wl.GATE_DIAG, True, 40,
                             v_outlier_channels=4), 40),
    "gdn_d64": (wl.Workload("g64", 2, 2, 4, 64, wl.GATE_SCALAR, False, 40), 40),
    "kda_d64_w8_k8_full": (wl.Workload("k64", 2, 1, 3, 64, wl.GATE_DIAG, False, 20, window=8,
                                       n_comp=8, smooth=1.0), 20),
    "naive_w1_k0": (wl.Workload("n", 1, 1, 2, 32, wl.GATE_SCALAR, False, 12, window=1,
                                n_comp=0, smooth=0.0), 12),
    "gdn_d128_f32": (wl.Workload("gf", 2, 2, 4, 128, wl.GATE_SCALAR, False, 36), 36),
    # windows above 16 tokens (the per-tile kernel): two folds of 32 tokens
    "gdn_gva_d128_w32": (wl.Workload("g32", 2, 2, 4, 128, wl.GATE_SCALAR, True, 70,
                                     window=32), 70),
    "kda_d64_w32_k8": (wl.Workload("k32", 2, 2, 2, 64, wl.GATE_DIAG, False, 40, window=32,
                                   n_comp=8), 40),
    # the quad path (d = 128, bf16 inputs) without compensators, with eight of
    # them (larger records, fewer CTAs per SM), and with smoothing off / full
    "gdn_gva_d128_k0": (wl.Workload("gk0", 2, 4, 8, 128, wl.GATE_SCALAR, True, 20, n_comp=0), 20),
    "kda_d128_k8_s1": (wl.Workload("kk8", 2, 4, 4, 128, wl.GATE_DIAG, True, 20, n_comp=8,
                                   smooth=1.0), 20),
    "gdn_gva_d128_s0": (wl.Workload("gs0", 2, 4, 8, 128, wl.GATE_SCALAR, True, 20,
                                    smooth=0.0), 20),
    "kda_d128_f32": (wl.Workload("kf", 2, 2, 2, 128, wl.GATE_DIAG, False, 36,
                                 v_outlier_channels=4), 36),
}


@pytest.mark.parametrize("case", sorted(CASES))
def test_decode_teacher_forced(case):
    w, T = CASES[case]
    rng = np.random.default_rng(0)
    S0, _, _ = wl.initial_states(rng, w.tiles, w.d, w.d)
    ti = wl.token_inputs(rng, w, T)
    cfg = B.config_for(w)
    ds = B.DeviceState(cfg)
    ocfg = P.orc_cfg(w)
    tiles = [oracle.Tile(ocfg, S0[t].astype(np.float64)) for t in range(w.tiles)]
    P.import_records(ds, [tl.rec for tl in tiles])
    dev = P.DeviceInputs(ti, w.io_bf16)
    out = torch.empty((w.batch, w.num_v_heads, w.d), dtype=torch.float32, device="cuda")
    worst = 0.0
    folds = 0
    for t in range(T):
        q, k, v, a, b = dev.token(t)
        B.lq_decode_step(cfg, q, k, v, a, b, ds.st, out)
        o_gpu = out.cpu().numpy().reshape(w.tiles, w.d)
        margins = np.zeros(w.tiles)
        for tile in range(w.tiles):
            tl = tiles[tile]
            tl.diag = oracle.new_diag()
            o = tl.run(*P.tile_inputs(ti, w, tile, t, t + 1))[0]
            err = P.normwise(o_gpu[tile].astype(np.float64), o)
            worst = max(worst, float(err))
            assert err <= P.REL_TOL, (case, t, tile, err)
            margins[tile] = tl.diag[oracle.D_MIN_MARGIN]
        if (t + 1) % w.window == 0:
            folds += 1
            diff = P.compare_records(P.gpu_records(ds), [tl.rec for tl in tiles], margins)
            P.assert_records_close(diff)
            P.import_records(ds, [tl.rec for tl in tiles])   # teacher forcing
    # buffered deltas of the last, partial window
    n = T % w.window
    if n:
        bd = ds.buf_d.cpu().numpy()[:w.tiles * w.window * w.d].reshape(w.tiles, w.window, w.d)
        for tile in range(w.tiles):
            np.testing.assert_array_equal(ds.buf_n.cpu().numpy()[tile], n)
            err = np.max(P.normwise(bd[tile, :n].astype(np.float64), tiles[tile].bd[:n]))
            assert err <= P.REL_TOL
    assert B.lq_get_last_error(ds.st) == B.LQ_OK
    print(f"{case}: worst output error {worst:.2e} over {T} tokens, {folds} folds")


def test_decode_free_running_tiny_workload():
    """The tiny GDN workload exactly as specified: 64 tokens, 4 windows, both
    sides quantizing on their own from the same initial state."""
    w = wl.TINY_GDN
    rng = np.random.default_rng(0)
    S0, _, _ = wl.initial_states(rng, 1, 32, 32)
    ti = wl.token_inputs(rng, w, w.steps)
    cfg = B.config_for(w)
    ds, tiles = _init_both(w, cfg, S0)
    dev = P.DeviceInputs(ti, w.io_bf16)
    out = torch.empty((1, 1, 32), dtype=torch.float32, device="cuda")
    o_ref = tiles[0].run(*P.tile_inputs(ti, w, 0, 0, w.steps))
    for t in range(w.steps):
        B.lq_decode_step(cfg, *dev.token(t), ds.st, out)
        assert P.normwise(out.cpu().numpy()[0, 0].astype(np.float64), o_ref[t]) <= P.REL_TOL, t
    diff = P.compare_records(P.gpu_records(ds), [tiles[0].rec], np.array([1.0]))
    P.assert_records_close(diff)


@pytest.mark.parametrize("d,gate", [(64, wl.GATE_SCALAR), (128, wl.GATE_SCALAR),
                                    (128, wl.GATE_DIAG)])
def test_bf16_output(d, gate):
    w = wl.Workload("g", 2, 2, 4, d, gate, True, 20)
    rng = np.random.default_rng(3)
    S0, _, _ = wl.initial_states(rng, w.tiles, w.d, w.d)
    ti = wl.token_inputs(rng, w, 20)
    cfg = B.config_for(w, out_bf16=True)
    ds, tiles = _init_both(w, cfg, S0)
    dev = P.DeviceInputs(ti, True)
    out = torch.empty((w.batch, w.num_v_heads, w.d), dtype=torch.bfloat16, device="cuda")
    refs = [tl.run(*P.tile_inputs(ti, w, t, 0, 20)) for t, tl in enumerate(tiles)]
    for t in range(20):
        B.lq_decode_step(cfg, *dev.token(t), ds.st, out)
        o = out.float().cpu().numpy().reshape(w.tiles, w.d)
        for tile in range(w.tiles):
            assert P.normwise(o[tile].astype(np.float64), refs[tile][t]) <= 2.0 ** -8


# --------------------------------------------------------------------------
# fp32-state comparison path
# --------------------------------------------------------------------------

@pytest.mark.parametrize("case", ["tiny_gdn_d32", "gdn_gva_d128", "kda_d128", "gdn_d64"])
def test_fp32_path_vs_exact(case):
    w, _ = CASES[case]
    T = 32
    rng = np.random.default_rng(1)
    S0, _, _ = wl.initial_states(rng, w.tiles, w.d, w.d)
    ti = wl.token_inputs(rng, w, T)
    cfg = B.config_for(w)
    S = torch.from_numpy(S0).cuda().contiguous()
    dev = P.DeviceInputs(ti, w.io_bf16)
    out = torch.empty((w.batch, w.num_v_heads, w.d), dtype=torch.float32, device="cuda")
    outs = []
    for t in range(T):
        B.lq_fp32_decode_step(cfg, *dev.token(t), S, out)
        outs.append(out.cpu().numpy().reshape(w.tiles, w.d).copy())
    S_gpu = S.cpu().numpy()
    ocfg = P.orc_cfg(w)
    for tile in range(w.tiles):
        S_ex, o_ex = oracle.exact_run(ocfg, S0[tile], *P.tile_inputs(ti, w, tile, 0, T))
        for t in range(T):
            assert P.normwise(outs[t][tile].astype(np.float64), o_ex[t]) <= 1e-4, (tile, t)
        assert P.normwise(S_gpu[tile].reshape(-1).astype(np.float64), S_ex.reshape(-1)) <= 1e-4


# --------------------------------------------------------------------------
# ragged batches: active masks and partial-window flushes
# --------------------------------------------------------------------------

RAGGED_CASES = {
    # the general path: KDA, bf16 inputs, d = 64
    "kda_d64_bf16": wl.Workload("r", 5, 2, 4, 64, wl.GATE_DIAG, True, 48),
    # the path the bench times for GDN: bf16 inputs, d = 128, grouped heads
    # (Hk = 16, Hv = 32), so tiles of one CTA sit in different window phases
    "gdn_gva_d128_bf16": wl.Workload("rg", 5, 16, 32, 128, wl.GATE_SCALAR, True, 48),
    # GDN with fp32 inputs at d = 128 (the general path at full width)
    "gdn_d128_f32": wl.Workload("rf", 6, 4, 8, 128, wl.GATE_SCALAR, False, 48),
    # KDA with bf16 inputs at d = 128 (the Kimi-Linear-like shape, fewer tiles)
    "kda_d128_bf16": wl.Workload("rk", 5, 8, 8, 128, wl.GATE_DIAG, True, 48,
                                 v_outlier_channels=4),
    # a 32-token window: decode on the per-tile kernel, flushes of up to 31
    # buffered tokens
    "gdn_d64_bf16_w32": wl.Workload("r32", 5, 2, 4, 64, wl.GATE_SCALAR, True, 48, window=32),
}


@pytest.mark.parametrize("case", sorted(RAGGED_CASES))
def test_active_mask_and_flush(case):
    """Ragged batch: random active masks and partial-window flushes, so that
    the tiles of one launch (and of one CTA) sit in different window phases.
    Each tile is teacher-forced at its own folds: whenever a tile's window
    closes (boundary or flush), its record is compared and the oracle's is
    written into the GPU state."""
    w = RAGGED_CASES[case]
    T = 48
    rng = np.random.default_rng(7)
    S0, _, _ = wl.initial_states(rng, w.tiles, w.d, w.d)
    ti = wl.token_inputs(rng, w, T)
    active = rng.random((T, w.batch)) < 0.7
    flush = rng.random((T, w.batch)) < 0.1
    cfg = B.config_for(w)
    ds, tiles = _init_both(w, cfg, S0)
    dev = P.DeviceInputs(ti, w.io_bf16)
    out = torch.empty((w.batch, w.num_v_heads, w.d), dtype=torch.float32, device="cuda")
    rv = ds.record_view()
    folds = 0

    def sync_folded(closed):
        nonlocal folds
        if not closed:
            return
        g = P.gpu_records(ds)
        recs = [tiles[t].rec for t in closed]
        margins = np.array([tiles[t].diag[oracle.D_MIN_MARGIN] for t in closed])
        P.assert_records_close(P.compare_records(g, recs, margins, tiles=closed))
        for t in closed:
            rv[t] = torch.from_numpy(P.pack_record(tiles[t].rec, ds.layout, w.d,
                                                   w.n_comp)).cuda()
        folds += len(closed)

    for t in range(T):
        out.fill_(float("nan"))
        act = torch.from_numpy(active[t].astype(np.int32)).cuda()
        B.lq_decode_step(cfg, *dev.token(t), ds.st, out, active=act)
        o = out.cpu().numpy().reshape(w.batch, w.num_v_heads, w.d)
        closed = []
        for tile in range(w.tiles):
            b, h = divmod(tile, w.num_v_heads)
            if not active[t, b]:
                assert np.all(np.isnan(o[b, h]))
                continue
            tiles[tile].diag = oracle.new_diag()
            ref = tiles[tile].run(*P.tile_inputs(ti, w, tile, t, t + 1))[0]
            assert P.normwise(o[b, h].astype(np.float64), ref) <= P.REL_TOL, (t, tile)
            if tiles[tile].n[0] == 0:
                closed.append(tile)
        sync_folded(closed)
        if flush[t].any():
            B.lq_window_flush(cfg, ds.st, mask=torch.from_numpy(flush[t].astype(np.int32)).cuda())
            closed = []
            for tile in range(w.tiles):
                if flush[t, tile // w.num_v_heads] and tiles[tile].n[0] > 0:
                    tiles[tile].diag = oracle.new_diag()
                    tiles[tile].flush()
                    closed.append(tile)
            sync_folded(closed)
        n_gpu = ds.buf_n.cpu().numpy()[:w.tiles]
        assert list(n_gpu) == [int(tl.n[0]) for tl in tiles], t
    assert folds > w.tiles
    assert B.lq_get_last_error(ds.st) == B.LQ_OK


PACKED_CASES = {
    "kda_d128_bf16": wl.Workload("pk", 6, 32, 32, 128, wl.GATE_DIAG, True, 20),
    "gdn_gva_d128_bf16": wl.Workload("pg", 6, 16, 32, 128, wl.GATE_SCALAR, True, 20),
    "gdn_d64_f32": wl.Workload("pf", 5, 2, 4, 64, wl.GATE_SCALAR, False, 20),
    "kda_d64_bf16": wl.Workload("pd", 5, 4, 4, 64, wl.GATE_DIAG, True, 20),
}


@pytest.mark.parametrize("case", sorted(PACKED_CASES))
def test_packed_inputs_match_separate_inputs(case):
    """lq_decode_step_packed on per-tile blocks and lq_decode_step on separate
    arrays: the same bits (outputs, phases, records, buffers) over 20 tokens,
    a fold and a random active mask included."""
    w = PACKED_CASES[case]
    rng = np.random.default_rng(12)
    S0, _, _ = wl.initial_states(rng, w.tiles, w.d, w.d)
    ti = wl.token_inputs(rng, w, w.steps)
    active = rng.random((w.steps, w.batch)) < 0.8
    cfg = B.config_for(w)
    S0_dev = torch.from_numpy(S0).cuda()
    a, b = B.DeviceState(cfg), B.DeviceState(cfg)
    for ds in (a, b):
        B.lq_state_init(cfg, S0_dev, ds.st)
    dev = P.DeviceInputs(ti, w.io_bf16)
    outs = [torch.empty((w.batch, w.num_v_heads, w.d), device="cuda") for _ in range(2)]
    kda = w.gate == wl.GATE_DIAG
    for t in range(w.steps):
        act = torch.from_numpy(active[t].astype(np.int32)).cuda()
        q, k, v, al, be = dev.token(t)
        blocks = B.pack_tile_inputs(cfg, q, k, v, al)
        for o in outs:
            o.fill_(float("nan"))
        B.lq_decode_step(cfg, q, k, v, al, be, a.st, outs[0], active=act)
        B.lq_decode_step_packed(cfg, blocks, None if kda else al, be, b.st, outs[1], active=act)
        assert torch.equal(outs[0].isnan(), outs[1].isnan())
        assert torch.equal(outs[0].nan_to_num(), outs[1].nan_to_num()), t
    for name in ("records", "buf_k", "buf_d", "buf_g", "buf_n"):
        assert torch.equal(getattr(a, name), getattr(b, name)), name
    for ds in (a, b):
        assert B.lq_get_last_error(ds.st) == B.LQ_OK


@pytest.mark.parametrize("window,T", [(16, 21), (32, 45)])
def test_dequantize_base_and_current_state(window, T):
    w = wl.Workload("q", 2, 2, 2, 64, wl.GATE_DIAG, False, T, window=window)
    rng = np.random.default_rng(9)
    S0, _, _ = wl.initial_states(rng, w.tiles, w.d, w.d)
    ti = wl.token_inputs(rng, w, T)
    cfg = B.config_for(w)
    ds, tiles = _init_both(w, cfg, S0)
    P.import_records(ds, [tl.rec for tl in tiles])     # one start record on both sides
    dev = P.DeviceInputs(ti, False)
    out = torch.empty((w.batch, w.num_v_heads, w.d), dtype=torch.float32, device="cuda")
    for t in range(T):
        B.lq_decode_step(cfg, *dev.token(t), ds.st, out)
    for tl_i, tl in enumerate(tiles):
        tl.run(*P.tile_inputs(ti, w, tl_i, 0, T))
    S_base = torch.empty((w.tiles, w.d, w.d), dtype=torch.float32, device="cuda")
    S_cur = torch.empty_like(S_base)
    B.lq_state_dequantize(cfg, ds.st, False, S_base)
    B.lq_state_dequantize(cfg, ds.st, True, S_cur)
    Sb, Sc = S_base.cpu().numpy(), S_cur.cpu().numpy()
    for t, tl in enumerate(tiles):
        assert P.normwise(Sb[t].reshape(-1).astype(np.float64), tl.base().reshape(-1)) <= P.REL_TOL
        assert P.normwise(Sc[t].reshape(-1).astype(np.float64), tl.state().reshape(-1)) <= P.REL_TOL


# --------------------------------------------------------------------------
# full-size workloads in the benchmark's launch configuration, sampled
# --------------------------------------------------------------------------

def _full_size_sampled(w, T, sample, init_pool=None):
    """All tiles on the GPU in the benchmark's launch configuration; the
    oracle runs the sampled tiles.  Teacher-forced per window: at every
    boundary the sampled tiles' records are compared, then the oracle's records
    are written into the GPU state for those tiles."""
    rng = np.random.default_rng(0)
    pool = w.tiles if init_pool is None else init_pool
    S0p, _, _ = wl.initial_states(rng, pool, w.d, w.d)
    ti = wl.token_inputs(rng, w, T)
    cfg = B.config_for(w)
    ds = B.DeviceState(cfg)
    S0_dev = torch.from_numpy(S0p).cuda()
    if pool != w.tiles:
        S0_dev = S0_dev[torch.arange(w.tiles, device="cuda") % pool].contiguous()
    B.lq_state_init(cfg, S0_dev, ds.st)
    del S0_dev
    dev = P.DeviceInputs(ti, w.io_bf16)
    out = torch.empty((w.batch, w.num_v_heads, w.d), dtype=torch.float32, device="cuda")
    idx = torch.tensor(sample, device="cuda")
    ocfg = P.orc_cfg(w)
    tiles = [oracle.Tile(ocfg, S0p[t % pool].astype(np.float64), wy_check=False) for t in sample]
    rv = ds.record_view()
    L = ds.layout
    t0 = 0
    worst = 0.0
    while t0 < T:
        t1 = min(T, t0 + w.window)
        outs = []
        for t in range(t0, t1):
            B.lq_decode_step(cfg, *dev.token(t), ds.st, out)
            outs.append(out.view(w.tiles, w.d)[idx].cpu().numpy())
        margins = []
        for i, tile in enumerate(sample):
            tl = tiles[i]
            tl.diag = oracle.new_diag()
            o = tl.run(*P.tile_inputs(ti, w, tile, t0, t1))
            for t in range(t1 - t0):
                err = P.normwise(outs[t][i].astype(np.float64), o[t])
                worst = max(worst, float(err))
                assert err <= P.REL_TOL, (tile, t0 + t, err)
            margins.append(tl.diag[oracle.D_MIN_MARGIN])
        if t1 - t0 == w.window:
            raw = rv[idx].cpu().numpy()
            g = P.unpack_records(raw, L, w.d, w.n_comp)
            P.assert_records_close(P.compare_records(g, [tl.rec for tl in tiles],
                                                     np.array(margins)))
            packed = np.stack([P.pack_record(tl.rec, L, w.d, w.n_comp) for tl in tiles])
            rv[idx] = torch.from_numpy(packed).cuda()
        t0 = t1
    assert B.lq_get_last_error(ds.st) == B.LQ_OK
    print(f"{w.name}: worst output error {worst:.2e} over {T} tokens")


def test_full_size_qwen35_9b_like_gdn_sampled():
    w = wl.QWEN35_9B_GDN
    _full_size_sampled(w, 48, [0, 1, 31, 32, 333, 1024, 1500, 2047])


def test_full_size_kimi_linear_like_kda_sampled():
    w = wl.KIMI_LINEAR_KDA
    _full_size_sampled(w, 33, [0, 5, 1000, 2222, 4095])


def test_max_sweep_size_sampled():
    """The largest sweep point (1024 sequences x 32 heads = 32,768 tiles)."""
    w = wl.sweep_workload(1024)
    _full_size_sampled(w, 17, [0, 4097, 20000, 32767], init_pool=64)


# --------------------------------------------------------------------------
# device-side checks and the host-buffer entry point
# --------------------------------------------------------------------------

def test_corrupt_phase_sets_error_word_and_skips_tile():
    w = wl.Workload("e", 2, 1, 2, 32, wl.GATE_SCALAR, False, 2)
    rng = np.random.default_rng(5)
    S0, _, _ = wl.initial_states(rng, w.tiles, 32, 32)
    ti = wl.token_inputs(rng, w, 2)
    cfg = B.config_for(w)
    ds, tiles = _init_both(w, cfg, S0)
    ds.buf_n[1] = 99                       # corrupt phase of tile 1 (checked before any access)
    dev = P.DeviceInputs(ti, False)
    out = torch.full((w.batch, w.num_v_heads, w.d), 7.0, device="cuda")
    B.lq_decode_step(cfg, *dev.token(0), ds.st, out)
    assert B.lq_get_last_error(ds.st) == B.LQ_ERR_DEVICE_BOUNDS
    assert B.lq_get_last_error(ds.st) == B.LQ_OK           # cleared
    o = out.cpu().numpy().reshape(w.tiles, w.d)
    assert np.all(o[1] == 7.0)
    ref = tiles[0].run(*P.tile_inputs(ti, w, 0, 0, 1))[0]
    assert P.normwise(o[0].astype(np.float64), ref) <= P.REL_TOL


@pytest.mark.parametrize("bf16,gate", [(True, wl.GATE_SCALAR), (True, wl.GATE_DIAG)])
def test_bounded_wait_expiry_reports_timeout(bf16, gate):
    """The first CTA withholds its first slot's copies: its wait expires after a
    few polls, the error word says LQ_ERR_TIMEOUT, its tiles are left alone,
    every other CTA's tiles match a normal step, and the context stays usable."""
    w = wl.Workload("t", 64, 16, 32, 128, gate, bf16, 1)
    rng = np.random.default_rng(9)
    S0, _, _ = wl.initial_states(rng, w.tiles, w.d, w.d)
    ti = wl.token_inputs(rng, w, 1)
    cfg = B.config_for(w)
    S0_dev = torch.from_numpy(S0).cuda()
    dev = P.DeviceInputs(ti, bf16)
    outs = []
    for faulted in (False, True):
        ds = B.DeviceState(cfg)
        B.lq_state_init(cfg, S0_dev, ds.st)
        out = torch.full((w.batch, w.num_v_heads, w.d), float("nan"), device="cuda")
        if faulted:
            B.lq_test_decode_step_timeout(cfg, *dev.token(0), ds.st, out, wait_limit=2000)
            assert B.lq_get_last_error(ds.st) == B.LQ_ERR_TIMEOUT
        else:
            B.lq_decode_step(cfg, *dev.token(0), ds.st, out)
            assert B.lq_get_last_error(ds.st) == B.LQ_OK
        outs.append(out.reshape(w.tiles, w.d).cpu().numpy())
    normal, faulted = outs
    assert np.all(np.isnan(faulted[0]))              # the first CTA's first tile: untouched
    done = ~np.isnan(faulted).any(axis=1)
    skipped = np.flatnonzero(~done)
    # only the first CTA's tiles (0, g, 2g, ... for a grid of g CTAs) are
    # skipped: tile 0 always, and those of its tiles that had not been
    # finished when its waits expired
    assert skipped[0] == 0 and len(skipped) < w.tiles // 100
    if len(skipped) > 1:
        g = int(np.gcd.reduce(skipped[1:]))
        assert g >= 100 and np.all(skipped % g == 0), skipped
    assert np.array_equal(faulted[done], normal[done])
    # the context is still usable: a normal step on a fresh state succeeds
    ds = B.DeviceState(cfg)
    B.lq_state_init(cfg, S0_dev, ds.st)
    out = torch.empty((w.batch, w.num_v_heads, w.d), device="cuda")
    B.lq_decode_step(cfg, *dev.token(0), ds.st, out)
    assert B.lq_get_last_error(ds.st) == B.LQ_OK
    assert torch.isfinite(out).all()


HOST_MODES = {
    # inputs in pinned memory: the gather kernel reads them over the host link
    "pinned": (wl.Workload("h", 4, 2, 4, 128, wl.GATE_SCALAR, True, 20), set("qkv") | {"alpha", "beta"}),
    # pageable memory: every input goes through cudaMemcpyAsync
    "pageable": (wl.Workload("h", 4, 2, 4, 128, wl.GATE_SCALAR, True, 20), set()),
    # some of each in one call
    "mixed": (wl.Workload("h", 4, 2, 4, 128, wl.GATE_SCALAR, True, 20), {"q", "v"}),
    # 9 tiles: alpha and beta of 36 bytes (a ragged tail), placed 4 bytes off
    # a 16-byte boundary in pinned memory (the bytewise path)
    "ragged_misaligned": (wl.Workload("h9", 3, 1, 3, 64, wl.GATE_SCALAR, True, 20),
                          set("qkv") | {"alpha", "beta"}),
    # each token's q, k, v, alpha, beta back to back in one pinned block (every
    # size a multiple of 256 bytes): one copy-engine copy per call; GDN and KDA
    "packed": (wl.Workload("hp", 16, 2, 4, 128, wl.GATE_SCALAR, True, 20), set()),
    "packed_kda": (wl.Workload("hpk", 16, 4, 4, 128, wl.GATE_DIAG, True, 20), set()),
}


def _packed_host_inputs(dev, T):
    """Per token, q, k, v, alpha, beta back to back in one pinned block."""
    names = ("q", "k", "v", "alpha", "beta")
    sizes = [getattr(dev, n)[0].numel() * getattr(dev, n)[0].element_size() for n in names]
    assert all(sz % 256 == 0 for sz in sizes)
    block = torch.empty((T, sum(sizes)), dtype=torch.uint8).pin_memory()
    host = {n: [] for n in names}
    for t in range(T):
        off = 0
        for n, sz in zip(names, sizes):
            x = getattr(dev, n)[t].cpu()
            view = block[t, off:off + sz].view(x.dtype).view(x.shape)
            view.copy_(x)
            host[n].append(view)
            off += sz
        assert host["k"][t].data_ptr() == host["q"][t].data_ptr() + sizes[0]
    return host


@pytest.mark.parametrize("mode", sorted(HOST_MODES))
def test_host_entry_point_matches_device_entry_point(mode):
    w, pinned = HOST_MODES[mode]
    rng = np.random.default_rng(6)
    S0, _, _ = wl.initial_states(rng, w.tiles, w.d, w.d)
    ti = wl.token_inputs(rng, w, 20)
    cfg = B.config_for(w)
    a = B.DeviceState(cfg)
    b = B.DeviceState(cfg)
    S0_dev = torch.from_numpy(S0).cuda()
    B.lq_state_init(cfg, S0_dev, a.st)
    B.lq_state_init(cfg, S0_dev, b.st)
    dev = P.DeviceInputs(ti, True)
    host = _packed_host_inputs(dev, 20) if mode.startswith("packed") else {}
    for n in ("q", "k", "v", "alpha", "beta") if not host else ():
        x = getattr(dev, n).cpu()
        if n in pinned and mode == "ragged_misaligned" and n in ("alpha", "beta"):
            buf = torch.empty(x.numel() + 1, dtype=x.dtype).pin_memory()
            view = buf[1:].view(x.shape)
            view.copy_(x)
            assert view.data_ptr() % 16 == 4
            x = view
        elif n in pinned:
            x = x.pin_memory()
        else:
            assert not x.is_pinned()
        host[n] = x
    staging = torch.empty(B.lq_state_layout(cfg).host_staging_bytes, dtype=torch.uint8,
                          device="cuda")
    out_d = torch.empty((w.batch, w.num_v_heads, w.d), device="cuda")
    out_h = torch.empty((w.batch, w.num_v_heads, w.d)).pin_memory()
    for t in range(20):
        B.lq_decode_step(cfg, *dev.token(t), a.st, out_d)
        B.lq_decode_step_host(cfg, host["q"][t], host["k"][t], host["v"][t], host["alpha"][t],
                              host["beta"][t], b.st, out_h, staging)
        _sync()
        np.testing.assert_array_equal(out_h.numpy(), out_d.cpu().numpy())
    assert torch.equal(a.records, b.records)
    assert B.lq_get_last_error(b.st) == B.LQ_OK
