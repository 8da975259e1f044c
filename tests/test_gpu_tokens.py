"""lq_decode_tokens: several decode tokens per tile in one launch (the verify
step of speculative decoding), against the CPU oracle token by token.

One launch keeps each tile in shared memory for all its tokens, so the stored
record is read once per launch.  The outputs must meet the decode step's bar
(max relative error 1e-3 normwise per tile vector) against the oracle, the
fold inside a launch must give the oracle's record (codes +-1 on at most 0.1 %
of the entries), and a launch must leave the state exactly as the same tokens
decoded one call at a time would, up to rounding: the next tokens agree."""
import numpy as np
import pytest
import torch

import oracle
from recurrent_state_quantization_decode_b200 import workloads as wl

pytestmark = pytest.mark.gpu

import _parity as P  # noqa: E402

B = P.B

CASES = {
    "gdn_gva_d128_bf16": wl.Workload("tg", 3, 2, 4, 128, wl.GATE_SCALAR, True, 1),
    "kda_d128_bf16": wl.Workload("tk", 2, 4, 4, 128, wl.GATE_DIAG, True, 1, v_outlier_channels=4),
    "gdn_d64_f32_w8": wl.Workload("tf", 2, 2, 2, 64, wl.GATE_SCALAR, False, 1, window=8),
    "kda_d64_bf16_w32": wl.Workload("tw", 2, 2, 2, 64, wl.GATE_DIAG, True, 1, window=32),
}


def _launch(cfg, dev, t0, ntok, ds, out_all, active=None):
    """Tokens t0 .. t0 + ntok - 1 in one lq_decode_tokens call."""
    sl = slice(t0, t0 + ntok)
    B.lq_decode_tokens(cfg, ntok, dev.q[sl].contiguous(), dev.k[sl].contiguous(),
                       dev.v[sl].contiguous(), dev.alpha[sl].contiguous(),
                       dev.beta[sl].contiguous(), ds.st, out_all[sl], active=active)


@pytest.mark.parametrize("case", sorted(CASES))
def test_decode_tokens_against_the_oracle(case):
    """Launch 1 runs from a random window phase up to the window's last token
    (so its last token folds); the record is compared and the oracle's written
    back (teacher forcing); launch 2 runs 7 more tokens with one sequence
    inactive.  Every output is compared with the oracle."""
    w = CASES[case]
    W = w.window
    rng = np.random.default_rng(51)
    S0, _, _ = wl.initial_states(rng, w.tiles, w.d, w.d)
    n0 = 3 if W > 4 else 1
    T = n0 + (W - n0) + 7
    ti = wl.token_inputs(rng, w, T)
    cfg = B.config_for(w)
    ds = B.DeviceState(cfg)
    ocfg = P.orc_cfg(w)
    tiles = [oracle.Tile(ocfg, S0[t].astype(np.float64)) for t in range(w.tiles)]
    P.import_records(ds, [tl.rec for tl in tiles])
    dev = P.DeviceInputs(ti, w.io_bf16)
    out_all = torch.full((T, w.batch, w.num_v_heads, w.d), float("nan"), device="cuda")
    # warm-up: n0 tokens one call at a time, the window phase becomes n0
    for t in range(n0):
        B.lq_decode_step(cfg, *dev.token(t), ds.st, out_all[t])
    for tile, tl in enumerate(tiles):
        tl.run(*P.tile_inputs(ti, w, tile, 0, n0))
    # launch 1: W - n0 tokens, ending in the fold
    _launch(cfg, dev, n0, W - n0, ds, out_all)
    o = out_all.cpu().numpy().reshape(T, w.tiles, w.d)
    margins = np.zeros(w.tiles)
    for tile, tl in enumerate(tiles):
        tl.diag = oracle.new_diag()
        ref = tl.run(*P.tile_inputs(ti, w, tile, n0, W))
        for i in range(W - n0):
            err = P.normwise(o[n0 + i, tile].astype(np.float64), ref[i])
            assert err <= P.REL_TOL, (case, n0 + i, tile, err)
        margins[tile] = tl.diag[oracle.D_MIN_MARGIN]
        assert tl.n[0] == 0
    assert np.all(ds.buf_n.cpu().numpy()[:w.tiles] == 0)
    P.assert_records_close(P.compare_records(P.gpu_records(ds), [tl.rec for tl in tiles],
                                             margins))
    P.import_records(ds, [tl.rec for tl in tiles])          # teacher forcing
    # launch 2: 7 tokens, sequence 1 inactive
    act = np.ones(w.batch, dtype=np.int32)
    act[1] = 0
    _launch(cfg, dev, W, 7, ds, out_all, active=torch.from_numpy(act).cuda())
    o = out_all.cpu().numpy().reshape(T, w.batch, w.num_v_heads, w.d)
    for tile, tl in enumerate(tiles):
        b, h = divmod(tile, w.num_v_heads)
        if not act[b]:
            assert np.all(np.isnan(o[W:, b, h]))
            continue
        ref = tl.run(*P.tile_inputs(ti, w, tile, W, T))
        for i in range(7):
            err = P.normwise(o[W + i, b, h].astype(np.float64), ref[i])
            assert err <= P.REL_TOL, (case, W + i, tile, err)
    n_gpu = ds.buf_n.cpu().numpy()[:w.tiles].reshape(w.batch, w.num_v_heads)
    assert np.all(n_gpu[act == 1] == 7) and np.all(n_gpu[act == 0] == 0)
    assert B.lq_get_last_error(ds.st) == B.LQ_OK


def test_decode_tokens_equals_single_steps_and_accepts_zero_tokens():
    """One launch of 20 tokens (a fold inside it) against 20 calls of
    lq_decode_step from the same state: same phases and, within the decode
    bar, the same outputs and records.  ntok = 0 changes nothing."""
    w = wl.Workload("te", 2, 2, 4, 128, wl.GATE_SCALAR, True, 1)
    rng = np.random.default_rng(52)
    S0, _, _ = wl.initial_states(rng, w.tiles, w.d, w.d)
    T = 20
    ti = wl.token_inputs(rng, w, T)
    cfg = B.config_for(w)
    a, b = B.DeviceState(cfg), B.DeviceState(cfg)
    S0_dev = torch.from_numpy(S0).cuda()
    B.lq_state_init(cfg, S0_dev, a.st)
    B.lq_state_init(cfg, S0_dev, b.st)
    dev = P.DeviceInputs(ti, True)
    out_a = torch.empty((T, w.batch, w.num_v_heads, w.d), device="cuda")
    out_b = torch.empty_like(out_a)
    before = b.records.clone()
    B.lq_decode_tokens(cfg, 0, dev.q, dev.k, dev.v, dev.alpha, dev.beta, b.st, out_b)
    assert torch.equal(b.records, before) and torch.all(b.buf_n == 0)
    for t in range(T):
        B.lq_decode_step(cfg, *dev.token(t), a.st, out_a[t])
    _launch(cfg, dev, 0, T, b, out_b)
    assert torch.equal(a.buf_n, b.buf_n)
    oa = out_a.cpu().numpy().reshape(T, w.tiles, w.d).astype(np.float64)
    ob = out_b.cpu().numpy().reshape(T, w.tiles, w.d).astype(np.float64)
    assert np.max(P.normwise(ob, oa)) <= P.REL_TOL
    g_a, g_b = P.gpu_records(a), P.gpu_records(b)
    same = np.all(g_a["cid"] == g_b["cid"], axis=1)      # a near tie may pick another line
    assert same.mean() >= 0.9
    dq = np.abs(g_a["Q"][same].astype(np.int32) - g_b["Q"][same].astype(np.int32))
    assert dq.max() <= 1 and np.count_nonzero(dq) <= 1e-3 * dq.size
    assert B.lq_get_last_error(b.st) == B.LQ_OK
