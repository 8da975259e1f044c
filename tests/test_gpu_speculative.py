"""lq_window_rewind: rejecting speculative draft tokens inside a window.

Within a window the record is fixed and decoded tokens are appended buffer
entries, so dropping the last ones must leave exactly the state that never
saw them: continuing from it reproduces, bit for bit, a run that decoded
only the accepted tokens.  A drop across a window boundary is refused."""
import os
import sys

import numpy as np
import pytest
import torch

import oracle
from recurrent_state_quantization_decode_b200 import workloads as wl

pytestmark = pytest.mark.gpu

sys.path.insert(0, os.path.dirname(os.path.abspath(__file__)))
import _parity as P  # noqa: E402

B = P.B


@pytest.mark.parametrize("gate", [wl.GATE_SCALAR, wl.GATE_DIAG])
def test_rewind_matches_decoding_only_the_accepted_tokens(gate):
    w = wl.Workload("sp", 3, 2, 4, 128, gate, True, 1)
    rng = np.random.default_rng(41)
    S0, _, _ = wl.initial_states(rng, w.tiles, w.d, w.d)
    ti = wl.token_inputs(rng, w, 12)
    cfg = B.config_for(w)
    spec, ref = B.DeviceState(cfg), B.DeviceState(cfg)
    S0_dev = torch.from_numpy(S0).cuda()
    B.lq_state_init(cfg, S0_dev, spec.st)
    B.lq_state_init(cfg, S0_dev, ref.st)
    dev = P.DeviceInputs(ti, True)
    out_s = torch.empty((w.batch, w.num_v_heads, w.d), device="cuda")
    out_r = torch.empty_like(out_s)

    def mask(bits):
        return torch.tensor(bits, dtype=torch.int32, device="cuda")

    for t in range(3):                                  # accepted history
        B.lq_decode_step(cfg, *dev.token(t), spec.st, out_s)
        B.lq_decode_step(cfg, *dev.token(t), ref.st, out_r)
    accepted = [0, 3, 5]                                # of the 5 draft tokens 3..7
    for t in range(3, 8):
        B.lq_decode_step(cfg, *dev.token(t), spec.st, out_s)
        B.lq_decode_step(cfg, *dev.token(t), ref.st, out_r,
                         active=mask([int(t - 3 < a) for a in accepted]))
    B.lq_window_rewind(cfg, spec.st, mask([5 - a for a in accepted]))
    assert torch.equal(spec.buf_n, ref.buf_n)
    for t in range(8, 12):                              # both continue alike
        B.lq_decode_step(cfg, *dev.token(t), spec.st, out_s)
        B.lq_decode_step(cfg, *dev.token(t), ref.st, out_r)
        assert torch.equal(out_s, out_r), t
    assert B.lq_get_last_error(spec.st) == B.LQ_OK
    assert B.lq_get_last_error(ref.st) == B.LQ_OK


@pytest.mark.parametrize("gate", [wl.GATE_SCALAR, wl.GATE_DIAG])
def test_rewind_then_continue_matches_the_oracle(gate):
    """Draft, reject, continue through the next fold, against the oracle run
    on the accepted tokens only.  Sequence b keeps `accepted[b]` of 6 draft
    tokens; the GPU decodes all drafts, rewinds the rest, then decodes 14
    more tokens, which closes every sequence's window.  Every output after
    the rewind must meet the decode bar against the oracle, and at each
    sequence's fold the record must match (teacher-forced afterwards)."""
    w = wl.Workload("spo", 3, 2, 4, 128, gate, True, 1)
    rng = np.random.default_rng(43)
    S0, _, _ = wl.initial_states(rng, w.tiles, w.d, w.d)
    T = 4 + 6 + 14
    ti = wl.token_inputs(rng, w, T)
    cfg = B.config_for(w)
    ds = B.DeviceState(cfg)
    ocfg = P.orc_cfg(w)
    tiles = [oracle.Tile(ocfg, S0[t].astype(np.float64)) for t in range(w.tiles)]
    P.import_records(ds, [tl.rec for tl in tiles])     # both sides start from one record
    dev = P.DeviceInputs(ti, True)
    out = torch.empty((w.batch, w.num_v_heads, w.d), device="cuda")
    accepted = [0, 4, 6]
    history, drafts, cont = range(0, 4), range(4, 10), range(10, T)
    for t in list(history) + list(drafts):
        B.lq_decode_step(cfg, *dev.token(t), ds.st, out)
    B.lq_window_rewind(cfg, ds.st,
                       torch.tensor([6 - a for a in accepted], dtype=torch.int32, device="cuda"))
    # the oracle sees the history and each sequence's accepted drafts only
    for tile in range(w.tiles):
        b = tile // w.num_v_heads
        toks = list(history) + list(drafts)[:accepted[b]]
        ins = [P.tile_inputs(ti, w, tile, t, t + 1) for t in toks]
        tiles[tile].run(*[np.concatenate([x[i] for x in ins]) for i in range(5)])
    n_gpu = ds.buf_n.cpu().numpy()[:w.tiles]
    assert list(n_gpu) == [int(tl.n[0]) for tl in tiles]
    rv = ds.record_view()
    folds = 0
    for t in cont:
        B.lq_decode_step(cfg, *dev.token(t), ds.st, out)
        o = out.cpu().numpy().reshape(w.tiles, w.d)
        closed = []
        for tile in range(w.tiles):
            tl = tiles[tile]
            tl.diag = oracle.new_diag()
            ref = tl.run(*P.tile_inputs(ti, w, tile, t, t + 1))[0]
            assert P.normwise(o[tile].astype(np.float64), ref) <= P.REL_TOL, (t, tile)
            if tl.n[0] == 0:
                closed.append(tile)
        if closed:
            g = P.gpu_records(ds)
            margins = np.array([tiles[c].diag[oracle.D_MIN_MARGIN] for c in closed])
            P.assert_records_close(P.compare_records(g, [tiles[c].rec for c in closed],
                                                     margins, tiles=closed))
            for c in closed:
                rv[c] = torch.from_numpy(P.pack_record(tiles[c].rec, ds.layout, w.d,
                                                       w.n_comp)).cuda()
            folds += len(closed)
    assert folds == w.tiles                       # every sequence folded once after the rewind
    assert B.lq_get_last_error(ds.st) == B.LQ_OK


def test_rewind_across_a_window_boundary_is_refused():
    w = wl.Workload("sp2", 2, 2, 4, 64, wl.GATE_SCALAR, True, 1, window=4)
    rng = np.random.default_rng(42)
    S0, _, _ = wl.initial_states(rng, w.tiles, w.d, w.d)
    ti = wl.token_inputs(rng, w, 6)
    cfg = B.config_for(w)
    ds = B.DeviceState(cfg)
    B.lq_state_init(cfg, torch.from_numpy(S0).cuda(), ds.st)
    dev = P.DeviceInputs(ti, True)
    out = torch.empty((w.batch, w.num_v_heads, w.d), device="cuda")
    for t in range(6):                                  # a fold after token 3
        B.lq_decode_step(cfg, *dev.token(t), ds.st, out)
    before = ds.buf_n.clone()
    assert int(before[0]) == 2
    B.lq_window_rewind(cfg, ds.st, torch.tensor([3, 1], dtype=torch.int32, device="cuda"))
    assert B.lq_get_last_error(ds.st) == B.LQ_ERR_DEVICE_BOUNDS
    after = ds.buf_n.cpu().numpy().reshape(w.batch, w.num_v_heads)
    assert np.all(after[0] == 2) and np.all(after[1] == 1)   # sequence 0 refused, 1 dropped one
