"""lq_prefill: the exact recurrence over a prompt in chunks of 16 tokens (WY
form, products with the state on the tf32 tensor path), then the quantizer.

Outputs are compared with the oracle's exact fp64 recurrence, the record with
the oracle's quantizer applied to the exact final state (codes within one
step on at most 0.1 % of entries, compensator ids equal except at near
ties), and a prefilled state must decode on like the oracle's."""
import numpy as np
import pytest
import torch

import oracle
from recurrent_state_quantization_decode_b200 import workloads as wl

pytestmark = pytest.mark.gpu

import sys, os  # noqa: E401,E402
sys.path.insert(0, os.path.dirname(os.path.abspath(__file__)))
import _parity as P  # noqa: E402

B = P.B
EXACT_TOL = 1e-4   # fp32 recurrence against fp64 over the prompt

CASES = {
    "gdn_bf16_d128": (wl.Workload("p", 3, 4, 8, 128, wl.GATE_SCALAR, True, 1), 96, True),
    "kda_bf16_d128": (wl.Workload("pk", 2, 8, 8, 128, wl.GATE_DIAG, True, 1,
                                  v_outlier_channels=4), 64, True),
    "gdn_f32_d64_zero_start": (wl.Workload("p64", 2, 2, 4, 64, wl.GATE_SCALAR, False, 1),
                               80, False),
    "tiny_d32": (wl.Workload("p32", 1, 1, 2, 32, wl.GATE_SCALAR, False, 1), 50, True),
    # a last chunk of one token, KDA at d = 32
    "kda_f32_d32_T17": (wl.Workload("pk32", 2, 1, 2, 32, wl.GATE_DIAG, False, 1), 17, True),
    # a prompt shorter than one chunk
    "gdn_bf16_d128_T5": (wl.Workload("p5", 1, 2, 4, 128, wl.GATE_SCALAR, True, 1), 5, True),
}


@pytest.mark.parametrize("case", sorted(CASES))
def test_prefill_matches_exact_recurrence_then_quantizes(case):
    w, T, with_s0 = CASES[case]
    rng = np.random.default_rng(31)
    S0, _, _ = wl.initial_states(rng, w.tiles, w.d, w.d)
    if not with_s0:
        S0 = np.zeros_like(S0)
    ti = wl.token_inputs(rng, w, T)
    cfg = B.config_for(w)
    ds = B.DeviceState(cfg)
    dev = P.DeviceInputs(ti, w.io_bf16)
    out = torch.full((T, w.batch, w.num_v_heads, w.d), float("nan"), device="cuda")
    B.lq_prefill(cfg, dev.q, dev.k, dev.v, dev.alpha, dev.beta, T,
                 torch.from_numpy(S0).cuda() if with_s0 else None, ds.st, out)
    assert B.lq_get_last_error(ds.st) == B.LQ_OK
    o_gpu = out.cpu().numpy().astype(np.float64)
    assert np.all(ds.buf_n.cpu().numpy() == 0)
    ocfg = P.orc_cfg(w)
    recs, margins, exact_states = [], [], []
    for tile in range(w.tiles):
        b, h = divmod(tile, w.num_v_heads)
        hk = h // (w.num_v_heads // w.num_k_heads)
        S_T, o_ex = oracle.exact_run(ocfg, S0[tile].astype(np.float64), ti.q[:, b, hk],
                                     ti.k[:, b, hk], ti.v[:, b, h], ti.alpha[:, b, h],
                                     ti.beta[:, b, h])
        err = P.normwise(o_gpu[:, b, h], o_ex)
        assert np.all(err <= EXACT_TOL), (case, tile, float(err.max()))
        diag = oracle.new_diag()
        recs.append(oracle.quantize(ocfg, S_T, diag))
        margins.append(diag[oracle.D_MIN_MARGIN])
        exact_states.append(S_T)
    P.assert_records_close(P.compare_records(P.gpu_records(ds), recs, np.array(margins)))

    # the prefilled state decodes on like the oracle started from S_T
    ti2 = wl.token_inputs(rng, w, 1)
    dev2 = P.DeviceInputs(ti2, w.io_bf16)
    o2 = torch.empty((w.batch, w.num_v_heads, w.d), device="cuda")
    B.lq_decode_step(cfg, *dev2.token(0), ds.st, o2)
    o2 = o2.cpu().numpy().reshape(w.tiles, w.d).astype(np.float64)
    g = P.gpu_records(ds)
    for tile in range(w.tiles):
        tl = oracle.Tile(ocfg, exact_states[tile])
        if w.n_comp and not np.array_equal(g["cid"][tile], tl.rec.cid[:w.n_comp]):
            continue            # a near-tie pick: the decode starts from another record
        ref = tl.run(*P.tile_inputs(ti2, w, tile, 0, 1))[0]
        assert P.normwise(o2[tile], ref) <= P.REL_TOL, (case, tile)


def test_prefill_of_zero_tokens_is_init():
    w = wl.Workload("p0", 2, 2, 4, 128, wl.GATE_SCALAR, True, 1)
    rng = np.random.default_rng(32)
    S0, _, _ = wl.initial_states(rng, w.tiles, w.d, w.d)
    cfg = B.config_for(w)
    a, b = B.DeviceState(cfg), B.DeviceState(cfg)
    S0_dev = torch.from_numpy(S0).cuda()
    B.lq_state_init(cfg, S0_dev, a.st)
    B.lq_prefill(cfg, None, None, None, None, None, 0, S0_dev, b.st)
    torch.cuda.synchronize()
    assert torch.equal(a.records, b.records)
    assert B.lq_get_last_error(b.st) == B.LQ_OK


def test_checkpoint_pool_roundtrip_errors_and_accounting():
    """lq_checkpoint_save / restore: a round trip is bit-exact and decodes on
    identically; a tile off a window boundary or a slot past the pool is
    refused through the error word; one checkpoint costs Hv records."""
    w = wl.Workload("ck", 4, 2, 4, 128, wl.GATE_SCALAR, True, 1)
    rng = np.random.default_rng(33)
    S0, _, _ = wl.initial_states(rng, w.tiles, w.d, w.d)
    ti = wl.token_inputs(rng, w, 3)
    cfg = B.config_for(w)
    L = B.lq_state_layout(cfg)
    pool = torch.zeros(2 * w.num_v_heads * L.record_bytes, dtype=torch.uint8, device="cuda")
    # one checkpoint: Hv records against Hv fp32 states
    assert L.record_bytes == 19472
    assert round(65536 / L.record_bytes, 2) == 3.37
    ds = B.DeviceState(cfg)
    B.lq_state_init(cfg, torch.from_numpy(S0).cuda(), ds.st)
    slots = torch.tensor([1, -1, 0, -1], dtype=torch.int32, device="cuda")
    B.lq_checkpoint_save(cfg, ds.st, slots, pool, 2)
    assert B.lq_get_last_error(ds.st) == B.LQ_OK
    rec = ds.record_view()
    pv = pool.view(2, w.num_v_heads, L.record_bytes)
    hv = w.num_v_heads
    assert torch.equal(pv[1], rec[0:hv]) and torch.equal(pv[0], rec[2 * hv:3 * hv])
    # restore into a fresh state: both decode the next tokens identically
    ds2 = B.DeviceState(cfg)
    B.lq_state_init(cfg, torch.zeros_like(torch.from_numpy(S0)).cuda(), ds2.st)
    B.lq_checkpoint_restore(cfg, pool, 2, slots, ds2.st)
    dev = P.DeviceInputs(ti, True)
    act = torch.tensor([1, 0, 1, 0], dtype=torch.int32, device="cuda")
    o1 = torch.empty((w.batch, hv, w.d), device="cuda")
    o2 = torch.empty_like(o1)
    for t in range(2):
        B.lq_decode_step(cfg, *dev.token(t), ds.st, o1, active=act)
        B.lq_decode_step(cfg, *dev.token(t), ds2.st, o2, active=act)
        assert torch.equal(o1[0], o2[0]) and torch.equal(o1[2], o2[2])
    # sequence 0 is now off a window boundary: its save is refused
    B.lq_checkpoint_save(cfg, ds.st, slots, pool, 2)
    assert B.lq_get_last_error(ds.st) == B.LQ_ERR_DEVICE_BOUNDS
    # a slot past the pool is refused too
    bad = torch.tensor([5, -1, -1, -1], dtype=torch.int32, device="cuda")
    B.lq_checkpoint_restore(cfg, pool, 2, bad, ds2.st)
    assert B.lq_get_last_error(ds2.st) == B.LQ_ERR_DEVICE_BOUNDS
