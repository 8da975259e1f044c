"""lq_decode_step_host_noalloc: the host-buffer decode step for callers that
cannot allocate device memory (for example a plugin inside an application that
owns all device allocations).  It stages through the library's own fixed
device array instead of a caller-provided buffer.

Collected last on purpose (file name), so that a run stopping at the first
failure has run everything else first.  Self-contained: it builds its own
states, so it passes alone in a fresh process and after the other tests."""
import numpy as np
import pytest
import torch

from recurrent_state_quantization_decode_b200 import workloads as wl

pytestmark = pytest.mark.gpu

REL_TOL = 1e-3  # the parity tolerance of the other decode tests


def _binding():
    from recurrent_state_quantization_decode_b200 import build

    build.build()
    from recurrent_state_quantization_decode_b200 import binding

    return binding


def test_noalloc_matches_staged_entry_point_on_two_calls():
    B = _binding()
    assert torch.cuda.is_available()
    w = wl.Workload("noalloc", 4, 2, 4, 128, wl.GATE_SCALAR, True, 2)
    rng = np.random.default_rng(21)
    S0, _, _ = wl.initial_states(rng, w.tiles, w.d, w.d)
    ti = wl.token_inputs(rng, w, 2)
    cfg = B.config_for(w)
    assert B.lq_state_layout(cfg).host_staging_bytes <= B.LQ_NOALLOC_STAGING_MAX_BYTES
    ref = B.DeviceState(cfg)
    new = B.DeviceState(cfg)
    S0_dev = torch.from_numpy(S0).cuda()
    B.lq_state_init(cfg, S0_dev, ref.st)
    B.lq_state_init(cfg, S0_dev, new.st)
    host = {n: torch.from_numpy(getattr(ti, n)).to(torch.bfloat16 if n in "qkv" else
                                                    torch.float32).pin_memory()
            for n in ("q", "k", "v", "alpha", "beta")}
    staging = torch.empty(B.lq_state_layout(cfg).host_staging_bytes, dtype=torch.uint8,
                          device="cuda")
    out_ref = torch.empty((w.batch, w.num_v_heads, w.d)).pin_memory()
    out_new = torch.full((w.batch, w.num_v_heads, w.d), float("nan")).pin_memory()
    for t in range(2):                      # two calls in a row
        args = (host["q"][t], host["k"][t], host["v"][t], host["alpha"][t], host["beta"][t])
        B.lq_decode_step_host(cfg, *args, ref.st, out_ref, staging)
        B.lq_decode_step_host_noalloc(cfg, *args, new.st, out_new)
        torch.cuda.synchronize()
        a = out_new.numpy().reshape(w.tiles, w.d).astype(np.float64)
        b = out_ref.numpy().reshape(w.tiles, w.d).astype(np.float64)
        err = np.max(np.abs(a - b), axis=1) / np.max(np.abs(b), axis=1)
        assert np.all(err <= REL_TOL), (t, err.max())
    assert torch.equal(ref.buf_n, new.buf_n)
    assert B.lq_get_last_error(new.st) == B.LQ_OK


def test_noalloc_rejects_problems_above_its_fixed_array():
    B = _binding()
    # KDA inputs of 512 sequences x 32 heads need far more than the fixed array
    cfg = B.make_config(512, 32, 32, 128, gate=B.LQ_GATE_DIAG, in_bf16=True)
    assert B.lq_state_layout(cfg).host_staging_bytes > B.LQ_NOALLOC_STAGING_MAX_BYTES
    good = 1 << 20
    st = B.lq_state(good, good, good, good, good, good)
    with pytest.raises(B.LQError) as ei:
        B.lq_decode_step_host_noalloc(cfg, good, good, good, good, good, st, good, stream=0)
    assert ei.value.status == B.LQ_ERR_TOO_LARGE
