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

def _binding():
    from recurrent_state_quantization_decode_b200 import build

    build.build()
    from recurrent_state_quantization_decode_b200 import binding

    return binding


def test_noalloc_matches_staged_entry_point_on_two_calls():
    """Two calls in a row, then a third with an active mask: the no-alloc
    step runs the same gather and decode kernels on the same bytes as the
    staged entry point, so outputs and states must agree bit for bit; rows
    of inactive sequences come back holding what the caller's buffer held."""
    B = _binding()
    assert torch.cuda.is_available()
    w = wl.Workload("noalloc", 4, 2, 4, 128, wl.GATE_SCALAR, True, 3)
    rng = np.random.default_rng(21)
    S0, _, _ = wl.initial_states(rng, w.tiles, w.d, w.d)
    ti = wl.token_inputs(rng, w, 3)
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
        assert torch.isfinite(out_new).all(), t
        np.testing.assert_array_equal(out_new.numpy(), out_ref.numpy(), err_msg=f"call {t}")
    # third call: sequences 1 and 3 inactive; their rows keep a marker value
    active = torch.tensor([1, 0, 1, 0], dtype=torch.int32, device="cuda")
    out_ref.fill_(-7.0)
    out_new.fill_(-7.0)
    args = (host["q"][2], host["k"][2], host["v"][2], host["alpha"][2], host["beta"][2])
    B.lq_decode_step_host(cfg, *args, ref.st, out_ref, staging, active=active)
    B.lq_decode_step_host_noalloc(cfg, *args, new.st, out_new, active=active)
    torch.cuda.synchronize()
    o = out_new.numpy()
    np.testing.assert_array_equal(o, out_ref.numpy())
    assert np.all(o[[1, 3]] == -7.0)
    assert np.all(np.isfinite(o[[0, 2]])) and not np.any(o[[0, 2]] == -7.0)
    assert torch.equal(ref.buf_n, new.buf_n)
    assert torch.equal(ref.records, new.records)
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
