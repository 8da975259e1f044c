"""The C-ABI library without a GPU: it loads, exports every symbol the header
declares, lays out the state as the pages account for it, and rejects bad
arguments on the host before launching anything."""
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def B():
    from recurrent_state_quantization_decode_b200 import build

    build.build()
    from recurrent_state_quantization_decode_b200 import binding

    return binding


def _declared():
    txt = open(os.path.join(ROOT, "include", "leapquant.h")).read()
    txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
    return sorted(set(re.findall(r"\b(lq_[a-z0-9_]+)\s*\(", txt)))


def test_exports_every_declared_symbol(B):
    names = _declared()
    assert len(names) == 19
    assert sorted(B.EXPORTED) == names
    for n in names:
        assert hasattr(B._lib, n), n
    assert B.lq_version() == 1


def test_layout_matches_page_accounting(B):
    cfg = B.make_config(1, 1, 1, 128, 16, 4)
    L = B.lq_state_layout(cfg)
    assert L.record_bytes == 19472
    assert (L.off_sigma, L.off_m, L.off_comp_vec, L.off_comp_id) == (16384, 16896, 17408, 19456)
    assert round(L.record_bytes / 128**2, 2) == 1.19
    total, tile, buf = B.lq_state_bytes(cfg)
    assert tile == 19472 and total == L.records_bytes + buf + 4
    # grouped heads: buffered keys are stored once per key head
    g = B.make_config(64, 16, 32, 128, 16, 4, in_bf16=True)
    L = B.lq_state_layout(g)
    assert L.buf_k_bytes == 64 * 16 * 16 * 128 * 2
    assert L.buf_d_bytes == 64 * 32 * 16 * 128 * 4
    assert L.buf_g_bytes == 64 * 32 * 16 * 4
    kda = B.make_config(2, 4, 4, 64, 16, 4, gate=B.LQ_GATE_DIAG)
    assert B.lq_state_layout(kda).buf_g_bytes == 2 * 4 * 16 * 64 * 4
    for d in (32, 64, 128):
        for K in range(9):
            assert B.lq_state_layout(B.make_config(1, 1, 1, d, 16, K)).record_bytes % 16 == 0


@pytest.mark.parametrize("field,value,status", [
    ("d", 96, 2), ("d", 256, 2), ("window", 0, 2), ("window", 33, 2), ("n_comp", 9, 2),
    ("n_comp", -1, 2), ("smooth", 0.25, 2), ("batch", -1, 1), ("num_k_heads", 0, 1),
    ("num_v_heads", 3, 1), ("gate", 2, 1), ("in_dtype", 5, 1),
])
def test_bad_config_rejected_on_host(B, field, value, status):
    cfg = B.make_config(2, 2, 4, 64)
    setattr(cfg, field, value)
    with pytest.raises(B.LQError) as ei:
        B.lq_state_layout(cfg)
    assert ei.value.status == status
    assert B.lq_state_bytes(cfg)[0] == 0


def test_bad_pointers_rejected_before_launch(B):
    cfg = B.make_config(2, 2, 4, 64)
    good = 1 << 20  # never dereferenced: validation fails first
    st = B.lq_state(good, good, good, good, good, good)
    with pytest.raises(B.LQError) as ei:
        B.lq_decode_step(cfg, good, good, good, good, good, st, None, stream=0)
    assert ei.value.status == B.LQ_ERR_INVALID_ARG
    st_bad = B.lq_state(good + 4, good, good, good, good, good)
    with pytest.raises(B.LQError) as ei:
        B.lq_decode_step(cfg, good, good, good, good, good, st_bad, good, stream=0)
    assert ei.value.status == B.LQ_ERR_MISALIGNED
    with pytest.raises(B.LQError) as ei:
        B.lq_decode_step(cfg, good + 2, good, good, good, good, st, good, stream=0)
    assert ei.value.status == B.LQ_ERR_MISALIGNED
    with pytest.raises(B.LQError) as ei:
        B.lq_fp32_decode_step(cfg, good, good, good, good, good, good + 8, good, stream=0)
    assert ei.value.status == B.LQ_ERR_MISALIGNED
    with pytest.raises(B.LQError) as ei:
        B.lq_state_init(cfg, None, st, stream=0)
    assert ei.value.status == B.LQ_ERR_INVALID_ARG
    with pytest.raises(B.LQError) as ei:
        B.lq_decode_step_host(cfg, good, good, good, good, good, st, good, None, stream=0)
    assert ei.value.status == B.LQ_ERR_INVALID_ARG
    assert B.lq_get_last_error(B.lq_state(0, 0, 0, 0, 0, 0), 0) == B.LQ_ERR_INVALID_ARG
    # packed inputs: the block pointer, GDN's separate gates and beta are required
    # and aligned; windows above 16 tokens are refused
    with pytest.raises(B.LQError) as ei:
        B.lq_decode_step_packed(cfg, None, good, good, st, good, stream=0)
    assert ei.value.status == B.LQ_ERR_INVALID_ARG
    with pytest.raises(B.LQError) as ei:
        B.lq_decode_step_packed(cfg, good, None, good, st, good, stream=0)
    assert ei.value.status == B.LQ_ERR_INVALID_ARG
    with pytest.raises(B.LQError) as ei:
        B.lq_decode_step_packed(cfg, good + 8, good, good, st, good, stream=0)
    assert ei.value.status == B.LQ_ERR_MISALIGNED
    kda = B.make_config(2, 2, 2, 64, gate=B.LQ_GATE_DIAG)
    with pytest.raises(B.LQError) as ei:                  # KDA: gates inside the blocks
        B.lq_decode_step_packed(kda, good, None, good + 2, st, good, stream=0)
    assert ei.value.status == B.LQ_ERR_MISALIGNED
    w32 = B.make_config(2, 2, 4, 64, 32)
    with pytest.raises(B.LQError) as ei:
        B.lq_decode_step_packed(w32, good, good, good, st, good, stream=0)
    assert ei.value.status == B.LQ_ERR_UNSUPPORTED


def test_empty_batch_is_a_no_op(B):
    cfg = B.make_config(0, 2, 4, 64)
    good = 1 << 20
    st = B.lq_state(good, good, good, good, good, good)
    # batch == 0 returns LQ_OK without touching the device
    B.lq_decode_step(cfg, good, good, good, good, good, st, good, stream=0)
    B.lq_window_flush(cfg, st, stream=0)
    B.lq_fp32_decode_step(cfg, good, good, good, good, good, good, good, stream=0)


def test_status_strings(B):
    for s in range(8):
        assert B.lq_status_string(s).startswith("LQ_")


def _err(B, fn, *args, **kw):
    with pytest.raises(B.LQError) as ei:
        fn(*args, **kw)
    return ei.value.status


def test_newer_entry_points_reject_bad_arguments_before_launch(B):
    """Prefill, checkpoint copies, rollback, the host-buffer step and the
    timeout test hook: argument errors come back on the host, with no device
    access (addresses below are never dereferenced)."""
    cfg = B.make_config(2, 2, 4, 64)
    good = 1 << 20
    st = B.lq_state(good, good, good, good, good, good)
    # prefill: negative length, missing inputs for a non-empty prompt, misaligned S0
    assert _err(B, B.lq_prefill, cfg, good, good, good, good, good, -1, None, st,
                stream=0) == B.LQ_ERR_INVALID_ARG
    assert _err(B, B.lq_prefill, cfg, None, good, good, good, good, 8, None, st,
                stream=0) == B.LQ_ERR_INVALID_ARG
    assert _err(B, B.lq_prefill, cfg, good, good, good, good, good, 8, good + 4, st,
                stream=0) == B.LQ_ERR_MISALIGNED
    assert _err(B, B.lq_prefill, cfg, good, good, good, good + 2, good, 8, None, st,
                stream=0) == B.LQ_ERR_MISALIGNED
    # checkpoint copies: missing slots or pool, negative pool size, misaligned pool
    for save in (True, False):
        def call(slots, pool, n):
            if save:
                return B.lq_checkpoint_save(cfg, st, slots, pool, n, stream=0)
            return B.lq_checkpoint_restore(cfg, pool, n, slots, st, stream=0)
        assert _err(B, call, None, good, 1) == B.LQ_ERR_INVALID_ARG
        assert _err(B, call, good, None, 1) == B.LQ_ERR_INVALID_ARG
        assert _err(B, call, good, good, -1) == B.LQ_ERR_INVALID_ARG
        assert _err(B, call, good, good + 8, 1) == B.LQ_ERR_MISALIGNED
        assert _err(B, call, good + 2, good, 1) == B.LQ_ERR_MISALIGNED
    # rollback: missing or misaligned drop counts
    assert _err(B, B.lq_window_rewind, cfg, st, None, stream=0) == B.LQ_ERR_INVALID_ARG
    assert _err(B, B.lq_window_rewind, cfg, st, good + 2, stream=0) == B.LQ_ERR_MISALIGNED
    # host-buffer step: misaligned staging or mask
    assert _err(B, B.lq_decode_step_host, cfg, good, good, good, good, good, st, good,
                good + 8, stream=0) == B.LQ_ERR_MISALIGNED
    assert _err(B, B.lq_decode_step_host, cfg, good, good, good, good, good, st, good, good,
                active=good + 1, stream=0) == B.LQ_ERR_MISALIGNED
    # the no-alloc host step checks every argument before it looks up or
    # touches its array: without a GPU these come back as argument errors,
    # not as a CUDA error from the lookup
    assert _err(B, B.lq_decode_step_host_noalloc, cfg, None, good, good, good, good, st,
                good, stream=0) == B.LQ_ERR_INVALID_ARG
    assert _err(B, B.lq_decode_step_host_noalloc, cfg, good, good, good, good, good, st,
                good, active=good + 1, stream=0) == B.LQ_ERR_MISALIGNED
    assert _err(B, B.lq_decode_step_host_noalloc, cfg, good + 4, good, good, good, good, st,
                good, stream=0) == B.LQ_ERR_MISALIGNED
    assert _err(B, B.lq_decode_step_host_noalloc, bad_cfg := B.make_config(2, 2, 4, 96), good,
                good, good, good, good, st, good, stream=0) == B.LQ_ERR_UNSUPPORTED
    big = B.make_config(4096, 32, 32, 128)        # staging above the fixed array
    assert B.lq_state_layout(big).host_staging_bytes > B.LQ_NOALLOC_STAGING_MAX_BYTES
    assert _err(B, B.lq_decode_step_host_noalloc, big, good, good, good, good, good, st, good,
                stream=0) == B.LQ_ERR_TOO_LARGE
    del bad_cfg
    # timeout hook: a zero poll limit or an empty batch is refused
    assert _err(B, B.lq_test_decode_step_timeout, cfg, good, good, good, good, good, st, good,
                0, stream=0) == B.LQ_ERR_INVALID_ARG
    empty = B.make_config(0, 2, 4, 64)
    assert _err(B, B.lq_test_decode_step_timeout, empty, good, good, good, good, good, st,
                good, 16, stream=0) == B.LQ_ERR_INVALID_ARG
    # a bad config is reported before anything else
    bad = B.make_config(2, 2, 4, 96)
    assert _err(B, B.lq_prefill, bad, good, good, good, good, good, 8, None, st,
                stream=0) == B.LQ_ERR_UNSUPPORTED
    assert _err(B, B.lq_window_rewind, bad, st, good, stream=0) == B.LQ_ERR_UNSUPPORTED


def test_newer_entry_points_accept_an_empty_batch(B):
    """batch == 0 returns LQ_OK without touching the device."""
    cfg = B.make_config(0, 2, 4, 64)
    good = 1 << 20
    st = B.lq_state(good, good, good, good, good, good)
    B.lq_prefill(cfg, good, good, good, good, good, 8, good, st, stream=0)
    B.lq_prefill(cfg, None, None, None, None, None, 0, None, st, stream=0)
    B.lq_checkpoint_save(cfg, st, good, good, 4, stream=0)
    B.lq_checkpoint_restore(cfg, good, 4, good, st, stream=0)
    B.lq_window_rewind(cfg, st, good, stream=0)
    B.lq_decode_step_host(cfg, good, good, good, good, good, st, good, good, stream=0)
    B.lq_decode_step_host_noalloc(cfg, good, good, good, good, good, st, good, stream=0)
    B.lq_state_init(cfg, good, st, stream=0)
