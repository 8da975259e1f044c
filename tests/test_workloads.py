"""The seeded input generator against the recipe it documents: shapes of the
named workloads, unit-norm q and k, the gate and beta ranges, bf16-exact
values, the planted outlier lines of the initial states (x20 once, also where
a planted row meets a planted column), the fixed x10 value channels of the KDA
workload, the ragged lengths and window phases, and determinism by seed."""
import numpy as np
import pytest

from recurrent_state_quantization_decode_b200 import workloads as wl


def test_named_workload_shapes():
    assert wl.TINY_GDN.tiles == 1 and wl.TINY_GDN.d == 32 and not wl.TINY_GDN.io_bf16
    q = wl.QWEN35_9B_GDN
    assert (q.batch, q.num_k_heads, q.num_v_heads, q.d, q.tiles) == (64, 16, 32, 128, 2048)
    assert q.gate == wl.GATE_SCALAR and q.io_bf16
    k = wl.KIMI_LINEAR_KDA
    assert (k.batch, k.num_k_heads, k.num_v_heads, k.tiles) == (128, 32, 32, 4096)
    assert k.gate == wl.GATE_DIAG and k.v_outlier_channels == 4
    assert [wl.sweep_workload(b).tiles for b in (8, 1024)] == [256, 32768]
    for w in (wl.TINY_GDN, q, k):
        assert (w.window, w.n_comp, w.smooth) == (16, 4, 0.5)


@pytest.mark.parametrize("w", [wl.TINY_GDN, wl.Workload("g", 3, 2, 4, 64, wl.GATE_SCALAR, True, 8),
                               wl.Workload("k", 2, 4, 4, 64, wl.GATE_DIAG, True, 8,
                                           v_outlier_channels=4)])
def test_token_inputs_follow_the_recipe(w):
    T = 40
    ti = wl.token_inputs(np.random.default_rng(3), w, T)
    B, Hk, Hv, d = w.batch, w.num_k_heads, w.num_v_heads, w.d
    assert ti.q.shape == ti.k.shape == (T, B, Hk, d) and ti.v.shape == (T, B, Hv, d)
    assert ti.beta.shape == (T, B, Hv)
    assert ti.alpha.shape == ((T, B, Hv) if w.gate == wl.GATE_SCALAR else (T, B, Hv, d))
    for x in (ti.q, ti.k, ti.v, ti.alpha, ti.beta):
        assert x.dtype == np.float32
    # q and k are unit vectors per head (bf16 rounding moves the norm by < 2^-8)
    tol = 2.0 ** -8 if w.io_bf16 else 1e-6
    for x in (ti.q, ti.k):
        assert np.allclose(np.linalg.norm(x.astype(np.float64), axis=-1), 1.0, atol=tol)
    # bf16 inputs hold bf16-representable values only
    if w.io_bf16:
        for x in (ti.q, ti.k, ti.v):
            np.testing.assert_array_equal(x, wl.to_bf16_values(x))
    assert np.all((ti.beta > 0) & (ti.beta < 1))
    if w.gate == wl.GATE_SCALAR:
        assert np.all((ti.alpha >= 0.9) & (ti.alpha <= 1.0))
    else:
        # exp(-softplus(z) / 20): in (0, 1), exp(-ln 2 / 20) at z = 0
        assert np.all((ti.alpha > 0) & (ti.alpha < 1))
        assert abs(np.median(ti.alpha) - np.exp(-np.log(2.0) * 0.05)) < 0.01


def test_kda_value_outlier_channels_are_fixed_and_ten_times_larger():
    w = wl.Workload("k", 4, 4, 4, 128, wl.GATE_DIAG, False, 8, v_outlier_channels=4)
    a = wl.token_inputs(np.random.default_rng(1), w, 64)
    b = wl.token_inputs(np.random.default_rng(2), w, 64)
    std_a = a.v.reshape(-1, w.d).std(axis=0)
    std_b = b.v.reshape(-1, w.d).std(axis=0)
    big_a = np.sort(np.argsort(std_a)[-4:])
    np.testing.assert_array_equal(big_a, np.sort(np.argsort(std_b)[-4:]))   # same channels
    others = np.setdiff1d(np.arange(w.d), big_a)
    assert np.all(np.abs(std_a[big_a] / 10.0 - 1.0) < 0.15)
    assert np.all(np.abs(std_a[others] - 1.0) < 0.15)


def test_initial_states_plant_rows_and_columns_once():
    rng = np.random.default_rng(5)
    tiles, d = 6, 64
    S, rows, cols = wl.initial_states(rng, tiles, d, d)
    assert S.shape == (tiles, d, d) and S.dtype == np.float32
    # the same draws without planting: the base state, then the chosen lines
    rng2 = np.random.default_rng(5)
    base = (rng2.standard_normal((tiles, d, d)) * 0.02).astype(np.float32)
    for t in range(tiles):
        r = rng2.choice(d, 2, replace=False)
        c = rng2.choice(d, 2, replace=False)
        np.testing.assert_array_equal(r, rows[t])
        np.testing.assert_array_equal(c, cols[t])
        assert len(set(r)) == 2 and len(set(c)) == 2
        planted = np.zeros((d, d), bool)
        planted[r, :] = True
        planted[:, c] = True
        expect = np.where(planted, base[t] * np.float32(20.0), base[t])
        np.testing.assert_array_equal(S[t], expect)       # x20 once, crossings included
    plain = [S[t][np.ix_(np.setdiff1d(np.arange(d), rows[t]), np.setdiff1d(np.arange(d), cols[t]))]
             for t in range(tiles)]
    assert abs(np.concatenate([p.ravel() for p in plain]).std() / 0.02 - 1.0) < 0.05


def test_ragged_lengths_and_phases():
    L, phase = wl.ragged_lengths(np.random.default_rng(9), 4000)
    assert L.dtype == np.int64 and phase.dtype == np.int64
    assert L.min() >= 1 and L.max() <= 32768
    assert set(np.unique(phase)) <= set(range(16)) and len(np.unique(phase)) == 16
    # LogNormal(7, 1): the median is e^7
    assert abs(np.log(np.median(L)) - 7.0) < 0.1
    L2, _ = wl.ragged_lengths(np.random.default_rng(9), 4000, max_len=512)
    assert L2.max() == 512


def test_same_seed_same_inputs():
    w = wl.Workload("g", 2, 2, 4, 32, wl.GATE_SCALAR, True, 4)
    a = wl.token_inputs(np.random.default_rng(7), w, 5)
    b = wl.token_inputs(np.random.default_rng(7), w, 5)
    for n in ("q", "k", "v", "alpha", "beta"):
        np.testing.assert_array_equal(getattr(a, n), getattr(b, n))


def test_device_generator_follows_the_recipe():
    """token_inputs_device (the draws for batches too large for the host) keeps
    the recipe of token_inputs: unit-norm q and k per head (bf16-rounded),
    beta in (0, 1), GDN alpha in [0.9, 1], KDA alpha in (0, 1], shapes, and
    the same stream for the same seed (checked on the CPU device)."""
    import torch

    for w in (wl.RAGGED, wl.KIMI_LINEAR_KDA):
        g1, g2 = torch.Generator(), torch.Generator()
        g1.manual_seed(3)
        g2.manual_seed(3)
        a = wl.token_inputs_device(g1, w, 3, "cpu", batch=2)
        b = wl.token_inputs_device(g2, w, 3, "cpu", batch=2)
        for n in a:
            assert torch.equal(a[n], b[n]), n
        assert a["q"].shape == (3, 2, w.num_k_heads, w.d)
        assert a["v"].shape == (3, 2, w.num_v_heads, w.d)
        assert a["q"].dtype == torch.bfloat16 and a["v"].dtype == torch.bfloat16
        nq = torch.linalg.vector_norm(a["q"].double(), dim=-1)
        assert torch.allclose(nq, torch.ones_like(nq), atol=1e-2)
        assert torch.all((a["beta"] > 0) & (a["beta"] < 1))
        if w.gate == wl.GATE_SCALAR:
            assert a["alpha"].shape == (3, 2, w.num_v_heads)
            assert torch.all((a["alpha"] >= 0.9) & (a["alpha"] <= 1.0))
        else:
            assert a["alpha"].shape == (3, 2, w.num_v_heads, w.d)
            assert torch.all((a["alpha"] > 0) & (a["alpha"] <= 1.0))
