"""Glue for GPU-vs-oracle parity tests: runs the same seeded inputs through
libleapquant (via the binding) and through the CPU oracle, and compares.

Tolerances (from the decode step's parity bar):
  * floating point: max relative error 1e-3, normwise per vector (max |diff|
    over a vector / max |reference| over it);
  * int8 codes: equal except +-1 on at most 0.1 % of the entries (rounding
    ties, since the GPU folds in fp32 and the oracle in fp64);
  * compensator ids: equal, unless the oracle's selection margin at that fold
    is below 1e-9 relative (a near tie), in which case either line is valid.
"""
from __future__ import annotations

import dataclasses

import numpy as np
import torch

import oracle
from recurrent_state_quantization_decode_b200 import binding as B
from recurrent_state_quantization_decode_b200 import workloads as wl

REL_TOL = 1e-3
CODE_MISMATCH_FRAC = 1e-3
NEAR_TIE_MARGIN = 1e-9


def orc_cfg(w: wl.Workload, quant: int = 1) -> oracle.Cfg:
    return oracle.Cfg(w.d, w.d, W=w.window, K=w.n_comp, gate=w.gate, quant=quant,
                      smooth=w.smooth)


def normwise(x: np.ndarray, ref: np.ndarray, axis=-1) -> np.ndarray:
    num = np.max(np.abs(x - ref), axis=axis)
    den = np.maximum(np.max(np.abs(ref), axis=axis), 1e-30)
    return num / den


# --------------------------------------------------------------------------
# Records in the public byte layout
# --------------------------------------------------------------------------

def unpack_records(raw: np.ndarray, layout, d: int, K: int) -> dict:
    """raw [tiles, record_bytes] uint8 -> dict of per-tile arrays."""
    raw = np.ascontiguousarray(raw)
    T = raw.shape[0]
    L = layout
    Q = raw[:, :d * d].copy().view(np.int8).reshape(T, d, d)
    sig = raw[:, L.off_sigma:L.off_sigma + 4 * d].copy().view(np.float32)
    m = raw[:, L.off_m:L.off_m + 4 * d].copy().view(np.float32)
    cv = raw[:, L.off_comp_vec:L.off_comp_vec + 4 * K * d].copy().view(np.float32)
    cid = raw[:, L.off_comp_id:L.off_comp_id + 4 * K].copy().view(np.int32)
    return {"Q": Q, "sig": sig, "m": m, "cv": cv.reshape(T, K, d), "cid": cid.reshape(T, K)}


def pack_record(rec: oracle.Record, layout, d: int, K: int) -> np.ndarray:
    out = np.zeros(layout.record_bytes, dtype=np.uint8)
    out[:d * d] = rec.Q.reshape(-1).view(np.uint8)
    out[layout.off_sigma:layout.off_sigma + 4 * d] = rec.sig.view(np.uint8)
    out[layout.off_m:layout.off_m + 4 * d] = rec.m.view(np.uint8)
    if K:
        out[layout.off_comp_vec:layout.off_comp_vec + 4 * K * d] = \
            np.ascontiguousarray(rec.cv[:K, :d]).view(np.uint8).reshape(-1)
        out[layout.off_comp_id:layout.off_comp_id + 4 * K] = rec.cid[:K].view(np.uint8)
    return out


def gpu_records(ds: B.DeviceState) -> dict:
    c = ds.cfg
    return unpack_records(ds.record_view().cpu().numpy(), ds.layout, c.d, c.n_comp)


def import_records(ds: B.DeviceState, recs: list) -> None:
    """Write oracle records for every tile and empty the buffers."""
    c = ds.cfg
    raw = np.stack([pack_record(r, ds.layout, c.d, c.n_comp) for r in recs])
    ds.record_view().copy_(torch.from_numpy(raw).to(ds.records.device))
    ds.buf_n.zero_()


@dataclasses.dataclass
class RecordDiff:
    max_code_diff: int
    code_mismatch: int
    entries: int
    max_sig_err: float
    max_m_err: float
    max_cv_err: float
    id_mismatch_tiles: list


def compare_records(g: dict, o: list, margins: np.ndarray, tiles=None) -> RecordDiff:
    """g: unpacked GPU records (all tiles); o: oracle Records for `tiles`."""
    tiles = list(range(len(o))) if tiles is None else list(tiles)
    maxd, mism, ent, es, em, ec, bad_ids = 0, 0, 0, 0.0, 0.0, 0.0, []
    for i, t in enumerate(tiles):
        r = o[i]
        K = g["cid"].shape[1]
        if K and not np.array_equal(g["cid"][t], r.cid[:K]):
            bad_ids.append((t, margins[i]))
            continue
        dq = np.abs(g["Q"][t].astype(np.int32) - r.Q.astype(np.int32))
        maxd = max(maxd, int(dq.max()))
        mism += int(np.count_nonzero(dq))
        ent += dq.size
        es = max(es, float(normwise(g["sig"][t].astype(np.float64), r.sig.astype(np.float64))))
        em = max(em, float(normwise(g["m"][t].astype(np.float64), r.m.astype(np.float64))))
        if K:
            ec = max(ec, float(np.max(normwise(g["cv"][t].astype(np.float64),
                                               r.cv[:K].astype(np.float64)))))
    return RecordDiff(maxd, mism, ent, es, em, ec, bad_ids)


def assert_records_close(diff: RecordDiff) -> None:
    for t, margin in diff.id_mismatch_tiles:
        assert margin < NEAR_TIE_MARGIN, f"tile {t}: compensator ids differ, margin {margin}"
    assert diff.max_code_diff <= 1, diff
    assert diff.code_mismatch <= CODE_MISMATCH_FRAC * max(diff.entries, 1), diff
    assert diff.max_sig_err <= REL_TOL and diff.max_m_err <= REL_TOL, diff
    assert diff.max_cv_err <= REL_TOL, diff


# --------------------------------------------------------------------------
# Inputs on the device
# --------------------------------------------------------------------------

class DeviceInputs:
    """All T tokens of a TokenInputs on the GPU, token-major."""

    def __init__(self, ti: wl.TokenInputs, in_bf16: bool, device="cuda"):
        dt = torch.bfloat16 if in_bf16 else torch.float32
        self.q = torch.from_numpy(ti.q).to(device=device, dtype=dt).contiguous()
        self.k = torch.from_numpy(ti.k).to(device=device, dtype=dt).contiguous()
        self.v = torch.from_numpy(ti.v).to(device=device, dtype=dt).contiguous()
        self.alpha = torch.from_numpy(ti.alpha).to(device=device).contiguous()
        self.beta = torch.from_numpy(ti.beta).to(device=device).contiguous()
        self.T = ti.q.shape[0]

    def token(self, t: int):
        return self.q[t], self.k[t], self.v[t], self.alpha[t], self.beta[t]


def tile_inputs(ti: wl.TokenInputs, w: wl.Workload, tile: int, t0: int, t1: int):
    """Oracle-side inputs of one tile for tokens t0..t1-1 (fp64)."""
    b, h = divmod(tile, w.num_v_heads)
    hk = h // (w.num_v_heads // w.num_k_heads)
    return (ti.q[t0:t1, b, hk], ti.k[t0:t1, b, hk], ti.v[t0:t1, b, h],
            ti.alpha[t0:t1, b, h], ti.beta[t0:t1, b, h])
