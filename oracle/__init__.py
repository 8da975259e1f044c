"""CPU oracle for the LeapQuant int8-state GDN/KDA decode step (ctypes wrapper).

TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and bench.py's
cpu_baseline / reference legs may import this package.  The product library
never imports it, and it imports nothing from the product package.

The arithmetic lives in leapquant_oracle.c (plain fp64 C); this module builds
it with gcc on first use and marshals numpy arrays.  Everything here is
per tile: one (sequence, value head) state S of shape d_v x d_k, with
o = S q.  See leapquant_oracle.c for the algorithm, its sources and the
readings taken where the pages are silent.

Parity status: every function is pinned by tests/test_oracle_pins.py except
the end-to-end model accuracy the pages report (75.5 % over 12 model-task
pairs), which needs trained weights and datasets: parity unpinned.
"""
from __future__ import annotations

import ctypes
import dataclasses
import os
import subprocess
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "leapquant_oracle.c")
_LIB = os.path.join(_HERE, "_leapquant_oracle.so")

GATE_SCALAR, GATE_DIAG = 0, 1
SMOOTH_CODES = {0.0: 0, 0.5: 1, 1.0: 2}
D_WY_RESIDUAL, D_MIN_MARGIN, D_FOLDS, D_SELECTIONS = 0, 1, 2, 3


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (no fast-math, no FMA contraction)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off",
               "-fno-fast-math", _SRC, "-o", _LIB + ".tmp", "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(_LIB + ".tmp", _LIB)
    return _LIB


_lib = None


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_LIB)
        if L.orc_version() != 1:
            raise RuntimeError("oracle library version mismatch")
        _lib = L
    return _lib


def _p(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _f64(x) -> np.ndarray:
    return np.ascontiguousarray(x, dtype=np.float64)


@dataclasses.dataclass(frozen=True)
class Cfg:
    dk: int
    dv: int
    W: int = 16
    K: int = 4
    gate: int = GATE_SCALAR
    quant: int = 1  # 1 = int8 LeapQuant, 0 = identity (no rounding anywhere)
    smooth: float = 0.5  # exponent of the column max: 0, 0.5 or 1

    @property
    def dmax(self) -> int:
        return max(self.dk, self.dv)

    @property
    def ga(self) -> int:
        return self.dk if self.gate == GATE_DIAG else 1

    def arr(self) -> np.ndarray:
        return np.array([self.dk, self.dv, self.W, self.K, self.gate, self.quant,
                         SMOOTH_CODES[float(self.smooth)]], dtype=np.int32)


def new_diag() -> np.ndarray:
    d = np.zeros(8, dtype=np.float64)
    d[D_MIN_MARGIN] = np.inf
    return d


def _check(rc: int, what: str) -> None:
    if rc < 0:
        raise ValueError(f"oracle {what} rejected its arguments (rc={rc})")


def exact_run(cfg: Cfg, S: np.ndarray, q, k, v, alpha, beta):
    """Exact recurrence over T tokens.  q, k: [T, dk]; v: [T, dv];
    alpha: [T] (GDN) or [T, dk] (KDA); beta: [T].  Returns (S_T, o [T, dv])."""
    S = _f64(S).copy()
    q, k, v, beta = _f64(q), _f64(k), _f64(v), _f64(beta)
    T = q.shape[0]
    alpha = _f64(alpha).reshape(T, cfg.ga)
    o = np.zeros((T, cfg.dv), dtype=np.float64)
    rc = lib().orc_exact_run(_p(cfg.arr()), ctypes.c_int(T), _p(S), _p(q), _p(k), _p(v),
                             _p(alpha), _p(beta), ctypes.c_long(cfg.dk), ctypes.c_long(cfg.dk),
                             ctypes.c_long(cfg.dv), ctypes.c_long(cfg.ga), ctypes.c_long(1),
                             _p(o), ctypes.c_long(cfg.dv))
    _check(rc, "exact_run")
    return S, o


@dataclasses.dataclass
class Record:
    """One stored tile.  int8: Q [dv, dk] int8, sig [dv], m [dk], cv [K, dmax]
    (float32), cid [K] int32.  identity: Rid [dv, dk] and cv64 [K, dmax] fp64."""
    cid: np.ndarray
    Q: Optional[np.ndarray] = None
    sig: Optional[np.ndarray] = None
    m: Optional[np.ndarray] = None
    cv: Optional[np.ndarray] = None
    Rid: Optional[np.ndarray] = None
    cv64: Optional[np.ndarray] = None

    @staticmethod
    def empty(cfg: Cfg) -> "Record":
        r = Record(cid=np.zeros(max(cfg.K, 1), dtype=np.int32))
        if cfg.quant:
            r.Q = np.zeros((cfg.dv, cfg.dk), dtype=np.int8)
            r.sig = np.zeros(cfg.dv, dtype=np.float32)
            r.m = np.zeros(cfg.dk, dtype=np.float32)
            r.cv = np.zeros((max(cfg.K, 1), cfg.dmax), dtype=np.float32)
        else:
            r.Rid = np.zeros((cfg.dv, cfg.dk), dtype=np.float64)
            r.cv64 = np.zeros((max(cfg.K, 1), cfg.dmax), dtype=np.float64)
        return r

    def ptrs(self):
        return (_p(self.Q), _p(self.sig), _p(self.m), _p(self.cv), _p(self.cid), _p(self.Rid),
                _p(self.cv64))

    def copy(self) -> "Record":
        return Record(**{f.name: (None if getattr(self, f.name) is None
                                  else getattr(self, f.name).copy())
                         for f in dataclasses.fields(self)})


def quantize(cfg: Cfg, S: np.ndarray, diag: Optional[np.ndarray] = None,
             want_xq: bool = False):
    """quantize(S): compensators, smoothing, per-row int8.  Returns the Record
    (and, with want_xq, each code's value before rounding, float32 [dv, dk])."""
    S = _f64(S).reshape(cfg.dv, cfg.dk)
    rec = Record.empty(cfg)
    xq = np.zeros((cfg.dv, cfg.dk), dtype=np.float32) if want_xq else None
    rc = lib().orc_quantize(_p(cfg.arr()), _p(S), *rec.ptrs(), _p(xq), _p(diag))
    _check(rc, "quantize")
    return (rec, xq) if want_xq else rec


def dequantize(cfg: Cfg, rec: Record) -> np.ndarray:
    S0 = np.zeros((cfg.dv, cfg.dk), dtype=np.float64)
    rc = lib().orc_dequantize(_p(cfg.arr()), *rec.ptrs(), _p(S0))
    _check(rc, "dequantize")
    return S0


class Tile:
    """One tile of the windowed quantized decode: a stored record plus the
    in-window buffer of (k_i, d_i, alpha_i) and, for the cross-check, the WY
    pair (u_i, w_i)."""

    def __init__(self, cfg: Cfg, S0: Optional[np.ndarray] = None, wy_check: bool = True):
        self.cfg = cfg
        self.diag = new_diag()
        self.rec = Record.empty(cfg)
        self.n = np.zeros(1, dtype=np.int32)
        self.bk = np.zeros((cfg.W, cfg.dk), dtype=np.float64)
        self.bd = np.zeros((cfg.W, cfg.dv), dtype=np.float64)
        self.ba = np.zeros((cfg.W, cfg.ga), dtype=np.float64)
        self.bu = np.zeros((cfg.W, cfg.dv), dtype=np.float64) if wy_check else None
        self.bw = np.zeros((cfg.W, cfg.dk), dtype=np.float64) if wy_check else None
        if S0 is not None:
            self.init(S0)

    def init(self, S0: np.ndarray) -> None:
        """init(S): quantize S and empty the buffer."""
        self.rec = quantize(self.cfg, S0, self.diag)
        self.n[0] = 0

    def run(self, q, k, v, alpha, beta) -> np.ndarray:
        """Decode T tokens (q, k: [T, dk]; v: [T, dv]; alpha: [T] or [T, dk];
        beta: [T]); returns o [T, dv].  Folds whenever the window fills."""
        cfg = self.cfg
        q, k, v, beta = _f64(q), _f64(k), _f64(v), _f64(beta)
        T = q.shape[0]
        alpha = _f64(alpha).reshape(T, cfg.ga)
        o = np.zeros((T, cfg.dv), dtype=np.float64)
        rc = lib().orc_lq_run(
            _p(cfg.arr()), ctypes.c_int(T), *self.rec.ptrs(), _p(self.n), _p(self.bk),
            _p(self.bd), _p(self.ba), _p(self.bu), _p(self.bw), _p(q), _p(k), _p(v), _p(alpha),
            _p(beta), ctypes.c_long(cfg.dk), ctypes.c_long(cfg.dk), ctypes.c_long(cfg.dv),
            ctypes.c_long(cfg.ga), ctypes.c_long(1), _p(o), ctypes.c_long(cfg.dv),
            _p(self.diag))
        _check(rc, "lq_run")
        return o

    def flush(self) -> None:
        """Fold a partially filled window now."""
        rc = lib().orc_lq_flush(_p(self.cfg.arr()), *self.rec.ptrs(), _p(self.n), _p(self.bk),
                                _p(self.bd), _p(self.ba), _p(self.diag))
        _check(rc, "lq_flush")

    def state(self) -> np.ndarray:
        """The current state: window base advanced by the buffered tokens."""
        S = np.zeros((self.cfg.dv, self.cfg.dk), dtype=np.float64)
        rc = lib().orc_lq_state(_p(self.cfg.arr()), *self.rec.ptrs(), ctypes.c_int(int(self.n[0])),
                                _p(self.bk), _p(self.bd), _p(self.ba), _p(S))
        _check(rc, "lq_state")
        return S

    def base(self) -> np.ndarray:
        """The window-base state S0 reconstructed from the record."""
        return dequantize(self.cfg, self.rec)


def batch_run(cfg: Cfg, B: int, Hk: int, Hv: int, T: int, rec: dict, buf: dict, inp: dict,
              nthreads: int = 0) -> int:
    """All tiles of a batch for T tokens (int8 records only), OpenMP across
    tiles.  rec: Q [tiles, dv, dk] int8, sig, m, cv [tiles, K, dmax], cid
    [tiles, K]; buf: n [tiles] int32, bk, bd, ba (fp64); inp: q, k [T, B, Hk, dk],
    v [T, B, Hv, dv], alpha [T, B, Hv(, dk)], beta [T, B, Hv] (fp64) and o
    [T, B, Hv, dv] (fp64, written).  Returns the number of threads used."""
    used = lib().orc_lq_batch(
        _p(cfg.arr()), ctypes.c_int(B), ctypes.c_int(Hk), ctypes.c_int(Hv), ctypes.c_int(T),
        _p(rec["Q"]), _p(rec["sig"]), _p(rec["m"]), _p(rec["cv"]), _p(rec["cid"]),
        _p(buf["n"]), _p(buf["bk"]), _p(buf["bd"]), _p(buf["ba"]),
        _p(inp["q"]), _p(inp["k"]), _p(inp["v"]), _p(inp["alpha"]), _p(inp["beta"]),
        _p(inp["o"]), ctypes.c_int(nthreads))
    _check(used, "lq_batch")
    return used
