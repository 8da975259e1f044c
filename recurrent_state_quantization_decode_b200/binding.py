"""Thin ctypes binding of libleapquant.so (include/leapquant.h).

Argument marshalling only: every step of the decode path runs in the library's
CUDA kernels.  Tensors are passed as device pointers (torch tensors are
accepted and must already live on the GPU, contiguous); PyTorch provides the
memory and the streams.  Importing this module fails loudly if the library
has not been built (python -m recurrent_state_quantization_decode_b200.build).
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libleapquant.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it with "
        "`python -m recurrent_state_quantization_decode_b200.build` (needs nvcc). "
        "There is no CPU fallback.")

_lib = ctypes.CDLL(LIB_PATH)

LQ_OK, LQ_ERR_INVALID_ARG, LQ_ERR_UNSUPPORTED, LQ_ERR_MISALIGNED, LQ_ERR_CUDA, \
    LQ_ERR_DEVICE_BOUNDS, LQ_ERR_TOO_LARGE, LQ_ERR_TIMEOUT = range(8)
LQ_NOALLOC_STAGING_MAX_BYTES = 8 << 20  # the fixed staging array of the no-alloc entry point
LQ_GATE_SCALAR, LQ_GATE_DIAG = 0, 1
LQ_DTYPE_F32, LQ_DTYPE_BF16 = 0, 1

# Every symbol include/leapquant.h declares.
EXPORTED = ("lq_version", "lq_status_string", "lq_state_layout", "lq_state_bytes",
            "lq_state_init", "lq_decode_step", "lq_decode_step_host",
            "lq_decode_step_host_noalloc", "lq_window_flush",
            "lq_fp32_decode_step", "lq_state_dequantize", "lq_get_last_error",
            "lq_test_decode_step_timeout", "lq_prefill", "lq_checkpoint_save",
            "lq_checkpoint_restore", "lq_window_rewind", "lq_decode_tokens",
            "lq_decode_step_packed")


class lq_config(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int32), ("num_k_heads", ctypes.c_int32),
                ("num_v_heads", ctypes.c_int32), ("d", ctypes.c_int32),
                ("window", ctypes.c_int32), ("n_comp", ctypes.c_int32),
                ("gate", ctypes.c_int32), ("in_dtype", ctypes.c_int32),
                ("out_dtype", ctypes.c_int32), ("smooth", ctypes.c_float)]


class lq_layout(ctypes.Structure):
    _fields_ = [(n, ctypes.c_size_t) for n in (
        "record_bytes", "off_sigma", "off_m", "off_comp_vec", "off_comp_id", "records_bytes",
        "buf_k_bytes", "buf_d_bytes", "buf_g_bytes", "buf_n_bytes", "err_bytes",
        "fp32_state_bytes", "host_staging_bytes")]


class lq_state(ctypes.Structure):
    _fields_ = [("records", ctypes.c_void_p), ("buf_k", ctypes.c_void_p),
                ("buf_d", ctypes.c_void_p), ("buf_g", ctypes.c_void_p),
                ("buf_n", ctypes.c_void_p), ("err", ctypes.c_void_p)]


_P = ctypes.c_void_p
_CFG = ctypes.POINTER(lq_config)
_ST = ctypes.POINTER(lq_state)
_sig = {
    "lq_version": ([], ctypes.c_int32),
    "lq_status_string": ([ctypes.c_int], ctypes.c_char_p),
    "lq_state_layout": ([_CFG, ctypes.POINTER(lq_layout)], ctypes.c_int),
    "lq_state_bytes": ([_CFG, ctypes.POINTER(ctypes.c_size_t),
                        ctypes.POINTER(ctypes.c_size_t)], ctypes.c_size_t),
    "lq_state_init": ([_CFG, _P, _ST, _P, _P], ctypes.c_int),
    "lq_decode_step": ([_CFG, _P, _P, _P, _P, _P, _ST, _P, _P, _P], ctypes.c_int),
    "lq_decode_step_packed": ([_CFG, _P, _P, _P, _ST, _P, _P, _P], ctypes.c_int),
    "lq_decode_step_host": ([_CFG, _P, _P, _P, _P, _P, _ST, _P, _P, _P, _P], ctypes.c_int),
    "lq_decode_step_host_noalloc": ([_CFG, _P, _P, _P, _P, _P, _ST, _P, _P, _P], ctypes.c_int),
    "lq_window_flush": ([_CFG, _ST, _P, _P], ctypes.c_int),
    "lq_fp32_decode_step": ([_CFG, _P, _P, _P, _P, _P, _P, _P, _P], ctypes.c_int),
    "lq_state_dequantize": ([_CFG, _ST, ctypes.c_int32, _P, _P], ctypes.c_int),
    "lq_get_last_error": ([_ST, _P], ctypes.c_int),
    "lq_test_decode_step_timeout": ([_CFG, _P, _P, _P, _P, _P, _ST, _P, ctypes.c_uint32, _P],
                                    ctypes.c_int),
    "lq_prefill": ([_CFG, _P, _P, _P, _P, _P, ctypes.c_int32, _P, _ST, _P, _P, _P],
                   ctypes.c_int),
    "lq_checkpoint_save": ([_CFG, _ST, _P, _P, ctypes.c_int32, _P], ctypes.c_int),
    "lq_checkpoint_restore": ([_CFG, _P, ctypes.c_int32, _P, _ST, _P], ctypes.c_int),
    "lq_window_rewind": ([_CFG, _ST, _P, _P], ctypes.c_int),
    "lq_decode_tokens": ([_CFG, ctypes.c_int32, _P, _P, _P, _P, _P, _ST, _P, _P, _P],
                         ctypes.c_int),
}
for _name, (_args, _res) in _sig.items():
    _f = getattr(_lib, _name)
    _f.argtypes = _args
    _f.restype = _res


class LQError(RuntimeError):
    def __init__(self, status: int, call: str):
        self.status = status
        super().__init__(f"{call}: {lq_status_string(status)}")


def _check(status: int, call: str) -> None:
    if status != LQ_OK:
        raise LQError(status, call)


def _ptr(x) -> Optional[int]:
    """Device (or host) address of a tensor / int / None."""
    if x is None:
        return None
    if isinstance(x, int):
        return x
    if hasattr(x, "data_ptr"):
        if hasattr(x, "is_contiguous") and not x.is_contiguous():
            raise ValueError("tensors passed to libleapquant must be contiguous")
        return x.data_ptr()
    raise TypeError(f"cannot pass {type(x).__name__} as a pointer")


def _stream(stream) -> Optional[int]:
    if stream is None:
        try:
            import torch
            if torch.cuda.is_available():
                return torch.cuda.current_stream().cuda_stream
        except ImportError:
            pass
        return None
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def make_config(batch: int, num_k_heads: int, num_v_heads: int, d: int, window: int = 16,
                n_comp: int = 4, gate: int = LQ_GATE_SCALAR, in_bf16: bool = False,
                out_bf16: bool = False, smooth: float = 0.5) -> lq_config:
    return lq_config(batch, num_k_heads, num_v_heads, d, window, n_comp, gate,
                     LQ_DTYPE_BF16 if in_bf16 else LQ_DTYPE_F32,
                     LQ_DTYPE_BF16 if out_bf16 else LQ_DTYPE_F32, smooth)


def config_for(workload, batch: Optional[int] = None, out_bf16: bool = False) -> lq_config:
    """lq_config of a workloads.Workload."""
    w = workload
    return make_config(w.batch if batch is None else batch, w.num_k_heads, w.num_v_heads, w.d,
                       w.window, w.n_comp, w.gate, w.io_bf16, out_bf16, w.smooth)


# ---------------------------------------------------------------------------
# The C entry points, same names
# ---------------------------------------------------------------------------

def lq_version() -> int:
    return _lib.lq_version()


def lq_status_string(status: int) -> str:
    return _lib.lq_status_string(status).decode()


def lq_state_layout(cfg: lq_config) -> lq_layout:
    out = lq_layout()
    _check(_lib.lq_state_layout(ctypes.byref(cfg), ctypes.byref(out)), "lq_state_layout")
    return out


def lq_state_bytes(cfg: lq_config) -> tuple[int, int, int]:
    """(total, tile_bytes, buffer_bytes); total 0 means a bad cfg."""
    tb, bb = ctypes.c_size_t(0), ctypes.c_size_t(0)
    total = _lib.lq_state_bytes(ctypes.byref(cfg), ctypes.byref(tb), ctypes.byref(bb))
    return total, tb.value, bb.value


def lq_state_init(cfg, S0, state: lq_state, mask=None, stream=None) -> None:
    _check(_lib.lq_state_init(ctypes.byref(cfg), _ptr(S0), ctypes.byref(state), _ptr(mask),
                              _stream(stream)), "lq_state_init")


def lq_decode_step(cfg, q, k, v, alpha, beta, state: lq_state, out, active=None,
                   stream=None) -> None:
    _check(_lib.lq_decode_step(ctypes.byref(cfg), _ptr(q), _ptr(k), _ptr(v), _ptr(alpha),
                               _ptr(beta), ctypes.byref(state), _ptr(out), _ptr(active),
                               _stream(stream)), "lq_decode_step")


def lq_decode_step_packed(cfg, qkva, alpha, beta, state: lq_state, out, active=None,
                          stream=None) -> None:
    """lq_decode_step with each tile's q, k, v (and KDA gate) packed back to
    back in qkva (see pack_tile_inputs); alpha: the GDN gates, None for KDA."""
    _check(_lib.lq_decode_step_packed(ctypes.byref(cfg), _ptr(qkva), _ptr(alpha), _ptr(beta),
                                      ctypes.byref(state), _ptr(out), _ptr(active),
                                      _stream(stream)), "lq_decode_step_packed")


def pack_tile_inputs(cfg, q, k, v, alpha):
    """The per-tile block layout of lq_decode_step_packed from q, k [B][Hk][d],
    v [B][Hv][d] and, for KDA, alpha [B][Hv][d] (torch tensors on one device):
    a uint8 tensor [B][Hv][block bytes]."""
    import torch

    B, Hk, Hv = cfg.batch, cfg.num_k_heads, cfg.num_v_heads
    g = Hv // Hk
    parts = [q.repeat_interleave(g, dim=1), k.repeat_interleave(g, dim=1), v]
    blocks = [x.contiguous().view(torch.uint8).reshape(B, Hv, -1) for x in parts]
    if cfg.gate == LQ_GATE_DIAG:
        blocks.append(alpha.contiguous().view(torch.uint8).reshape(B, Hv, -1))
    return torch.cat(blocks, dim=2).contiguous()


def lq_decode_tokens(cfg, ntok: int, q, k, v, alpha, beta, state: lq_state, out, active=None,
                     stream=None) -> None:
    """ntok consecutive decode tokens in one launch (token-major inputs and
    outputs, each token laid out as for lq_decode_step)."""
    _check(_lib.lq_decode_tokens(ctypes.byref(cfg), ctypes.c_int32(ntok), _ptr(q), _ptr(k),
                                 _ptr(v), _ptr(alpha), _ptr(beta), ctypes.byref(state),
                                 _ptr(out), _ptr(active), _stream(stream)), "lq_decode_tokens")


def lq_prefill(cfg, q, k, v, alpha, beta, T: int, S0, state: lq_state, out=None, mask=None,
               stream=None) -> None:
    """Exact recurrence over a T-token prompt (token-major inputs), outputs to
    `out` ([T, B, Hv, d], optional), then the quantizer into `state`."""
    _check(_lib.lq_prefill(ctypes.byref(cfg), _ptr(q), _ptr(k), _ptr(v), _ptr(alpha),
                           _ptr(beta), ctypes.c_int32(T), _ptr(S0), ctypes.byref(state),
                           _ptr(out), _ptr(mask), _stream(stream)), "lq_prefill")


def lq_checkpoint_save(cfg, state: lq_state, slots, pool, num_slots: int,
                       stream=None) -> None:
    """Copy the records of the sequences with slots[b] >= 0 into pool slot
    slots[b] (tiles must be on a window boundary)."""
    _check(_lib.lq_checkpoint_save(ctypes.byref(cfg), ctypes.byref(state), _ptr(slots),
                                   _ptr(pool), ctypes.c_int32(num_slots), _stream(stream)),
           "lq_checkpoint_save")


def lq_checkpoint_restore(cfg, pool, num_slots: int, slots, state: lq_state,
                          stream=None) -> None:
    """Copy pool slot slots[b] into sequence b's records (buf_n = 0)."""
    _check(_lib.lq_checkpoint_restore(ctypes.byref(cfg), _ptr(pool), ctypes.c_int32(num_slots),
                                      _ptr(slots), ctypes.byref(state), _stream(stream)),
           "lq_checkpoint_restore")


def lq_window_rewind(cfg, state: lq_state, drop, stream=None) -> None:
    """Drop the last drop[b] decoded tokens of sequence b (inside a window)."""
    _check(_lib.lq_window_rewind(ctypes.byref(cfg), ctypes.byref(state), _ptr(drop),
                                 _stream(stream)), "lq_window_rewind")


def lq_test_decode_step_timeout(cfg, q, k, v, alpha, beta, state: lq_state, out,
                                wait_limit: int, stream=None) -> None:
    """Testing only: lq_decode_step in which the first CTA withholds the copies
    of its first ring slot, so that its bounded wait (wait_limit polls) expires
    and the error word reports LQ_ERR_TIMEOUT."""
    _check(_lib.lq_test_decode_step_timeout(ctypes.byref(cfg), _ptr(q), _ptr(k), _ptr(v),
                                            _ptr(alpha), _ptr(beta), ctypes.byref(state),
                                            _ptr(out), ctypes.c_uint32(wait_limit),
                                            _stream(stream)), "lq_test_decode_step_timeout")


def lq_decode_step_host(cfg, q_host, k_host, v_host, alpha_host, beta_host, state: lq_state,
                        out_host, staging, active=None, stream=None) -> None:
    _check(_lib.lq_decode_step_host(ctypes.byref(cfg), _ptr(q_host), _ptr(k_host),
                                    _ptr(v_host), _ptr(alpha_host), _ptr(beta_host),
                                    ctypes.byref(state), _ptr(out_host), _ptr(staging),
                                    _ptr(active), _stream(stream)), "lq_decode_step_host")


def lq_decode_step_host_noalloc(cfg, q_host, k_host, v_host, alpha_host, beta_host,
                                state: lq_state, out_host, active=None, stream=None) -> None:
    """lq_decode_step_host without a staging argument, for callers that cannot
    allocate device memory: the library stages through its own fixed array of
    LQ_NOALLOC_STAGING_MAX_BYTES (shared by all calls; overlapping calls race)."""
    _check(_lib.lq_decode_step_host_noalloc(ctypes.byref(cfg), _ptr(q_host), _ptr(k_host),
                                            _ptr(v_host), _ptr(alpha_host), _ptr(beta_host),
                                            ctypes.byref(state), _ptr(out_host), _ptr(active),
                                            _stream(stream)), "lq_decode_step_host_noalloc")


def lq_window_flush(cfg, state: lq_state, mask=None, stream=None) -> None:
    _check(_lib.lq_window_flush(ctypes.byref(cfg), ctypes.byref(state), _ptr(mask),
                                _stream(stream)), "lq_window_flush")


def lq_fp32_decode_step(cfg, q, k, v, alpha, beta, S, out, stream=None) -> None:
    _check(_lib.lq_fp32_decode_step(ctypes.byref(cfg), _ptr(q), _ptr(k), _ptr(v), _ptr(alpha),
                                    _ptr(beta), _ptr(S), _ptr(out), _stream(stream)),
           "lq_fp32_decode_step")


def lq_state_dequantize(cfg, state: lq_state, include_buffer: bool, S_out, stream=None) -> None:
    _check(_lib.lq_state_dequantize(ctypes.byref(cfg), ctypes.byref(state),
                                    1 if include_buffer else 0, _ptr(S_out), _stream(stream)),
           "lq_state_dequantize")


def lq_get_last_error(state: lq_state, stream=None) -> int:
    """Status word of the device-side checks (LQ_OK or LQ_ERR_DEVICE_BOUNDS)."""
    return _lib.lq_get_last_error(ctypes.byref(state), _stream(stream))


# ---------------------------------------------------------------------------
# Device memory for a state (plumbing: torch allocates, the layout decides)
# ---------------------------------------------------------------------------

class DeviceState:
    """Device buffers of one layer's stored state, allocated with torch per
    lq_state_layout.  .st is the lq_state to pass to the C calls."""

    def __init__(self, cfg: lq_config, device="cuda"):
        import torch

        self.cfg = cfg
        self.layout = L = lq_state_layout(cfg)
        u8 = torch.uint8
        self.records = torch.zeros(max(L.records_bytes, 16), dtype=u8, device=device)
        self.buf_k = torch.zeros(max(L.buf_k_bytes, 16), dtype=u8, device=device)
        self.buf_d = torch.zeros(max(L.buf_d_bytes // 4, 4), dtype=torch.float32, device=device)
        self.buf_g = torch.zeros(max(L.buf_g_bytes // 4, 4), dtype=torch.float32, device=device)
        self.buf_n = torch.zeros(max(L.buf_n_bytes // 4, 1), dtype=torch.int32, device=device)
        self.err = torch.zeros(4, dtype=torch.int32, device=device)
        self.st = lq_state(self.records.data_ptr(), self.buf_k.data_ptr(),
                           self.buf_d.data_ptr(), self.buf_g.data_ptr(),
                           self.buf_n.data_ptr(), self.err.data_ptr())

    def record_view(self):
        """[tiles, record_bytes] uint8 view of the records."""
        L, c = self.layout, self.cfg
        return self.records[:L.records_bytes].view(c.batch * c.num_v_heads, L.record_bytes)
