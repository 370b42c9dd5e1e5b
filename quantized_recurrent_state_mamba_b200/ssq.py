"""Thin Python binding over libssq (include/ssq.h).

Argument marshalling only: every function checks that the tensors it is given
are CUDA tensors of the documented dtype, contiguity and size (the C ABI sees
only pointers, so the sizes are checked here), and calls the C entry point of
the same name on the current torch stream.  All arithmetic runs in the CUDA
kernels of libssq.so; importing this module fails loudly when the library is
missing.
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libssq.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"libssq.so is missing at {LIB_PATH}: build it with "
        "`python -m quantized_recurrent_state_mamba_b200.build`")
_lib = ctypes.CDLL(LIB_PATH)

SSQ_OK, SSQ_ERR_INVALID_ARG, SSQ_ERR_UNSUPPORTED, SSQ_ERR_ALIGNMENT, SSQ_ERR_CUDA = range(5)
SSQ_F32, SSQ_BF16, SSQ_I8_SYM, SSQ_I8_ASYM, SSQ_I4_SYM, SSQ_I4_ASYM = range(6)
FORMATS = {"f32": SSQ_F32, "bf16": SSQ_BF16, "i8s": SSQ_I8_SYM, "i8a": SSQ_I8_ASYM,
           "i4s": SSQ_I4_SYM, "i4a": SSQ_I4_ASYM}
SSQ_DEVERR_SLOT = 0x1
SSQ_DEVERR_NONFINITE = 0x2
SSQ_DEVERR_TIMEOUT = 0x4
SSQ_DEVERR_CHANNEL = 0x8
SSQ_MAX_HEADS = 512
SSQ_POOL_HEADER_BYTES = 256
SSQ_POOL_ALIGN = 256


class SsqError(RuntimeError):
    def __init__(self, status, detail):
        super().__init__(f"{_status_string(status)}: {detail}")
        self.status = status


class ssq_config(ctypes.Structure):
    _fields_ = [("n_layers", ctypes.c_int), ("n_slots", ctypes.c_int),
                ("nheads", ctypes.c_int), ("headdim", ctypes.c_int),
                ("d_state", ctypes.c_int), ("ngroups", ctypes.c_int),
                ("fmt", ctypes.c_int), ("head_mask", ctypes.POINTER(ctypes.c_uint8))]


class ssq_layout(ctypes.Structure):
    _fields_ = [(n, ctypes.c_size_t) for n in (
        "pool_bytes", "header_bytes", "slot_bytes", "codes_off", "meta_off", "fp_off",
        "codes_layer_bytes", "meta_layer_bytes", "fp_layer_bytes", "row_code_bytes",
        "row_meta_bytes", "fp_elem_bytes")] + [
        ("n_quant_heads", ctypes.c_int), ("n_fp_heads", ctypes.c_int)]


class ssq_damp_config(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int) for n in (
        "n_layers", "n_slots", "nheads", "headdim", "d_state", "ngroups", "n_protected")]


class ssq_damp_layout(ctypes.Structure):
    _fields_ = [(n, ctypes.c_size_t) for n in (
        "pool_bytes", "header_bytes", "slot_bytes", "layer_bytes", "head_bytes", "hi_off",
        "codes_off", "meta_off")] + [("bits_per_value", ctypes.c_double)]


_P = ctypes.c_void_p
_CFG = ctypes.POINTER(ssq_config)
_I = ctypes.c_int
_lib.ssq_status_string.restype = ctypes.c_char_p
_lib.ssq_status_string.argtypes = [_I]
_lib.ssq_last_error_detail.restype = ctypes.c_char_p
_lib.ssq_last_error_detail.argtypes = []
_lib.ssq_pool_layout.argtypes = [_CFG, ctypes.POINTER(ssq_layout), ctypes.POINTER(ctypes.c_int32)]
_lib.ssq_pool_init.argtypes = [_CFG, _P, _P]
_lib.ssq_pool_error.argtypes = [_CFG, _P, ctypes.POINTER(ctypes.c_uint32), _P]
_lib.ssq_quantize_rows.argtypes = [_CFG, _P, _P, _I, _I, _I, _P, _P]
_lib.ssq_dequantize_rows.argtypes = [_CFG, _P, _P, _I, _I, _I, _P, _P]
_lib.ssq_decode_step.argtypes = [_CFG, _P, _P, _I, _I, _I] + [_P] * 7 + [_P]
_lib.ssq_scan.argtypes = [_CFG, _P, _P, _I, _I, _I] + [_P] * 7 + [_P]
_lib.ssq_prefill.argtypes = [_CFG, _P, _P, _I, _I, _I] + [_P] * 7 + [_P]
_lib.ssq_decode_step_sr.argtypes = [_CFG, _P, _P, _I, _I, _I] + [_P] * 7 + [ctypes.c_uint64, ctypes.c_uint32, _P]
_lib.ssq_scan_sr.argtypes = [_CFG, _P, _P, _I, _I, _I] + [_P] * 7 + [ctypes.c_uint64, ctypes.c_uint32, _P]
_lib.ssq_decode_diag.argtypes = [_CFG, _P, _P, _I, _I, _I] + [_P] * 6 + [_P]
_DCFG = ctypes.POINTER(ssq_damp_config)
_lib.ssq_damp_pool_layout.argtypes = [_DCFG, ctypes.POINTER(ssq_damp_layout)]
_lib.ssq_damp_quantize.argtypes = [_DCFG, _P, _P, _P, _I, _I, _I, _P, _P]
_lib.ssq_damp_dequantize.argtypes = [_DCFG, _P, _P, _P, _I, _I, _I, _P, _P]
_lib.ssq_damp_decode_step.argtypes = [_DCFG, _P, _P, _P, _I, _I, _I] + [_P] * 7 + [_P]
_lib.ssq_damp_pool_error.argtypes = [_DCFG, _P, ctypes.POINTER(ctypes.c_uint32), _P]
_lib.ssq_test_hooks.argtypes = [_I, ctypes.c_longlong]
for _f in ("ssq_test_hooks", "ssq_pool_layout", "ssq_pool_init", "ssq_pool_error", "ssq_quantize_rows",
           "ssq_dequantize_rows", "ssq_decode_step", "ssq_scan", "ssq_prefill",
           "ssq_decode_step_sr", "ssq_scan_sr", "ssq_decode_diag", "ssq_damp_pool_layout",
           "ssq_damp_quantize", "ssq_damp_dequantize", "ssq_damp_decode_step",
           "ssq_damp_pool_error"):
    getattr(_lib, _f).restype = _I


def _status_string(s):
    return _lib.ssq_status_string(int(s)).decode()


def _check(status):
    if status != SSQ_OK:
        raise SsqError(status, _lib.ssq_last_error_detail().decode())


class Config:
    """A pool configuration (ssq_config) that owns its head mask buffer."""

    def __init__(self, n_layers, n_slots, nheads, headdim, d_state, ngroups=1,
                 fmt="i8a", head_mask=None):
        fmt_id = FORMATS[fmt] if isinstance(fmt, str) else int(fmt)
        self.c = ssq_config(int(n_layers), int(n_slots), int(nheads), int(headdim),
                            int(d_state), int(ngroups), fmt_id, None)
        self._mask = None
        if head_mask is not None:
            m = [int(bool(v)) for v in list(head_mask)]
            self._mask = (ctypes.c_uint8 * len(m))(*m)
            self.c.head_mask = ctypes.cast(self._mask, ctypes.POINTER(ctypes.c_uint8))
        self.head_mask = None if head_mask is None else [int(bool(v)) for v in head_mask]
        self.fmt = fmt_id

    def __getattr__(self, name):
        return getattr(self.__dict__["c"], name)

    @property
    def ref(self):
        return ctypes.byref(self.c)


def _ptr(t, name, dtype, numel, allow_none=False):
    if t is None:
        if allow_none:
            return None
        raise ValueError(f"{name} is required")
    if isinstance(t, int):
        return t
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name}: expected a torch tensor")
    if not t.is_cuda:
        raise ValueError(f"{name}: expected a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name}: expected {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name}: expected a contiguous tensor")
    if numel is not None and t.numel() < numel:
        raise ValueError(f"{name}: {t.numel()} elements, need {numel}")
    return t.data_ptr()


def _stream(stream):
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def ssq_pool_layout(cfg: Config):
    """Layout of the pool (dict of ssq_layout fields) and the region order of
    the heads (list: region position -> head index)."""
    L = ssq_layout()
    perm = (ctypes.c_int32 * cfg.nheads)()
    _check(_lib.ssq_pool_layout(cfg.ref, ctypes.byref(L), perm))
    d = {name: getattr(L, name) for name, _ in ssq_layout._fields_}
    return d, list(perm)


def alloc_pool(cfg: Config, device="cuda"):
    """A zeroed pool of layout.pool_bytes bytes (torch allocations are at
    least 256-byte aligned)."""
    L, _ = ssq_pool_layout(cfg)
    pool = torch.empty(L["pool_bytes"], dtype=torch.uint8, device=device)
    ssq_pool_init(cfg, pool)
    return pool


def _pool_ptr(cfg, pool):
    L, _ = ssq_pool_layout(cfg)
    return _ptr(pool, "pool", torch.uint8, L["pool_bytes"])


def ssq_pool_init(cfg: Config, pool, stream=None):
    _check(_lib.ssq_pool_init(cfg.ref, _pool_ptr(cfg, pool), _stream(stream)))


def ssq_pool_error(cfg: Config, pool, stream=None) -> int:
    """Read and clear the pool's device error word (synchronises the stream)."""
    v = ctypes.c_uint32(0)
    _check(_lib.ssq_pool_error(cfg.ref, _pool_ptr(cfg, pool), ctypes.byref(v), _stream(stream)))
    return int(v.value)


def ssq_test_hooks(withhold_first_tile: bool, wait_limit_cycles: int = 0):
    """Test support for the decode step's failure path (see include/ssq.h):
    the pipeline wait bound in SM clock cycles (0: the default) and whether
    the first thread block withholds its first tile's copy."""
    _check(_lib.ssq_test_hooks(1 if withhold_first_tile else 0, int(wait_limit_cycles)))


def _slots(slot_idx, batch):
    return _ptr(slot_idx, "slot_idx", torch.int32, batch, allow_none=True)


def ssq_quantize_rows(cfg: Config, pool, slot_idx, batch, layer0, nl, S, stream=None):
    """S: fp32 [nl][batch][nheads][headdim][d_state] -> pool slots."""
    n = nl * batch * cfg.nheads * cfg.headdim * cfg.d_state
    _check(_lib.ssq_quantize_rows(cfg.ref, _pool_ptr(cfg, pool), _slots(slot_idx, batch),
                                  batch, layer0, nl, _ptr(S, "S", torch.float32, n),
                                  _stream(stream)))


def ssq_dequantize_rows(cfg: Config, pool, slot_idx, batch, layer0, nl, S_out, stream=None):
    n = nl * batch * cfg.nheads * cfg.headdim * cfg.d_state
    _check(_lib.ssq_dequantize_rows(cfg.ref, _pool_ptr(cfg, pool), _slots(slot_idx, batch),
                                    batch, layer0, nl, _ptr(S_out, "S_out", torch.float32, n),
                                    _stream(stream)))


def ssq_decode_step(cfg: Config, pool, slot_idx, batch, layer0, nl, x, B, C, dt, A, D, y,
                    stream=None):
    """One decode token: x/y [nl][batch][H][P], B/C [nl][batch][G][N],
    dt [nl][batch][H], A/D [nl][H] (fp32 CUDA tensors)."""
    H, P, N, G = cfg.nheads, cfg.headdim, cfg.d_state, cfg.ngroups
    f = torch.float32
    _check(_lib.ssq_decode_step(
        cfg.ref, _pool_ptr(cfg, pool), _slots(slot_idx, batch), batch, layer0, nl,
        _ptr(x, "x", f, nl * batch * H * P), _ptr(B, "B", f, nl * batch * G * N),
        _ptr(C, "C", f, nl * batch * G * N), _ptr(dt, "dt", f, nl * batch * H),
        _ptr(A, "A", f, nl * H), _ptr(D, "D", f, nl * H),
        _ptr(y, "y", f, nl * batch * H * P), _stream(stream)))


def ssq_decode_diag(cfg: Config, pool, slot_idx, batch, layer0, nl, x, B, C, dt, A, diag,
                    stream=None):
    """Read-only diagnostics of one decode step: diag [nl][batch][H][P][4] =
    (reversals, reversal error seen by the readout, total rounding error
    seen by the readout, readout signal).  Other layouts as ssq_decode_step."""
    H, P, N, G = cfg.nheads, cfg.headdim, cfg.d_state, cfg.ngroups
    f = torch.float32
    _check(_lib.ssq_decode_diag(
        cfg.ref, _pool_ptr(cfg, pool), _slots(slot_idx, batch), batch, layer0, nl,
        _ptr(x, "x", f, nl * batch * H * P), _ptr(B, "B", f, nl * batch * G * N),
        _ptr(C, "C", f, nl * batch * G * N), _ptr(dt, "dt", f, nl * batch * H),
        _ptr(A, "A", f, nl * H), _ptr(diag, "diag", f, nl * batch * H * P * 4),
        _stream(stream)))


def ssq_scan(cfg: Config, pool, slot_idx, batch, layer, T, x, B, C, dt, A, D, y, stream=None):
    """T tokens of one layer: x/y [batch][T][H][P], B/C [batch][T][G][N],
    dt [batch][T][H], A/D [H]."""
    H, P, N, G = cfg.nheads, cfg.headdim, cfg.d_state, cfg.ngroups
    f = torch.float32
    _check(_lib.ssq_scan(
        cfg.ref, _pool_ptr(cfg, pool), _slots(slot_idx, batch), batch, layer, T,
        _ptr(x, "x", f, batch * T * H * P), _ptr(B, "B", f, batch * T * G * N),
        _ptr(C, "C", f, batch * T * G * N), _ptr(dt, "dt", f, batch * T * H),
        _ptr(A, "A", f, H), _ptr(D, "D", f, H), _ptr(y, "y", f, batch * T * H * P),
        _stream(stream)))


def ssq_decode_step_sr(cfg: Config, pool, slot_idx, batch, layer0, nl, x, B, C, dt, A, D, y,
                       seed, step, stream=None):
    """ssq_decode_step with stochastic rounding (draws keyed by seed, step)."""
    H, P, N, G = cfg.nheads, cfg.headdim, cfg.d_state, cfg.ngroups
    f = torch.float32
    _check(_lib.ssq_decode_step_sr(
        cfg.ref, _pool_ptr(cfg, pool), _slots(slot_idx, batch), batch, layer0, nl,
        _ptr(x, "x", f, nl * batch * H * P), _ptr(B, "B", f, nl * batch * G * N),
        _ptr(C, "C", f, nl * batch * G * N), _ptr(dt, "dt", f, nl * batch * H),
        _ptr(A, "A", f, nl * H), _ptr(D, "D", f, nl * H), _ptr(y, "y", f, nl * batch * H * P),
        ctypes.c_uint64(int(seed)), ctypes.c_uint32(int(step)), _stream(stream)))


def ssq_scan_sr(cfg: Config, pool, slot_idx, batch, layer, T, x, B, C, dt, A, D, y, seed,
                step0, stream=None):
    """ssq_scan with stochastic rounding, token t at step0 + t."""
    H, P, N, G = cfg.nheads, cfg.headdim, cfg.d_state, cfg.ngroups
    f = torch.float32
    _check(_lib.ssq_scan_sr(
        cfg.ref, _pool_ptr(cfg, pool), _slots(slot_idx, batch), batch, layer, T,
        _ptr(x, "x", f, batch * T * H * P), _ptr(B, "B", f, batch * T * G * N),
        _ptr(C, "C", f, batch * T * G * N), _ptr(dt, "dt", f, batch * T * H),
        _ptr(A, "A", f, H), _ptr(D, "D", f, H), _ptr(y, "y", f, batch * T * H * P),
        ctypes.c_uint64(int(seed)), ctypes.c_uint32(int(step0)), _stream(stream)))


def ssq_prefill(cfg: Config, pool, slot_idx, batch, layer, T, x, B, C, dt, A, D, y,
                stream=None):
    """Prefill hand-off: T tokens of one layer in fp32, the final state
    quantized once.  Layouts as ssq_scan."""
    H, P, N, G = cfg.nheads, cfg.headdim, cfg.d_state, cfg.ngroups
    f = torch.float32
    _check(_lib.ssq_prefill(
        cfg.ref, _pool_ptr(cfg, pool), _slots(slot_idx, batch), batch, layer, T,
        _ptr(x, "x", f, batch * T * H * P), _ptr(B, "B", f, batch * T * G * N),
        _ptr(C, "C", f, batch * T * G * N), _ptr(dt, "dt", f, batch * T * H),
        _ptr(A, "A", f, H), _ptr(D, "D", f, H), _ptr(y, "y", f, batch * T * H * P),
        _stream(stream)))


# ---------------------------------------------------------------------------
# DAMP mixed-tier pool
# ---------------------------------------------------------------------------

class DampConfig:
    """A DAMP pool configuration (ssq_damp_config)."""

    def __init__(self, n_layers, n_slots, nheads, headdim, d_state, ngroups=1, n_protected=16):
        self.c = ssq_damp_config(int(n_layers), int(n_slots), int(nheads), int(headdim),
                                 int(d_state), int(ngroups), int(n_protected))

    def __getattr__(self, name):
        return getattr(self.__dict__["c"], name)

    @property
    def ref(self):
        return ctypes.byref(self.c)


def ssq_damp_pool_layout(cfg: DampConfig):
    L = ssq_damp_layout()
    _check(_lib.ssq_damp_pool_layout(cfg.ref, ctypes.byref(L)))
    return {name: getattr(L, name) for name, _ in ssq_damp_layout._fields_}


def damp_alloc_pool(cfg: DampConfig, device="cuda"):
    """A zeroed DAMP pool (the all-zero state)."""
    L = ssq_damp_pool_layout(cfg)
    return torch.zeros(L["pool_bytes"], dtype=torch.uint8, device=device)


def _damp_ptrs(cfg, pool, chan):
    L = ssq_damp_pool_layout(cfg)
    return (_ptr(pool, "pool", torch.uint8, L["pool_bytes"]),
            _ptr(chan, "chan", torch.int32, cfg.n_layers * cfg.nheads * cfg.d_state))


def ssq_damp_quantize(cfg: DampConfig, pool, chan, slot_idx, batch, layer0, nl, S, stream=None):
    """S: fp32 [nl][batch][nheads][headdim][d_state] -> DAMP pool slots."""
    pp, cp = _damp_ptrs(cfg, pool, chan)
    n = nl * batch * cfg.nheads * cfg.headdim * cfg.d_state
    _check(_lib.ssq_damp_quantize(cfg.ref, pp, cp, _slots(slot_idx, batch), batch, layer0, nl,
                                  _ptr(S, "S", torch.float32, n), _stream(stream)))


def ssq_damp_dequantize(cfg: DampConfig, pool, chan, slot_idx, batch, layer0, nl, S_out,
                        stream=None):
    pp, cp = _damp_ptrs(cfg, pool, chan)
    n = nl * batch * cfg.nheads * cfg.headdim * cfg.d_state
    _check(_lib.ssq_damp_dequantize(cfg.ref, pp, cp, _slots(slot_idx, batch), batch, layer0,
                                    nl, _ptr(S_out, "S_out", torch.float32, n),
                                    _stream(stream)))


def ssq_damp_decode_step(cfg: DampConfig, pool, chan, slot_idx, batch, layer0, nl, x, B, C, dt,
                         A, D, y, stream=None):
    """One decode token on DAMP slots; layouts as ssq_decode_step."""
    H, P, N, G = cfg.nheads, cfg.headdim, cfg.d_state, cfg.ngroups
    f = torch.float32
    pp, cp = _damp_ptrs(cfg, pool, chan)
    _check(_lib.ssq_damp_decode_step(
        cfg.ref, pp, cp, _slots(slot_idx, batch), batch, layer0, nl,
        _ptr(x, "x", f, nl * batch * H * P), _ptr(B, "B", f, nl * batch * G * N),
        _ptr(C, "C", f, nl * batch * G * N), _ptr(dt, "dt", f, nl * batch * H),
        _ptr(A, "A", f, nl * H), _ptr(D, "D", f, nl * H), _ptr(y, "y", f, nl * batch * H * P),
        _stream(stream)))


def ssq_damp_pool_error(cfg: DampConfig, pool, stream=None) -> int:
    v = ctypes.c_uint32(0)
    L = ssq_damp_pool_layout(cfg)
    _check(_lib.ssq_damp_pool_error(cfg.ref, _ptr(pool, "pool", torch.uint8, L["pool_bytes"]),
                                    ctypes.byref(v), _stream(stream)))
    return int(v.value)


def ssq_status_string(status) -> str:
    return _status_string(status)


def ssq_last_error_detail() -> str:
    return _lib.ssq_last_error_detail().decode()


def raw():
    """The ctypes handle of libssq.so (for tests that call the C ABI with
    explicit pointers)."""
    return _lib
