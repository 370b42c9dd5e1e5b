"""CPU oracle for the quantized Mamba-2 recurrent-state update.

TEST INFRASTRUCTURE ONLY.  The tests, the package smoke check and the
benchmark's CPU-baseline leg may import this package; the library and its
Python binding never do.  It wraps ``ssq_oracle.c`` (plain scalar C, built
with ``-ffp-contract=off``) through ctypes and works on a *logical* state:
integer codes, per-row step and zero point, and fp32 values for fp rows.  It
knows nothing of the library's pool byte layout.

Every function states the passage of the pages it follows in ``ssq_oracle.c``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "ssq_oracle.c")
_LIB = os.path.join(_HERE, "liboref.so")

F32, BF16, I8_SYM, I8_ASYM, I4_SYM, I4_ASYM = range(6)
FORMATS = {"f32": F32, "bf16": BF16, "i8s": I8_SYM, "i8a": I8_ASYM,
           "i4s": I4_SYM, "i4a": I4_ASYM}


def build(force: bool = False) -> str:
    """Compile the oracle into ``oracle/liboref.so`` (gcc, scalar, no FMA
    contraction).  Rebuilds when the source is newer than the library."""
    hdr = os.path.join(_HERE, "ssq_oracle.h")
    stale = (not os.path.exists(_LIB)
             or os.path.getmtime(_LIB) < max(os.path.getmtime(_SRC),
                                             os.path.getmtime(hdr)))
    if force or stale:
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call([
            "gcc", "-O2", "-ffp-contract=off", "-fno-fast-math", "-std=c11",
            "-shared", "-fPIC", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


class _Cfg(ctypes.Structure):
    _fields_ = [("fmt", ctypes.c_int), ("nheads", ctypes.c_int),
                ("headdim", ctypes.c_int), ("d_state", ctypes.c_int),
                ("ngroups", ctypes.c_int),
                ("head_mask", ctypes.POINTER(ctypes.c_uint8))]


class _State(ctypes.Structure):
    _fields_ = [("q", ctypes.POINTER(ctypes.c_int32)),
                ("delta", ctypes.POINTER(ctypes.c_float)),
                ("zero", ctypes.POINTER(ctypes.c_float)),
                ("val", ctypes.POINTER(ctypes.c_float))]


def lib():
    global _lib
    if _lib is None:
        # SSQ_ORACLE_LIB points the tests' mutation check at a deliberately
        # broken build of the oracle; normally the library is built here.
        path = os.environ.get("SSQ_ORACLE_LIB") or build()
        _lib = ctypes.CDLL(path)
        _lib.oref_lambda.restype = ctypes.c_float
        _lib.oref_lambda.argtypes = [ctypes.c_float, ctypes.c_float]
        _lib.oref_bf16_round.restype = ctypes.c_float
        _lib.oref_bf16_round.argtypes = [ctypes.c_float]
        _lib.oref_sr_u16.restype = ctypes.c_uint32
        _lib.oref_sr_u16.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.c_int, ctypes.c_int]
        _lib.oref_fp16_round.restype = ctypes.c_float
        _lib.oref_fp16_round.argtypes = [ctypes.c_float]
    return _lib


def _p(a, ct):
    return a.ctypes.data_as(ctypes.POINTER(ct))


def _f32(a):
    return np.ascontiguousarray(a, dtype=np.float32)


@dataclass
class Cfg:
    """Shape and format of one layer's state: nheads x headdim rows of
    d_state entries, ngroups B/C groups, optional per-head quantize mask."""
    fmt: int
    nheads: int
    headdim: int
    d_state: int
    ngroups: int = 1
    head_mask: np.ndarray | None = None

    def c(self):
        cfg = _Cfg(self.fmt, self.nheads, self.headdim, self.d_state,
                   self.ngroups, None)
        if self.head_mask is not None:
            self._mask = np.ascontiguousarray(self.head_mask, dtype=np.uint8)
            cfg.head_mask = _p(self._mask, ctypes.c_uint8)
        return cfg

    @property
    def rows(self):
        return self.nheads * self.headdim

    def row_is_quant(self, h):
        if self.fmt in (F32, BF16):
            return False
        return self.head_mask is None or bool(self.head_mask[h])


class State:
    """Logical state of ``count`` (layer, request) pairs."""

    def __init__(self, cfg: Cfg, count: int = 1):
        R, N = cfg.rows, cfg.d_state
        self.cfg = cfg
        self.count = count
        self.q = np.zeros((count, R, N), np.int32)
        self.delta = np.zeros((count, R), np.float32)
        self.zero = np.zeros((count, R), np.float32)
        self.val = np.zeros((count, R, N), np.float32)

    def c(self, i):
        return _State(_p(self.q[i], ctypes.c_int32),
                      _p(self.delta[i], ctypes.c_float),
                      _p(self.zero[i], ctypes.c_float),
                      _p(self.val[i], ctypes.c_float))

    def copy(self):
        s = State(self.cfg, self.count)
        s.q[...] = self.q
        s.delta[...] = self.delta
        s.zero[...] = self.zero
        s.val[...] = self.val
        return s


def lam(dt, A):
    return float(lib().oref_lambda(float(dt), float(A)))


def bf16_round(v):
    v = _f32(v)
    out = np.empty_like(v)
    f = lib().oref_bf16_round
    for i, x in enumerate(v.reshape(-1)):
        out.reshape(-1)[i] = f(float(x))
    return out


def quantize_row(fmt, v):
    """Refit and round one row.  Returns (codes, delta, zero, pre) where pre
    is the pre-rounding value v*inv of each entry (the exact product,
    stored as float32)."""
    v = _f32(v)
    N = v.shape[0]
    q = np.zeros(N, np.int32)
    pre = np.zeros(N, np.float32)
    d = ctypes.c_float()
    z = ctypes.c_float()
    lib().oref_quantize_row_dbg(fmt, N, _p(v, ctypes.c_float),
                                _p(q, ctypes.c_int32), ctypes.byref(d),
                                ctypes.byref(z), _p(pre, ctypes.c_float))
    return q, np.float32(d.value), np.float32(z.value), pre


def dequantize_row(fmt, q, delta, zero):
    q = np.ascontiguousarray(q, dtype=np.int32)
    out = np.zeros(q.shape[0], np.float32)
    lib().oref_dequantize_row(fmt, q.shape[0], _p(q, ctypes.c_int32),
                              ctypes.c_float(delta), ctypes.c_float(zero),
                              _p(out, ctypes.c_float))
    return out


def state_from_f32(cfg: Cfg, S):
    """S[count][H][P][N] (or [H][P][N]) fp32 -> logical State."""
    S = _f32(S)
    if S.ndim == 3:
        S = S[None]
    st = State(cfg, S.shape[0])
    c = cfg.c()
    for i in range(S.shape[0]):
        Si = np.ascontiguousarray(S[i])
        lib().oref_state_from_f32(ctypes.byref(c), _p(Si, ctypes.c_float),
                                  ctypes.byref(st.c(i)))
    return st


def state_to_f32(st: State):
    cfg = st.cfg
    out = np.zeros((st.count, cfg.nheads, cfg.headdim, cfg.d_state),
                   np.float32)
    c = cfg.c()
    for i in range(st.count):
        lib().oref_state_to_f32(ctypes.byref(c), ctypes.byref(st.c(i)),
                                _p(out[i], ctypes.c_float))
    return out


def step(cfg: Cfg, st: State, i, x, B, C, dt, A, D, want_pre=False):
    """One decode step of state pair i.  x[H][P], B/C[G][N], dt/A/D[H].
    Returns y[H][P] (and pre[H*P][N] when want_pre)."""
    x, B, C, dt, A, D = map(_f32, (x, B, C, dt, A, D))
    y = np.zeros((cfg.nheads, cfg.headdim), np.float32)
    pre = np.zeros((cfg.rows, cfg.d_state), np.float32) if want_pre else None
    c = cfg.c()
    lib().oref_step(ctypes.byref(c), ctypes.byref(st.c(i)),
                    _p(x, ctypes.c_float), _p(B, ctypes.c_float),
                    _p(C, ctypes.c_float), _p(dt, ctypes.c_float),
                    _p(A, ctypes.c_float), _p(D, ctypes.c_float),
                    _p(y, ctypes.c_float),
                    _p(pre, ctypes.c_float) if want_pre else None)
    return (y, pre) if want_pre else y


def scan(cfg: Cfg, st: State, i, x, B, C, dt, A, D):
    """T steps on state pair i.  x[T][H][P], B/C[T][G][N], dt[T][H]."""
    x, B, C, dt, A, D = map(_f32, (x, B, C, dt, A, D))
    T = x.shape[0]
    y = np.zeros((T, cfg.nheads, cfg.headdim), np.float32)
    c = cfg.c()
    lib().oref_scan(ctypes.byref(c), ctypes.byref(st.c(i)), T,
                    _p(x, ctypes.c_float), _p(B, ctypes.c_float),
                    _p(C, ctypes.c_float), _p(dt, ctypes.c_float),
                    _p(A, ctypes.c_float), _p(D, ctypes.c_float),
                    _p(y, ctypes.c_float))
    return y


def step_diag(cfg: Cfg, st: State, i, x, B, C, dt, A, D):
    """Diagnostics of the decode step pair i would take (state unchanged):
    [H][P][4] = reversals, readout reversal error, readout rounding error,
    readout signal."""
    x, B, C, dt, A, D = map(_f32, (x, B, C, dt, A, D))
    out = np.zeros((cfg.nheads, cfg.headdim, 4), np.float32)
    c = cfg.c()
    lib().oref_step_diag(ctypes.byref(c), ctypes.byref(st.c(i)), _p(x, ctypes.c_float),
                         _p(B, ctypes.c_float), _p(C, ctypes.c_float), _p(dt, ctypes.c_float),
                         _p(A, ctypes.c_float), _p(D, ctypes.c_float), _p(out, ctypes.c_float))
    return out


class _SR(ctypes.Structure):
    _fields_ = [("seed", ctypes.c_uint64), ("step", ctypes.c_uint32),
                ("layer", ctypes.c_uint32), ("slot", ctypes.c_uint32)]


def philox4x32_10(ctr, key):
    """Philox4x32-10 of a 4-word counter and 2-word key (uint32 each)."""
    c = (ctypes.c_uint32 * 4)(*[int(v) & 0xFFFFFFFF for v in ctr])
    k = (ctypes.c_uint32 * 2)(*[int(v) & 0xFFFFFFFF for v in key])
    out = (ctypes.c_uint32 * 4)()
    lib().oref_philox4x32_10(c, k, out)
    return [int(v) for v in out]


def sr_draws(seed, step, layer, slot, rows, N):
    """The 16-bit draws of every entry of `rows` rows: uint32 [rows][N]."""
    r = _SR(seed, step, layer, slot)
    u = np.zeros((rows, N), np.uint32)
    for row in range(rows):
        for n in range(N):
            u[row, n] = lib().oref_sr_u16(ctypes.byref(r), row, n, N)
    return u


def quantize_row_sr(fmt, v, u16):
    """Refit one row and round it stochastically with the given 16-bit
    draws.  Returns (codes, delta, zero)."""
    v = _f32(v)
    N = v.shape[0]
    u = np.ascontiguousarray(u16, dtype=np.uint32)
    q = np.zeros(N, np.int32)
    d = ctypes.c_float()
    z = ctypes.c_float()
    lib().oref_quantize_row_sr(fmt, N, _p(v, ctypes.c_float), _p(u, ctypes.c_uint32),
                               _p(q, ctypes.c_int32), ctypes.byref(d), ctypes.byref(z))
    return q, np.float32(d.value), np.float32(z.value)


def step_sr(cfg: Cfg, st: State, i, x, B, C, dt, A, D, seed, step, layer, slot):
    """One decode step on pair i with stochastic rounding."""
    x, B, C, dt, A, D = map(_f32, (x, B, C, dt, A, D))
    y = np.zeros((cfg.nheads, cfg.headdim), np.float32)
    r = _SR(seed, step, layer, slot)
    c = cfg.c()
    lib().oref_step_sr(ctypes.byref(c), ctypes.byref(st.c(i)), ctypes.byref(r),
                       _p(x, ctypes.c_float), _p(B, ctypes.c_float), _p(C, ctypes.c_float),
                       _p(dt, ctypes.c_float), _p(A, ctypes.c_float), _p(D, ctypes.c_float),
                       _p(y, ctypes.c_float))
    return y


def scan_sr(cfg: Cfg, st: State, i, x, B, C, dt, A, D, seed, step0, layer, slot):
    """T steps on pair i with stochastic rounding, token t at step0 + t."""
    x, B, C, dt, A, D = map(_f32, (x, B, C, dt, A, D))
    T = x.shape[0]
    y = np.zeros((T, cfg.nheads, cfg.headdim), np.float32)
    r = _SR(seed, step0, layer, slot)
    c = cfg.c()
    lib().oref_scan_sr(ctypes.byref(c), ctypes.byref(st.c(i)), ctypes.byref(r), T,
                       _p(x, ctypes.c_float), _p(B, ctypes.c_float), _p(C, ctypes.c_float),
                       _p(dt, ctypes.c_float), _p(A, ctypes.c_float), _p(D, ctypes.c_float),
                       _p(y, ctypes.c_float))
    return y


def prefill(cfg: Cfg, st: State, i, x, B, C, dt, A, D):
    """Prefill hand-off on state pair i: T tokens of the fp32 recurrence with
    no rounding between tokens, y from the fp32 state, one quantization of
    the final state.  x[T][H][P], B/C[T][G][N], dt[T][H]."""
    x, B, C, dt, A, D = map(_f32, (x, B, C, dt, A, D))
    T = x.shape[0]
    y = np.zeros((T, cfg.nheads, cfg.headdim), np.float32)
    c = cfg.c()
    lib().oref_prefill(ctypes.byref(c), ctypes.byref(st.c(i)), T,
                       _p(x, ctypes.c_float), _p(B, ctypes.c_float),
                       _p(C, ctypes.c_float), _p(dt, ctypes.c_float),
                       _p(A, ctypes.c_float), _p(D, ctypes.c_float),
                       _p(y, ctypes.c_float))
    return y


def scan_f64(cfg: Cfg, S0, x, B, C, dt, A, D):
    """Unquantized fp64 trajectory from S0[H][P][N]; returns (S_T, y[T])."""
    x, B, C, dt, A, D = map(_f32, (x, B, C, dt, A, D))
    S = np.ascontiguousarray(S0, dtype=np.float64).copy()
    T = x.shape[0]
    y = np.zeros((T, cfg.nheads, cfg.headdim), np.float64)
    c = cfg.c()
    lib().oref_scan_f64(ctypes.byref(c), _p(S, ctypes.c_double), T,
                        _p(x, ctypes.c_float), _p(B, ctypes.c_float),
                        _p(C, ctypes.c_float), _p(dt, ctypes.c_float),
                        _p(A, ctypes.c_float), _p(D, ctypes.c_float),
                        _p(y, ctypes.c_double))
    return S, y


def decode_batch(cfg: Cfg, st: State, nl, batch, x, B, C, dt, A, D):
    """One decode step for nl layers x batch requests; st holds nl*batch
    pairs ordered [l][b].  x[nl][batch][H][P], B/C[nl][batch][G][N],
    dt[nl][batch][H], A/D[nl][H].  Returns y[nl][batch][H][P]."""
    assert st.count == nl * batch
    x, B, C, dt, A, D = map(_f32, (x, B, C, dt, A, D))
    y = np.zeros((nl, batch, cfg.nheads, cfg.headdim), np.float32)
    arr = (_State * st.count)(*[st.c(i) for i in range(st.count)])
    c = cfg.c()
    lib().oref_decode_batch(ctypes.byref(c), nl, batch, arr,
                            _p(x, ctypes.c_float), _p(B, ctypes.c_float),
                            _p(C, ctypes.c_float), _p(dt, ctypes.c_float),
                            _p(A, ctypes.c_float), _p(D, ctypes.c_float),
                            _p(y, ctypes.c_float))
    return y


# ---------------------------------------------------------------------------
# DAMP mixed-tier state ("Mamba state quantization for inference", "Mixed
# precision spends bits on persistent channels")
# ---------------------------------------------------------------------------

class _DampCfg(ctypes.Structure):
    _fields_ = [("nheads", ctypes.c_int), ("headdim", ctypes.c_int),
                ("d_state", ctypes.c_int), ("ngroups", ctypes.c_int),
                ("n_protected", ctypes.c_int), ("chan", ctypes.POINTER(ctypes.c_int32))]


class _DampState(ctypes.Structure):
    _fields_ = [("hi", ctypes.POINTER(ctypes.c_float)),
                ("q", ctypes.POINTER(ctypes.c_int32)),
                ("delta", ctypes.POINTER(ctypes.c_float)),
                ("zero", ctypes.POINTER(ctypes.c_float))]


@dataclass
class DampCfg:
    """One layer's tiered state: nheads heads of d_state key channels, each a
    rotated value vector of headdim entries; chan[h][m] = key channel at
    position m, the first n_protected positions in FP16."""
    nheads: int
    headdim: int
    d_state: int
    ngroups: int
    n_protected: int
    chan: np.ndarray

    def c(self):
        self._chan = np.ascontiguousarray(self.chan, dtype=np.int32).reshape(
            self.nheads, self.d_state)
        return _DampCfg(self.nheads, self.headdim, self.d_state, self.ngroups,
                        self.n_protected, _p(self._chan, ctypes.c_int32))


class DampState:
    """Tiered state of ``count`` (layer, request) pairs."""

    def __init__(self, cfg: DampCfg, count: int = 1):
        H, P, N, K = cfg.nheads, cfg.headdim, cfg.d_state, cfg.n_protected
        self.cfg = cfg
        self.count = count
        self.hi = np.zeros((count, H, K, P), np.float32)
        self.q = np.zeros((count, H, N - K, P), np.int32)
        self.delta = np.zeros((count, H, N - K), np.float32)
        self.zero = np.zeros((count, H, N - K), np.float32)

    def c(self, i):
        return _DampState(_p(self.hi[i], ctypes.c_float), _p(self.q[i], ctypes.c_int32),
                          _p(self.delta[i], ctypes.c_float), _p(self.zero[i], ctypes.c_float))

    def copy(self):
        s = DampState(self.cfg, self.count)
        for k in ("hi", "q", "delta", "zero"):
            getattr(s, k)[...] = getattr(self, k)
        return s


def hadamard(v):
    """Sylvester-Hadamard rotation of a vector of power-of-two length:
    out[k] = sum_p (-1)^popcount(k&p) v[p], summed in double, rounded once."""
    v = _f32(v)
    out = np.zeros_like(v)
    lib().oref_hadamard(v.shape[0], _p(v, ctypes.c_float), 1, _p(out, ctypes.c_float))
    return out


def fp16_round(v):
    v = _f32(v)
    out = np.empty_like(v)
    f = lib().oref_fp16_round
    for i, x in enumerate(v.reshape(-1)):
        out.reshape(-1)[i] = f(float(x))
    return out


def damp_from_f32(cfg: DampCfg, S):
    """S[count][H][P][N] (or [H][P][N]) fp32 -> DampState."""
    S = _f32(S)
    if S.ndim == 3:
        S = S[None]
    st = DampState(cfg, S.shape[0])
    c = cfg.c()
    for i in range(S.shape[0]):
        lib().oref_damp_from_f32(ctypes.byref(c), _p(S[i], ctypes.c_float),
                                 ctypes.byref(st.c(i)))
    return st


def damp_to_f32(st: DampState):
    cfg = st.cfg
    out = np.zeros((st.count, cfg.nheads, cfg.headdim, cfg.d_state), np.float32)
    c = cfg.c()
    for i in range(st.count):
        lib().oref_damp_to_f32(ctypes.byref(c), ctypes.byref(st.c(i)), _p(out[i], ctypes.c_float))
    return out


def damp_step(cfg: DampCfg, st: DampState, i, x, B, C, dt, A, D):
    """One decode step of pair i on the tiered state.  x[H][P], B/C[G][N],
    dt/A/D[H]; returns y[H][P]."""
    x, B, C, dt, A, D = map(_f32, (x, B, C, dt, A, D))
    y = np.zeros((cfg.nheads, cfg.headdim), np.float32)
    c = cfg.c()
    lib().oref_damp_step(ctypes.byref(c), ctypes.byref(st.c(i)), _p(x, ctypes.c_float),
                         _p(B, ctypes.c_float), _p(C, ctypes.c_float), _p(dt, ctypes.c_float),
                         _p(A, ctypes.c_float), _p(D, ctypes.c_float), _p(y, ctypes.c_float))
    return y
