"""Seeded synthetic inputs for the quantized state update.

This module holds no arithmetic of the method: it only draws the random
tensors that both the CUDA library and the CPU oracle consume.  Shapes and
distributions follow the workloads the pages describe (Mamba-2 130M / 370M /
8B state shapes, "ssm-state-quantization" README, Setup; the 30-layer,
batch-256 serving pool of "Mamba state quantization for inference",
"Recurrent state is fixed per request, not free"):

  x ~ N(0, 1);  B, C ~ N(0, 1/16);  dt = softplus(N(-2, 1));
  A_h = -exp(U(ln 0.5, ln 16));  D ~ N(0, 1);  initial state 0 or N(0, 1).

Every tensor comes from its own PCG64 stream keyed by (seed, tag), and the
initial state of each (layer, request) pair from its own stream keyed by
(seed, tag, layer, request), so that any pair can be regenerated on its own
without drawing the whole pool.
"""
from __future__ import annotations

import concurrent.futures as _cf
import math
import os
from dataclasses import dataclass, field

import numpy as np

_TAGS = {"x": 1, "B": 2, "C": 3, "dt": 4, "A": 5, "D": 6, "S0": 7,
         "Aband": 8, "chan": 9}

# softplus(-2): the median of dt = softplus(N(-2, 1)).
MEDIAN_DT = math.log1p(math.exp(-2.0))


def _rng(seed, tag, *extra):
    return np.random.Generator(np.random.PCG64([seed, _TAGS[tag], *extra]))


def normal(seed, tag, shape, std=1.0):
    a = _rng(seed, tag).standard_normal(shape, dtype=np.float32)
    if std != 1.0:
        a *= np.float32(std)
    return a


def dt_draw(seed, shape):
    z = _rng(seed, "dt").standard_normal(shape, dtype=np.float64) - 2.0
    return np.log1p(np.exp(z)).astype(np.float32)


def A_draw(seed, shape):
    u = _rng(seed, "A").uniform(math.log(0.5), math.log(16.0), size=shape)
    return (-np.exp(u)).astype(np.float32)


def A_banded(seed, nheads):
    """Per-head A whose typical decay lambda_bar = exp(A * median dt) falls in
    the three bands of "ssm-state-quantization" (<= 0.9, (0.9, 0.99],
    > 0.99), in equal thirds (the first bands get the remainder), lambda_bar
    log-uniform inside each band ([0.5, 0.9], (0.9, 0.99], (0.99, 0.999])."""
    r = _rng(seed, "Aband")
    n0 = (nheads + 2) // 3
    n1 = (nheads + 1) // 3
    n2 = nheads - n0 - n1
    bands = [(0.5, 0.9, n0), (0.9, 0.99, n1), (0.99, 0.999, n2)]
    lam = []
    for lo, hi, n in bands:
        lam.append(np.exp(r.uniform(math.log(lo), math.log(hi), size=n)))
    lam = np.concatenate(lam)
    A = (np.log(lam) / MEDIAN_DT).astype(np.float32)
    band = np.concatenate([np.full(n, i) for i, (_, _, n) in enumerate(bands)])
    return A, band


def state_pair(seed, l, b, rows, N):
    """Initial state of one (layer, request) pair, N(0, 1), [rows][N]."""
    return _rng(seed, "S0", l, b).standard_normal((rows, N), dtype=np.float32)


def state_all(seed, nl, batch, rows, N, threads=None):
    """Initial state of all pairs, [nl][batch][rows][N], drawn pair by pair
    (identical to state_pair for every pair), in host threads."""
    out = np.empty((nl, batch, rows, N), np.float32)

    def fill(lb):
        l, b = divmod(lb, batch)
        out[l, b] = state_pair(seed, l, b, rows, N)

    threads = threads or min(32, os.cpu_count() or 1)
    with _cf.ThreadPoolExecutor(threads) as ex:
        list(ex.map(fill, range(nl * batch)))
    return out


@dataclass
class Decode:
    """One decode step over nl layers and a batch of requests."""
    name: str
    seed: int
    nl: int
    batch: int
    nheads: int
    headdim: int
    d_state: int
    ngroups: int
    fmt: str
    init: str = "normal"          # "zero" or "normal"
    head_mask: np.ndarray | None = None
    extra: dict = field(default_factory=dict)

    @property
    def rows(self):
        return self.nheads * self.headdim

    def inputs(self):
        nl, Bt, H, P, N, G = (self.nl, self.batch, self.nheads, self.headdim,
                              self.d_state, self.ngroups)
        s = self.seed
        return dict(
            x=normal(s, "x", (nl, Bt, H, P)),
            B=normal(s, "B", (nl, Bt, G, N), 0.25),
            C=normal(s, "C", (nl, Bt, G, N), 0.25),
            dt=dt_draw(s, (nl, Bt, H)),
            A=A_draw(s, (nl, H)),
            D=normal(s, "D", (nl, H)),
        )

    def state_pair(self, l, b):
        if self.init == "zero":
            return np.zeros((self.rows, self.d_state), np.float32)
        return state_pair(self.seed, l, b, self.rows, self.d_state)

    def state_all(self):
        if self.init == "zero":
            return np.zeros((self.nl, self.batch, self.rows, self.d_state),
                            np.float32)
        return state_all(self.seed, self.nl, self.batch, self.rows,
                         self.d_state)


@dataclass
class Scan:
    """T tokens of one layer for a batch of requests."""
    name: str
    seed: int
    batch: int
    T: int
    nheads: int
    headdim: int
    d_state: int
    ngroups: int
    fmt: str
    banded: bool = False
    init: str = "zero"
    head_mask: np.ndarray | None = None

    @property
    def rows(self):
        return self.nheads * self.headdim

    def inputs(self):
        Bt, T, H, P, N, G = (self.batch, self.T, self.nheads, self.headdim,
                             self.d_state, self.ngroups)
        s = self.seed
        if self.banded:
            A, _ = A_banded(s, H)
        else:
            A = A_draw(s, (H,))
        return dict(
            x=normal(s, "x", (Bt, T, H, P)),
            B=normal(s, "B", (Bt, T, G, N), 0.25),
            C=normal(s, "C", (Bt, T, G, N), 0.25),
            dt=dt_draw(s, (Bt, T, H)),
            A=A,
            D=normal(s, "D", (H,)),
        )

    def bands(self):
        return A_banded(self.seed, self.nheads)[1]


def mid_band_mask(nheads, seed=2):
    """Mask that quantizes only the mid band (0.9 < lambda_bar <= 0.99)."""
    band = A_banded(seed, nheads)[1]
    return (band == 1).astype(np.uint8)


# The five workloads: the tiny parity case, the 130M-shaped decode step, the
# 370M-shaped scan, the 8B-shaped decode and the serving-scale format sweep.
def tiny(T=64):
    return Scan("tiny L1 b1 H2 P8 N16 T64 i8a", seed=0, batch=1, T=T,
                nheads=2, headdim=8, d_state=16, ngroups=1, fmt="i8a")


def decode_130m(fmt="i8a", batch=256, nl=24):
    return Decode(f"mamba2-130m decode L{nl} b{batch} H24 P64 N128 {fmt}",
                  seed=1, nl=nl, batch=batch, nheads=24, headdim=64,
                  d_state=128, ngroups=1, fmt=fmt)


def scan_370m(mask="all", batch=8, T=2048):
    m = None if mask == "all" else mid_band_mask(32)
    return Scan(f"mamba2-370m scan b{batch} T{T} H32 P64 N128 i4a {mask}",
                seed=2, batch=batch, T=T, nheads=32, headdim=64, d_state=128,
                ngroups=1, fmt="i4a", banded=True, head_mask=m)


def decode_8b(fmt="i8a", batch=64):
    return Decode(f"mamba2-8b decode L1 b{batch} H128 P64 N128 G8 {fmt}",
                  seed=3, nl=1, batch=batch, nheads=128, headdim=64,
                  d_state=128, ngroups=8, fmt=fmt)


def sweep_serving(fmt="i8a", batch=256, nl=30):
    # The serving-scale pool starts from the zero state (the workload names
    # no initial state); a few steps of input make it non-zero.
    return Decode(f"serving sweep L{nl} b{batch} H32 P128 N128 {fmt}",
                  seed=4, nl=nl, batch=batch, nheads=32, headdim=128,
                  d_state=128, ngroups=1, fmt=fmt, init="zero")


def damp_channels(seed, n_layers, nheads, d_state):
    """A channel map per (layer, head) for the DAMP mixed-tier layout:
    int32 [n_layers][nheads][d_state], a seeded random permutation each (the
    calibration that would rank channels needs data; any permutation costs
    the same)."""
    rng = _rng(seed, "chan")
    return np.stack([np.stack([rng.permutation(d_state) for _ in range(nheads)])
                     for _ in range(n_layers)]).astype(np.int32)


def decode_130m_damp(batch=256, nl=24):
    """The 130M decode shape for the DAMP layout (16 of 128 key channels in
    FP16, the rest INT8)."""
    return Decode(f"mamba2-130m decode L{nl} b{batch} H24 P64 N128 damp K16",
                  seed=1, nl=nl, batch=batch, nheads=24, headdim=64,
                  d_state=128, ngroups=1, fmt="i8a")
