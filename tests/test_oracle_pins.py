"""Pins of the CPU oracle against what the pages and the mathematics fix.

Nothing here re-types the oracle's own formulas: each test checks the oracle
against an independent closed form, an invariant of the grid, a brute-force
search, a library routine, or a value worked out by hand from the pages'
definitions (tests/golden/).  A plausible slip in the oracle (a dropped term,
a wrong sign or index, a transposed operand, an off-by-one grid) fails at
least one of them.

Sources: "ssm-state-quantization" README, Setup (lambda = exp(dt*A); one scale
per (head, head_dim) row over the d_state entries, refit every step;
symmetric grid [-amax, amax] with step amax/(2^(b-1)-1); asymmetric grid
[min, max] with an integer zero point and step (max-min)/(2^b-1); output read
from the quantized state) and Findings 1 (nearest rounding); "Mamba state
quantization for inference", "Quantization error returns on the next token"
(S_t = A_t S_(t-1) + W_t, and with rounding S_q,t = A_t S_q,(t-1) + W_t + R_t).
"""
import math
import os

import numpy as np
import pytest

import oracle as O
from quantized_recurrent_state_mamba_b200 import workloads as W

QFMTS = [O.I8_SYM, O.I8_ASYM, O.I4_SYM, O.I4_ASYM]
BITS = {O.I8_SYM: 8, O.I8_ASYM: 8, O.I4_SYM: 4, O.I4_ASYM: 4}
GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def qrange(fmt):
    b = BITS[fmt]
    if fmt in (O.I8_SYM, O.I4_SYM):
        qs = 2 ** (b - 1) - 1
        return -qs, qs
    return 0, 2 ** b - 1


def deq64(fmt, q, delta, zero):
    """(q - z) * Delta in double: exact for the ranges involved."""
    return (np.asarray(q, np.float64) - np.float64(zero)) * np.float64(delta)


def rows_zoo(rng, N):
    """Rows of many shapes: normal, shifted all-positive / all-negative, heavy
    tailed, tiny, constant, single outlier, near-constant."""
    out = [
        rng.standard_normal(N),
        rng.standard_normal(N) * 1e-3 + 5.0,
        -np.abs(rng.standard_normal(N)) - 0.5,
        rng.standard_cauchy(N),
        rng.standard_normal(N) * 1e-20,
        np.full(N, 0.75),
        np.full(N, -3.0),
        np.where(np.arange(N) == 3, 100.0, rng.standard_normal(N) * 0.01),
        1.0 + rng.standard_normal(N) * 1e-6,
        rng.uniform(0, 1, N),
    ]
    return [np.asarray(r, np.float32) for r in out]


# ---------------------------------------------------------------------------
# The quantizer (ssm-state-quantization README, Setup; Findings 1)
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("fmt", QFMTS)
@pytest.mark.parametrize("N", [1, 2, 5, 16, 128])
def test_codes_are_nearest_by_enumeration(oref, fmt, N):
    """Every chosen code is a nearest grid level: enumerate every code of the
    format and check none reconstructs closer (ties may go either way)."""
    rng = np.random.default_rng(100 + N + 7 * fmt)
    lo_c, hi_c = qrange(fmt)
    cand = np.arange(lo_c, hi_c + 1, dtype=np.float64)
    for v in rows_zoo(rng, N):
        q, d, z, _ = O.quantize_row(fmt, v)
        assert q.min() >= lo_c and q.max() <= hi_c
        if d == 0:
            assert np.all(np.abs(v) < 1e-30)
            continue
        levels = deq64(fmt, cand, d, z)                    # [ncodes]
        err_all = np.abs(levels[None, :] - v[:, None].astype(np.float64))
        best = err_all.min(axis=1)
        chosen = np.abs(deq64(fmt, q, d, z) - v.astype(np.float64))
        # within a few fp32 ulps of the scaled value (rounding of v*inv)
        slack = 4 * np.finfo(np.float32).eps * np.abs(v.astype(np.float64)) \
            + 1e-12 * d
        assert np.all(chosen <= best + slack), (fmt, v, q, d, z)


@pytest.mark.parametrize("fmt", QFMTS)
def test_reconstruction_within_half_step(oref, fmt):
    """|deq - v| <= Delta/2 + 2 ulp(max|row|) for every entry."""
    rng = np.random.default_rng(7 + fmt)
    for N in (16, 64, 128):
        for v in rows_zoo(rng, N):
            q, d, z, _ = O.quantize_row(fmt, v)
            s = O.dequantize_row(fmt, q, d, z).astype(np.float64)
            ulp = np.spacing(np.float32(np.max(np.abs(v)))).astype(np.float64)
            assert np.all(np.abs(s - v) <= d / 2 + 2 * ulp + 1e-38)


@pytest.mark.parametrize("fmt", [O.I8_ASYM, O.I4_ASYM])
def test_asym_grid_spans_min_max(oref, fmt):
    """Asymmetric grid [min, max] with an integer zero point: the row minimum
    takes code 0 (always), the maximum takes the top code (unless it lies on a
    rounding boundary), and both are reconstructed within Delta/2."""
    rng = np.random.default_rng(11 + fmt)
    qa = 2 ** BITS[fmt] - 1
    for _ in range(300):
        N = int(rng.integers(2, 129))
        v = (rng.standard_normal(N) * rng.uniform(0.01, 10)
             + rng.uniform(-5, 5)).astype(np.float32)
        q, d, z, pre = O.quantize_row(fmt, v)
        i_lo, i_hi = int(np.argmin(v)), int(np.argmax(v))
        assert q[i_lo] == 0
        near_half = abs(abs(pre[i_hi] - np.floor(pre[i_hi])) - 0.5) < 1e-3
        assert q[i_hi] == qa or near_half
        assert float(z) == round(float(z))                # integer zero point
        s = O.dequantize_row(fmt, q, d, z)
        assert abs(float(s[i_lo]) - float(v[i_lo])) <= d / 2 * (1 + 1e-5)
        assert abs(float(s[i_hi]) - float(v[i_hi])) <= d / 2 * (1 + 1e-5)
        # the grid is exactly qa steps wide around [min, max]
        assert abs((qa * float(d)) - (float(v.max()) - float(v.min()))) \
            <= 1e-5 * (float(v.max()) - float(v.min())) + 1e-30


@pytest.mark.parametrize("fmt", [O.I8_SYM, O.I4_SYM])
def test_sym_grid_spans_amax(oref, fmt):
    """Symmetric grid [-amax, amax], step amax/(2^(b-1)-1): the largest
    magnitude takes code +-qs and codes are odd under a sign flip."""
    rng = np.random.default_rng(13 + fmt)
    qs = 2 ** (BITS[fmt] - 1) - 1
    for _ in range(300):
        N = int(rng.integers(1, 129))
        v = (rng.standard_normal(N) * rng.uniform(0.01, 10)).astype(np.float32)
        q, d, z, _ = O.quantize_row(fmt, v)
        assert z == 0
        i = int(np.argmax(np.abs(v)))
        assert q[i] == (qs if v[i] > 0 else -qs)
        assert abs(qs * float(d) - float(np.abs(v).max())) \
            <= 1e-6 * float(np.abs(v).max())
        qn, dn, _, _ = O.quantize_row(fmt, -v)
        assert dn == d and np.array_equal(qn, -q)


@pytest.mark.parametrize("fmt", [O.I8_ASYM, O.I4_ASYM])
def test_asym_dyadic_rows_exact(oref, fmt):
    """Rows built on the grid itself (dyadic values with max - min =
    qa*2^-e and min = -k*2^-e) reconstruct bit-exactly: codes equal the
    construction, Delta = 2^-e, z = k."""
    rng = np.random.default_rng(17 + fmt)
    qa = 2 ** BITS[fmt] - 1
    for _ in range(200):
        e = int(rng.integers(-4, 12))
        k = int(rng.integers(-3 * qa, 3 * qa))
        N = int(rng.integers(2, 129))
        j = rng.integers(0, qa + 1, N)
        j[0], j[-1] = 0, qa
        step = 2.0 ** -e
        v = ((j - k) * step).astype(np.float32)
        q, d, z, _ = O.quantize_row(fmt, v)
        assert d == np.float32(step)
        assert z == k
        assert np.array_equal(q, j)
        assert np.array_equal(O.dequantize_row(fmt, q, d, z), v)


@pytest.mark.parametrize("fmt", QFMTS)
def test_idempotent(oref, fmt):
    """Quantizing a reconstructed row gives back the same codes and zero
    point, and the step within 1 ulp.  This holds while the reconstruction
    (q - z)*Delta is fine compared with the step, i.e. the row's offset is a
    modest number of steps (|z| <= 2^12).  A near-constant row far from zero
    has a zero point of millions of steps; its reconstruction is rounded to
    the ulp of its offset, which can be a visible fraction of a step, and only
    the reconstruction bound above applies to it."""
    rng = np.random.default_rng(19 + fmt)
    for N in (16, 128):
        for v in rows_zoo(rng, N):
            q, d, z, _ = O.quantize_row(fmt, v)
            if abs(float(z)) > 2 ** 12:
                continue
            s = O.dequantize_row(fmt, q, d, z)
            q2, d2, z2, _ = O.quantize_row(fmt, s)
            if d == 0:
                assert d2 == 0 and np.all(q2 == q)
                continue
            assert abs(float(d2) - float(d)) <= np.spacing(np.float32(d))
            assert z2 == z
            assert np.array_equal(q2, q)


@pytest.mark.parametrize("fmt", QFMTS)
def test_power_of_two_scale_equivariance(oref, fmt):
    """Scaling a row by 2^k scales the step by 2^k exactly and leaves codes
    and zero point unchanged (a pure decay step with lambda = 2^k, w = 0)."""
    rng = np.random.default_rng(23 + fmt)
    for v in rows_zoo(rng, 64):
        q, d, z, _ = O.quantize_row(fmt, v)
        if d == 0 or float(np.abs(v).max()) < 1e-30:
            continue
        for k in (-3, -1, 2):
            q2, d2, z2, _ = O.quantize_row(fmt, v * np.float32(2.0 ** k))
            assert d2 == np.float32(d * 2.0 ** k)
            assert z2 == z and np.array_equal(q2, q)


@pytest.mark.parametrize("fmt", QFMTS)
def test_general_scale_equivariance(oref, fmt):
    """For a decay lambda in (0, 1] and rows whose spread is large against
    their fp32 spacing, the codes are unchanged except entries on a rounding
    boundary, and the step scales by lambda up to the fp32 rounding of the
    scaled extremes."""
    rng = np.random.default_rng(29 + fmt)
    qm = qrange(fmt)[1]
    zoo = rows_zoo(rng, 128)
    for v in (zoo[0], zoo[3], zoo[9]):
        q, d, z, pre = O.quantize_row(fmt, v)
        for lam in (0.93, 0.5001, 0.999):
            v2 = (v * np.float32(lam)).astype(np.float32)
            q2, d2, z2, pre2 = O.quantize_row(fmt, v2)
            ext = np.spacing(np.float32(lam * np.abs(v).max())).astype(np.float64)
            tol = 4 * ext / qm + 2 * np.spacing(np.float32(d2)) \
                + 2e-7 * lam * float(d)
            assert abs(float(d2) - lam * float(d)) <= tol
            frac = np.abs(np.abs(pre - np.floor(pre)) - 0.5)
            diff = q2 != q
            assert np.all(frac[diff] < 1e-3)


def test_degenerate_rows(oref):
    """All-zero rows store Delta = 0 and codes 0; constant rows reconstruct
    exactly; rows too small for a normal fp32 step flush to zero."""
    for fmt in QFMTS:
        q, d, z, _ = O.quantize_row(fmt, np.zeros(16, np.float32))
        assert d == 0 and z == 0 and np.all(q == 0)
        for c in (0.75, -3.0, 1e-3):
            v = np.full(16, c, np.float32)
            q, d, z, _ = O.quantize_row(fmt, v)
            s = O.dequantize_row(fmt, q, d, z)
            if fmt in (O.I8_ASYM, O.I4_ASYM):
                assert np.array_equal(s, v)
            else:
                assert np.allclose(s, v, rtol=2e-7, atol=0)
        tiny = np.full(16, 1e-40, np.float32)
        q, d, z, _ = O.quantize_row(fmt, tiny)
        assert d == 0 and np.all(O.dequantize_row(fmt, q, d, z) == 0)


def _golden_rows():
    out = []
    with open(os.path.join(GOLDEN, "quantizer_worked_examples.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            fmt, vals, delta, zero, codes = [t.strip() for t in line.split("|")]
            out.append((O.FORMATS[fmt],
                        np.array([float(t) for t in vals.split()], np.float32),
                        float(delta), float(zero),
                        np.array([int(t) for t in codes.split()], np.int32)))
    return out


def test_worked_examples(oref):
    """Rows quantized by hand from the grid definitions (tests/golden)."""
    rows = _golden_rows()
    assert len(rows) >= 6
    for fmt, v, delta, zero, codes in rows:
        q, d, z, _ = O.quantize_row(fmt, v)
        assert np.array_equal(q, codes), (fmt, v, q, codes)
        assert z == zero
        assert abs(float(d) - delta) <= 1e-6 * abs(delta) + 1e-38


# ---------------------------------------------------------------------------
# The recurrence and the readout
# ---------------------------------------------------------------------------

def _closed_form(S0, x, B, C, dt, A, D, G):
    """Unrolled recurrence in fp64 without any recursion:
    S_T = (prod_t lam_t) S0 + sum_t (prod_{s>t} lam_s) dt_t x_t B_t, and
    y_t = C_t . S_t + D x_t, with lam_t = exp(dt_t A) per head and B/C taken
    from group g(h) = h // (H/G)."""
    T, H, P = x.shape
    N = S0.shape[-1]
    hpg = H // G
    S0 = S0.astype(np.float64)
    lam = np.exp(dt.astype(np.float64) * A.astype(np.float64)[None, :])  # [T][H]
    g_of = np.arange(H) // hpg
    Bh = B.astype(np.float64)[:, g_of, :]                                # [T][H][N]
    Ch = C.astype(np.float64)[:, g_of, :]
    ys = np.zeros((T, H, P))
    S_t = None
    for t_end in range(1, T + 1):
        # decay products over (s, t_end]
        logl = np.log(lam[:t_end])                                       # [t][H]
        suffix = np.exp(np.cumsum(logl[::-1], axis=0)[::-1])            # prod_{s>=t}
        after = np.concatenate([suffix[1:], np.ones((1, H))], axis=0)    # prod_{s>t}
        S_t = suffix[0][:, None, None] * S0
        u = (dt.astype(np.float64)[:t_end] * after)                      # [t][H]
        S_t = S_t + np.einsum("th,thp,thn->hpn", u,
                              x.astype(np.float64)[:t_end], Bh[:t_end])
        ys[t_end - 1] = np.einsum("hpn,hn->hp", S_t, Ch[t_end - 1]) \
            + D.astype(np.float64)[:, None] * x.astype(np.float64)[t_end - 1]
    return S_t, ys


@pytest.mark.parametrize("G", [1, 2])
def test_recurrence_matches_unrolled_closed_form(oref, G):
    """Quantization off (f32 state): T=64 steps of the oracle equal the
    unrolled recurrence within 1e-5 normwise, state and every y_t; the fp64
    trajectory matches it within 1e-12."""
    H, P, N, T = 2 * G, 8, 16, 64
    wl = W.Scan("pin", seed=5, batch=1, T=T, nheads=H, headdim=P,
                d_state=N, ngroups=G, fmt="f32")
    inp = wl.inputs()
    x, B, C, dt = (inp[k][0] for k in ("x", "B", "C", "dt"))
    A, D = inp["A"], inp["D"]
    S0 = W.state_pair(5, 0, 0, H * P, N).reshape(H, P, N)
    cfg = O.Cfg(O.F32, H, P, N, G)
    st = O.state_from_f32(cfg, S0)
    y = O.scan(cfg, st, 0, x, B, C, dt, A, D)
    S_T = O.state_to_f32(st)[0]
    S_ref, y_ref = _closed_form(S0, x, B, C, dt, A, D, G)
    assert np.linalg.norm(S_T - S_ref) <= 1e-5 * np.linalg.norm(S_ref)
    for t in range(T):
        assert np.linalg.norm(y[t] - y_ref[t]) <= 1e-5 * np.linalg.norm(y_ref[t]) + 1e-6
    S64, y64 = O.scan_f64(cfg, S0, x, B, C, dt, A, D)
    assert np.linalg.norm(S64 - S_ref) <= 1e-12 * np.linalg.norm(S_ref)
    assert np.linalg.norm(y64 - y_ref) <= 1e-12 * np.linalg.norm(y_ref)


def test_readout_closed_form_first_token(oref):
    """From the zero state, one step gives S = dt x B and
    y = (dt x)(C . B) + D x: exactly (to fp32 rounding) with an f32 state, and
    within sum_n |C_n| Delta/2 with a quantized state (the output is read from
    the quantized state)."""
    H, P, N = 4, 8, 16
    wl = W.Scan("pin", seed=9, batch=1, T=1, nheads=H, headdim=P,
                d_state=N, ngroups=1, fmt="f32")
    inp = wl.inputs()
    x, B, C, dt = (inp[k][0, 0] for k in ("x", "B", "C", "dt"))
    A, D = inp["A"], inp["D"]
    xd = x.astype(np.float64)
    cb = float(np.dot(C[0].astype(np.float64), B[0].astype(np.float64)))
    y_ref = dt.astype(np.float64)[:, None] * xd * cb + D.astype(np.float64)[:, None] * xd
    for fmt in [O.F32] + QFMTS:
        cfg = O.Cfg(fmt, H, P, N, 1)
        st = O.State(cfg)
        y = O.step(cfg, st, 0, x, B, C, dt, A, D)
        if fmt == O.F32:
            assert np.allclose(y, y_ref, rtol=1e-6, atol=1e-7)
        else:
            bound = np.sum(np.abs(C[0])) * st.delta[0].reshape(H, P) / 2
            assert np.all(np.abs(y - y_ref) <= bound * (1 + 1e-4) + 1e-6)


def test_special_cases(oref):
    """dt = 0 leaves an f32 state unchanged and a quantized state's codes
    unchanged (lambda = 1, no input); x = 0 is a pure decay; A = -inf forgets
    the past (S = dt x B)."""
    H, P, N = 2, 8, 16
    rng = np.random.default_rng(3)
    S0 = rng.standard_normal((H, P, N)).astype(np.float32)
    x = rng.standard_normal((H, P)).astype(np.float32)
    B = (rng.standard_normal((1, N)) * 0.25).astype(np.float32)
    C = (rng.standard_normal((1, N)) * 0.25).astype(np.float32)
    A = np.array([-1.0, -4.0], np.float32)
    D = np.zeros(H, np.float32)
    dt = np.array([0.3, 0.05], np.float32)

    cfg = O.Cfg(O.F32, H, P, N)
    st = O.state_from_f32(cfg, S0)
    O.step(cfg, st, 0, x, B, C, np.zeros(H, np.float32), A, D)
    assert np.array_equal(O.state_to_f32(st)[0], S0)

    for fmt in QFMTS:
        cq = O.Cfg(fmt, H, P, N)
        st = O.state_from_f32(cq, S0)
        q0, d0, z0 = st.q.copy(), st.delta.copy(), st.zero.copy()
        O.step(cq, st, 0, x, B, C, np.zeros(H, np.float32), A, D)
        assert np.array_equal(st.q, q0) and np.array_equal(st.zero, z0)
        assert np.all(np.abs(st.delta - d0) <= np.spacing(d0))

    st = O.state_from_f32(cfg, S0)
    O.step(cfg, st, 0, np.zeros_like(x), B, C, dt, A, D)
    lam = np.exp(dt.astype(np.float64) * A)[:, None, None]
    assert np.allclose(O.state_to_f32(st)[0], lam * S0, rtol=2e-7, atol=0)

    st = O.state_from_f32(cfg, S0)
    O.step(cfg, st, 0, x, B, C, dt, np.full(H, -np.inf, np.float32), D)
    w = dt.astype(np.float64)[:, None, None] * x[:, :, None] * B[0][None, None, :]
    assert np.allclose(O.state_to_f32(st)[0], w, rtol=2e-7, atol=0)


def test_mask_keeps_fp32_rows(oref):
    """Heads with mask 0 keep an unrounded fp32 row: their trajectory equals
    the f32-format run, while masked-in heads are rounded."""
    H, P, N, T = 3, 8, 16, 8
    wl = W.Scan("pin", seed=12, batch=1, T=T, nheads=H, headdim=P,
                d_state=N, ngroups=1, fmt="i4a")
    inp = wl.inputs()
    x, B, C, dt = (inp[k][0] for k in ("x", "B", "C", "dt"))
    A, D = inp["A"], inp["D"]
    mask = np.array([0, 1, 0], np.uint8)
    cm = O.Cfg(O.I4_ASYM, H, P, N, 1, mask)
    cf = O.Cfg(O.F32, H, P, N, 1)
    sm, sf = O.State(cm), O.State(cf)
    O.scan(cm, sm, 0, x, B, C, dt, A, D)
    O.scan(cf, sf, 0, x, B, C, dt, A, D)
    Sm, Sf = O.state_to_f32(sm)[0], O.state_to_f32(sf)[0]
    assert np.array_equal(Sm[0], Sf[0]) and np.array_equal(Sm[2], Sf[2])
    assert not np.array_equal(Sm[1], Sf[1])


def test_error_feedback_law(oref):
    """With rounding, the stored state obeys S_q,t = lam_t S_q,(t-1) + W_t +
    R_t ("Quantization error returns on the next token"), so the error
    against the exact trajectory is the unrolled sum of the residuals:
    S_q,T - S_T = sum_t (prod_{s>t} lam_s) R_t.  Each R_t is bounded by half a
    step per entry plus the fp32 rounding of the update."""
    H, P, N, T = 2, 8, 16, 32
    wl = W.Scan("pin", seed=21, batch=1, T=T, nheads=H, headdim=P,
                d_state=N, ngroups=1, fmt="i8a")
    inp = wl.inputs()
    x, B, C, dt = (inp[k][0] for k in ("x", "B", "C", "dt"))
    A, D = inp["A"], inp["D"]
    cfg = O.Cfg(O.I8_ASYM, H, P, N)
    st = O.State(cfg)
    S_prev = np.zeros((H, P, N))
    lam = np.array([[O.lam(dt[t, h], A[h]) for h in range(H)]
                    for t in range(T)], np.float64)
    err = np.zeros((H, P, N))
    for t in range(T):
        O.step(cfg, st, 0, x[t], B[t], C[t], dt[t], A, D)
        S_q = O.state_to_f32(st)[0].astype(np.float64)
        Wt = (dt[t].astype(np.float64)[:, None, None]
              * x[t].astype(np.float64)[:, :, None] * B[t][0][None, None, :])
        R = S_q - (lam[t][:, None, None] * S_prev + Wt)
        half = st.delta[0].reshape(H, P)[:, :, None].astype(np.float64) / 2
        assert np.all(np.abs(R) <= half + 1e-6 * (np.abs(S_q) + 1e-30))
        err = lam[t][:, None, None] * err + R
        S_prev = S_q
    S_exact, _ = O.scan_f64(cfg, np.zeros((H, P, N)), x, B, C, dt, A, D)
    lam_err = np.abs(lam - np.exp(dt.astype(np.float64) * A)).max()
    assert lam_err < 1e-7
    assert np.allclose(S_prev - S_exact, err, atol=1e-5, rtol=1e-4)


def test_bf16_rounding_matches_torch(oref):
    """bf16 storage rounds to nearest even: same as torch's CPU conversion."""
    torch = pytest.importorskip("torch")
    rng = np.random.default_rng(31)
    v = np.concatenate([rng.standard_normal(2000).astype(np.float32),
                        np.array([1.0, -0.0, 0.0, 1.00390625, 1.01171875,
                                  3.0e38, -1e-38, 65504.0], np.float32)])
    ours = O.bf16_round(v)
    ref = torch.from_numpy(v).to(torch.bfloat16).to(torch.float32).numpy()
    assert np.array_equal(ours.view(np.uint32), ref.view(np.uint32))


def test_lambda_bands_of_scan_workload():
    """The 370M-shaped scan workload puts its heads in the three lambda bands
    of "ssm-state-quantization" (<= 0.9, (0.9, 0.99], > 0.99) in thirds."""
    A, band = W.A_banded(2, 32)
    lam_bar = np.exp(A.astype(np.float64) * W.MEDIAN_DT)
    assert np.all(lam_bar[band == 0] <= 0.9) and np.all(lam_bar[band == 0] >= 0.5 - 1e-9)
    assert np.all((lam_bar[band == 1] > 0.9) & (lam_bar[band == 1] <= 0.99))
    assert np.all((lam_bar[band == 2] > 0.99) & (lam_bar[band == 2] <= 0.999))
    assert [int((band == i).sum()) for i in range(3)] == [11, 11, 10]
    assert abs(W.MEDIAN_DT - 0.126928) < 1e-6


@pytest.mark.parametrize("fmt", QFMTS)
def test_output_read_from_quantized_state(oref, fmt):
    """The output is read from the state as stored after rounding
    ("ssm-state-quantization" README, Setup: unlike the INT4 baseline it
    cites, the output comes from the quantized state): y equals
    C . S_stored + D x for the stored (dequantized) state, and differs from
    the readout of the unrounded update by about the rounding error."""
    H, P, N = 4, 8, 16
    rng = np.random.default_rng(37 + fmt)
    S0 = rng.standard_normal((H, P, N)).astype(np.float32)
    x = rng.standard_normal((H, P)).astype(np.float32)
    B = (rng.standard_normal((1, N)) * 0.25).astype(np.float32)
    C = (rng.standard_normal((1, N)) * 0.25).astype(np.float32)
    dt = np.full(H, 0.2, np.float32)
    A = np.array([-1.0, -2.0, -0.5, -4.0], np.float32)
    D = rng.standard_normal(H).astype(np.float32)
    cq = O.Cfg(fmt, H, P, N)
    st = O.state_from_f32(cq, S0)
    Sdeq = O.state_to_f32(st)[0]
    y = O.step(cq, st, 0, x, B, C, dt, A, D)
    Ss = O.state_to_f32(st)[0].astype(np.float64)
    y_stored = np.einsum("hpn,n->hp", Ss, C[0].astype(np.float64)) \
        + D.astype(np.float64)[:, None] * x
    scale = np.einsum("hpn,n->hp", np.abs(Ss), np.abs(C[0])) + np.abs(D[:, None] * x)
    assert np.all(np.abs(y - y_stored) <= 1e-6 * scale)
    # the unrounded update from the same starting values reads differently
    cf = O.Cfg(O.F32, H, P, N)
    sf = O.state_from_f32(cf, Sdeq)
    y_f = O.step(cf, sf, 0, x, B, C, dt, A, D)
    assert np.max(np.abs(y_f - y) / scale) > 1e-5


# ---------------------------------------------------------------------------
# Prefill hand-off ("Mamba state quantization for inference", phase-aware
# benchmarks: prefill in FP32, then the final state written into the packed
# cache)
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("fmt", [O.F32] + QFMTS)
def test_prefill_matches_unrolled_closed_form(oref, fmt):
    """T=64 tokens of the prefill from an N(0,1) state: every y_t equals the
    unrolled fp64 recurrence within 1e-5 normwise (y is read from the fp32
    state, not the codes), and the stored state is the closed-form S_T
    quantized once: within half a step of S_T per entry (fp32 format: within
    1e-5 normwise)."""
    G, H, P, N, T = 2, 4, 8, 16, 64
    wl = W.Scan("pin", seed=6, batch=1, T=T, nheads=H, headdim=P,
                d_state=N, ngroups=G, fmt="f32")
    inp = wl.inputs()
    x, B, C, dt = (inp[k][0] for k in ("x", "B", "C", "dt"))
    A, D = inp["A"], inp["D"]
    S0 = W.state_pair(6, 0, 0, H * P, N).reshape(H, P, N)
    # the starting state is what the pool holds: S0 in the target format
    cfg = O.Cfg(fmt, H, P, N, G)
    st = O.state_from_f32(cfg, S0)
    S0_stored = O.state_to_f32(st)[0]
    y = O.prefill(cfg, st, 0, x, B, C, dt, A, D)
    S_ref, y_ref = _closed_form(S0_stored, x, B, C, dt, A, D, G)
    for t in range(T):
        assert np.linalg.norm(y[t] - y_ref[t]) <= 1e-5 * np.linalg.norm(y_ref[t]) + 1e-6
    S_T = O.state_to_f32(st)[0]
    if fmt == O.F32:
        assert np.linalg.norm(S_T - S_ref) <= 1e-5 * np.linalg.norm(S_ref)
    else:
        half = st.delta[0].reshape(H, P, 1) / 2
        rng = np.abs(S_ref).max(axis=-1, keepdims=True)
        assert np.all(np.abs(S_T - S_ref) <= half * (1 + 1e-3) + 1e-5 * rng)


@pytest.mark.parametrize("fmt", QFMTS)
def test_prefill_one_token_from_zero(oref, fmt):
    """One token from the zero state: the fp32 state is w = fl(dt x) B
    exactly, so the stored codes are the quantizer applied to that row and
    y = (dt x)(C . B) + D x within fp64 accumulation of fp32 terms."""
    H, P, N = 4, 8, 16
    wl = W.Scan("pin", seed=10, batch=1, T=1, nheads=H, headdim=P,
                d_state=N, ngroups=1, fmt="f32")
    inp = wl.inputs()
    x, B, C, dt = (inp[k][0] for k in ("x", "B", "C", "dt"))
    A, D = inp["A"], inp["D"]
    cfg = O.Cfg(fmt, H, P, N, 1)
    st = O.State(cfg)
    y = O.prefill(cfg, st, 0, x, B, C, dt, A, D)
    for h in range(H):
        for p in range(P):
            dtx = np.float32(dt[0, h]) * np.float32(x[0, h, p])
            w = (dtx * B[0, 0]).astype(np.float32)
            q, d, z, _ = O.quantize_row(fmt, w)
            r = h * P + p
            assert np.array_equal(st.q[0, r], q)
            assert st.delta[0, r] == d and st.zero[0, r] == z
            yref = float(np.dot(C[0, 0].astype(np.float64), w.astype(np.float64))) \
                + float(D[h]) * float(x[0, h, p])
            assert abs(float(y[0, h, p]) - yref) <= 1e-6 * (abs(yref) + 1.0)


def test_prefill_closer_to_exact_than_rounding_every_token(oref):
    """The point of the FP32 prefill: over T=256 tokens its final state is
    nearer the exact trajectory than the per-token rounded scan (int4, where
    the per-step rounding error is large): no worse on any head (a fast-
    decaying head forgets all but the last rounding either way) and clearly
    better on average."""
    H, P, N, T = 4, 8, 32, 256
    wl = W.Scan("pin", seed=12, batch=1, T=T, nheads=H, headdim=P,
                d_state=N, ngroups=1, fmt="f32")
    inp = wl.inputs()
    x, B, C, dt = (inp[k][0] for k in ("x", "B", "C", "dt"))
    A, D = inp["A"], inp["D"]
    cfg = O.Cfg(O.I4_ASYM, H, P, N, 1)
    st_p, st_s = O.State(cfg), O.State(cfg)
    O.prefill(cfg, st_p, 0, x, B, C, dt, A, D)
    O.scan(cfg, st_s, 0, x, B, C, dt, A, D)
    S64, _ = O.scan_f64(cfg, np.zeros((H, P, N)), x, B, C, dt, A, D)
    ep = np.abs(O.state_to_f32(st_p)[0] - S64).reshape(H, -1).mean(axis=1)
    es = np.abs(O.state_to_f32(st_s)[0] - S64).reshape(H, -1).mean(axis=1)
    assert np.all(ep <= es * 1.01), (ep, es)
    assert ep.mean() < 0.9 * es.mean(), (ep, es)


# ---------------------------------------------------------------------------
# Stochastic rounding ("ssm-state-quantization" README, Findings 9)
# ---------------------------------------------------------------------------

def _levels(fmt, delta, z):
    qm = {O.I8_ASYM: 255, O.I4_ASYM: 15, O.I8_SYM: 127, O.I4_SYM: 7}[fmt]
    codes = np.arange(-qm, qm + 1) if fmt in (O.I8_SYM, O.I4_SYM) else np.arange(0, qm + 1)
    deq = np.array([O.dequantize_row(fmt, np.array([c], np.int32), delta, z)[0]
                    for c in codes], np.float64)
    return codes, deq


@pytest.mark.parametrize("fmt", QFMTS)
def test_sr_rounds_to_a_bracketing_level(oref, fmt):
    """Every stochastically rounded entry lands on one of the two grid
    levels around it (or the end of the code range), whatever the draw."""
    rng = np.random.default_rng(41)
    for trial in range(40):
        v = (rng.standard_normal(32) * rng.uniform(0.01, 10)).astype(np.float32)
        if trial % 4 == 1:
            v = np.abs(v) + 1.0
        u = rng.integers(0, 65536, 32).astype(np.uint32)
        q, d, z = O.quantize_row_sr(fmt, v, u)
        codes, deq = _levels(fmt, d, z)
        for n in range(32):
            below = deq[deq <= v[n] * (1 + 1e-6) + 1e-30]
            above = deq[deq >= v[n] * (1 - 1e-6) - 1e-30]
            lo = below.max() if below.size else deq.min()
            hi = above.min() if above.size else deq.max()
            got = O.dequantize_row(fmt, q[n:n + 1], d, z)[0]
            assert lo - 1e-6 * abs(lo) <= got <= hi + 1e-6 * abs(hi), (fmt, n, v[n], got, lo, hi)


@pytest.mark.parametrize("fmt", QFMTS)
def test_sr_with_half_draw_is_nearest_off_ties(oref, fmt):
    """A draw of exactly 1/2 turns floor(p + u) into round-half-up: equal to
    the nearest rounding on every entry that is not an exact tie."""
    rng = np.random.default_rng(43)
    for _ in range(30):
        v = (rng.standard_normal(64) * 3).astype(np.float32)
        q_rtn, d, z, pre = O.quantize_row(fmt, v)
        q_sr, d2, z2 = O.quantize_row_sr(fmt, v, np.full(64, 32768, np.uint32))
        assert d == d2 and z == z2
        ties = np.abs(np.abs(pre - np.floor(pre)) - 0.5) == 0
        assert np.array_equal(q_rtn[~ties], q_sr[~ties])


@pytest.mark.parametrize("fmt", [O.I8_ASYM, O.I4_ASYM])
def test_sr_keeps_grid_points(oref, fmt):
    """Rows built on the grid reconstruct exactly under any draws (the
    fractional part is 0, so floor(p + u) = p)."""
    qa = 255 if fmt == O.I8_ASYM else 15
    rng = np.random.default_rng(45)
    e = -6
    codes = rng.integers(0, qa + 1, 48)
    codes[0], codes[1] = 0, qa
    k = 37
    v = ((codes - k) * 2.0 ** e).astype(np.float32)
    for _ in range(5):
        u = rng.integers(0, 65536, 48).astype(np.uint32)
        q, d, z = O.quantize_row_sr(fmt, v, u)
        assert np.array_equal(O.dequantize_row(fmt, q, d, z), v)


@pytest.mark.parametrize("fmt", QFMTS)
def test_sr_is_unbiased(oref, fmt):
    """Averaged over independent draws (Philox at 3000 steps) the
    stochastically rounded row equals the row: within 5 standard errors
    (each draw errs by at most one step), for every entry between the end
    levels of the grid.  (An extreme entry beyond the last level, which the
    integer zero point allows by up to half a step, is clamped and so
    biased by as much.)"""
    rng = np.random.default_rng(47)
    N = 32
    v = (rng.standard_normal(N) * 2).astype(np.float32)
    K = 3000
    acc = np.zeros(N)
    for step in range(K):
        u = O.sr_draws(123, step, 0, 0, 1, N)[0]
        q, d, z = O.quantize_row_sr(fmt, v, u)
        acc += O.dequantize_row(fmt, q, d, z)
    _, d, z, _ = O.quantize_row(fmt, v)
    _, deq = _levels(fmt, d, z)
    inside = (v >= deq.min()) & (v <= deq.max())
    assert inside.sum() >= N - 2
    mean = acc / K
    err = np.abs(mean - v)[inside]
    assert np.all(err <= 5 * (float(d) / 2) / np.sqrt(K)), err.max()


def test_sr_draws_are_uniform_and_keyed(oref):
    """The 16-bit draws: uniform over 16 bins (chi-square, 15 dof, p > 1e-4),
    mean within 5 sigma, and different for a different seed, step, layer,
    slot or row."""
    u = O.sr_draws(7, 11, 2, 5, 64, 128).reshape(-1).astype(np.float64)
    n = u.size
    assert abs(u.mean() - 32767.5) <= 5 * 18918.6 / np.sqrt(n)
    counts = np.bincount((u // 4096).astype(int), minlength=16)
    chi2 = float(((counts - n / 16) ** 2 / (n / 16)).sum())
    assert chi2 < 50.0, chi2                      # 15 dof: p(chi2 > 50) < 1e-5
    base = O.sr_draws(7, 11, 2, 5, 2, 16)
    for other in (O.sr_draws(8, 11, 2, 5, 2, 16), O.sr_draws(7, 12, 2, 5, 2, 16),
                  O.sr_draws(7, 11, 3, 5, 2, 16), O.sr_draws(7, 11, 2, 6, 2, 16)):
        assert np.mean(other == base) < 0.01
    assert np.mean(base[0] == base[1]) < 0.2


def test_sr_scan_is_steps_with_advancing_counter(oref):
    """T tokens of the SR scan equal T SR decode steps at steps step0 .. step0+T-1."""
    H, P, N, T = 2, 8, 16, 12
    wl = W.Scan("pin", seed=13, batch=1, T=T, nheads=H, headdim=P, d_state=N,
                ngroups=1, fmt="i8a")
    inp = wl.inputs()
    x, B, C, dt = (inp[k][0] for k in ("x", "B", "C", "dt"))
    cfg = O.Cfg(O.I8_ASYM, H, P, N, 1)
    a, b = O.State(cfg), O.State(cfg)
    ya = O.scan_sr(cfg, a, 0, x, B, C, dt, inp["A"], inp["D"], 99, 1000, 3, 4)
    yb = np.stack([O.step_sr(cfg, b, 0, x[t], B[t], C[t], dt[t], inp["A"], inp["D"],
                             99, 1000 + t, 3, 4) for t in range(T)])
    assert np.array_equal(a.q, b.q) and np.array_equal(ya, yb)
    # and it differs from nearest rounding somewhere
    c = O.State(cfg)
    O.scan(cfg, c, 0, x, B, C, dt, inp["A"], inp["D"])
    assert not np.array_equal(a.q, c.q)


# ---------------------------------------------------------------------------
# Step diagnostics ("ssm-state-quantization" README, Findings 4 and 5)
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("fmt", QFMTS)
def test_diag_readout_error_is_the_y_difference(oref, fmt):
    """The readout-visible rounding error of a row is y read from the stored
    state minus y read from the unrounded update (the step's y and the f32
    state's y), and the signal is the latter minus D x."""
    H, P, N = 3, 8, 32
    wl = W.Decode("pin", 21, 1, 1, H, P, N, 1, "i8a")
    inp = wl.inputs()
    S0 = W.state_pair(21, 0, 0, H * P, N).reshape(1, H, P, N)
    cfg = O.Cfg(fmt, H, P, N, 1)
    st = O.state_from_f32(cfg, S0)
    x, B, C, dt = (inp[k][0, 0] for k in ("x", "B", "C", "dt"))
    A, D = inp["A"][0], inp["D"][0]
    diag = O.step_diag(cfg, st, 0, x, B, C, dt, A, D)
    # the unrounded update: the same step with an f32 state holding deq(q)
    cf = O.Cfg(O.F32, H, P, N, 1)
    sf = O.state_from_f32(cf, O.state_to_f32(st))
    y_unrounded = O.step(cf, sf, 0, x, B, C, dt, A, D)
    y_stored = O.step(cfg, st, 0, x, B, C, dt, A, D)
    scale = np.abs(y_unrounded) + 1e-3
    assert np.all(np.abs((y_stored - y_unrounded) - diag[..., 2]) <= 1e-4 * scale)
    assert np.all(np.abs(y_unrounded - D[:, None] * x - diag[..., 3]) <= 1e-4 * scale)
    assert np.all(np.abs(diag[..., 1]) <= np.abs(C).sum() * st.delta.max() + 1e-6)


def test_diag_reversal_cases(oref):
    """Hand-built rows on the int8 asymmetric grid: with the zero state
    (lambda irrelevant) the update is s' = w, the applied increment is
    e + w = deq(s') and a reversal is deq of the other sign than w: never,
    since rounding keeps signs on a grid through 0.  A pure requantize
    (dt = 0, so w = 0) has no reversals by definition."""
    H, P, N = 1, 1, 16
    cfg = O.Cfg(O.I8_ASYM, H, P, N, 1)
    x = np.ones((H, P), np.float32)
    A = np.full(H, -1.0, np.float32)
    D = np.zeros(H, np.float32)
    C = np.ones((1, N), np.float32)
    dt = np.ones(H, np.float32)
    rng = np.random.default_rng(3)
    B = rng.standard_normal((1, N)).astype(np.float32)
    st = O.State(cfg)
    diag = O.step_diag(cfg, st, 0, x, B, C, dt, A, D)
    assert diag[0, 0, 0] == 0
    st2 = O.state_from_f32(cfg, rng.standard_normal((1, H, P, N)).astype(np.float32))
    diag2 = O.step_diag(cfg, st2, 0, x, B, C, np.zeros(H, np.float32), A, D)
    assert diag2[0, 0, 0] == 0 and diag2[0, 0, 1] == 0


@pytest.mark.parametrize("fmt", QFMTS)
def test_diag_reversals_from_the_step_results(oref, fmt):
    """Reversal count and reversal readout error recomputed from what the
    plain step produces (the stored state after oref_step, the unrounded
    update of an f32 state, and w = fl(dt x) B): an entry reverses when the
    applied increment (stored - s') + w has the other sign than w."""
    H, P, N = 4, 8, 32
    wl = W.Decode("pin", 22, 1, 1, H, P, N, 1, "i8a")
    inp = wl.inputs()
    S0 = (W.state_pair(22, 0, 0, H * P, N).reshape(1, H, P, N) * 0.05).astype(np.float32)
    cfg = O.Cfg(fmt, H, P, N, 1)
    st = O.state_from_f32(cfg, S0)
    x, B, C, dt = (inp[k][0, 0] for k in ("x", "B", "C", "dt"))
    A, D = inp["A"][0], inp["D"][0]
    diag = O.step_diag(cfg, st, 0, x, B, C, dt, A, D)
    cf = O.Cfg(O.F32, H, P, N, 1)
    sf = O.state_from_f32(cf, O.state_to_f32(st))
    O.step(cf, sf, 0, x, B, C, dt, A, D)
    s_new = O.state_to_f32(sf)[0]                       # s' per entry
    O.step(cfg, st, 0, x, B, C, dt, A, D)
    stored = O.state_to_f32(st)[0]
    w = (dt[:, None].astype(np.float32) * x).astype(np.float32)[..., None] * B[0][None, None, :]
    w = w.astype(np.float32)
    e = (stored - s_new).astype(np.float32)
    inc = (e + w).astype(np.float32)
    rev = ((w > 0) & (inc < 0)) | ((w < 0) & (inc > 0))
    assert np.array_equal(rev.sum(axis=-1), diag[..., 0].astype(int))
    rev_err = np.where(rev, C[0][None, None, :].astype(np.float64) * e, 0.0).sum(axis=-1)
    assert np.all(np.abs(rev_err - diag[..., 1]) <= 1e-5 * (np.abs(diag[..., 3]) + 1e-3))
    assert rev.sum() > 0                     # the small state makes reversals common


def test_decode_batch_is_the_step_of_every_pair(oref):
    """One decode step over nl layers x batch requests (the batched entry the
    decode call mirrors) equals the single-pair step of each (layer,
    request) pair with that pair's own inputs and its layer's A and D."""
    nl, batch = 2, 3
    cfg = O.Cfg(O.I8_ASYM, 4, 4, 16, 2)
    wl = W.Decode("pin", seed=5, nl=nl, batch=batch, nheads=4, headdim=4, d_state=16,
                  ngroups=2, fmt="i8a")
    inp = wl.inputs()
    S0 = np.stack([wl.state_pair(l, b).reshape(4, 4, 16)
                   for l in range(nl) for b in range(batch)])
    st_b = O.state_from_f32(cfg, S0)
    st_p = st_b.copy()
    y_b = O.decode_batch(cfg, st_b, nl, batch, inp["x"], inp["B"], inp["C"], inp["dt"],
                         inp["A"], inp["D"])
    for l in range(nl):
        for b in range(batch):
            i = l * batch + b
            y = O.step(cfg, st_p, i, inp["x"][l, b], inp["B"][l, b], inp["C"][l, b],
                       inp["dt"][l, b], inp["A"][l], inp["D"][l])
            assert np.array_equal(y, y_b[l, b]), (l, b)
    assert np.array_equal(st_b.q, st_p.q)
    assert np.array_equal(st_b.delta, st_p.delta)
    assert np.array_equal(st_b.zero, st_p.zero)
    assert not np.array_equal(inp["A"][0], inp["A"][1])
