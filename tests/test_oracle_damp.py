"""Pins of the oracle's DAMP mixed-tier state against what the pages and the
mathematics fix.

"Mamba state quantization for inference", "Mixed precision spends bits on
persistent channels": each key channel's vector over head_dim is rotated by
a Hadamard matrix; chosen channels stay in FP16, the others become 8-bit
codes with a step and an offset; every token decodes, updates in fp32, fits
new steps and stores the packed state; with 16 channels of 128 in FP16 the
page counts 9.875 bits per value.

The checks: the rotation against scipy's Hadamard matrix and a hand-written
H_4; fp16 rounding against numpy's conversion; the step against the exact
(double) recurrence on the un-rotated state within the tiers' rounding
bounds; y against the readout of the stored state; a one-entry value vector
(P = 1, the rotation the identity) reduces the step to the plain fp32 step,
bit for bit; the order of the INT8 positions does not matter; a full-FP16
and a full-INT8 layout round-trip within their bounds.
"""
import numpy as np
import pytest
import scipy.linalg

import oracle as O
from quantized_recurrent_state_mamba_b200 import workloads as W

H4 = np.array([[1, 1, 1, 1],
               [1, -1, 1, -1],
               [1, 1, -1, -1],
               [1, -1, -1, 1]], np.float64)   # Sylvester H_2 (x) H_2, written out


def test_hadamard_small_written_out(oref):
    for j in range(4):
        e = np.zeros(4, np.float32)
        e[j] = 1.0
        assert np.array_equal(O.hadamard(e), H4[:, j].astype(np.float32))


@pytest.mark.parametrize("P", [1, 2, 16, 64, 128])
def test_hadamard_matches_scipy(oref, P):
    rng = np.random.default_rng(P)
    v = rng.standard_normal(P).astype(np.float32)
    ref = (scipy.linalg.hadamard(P).astype(np.float64) @ v.astype(np.float64)).astype(np.float32)
    got = O.hadamard(v)
    # the double sums of P fp32 values are exact here: equal after rounding
    assert np.array_equal(got, ref)
    # H H = P I
    back = O.hadamard(got).astype(np.float64) / P
    assert np.allclose(back, v, rtol=0, atol=1e-6 * np.abs(v).max())


def test_fp16_rounding_matches_numpy(oref):
    rng = np.random.default_rng(4)
    v = np.concatenate([rng.standard_normal(2000) * 10.0 ** rng.integers(-9, 5, 2000),
                        [65504.0, 65519.9, 65520.0, 1e9, -1e9, 2.0 ** -24, 2.0 ** -25,
                         3 * 2.0 ** -26, 0.0, -0.0]]).astype(np.float32)
    ref = v.astype(np.float16).astype(np.float32)
    got = O.fp16_round(v)
    assert np.array_equal(got.view(np.uint32), ref.view(np.uint32))


def damp_case(seed, H, P, N, G, K, scale=1.0):
    rng = np.random.default_rng(seed)
    chan = np.stack([rng.permutation(N) for _ in range(H)]).astype(np.int32)
    cfg = O.DampCfg(H, P, N, G, K, chan)
    S0 = (W.state_pair(seed, 0, 0, H * P, N).reshape(H, P, N) * scale).astype(np.float32)
    wl = W.Decode("damp", seed, 1, 1, H, P, N, G, "i8a")
    inp = wl.inputs()
    args = tuple(inp[k][0, 0] for k in ("x", "B", "C", "dt")) + (inp["A"][0], inp["D"][0])
    return cfg, S0, args


def exact_step(S, args, H, P, N, G):
    """The recurrence on the un-rotated state, in double: lambda from the
    oracle's own scalar (the decay is pinned elsewhere)."""
    x, B, C, dt, A, D = args
    hpg = H // G
    S1 = np.zeros((H, P, N))
    for h in range(H):
        g = h // hpg
        lam = O.lam(dt[h], A[h])
        S1[h] = lam * S[h].astype(np.float64) + (float(dt[h]) * x[h].astype(np.float64))[:, None] \
            * B[g].astype(np.float64)[None, :]
    return S1


@pytest.mark.parametrize("K", [0, 16, 128])
def test_step_tracks_exact_recurrence(oref, K):
    """After one step the stored state, rotated back, is the exact update of
    the stored state before it within the rounding of each tier: an INT8
    position adds at most Delta/2 per rotated entry, an FP16 position a
    relative 2^-11, and the un-rotation averages P such errors."""
    H, P, N, G = 4, 64, 128, 2
    cfg, S0, args = damp_case(11, H, P, N, G, K)
    st = O.damp_from_f32(cfg, S0)
    Sq0 = O.damp_to_f32(st)[0]
    y = O.damp_step(cfg, st, 0, *args)
    Sq1 = O.damp_to_f32(st)[0].astype(np.float64)
    S1 = exact_step(Sq0, args, H, P, N, G)
    # per key channel: bound from the stored tiers
    for h in range(H):
        for m in range(N):
            n = cfg.chan[h, m]
            if m < K:
                t = st.hi[0, h, m].astype(np.float64)
                bound = np.abs(t).sum() / P * 2.0 ** -11
            else:
                bound = float(st.delta[0, h, m - K]) / 2.0
            # fp32 arithmetic of the update (a few ulps of the entries)
            slack = 1e-6 * (np.abs(S1[h, :, n]).max() + np.abs(Sq0[h, :, n]).max() + 1e-30)
            err = np.abs(Sq1[h, :, n] - S1[h, :, n]).max()
            assert err <= bound * 1.0001 + slack, (h, m, err, bound)
    # y is read from the stored state: D x + sum_n C_n S_q1[p, n]
    x, B, C, dt, A, D = args
    hpg = H // G
    for h in range(H):
        g = h // hpg
        yref = Sq1[h] @ C[g].astype(np.float64) + D[h] * x[h].astype(np.float64)
        sc = np.abs(Sq1[h]) @ np.abs(C[g].astype(np.float64)) + np.abs(D[h] * x[h])
        assert np.all(np.abs(y[h] - yref) <= 1e-5 * sc + 1e-30)


def test_one_entry_value_vector_is_the_fp32_step(oref):
    """P = 1: the rotation is the identity and every INT8 position holds one
    value, which the grid stores exactly (a constant group); with the
    identity channel order the step is the plain fp32 step bit for bit,
    y included."""
    H, P, N, G = 6, 1, 32, 2
    rng = np.random.default_rng(5)
    chan = np.tile(np.arange(N, dtype=np.int32), (H, 1))
    S0 = rng.standard_normal((H, P, N)).astype(np.float32)
    wl = W.Decode("p1", 5, 1, 1, H, P, N, G, "i8a")
    inp = wl.inputs()
    args = tuple(inp[k][0, 0] for k in ("x", "B", "C", "dt")) + (inp["A"][0], inp["D"][0])
    for K in (0, 7):
        cfg = O.DampCfg(H, P, N, G, K, chan)
        st = O.damp_from_f32(cfg, S0)
        if K == 0:
            assert np.array_equal(O.damp_to_f32(st)[0], S0)
        cf = O.Cfg(O.F32, H, P, N, G)
        sf = O.state_from_f32(cf, O.damp_to_f32(st)[0])
        y_ref = O.step(cf, sf, 0, *args)
        y = O.damp_step(cfg, st, 0, *args)
        got = O.damp_to_f32(st)[0]
        ref = O.state_to_f32(sf)[0]
        if K == 0:
            assert np.array_equal(got.view(np.uint32), ref.view(np.uint32))
            assert np.array_equal(y.view(np.uint32), y_ref.view(np.uint32))
        else:
            # protected positions are FP16: equal to the fp32 step's values
            # rounded to fp16
            assert np.array_equal(got[:, :, K:].view(np.uint32), ref[:, :, K:].view(np.uint32))
            assert np.array_equal(got[:, :, :K], O.fp16_round(ref[:, :, :K]))


def test_int8_position_order_does_not_matter(oref):
    """Permuting the INT8 positions (the protected set unchanged) stores the
    same group for each key channel; y changes only by summation order."""
    H, P, N, G, K = 2, 64, 128, 1, 16
    cfg, S0, args = damp_case(12, H, P, N, G, K)
    rng = np.random.default_rng(1)
    chan2 = cfg.chan.copy()
    for h in range(H):
        chan2[h, K:] = chan2[h, K:][rng.permutation(N - K)]
    cfg2 = O.DampCfg(H, P, N, G, K, chan2)
    st1, st2 = O.damp_from_f32(cfg, S0), O.damp_from_f32(cfg2, S0)
    y1 = O.damp_step(cfg, st1, 0, *args)
    y2 = O.damp_step(cfg2, st2, 0, *args)
    assert np.array_equal(O.damp_to_f32(st1), O.damp_to_f32(st2))
    assert np.allclose(y1, y2, rtol=1e-6, atol=1e-6 * np.abs(y1).max())


@pytest.mark.parametrize("K", [0, 128])
def test_round_trip_bounds(oref, K):
    """Rotate, store, reconstruct, rotate back: FP16 within a relative 2^-11
    of the rotated entries; INT8 within Delta/2 per rotated entry."""
    H, P, N, G = 3, 64, 128, 1
    cfg, S0, _ = damp_case(13, H, P, N, G, K, scale=3.0)
    st = O.damp_from_f32(cfg, S0)
    back = O.damp_to_f32(st)[0]
    for h in range(H):
        for m in range(N):
            n = cfg.chan[h, m]
            t = scipy.linalg.hadamard(P) @ S0[h, :, n].astype(np.float64)
            bound = (np.abs(t).sum() / P * 2.0 ** -11 if m < K
                     else float(st.delta[0, h, m - K]) / 2.0)
            err = np.abs(back[h, :, n].astype(np.float64) - S0[h, :, n]).max()
            assert err <= bound * 1.0001 + 1e-6 * np.abs(S0[h, :, n]).max()
    if K == 0:
        # every group spans its grid: 255 steps between min and max
        t = np.stack([scipy.linalg.hadamard(P) @ S0[0, :, cfg.chan[0, m]].astype(np.float64)
                      for m in range(N)])
        span = t.max(1) - t.min(1)
        assert np.allclose(st.delta[0, 0], span / 255.0, rtol=1e-5)
