"""Multi-step drift of the GPU path, reported.

Two free-running trajectories ("ssm-state-quantization" README, Findings 8:
the relative state error of a rounded recurrence grows like
1/sqrt(1 - lambda^2) and stays bounded at 8 bits; "Mamba state quantization
for inference", "Quantization error returns on the next token": the error
of step t is carried into every later step by the decay):

  - the tiny workload: 64 decode steps (1 layer, batch 1, 2 heads x 8 x 16,
    int8 asymmetric, zero initial state);
  - the 370M-shaped scan: batch 8, T 2048, 32 heads in three decay bands,
    int4 asymmetric, every head rounded and the mid band only.  The scan
    runs in chunks of 64 tokens (bit for bit the same as one scan of 2048:
    the state between tokens is the stored one), the pool read back after
    each chunk.

Curves against t: the fraction of codes that differ from the oracle's (the
oracle advancing its own state), the largest |dequantized difference| over
the row's range, the y error relative to the readout scale, and the error
of the stored state against the unrounded fp64 trajectory, per decay band.
The GPU-oracle comparison follows requests 0 and 1 and two heads of each
band (heads are independent with one group); the fp64 comparison covers
every head of requests 0 to 3.

The curves are written as JSON to the path in SSQ_DRIFT_REPORT (when set)
and printed.  Asserted: the codes never differ from the oracle's and y stays
within the readout tolerance; the drift itself is reported, with one loose
check of the law above (the state error times sqrt(1 - lambda_bar^2) within
a factor of 2 across the rounded bands).
"""
import json
import os

import numpy as np
import pytest
import torch

import oracle as O
from gpu_harness import Y_TOL, make_cfg, require_gpu, y_scale
from quantized_recurrent_state_mamba_b200 import workloads as W

pytestmark = pytest.mark.gpu

CHUNK = 64
FP64_REQUESTS = 4
ORACLE_REQUESTS = 2
_REPORT = {}


def cuda(a, dtype=torch.float32):
    return torch.from_numpy(np.ascontiguousarray(a)).to(device="cuda", dtype=dtype)


def _write_report():
    path = os.environ.get("SSQ_DRIFT_REPORT")
    if path:
        with open(path, "w") as f:
            json.dump(_REPORT, f, indent=1)


def _rel(a, b):
    d = np.linalg.norm((a - b).ravel())
    n = np.linalg.norm(b.ravel())
    return float(d / n) if n > 0 else float(d)


def _code_stats(ocfg, got, ref):
    """Fraction of differing codes and max |deq diff| / row range over the
    quantized rows of the states (GPU `got`, oracle `ref`)."""
    H, P = ocfg.nheads, ocfg.headdim
    n = diff = 0
    worst = 0.0
    Sg, Sr = O.state_to_f32(got), O.state_to_f32(ref)
    qa = 255.0 if ocfg.fmt == O.I8_ASYM else 15.0
    for i in range(ref.count):
        for h in range(H):
            if not ocfg.row_is_quant(h):
                continue
            rows = slice(h * P, (h + 1) * P)
            n += ref.q[i, rows].size
            diff += int((got.q[i, rows] != ref.q[i, rows]).sum())
            rng = qa * ref.delta[i, rows].astype(np.float64)[:, None]
            dd = np.abs(Sg[i, h].astype(np.float64) - Sr[i, h].astype(np.float64))
            worst = max(worst, float(np.max(dd / np.maximum(rng, 1e-30))))
    return diff / max(n, 1), worst


def test_drift_tiny_decode():
    """The tiny workload, 64 free-running decode steps."""
    from gpu_harness import download
    ssq = require_gpu()
    wl = W.tiny()
    inp = wl.inputs()
    H, P, N, T = wl.nheads, wl.headdim, wl.d_state, wl.T
    cfg, L, codec, ocfg = make_cfg(ssq, "i8a", 1, 1, H, P, N, 1)
    st = O.State(ocfg, 1)
    pool = ssq.alloc_pool(cfg)
    S64 = np.zeros((H, P, N))
    curve = []
    for t in range(T):
        x, B, C, dt = (inp[k][0, t] for k in ("x", "B", "C", "dt"))
        y = torch.empty((1, 1, H, P), device="cuda")
        ssq.ssq_decode_step(cfg, pool, None, 1, 0, 1, cuda(x[None, None]), cuda(B[None, None]),
                            cuda(C[None, None]), cuda(dt[None, None]), cuda(inp["A"][None]),
                            cuda(inp["D"][None]), y)
        y_ref = O.step(ocfg, st, 0, x, B, C, dt, inp["A"], inp["D"])
        got = download(codec, pool, [(0, 0)], ocfg)
        frac, dq = _code_stats(ocfg, got, st)
        scale = y_scale(ocfg, st, C[None], inp["D"][None], x[None])[0]
        yerr = float(np.max(np.abs(y.cpu().numpy()[0, 0].astype(np.float64) - y_ref)
                            / np.maximum(scale, 1e-30)))
        S64, _ = O.scan_f64(ocfg, S64, x[None], B[None], C[None], dt[None], inp["A"], inp["D"])
        curve.append({"t": t + 1, "code_diff_frac": frac, "deq_diff_over_range": dq,
                      "y_rel_err": yerr,
                      "state_rel_err_vs_fp64": _rel(O.state_to_f32(got)[0], S64)})
        assert frac == 0.0, f"step {t}: codes differ from the oracle's"
        assert yerr <= Y_TOL, f"step {t}: y error {yerr:.3e}"
    _REPORT["tiny_decode_T64_i8a"] = curve
    _write_report()
    print("tiny drift (t, state error vs fp64):",
          " ".join(f"{c['t']}:{c['state_rel_err_vs_fp64']:.2e}" for c in curve[7::8]))


@pytest.mark.parametrize("mask", ["all", "mid"])
def test_drift_scan_370m(mask):
    """The 370M scan over T 2048 in 64-token chunks; curves per decay band."""
    ssq = require_gpu()
    wl = W.scan_370m(mask)
    H, P, N, T, Bt = wl.nheads, wl.headdim, wl.d_state, wl.T, wl.batch
    inp = wl.inputs()
    band = wl.bands()
    A = inp["A"]
    lam_bar = np.exp(A.astype(np.float64) * W.MEDIAN_DT)
    cfg, L, codec, ocfg_full = make_cfg(ssq, "i4a", 1, Bt, H, P, N, 1, wl.head_mask)
    pool = ssq.alloc_pool(cfg)
    # the oracle follows two heads of each band
    heads = [int(h) for b in range(3) for h in np.nonzero(band == b)[0][:2]]
    sub_mask = None if wl.head_mask is None else wl.head_mask[heads]
    ocfg = O.Cfg(O.I4_ASYM, len(heads), P, N, 1, sub_mask)
    st = O.State(ocfg, ORACLE_REQUESTS)
    ocfg64 = O.Cfg(O.F32, H, P, N, 1)
    S64 = [np.zeros((H, P, N)) for _ in range(FP64_REQUESTS)]
    S_out = torch.empty((1, Bt, H, P, N), device="cuda")
    curve = []
    for c0 in range(0, T, CHUNK):
        sl = slice(c0, c0 + CHUNK)
        y = torch.empty((Bt, CHUNK, H, P), device="cuda")
        ssq.ssq_scan(cfg, pool, None, Bt, 0, CHUNK, cuda(inp["x"][:, sl]), cuda(inp["B"][:, sl]),
                     cuda(inp["C"][:, sl]), cuda(inp["dt"][:, sl]), cuda(A), cuda(inp["D"]), y)
        ssq.ssq_dequantize_rows(cfg, pool, None, Bt, 0, 1, S_out)
        Sg = S_out.cpu().numpy()[0]                      # [Bt][H][P][N]
        yh = y.cpu().numpy()
        # GPU against the oracle on the followed requests and heads
        yerr = 0.0
        for b in range(ORACLE_REQUESTS):
            for t in range(c0, c0 + CHUNK):
                y_ref = O.step(ocfg, st, b, inp["x"][b, t, heads], inp["B"][b, t],
                               inp["C"][b, t], inp["dt"][b, t, heads], A[heads],
                               inp["D"][heads])
                scale = y_scale(ocfg, _one(st, b, ocfg), inp["C"][b, t][None],
                                inp["D"][heads][None], inp["x"][b, t, heads][None])[0]
                e = np.abs(yh[b, t - c0][heads].astype(np.float64) - y_ref) / np.maximum(scale, 1e-30)
                yerr = max(yerr, float(e.max()))
        got = O.State(ocfg, ORACLE_REQUESTS)
        for b in range(ORACLE_REQUESTS):
            _read_heads(got, b, ocfg, codec, pool, b, heads)
        frac, dq = _code_stats(ocfg, got, st)
        # the stored state against the unrounded fp64 trajectory
        per_band = []
        for b in range(FP64_REQUESTS):
            S64[b], _ = O.scan_f64(ocfg64, S64[b], inp["x"][b, sl], inp["B"][b, sl],
                                   inp["C"][b, sl], inp["dt"][b, sl], A, inp["D"])
        for k in range(3):
            hb = np.nonzero(band == k)[0]
            per_band.append(_rel(np.stack([Sg[b][hb] for b in range(FP64_REQUESTS)]).astype(np.float64),
                                 np.stack([S64[b][hb] for b in range(FP64_REQUESTS)])))
        curve.append({"t": c0 + CHUNK, "code_diff_frac": frac, "deq_diff_over_range": dq,
                      "y_rel_err": yerr, "state_rel_err_vs_fp64_by_band": per_band})
        assert frac == 0.0, f"t {c0 + CHUNK}: codes differ from the oracle's"
        assert yerr <= Y_TOL, f"t {c0 + CHUNK}: y error {yerr:.3e}"
    lam_band = [float(np.mean(lam_bar[band == k])) for k in range(3)]
    last = curve[-1]["state_rel_err_vs_fp64_by_band"]
    _REPORT[f"scan_370m_T2048_i4a_{mask}"] = {
        "curve": curve, "lambda_bar_by_band": lam_band,
        "quantized_bands": [int(k) for k in range(3)
                            if wl.head_mask is None or np.all(wl.head_mask[band == k] != 0)],
        "final_err_times_sqrt_1_minus_lambda2": [
            e * float(np.sqrt(1.0 - l * l)) for e, l in zip(last, lam_band)]}
    _write_report()
    print(f"scan 370m {mask}: final state error vs fp64 by band {last}, lambda_bar {lam_band}")
    assert ssq.ssq_pool_error(cfg, pool) == 0
    # the reported law: across the rounded bands, the state error times
    # sqrt(1 - lambda_bar^2) stays within a factor of 2 (it grows like
    # 1/sqrt(1 - lambda^2); at 4 bits the slowest band's error exceeds the
    # state itself, the page's "fails at 4 bits")
    scaled = [e * np.sqrt(1.0 - l * l) for k, (e, l) in enumerate(zip(last, lam_band))
              if k in _REPORT[f"scan_370m_T2048_i4a_{mask}"]["quantized_bands"]]
    assert max(scaled) < 2.0 * min(scaled)


def _one(st, b, ocfg):
    """State pair b of `st` as a one-pair State (for y_scale)."""
    s = O.State(ocfg, 1)
    s.q[0], s.delta[0], s.zero[0], s.val[0] = st.q[b], st.delta[b], st.zero[b], st.val[b]
    return s


def _read_heads(got, i, ocfg, codec, pool, slot, heads):
    """The GPU's stored codes, steps and zero points of the followed heads of
    one request, read from the pool bytes."""
    buf_off, n = codec.slot_range(slot)
    buf = pool[buf_off:buf_off + n].cpu().numpy()
    codec.buf_offset = buf_off
    try:
        q, d, z, v = codec.read(buf, slot, 0)
    finally:
        codec.buf_offset = 0
    P = ocfg.headdim
    for k, h in enumerate(heads):
        rows = slice(h * P, (h + 1) * P)
        sub = slice(k * P, (k + 1) * P)
        got.q[i, sub], got.delta[i, sub], got.zero[i, sub], got.val[i, sub] = \
            q[rows], d[rows], z[rows], v[rows]
