"""Shared machinery of the GPU parity tests: set up a pool from oracle
states, run a library call, read the pool back, and compare with the oracle
under the acceptance rule.

Acceptance rule for one step from identical stored state and inputs:
  - quantized rows: zero point equal bitwise, step within 2 ulp; codes
    bit-exact except entries whose oracle pre-rounding value s'*inv lies
    within 1e-3 of a .5 boundary, which may differ by 1 and must be at most
    1e-4 of the entries;
  - fp rows (fp32 / bf16 state, masked heads): bit-exact;
  - y within 1e-4 normwise: |y - y_ref| <= 1e-4 (sum_n |C_n deq_n| + |D x|).
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle as O
from poolcodec import Codec

CODE_TOL_FRAC = 1e-4
Y_TOL = 1e-4


def require_gpu():
    if not torch.cuda.is_available():
        pytest.fail("GPU test run without a CUDA device")
    from quantized_recurrent_state_mamba_b200 import ssq
    return ssq


def make_cfg(ssq, fmt, n_layers, n_slots, H, P, N, G, mask=None):
    cfg = ssq.Config(n_layers=n_layers, n_slots=n_slots, nheads=H, headdim=P, d_state=N,
                     ngroups=G, fmt=fmt, head_mask=mask)
    L, perm = ssq.ssq_pool_layout(cfg)
    codec = Codec(cfg.fmt, H, P, N, L, perm)
    ocfg = O.Cfg(cfg.fmt, H, P, N, G, None if mask is None else np.asarray(mask, np.uint8))
    return cfg, L, codec, ocfg


def upload(ssq, cfg, L, codec, st, pairs):
    """Pool on the GPU holding oracle state pair i at (slot, layer) =
    pairs[i]; the rest of the pool is zero."""
    buf = np.zeros(L["pool_bytes"], np.uint8)
    for i, (slot, layer) in enumerate(pairs):
        codec.write(buf, slot, layer, st.q[i], st.delta[i], st.zero[i], st.val[i])
    return torch.from_numpy(buf).cuda()


def download(codec, pool, pairs, ocfg):
    buf = pool.cpu().numpy()
    st = O.State(ocfg, len(pairs))
    for i, (slot, layer) in enumerate(pairs):
        q, d, z, v = codec.read(buf, slot, layer)
        st.q[i], st.delta[i], st.zero[i], st.val[i] = q, d, z, v
    return st


def ulp_diff(a, b):
    a = np.asarray(a, np.float32).view(np.int32).astype(np.int64)
    b = np.asarray(b, np.float32).view(np.int32).astype(np.int64)
    return np.abs(a - b)


def compare_states(ocfg, got, ref, pre=None, where=""):
    """Check the acceptance rule on every row; return mismatch statistics."""
    H, P, N = ocfg.nheads, ocfg.headdim, ocfg.d_state
    stats = dict(entries=0, code_mismatch=0, boundary=0, rows=0)
    for i in range(ref.count):
        for h in range(H):
            rows = slice(h * P, (h + 1) * P)
            if ocfg.row_is_quant(h):
                stats["rows"] += P
                assert np.array_equal(got.zero[i, rows].view(np.uint32),
                                      ref.zero[i, rows].view(np.uint32)), \
                    f"{where} zero point differs (pair {i}, head {h})"
                ud = ulp_diff(got.delta[i, rows], ref.delta[i, rows])
                assert np.all(ud <= 2), f"{where} step differs by > 2 ulp (pair {i}, head {h})"
                stats["delta_ulp_max"] = max(stats.get("delta_ulp_max", 0), int(ud.max()))
                gq, rq = got.q[i, rows], ref.q[i, rows]
                diff = gq != rq
                stats["entries"] += gq.size
                if diff.any():
                    stats["code_mismatch"] += int(diff.sum())
                    assert np.all(np.abs(gq[diff] - rq[diff]) <= 1), where
                    assert pre is not None, f"{where} codes differ and no boundary info"
                    pr = pre[i, rows][diff].astype(np.float64)
                    frac = np.abs(np.abs(pr - np.floor(pr)) - 0.5)
                    assert np.all(frac < 1e-3), f"{where} code differs off a boundary"
                    stats["boundary"] += int(diff.sum())
            else:
                g, r = got.val[i, rows], ref.val[i, rows]
                assert np.array_equal(g.view(np.uint32), r.view(np.uint32)), \
                    f"{where} fp row differs (pair {i}, head {h})"
    if stats["entries"]:
        assert stats["code_mismatch"] <= CODE_TOL_FRAC * stats["entries"], stats
    return stats


def y_scale(ocfg, st_after, C, D, x):
    """sum_n |C_n deq_n| + |D x| per (pair, h, p), from the oracle state."""
    S = O.state_to_f32(st_after).astype(np.float64)      # [count][H][P][N]
    H = ocfg.nheads
    g_of = np.arange(H) // (H // ocfg.ngroups)
    Ch = np.abs(np.asarray(C, np.float64))[:, g_of, :]     # [count][H][N]
    return np.einsum("chpn,chn->chp", np.abs(S), Ch) + np.abs(
        np.asarray(D, np.float64)[:, :, None] * np.asarray(x, np.float64))


def check_y(y_gpu, y_ref, scale, where=""):
    err = np.abs(np.asarray(y_gpu, np.float64) - np.asarray(y_ref, np.float64))
    worst = float(np.max(err / np.maximum(scale, 1e-30)))
    assert np.all(err <= Y_TOL * scale + 1e-30), f"{where} y error {worst:.3e}"
    return worst
