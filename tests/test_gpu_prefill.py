"""GPU parity of the prefill hand-off (ssq_prefill through the C ABI) against
the CPU oracle: T tokens of the fp32 recurrence from the stored state, y
read from the fp32 state, the final state quantized once ("Mamba state
quantization for inference", "Mamba state quantization needs phase-aware
benchmarks": the prefill stays in fp32 and only its last state is packed).

The stored codes and metadata must be bit-identical to the oracle's (the
fp32 recurrence is one IEEE operation per step in both); y within the
readout tolerance of gpu_harness.py.
"""
import numpy as np
import pytest
import torch

import oracle as O
from gpu_harness import check_y, compare_states, download, make_cfg, require_gpu, upload
from quantized_recurrent_state_mamba_b200 import workloads as W

pytestmark = pytest.mark.gpu

ALL_FMTS = ["f32", "bf16", "i8s", "i8a", "i4s", "i4a"]


def cuda(a, dtype=torch.float32):
    return torch.from_numpy(np.ascontiguousarray(a)).to(device="cuda", dtype=dtype)


def prefill_scale(ocfg, C, D, x, S_traj):
    """sum_n |C_n s_n| + |D x| per (b, t, h, p) from the fp64 trajectory."""
    H = ocfg.nheads
    g_of = np.arange(H) // (H // ocfg.ngroups)
    Ch = np.abs(C.astype(np.float64))[:, :, g_of, :]              # [b][t][h][n]
    return np.einsum("bthn,bthpn->bthp", Ch, np.abs(S_traj)) \
        + np.abs(D.astype(np.float64))[None, None, :, None] * np.abs(x.astype(np.float64))


def run_prefill(fmt, H, P, N, G, batch, T, mask=None, seed=0, banded=False, init="normal"):
    ssq = require_gpu()
    cfg, L, codec, ocfg = make_cfg(ssq, fmt, 2, batch + 1, H, P, N, G, mask)
    wl = W.Scan("prefill", seed, batch, T, H, P, N, G, fmt, banded=banded, init=init)
    inp = wl.inputs()
    if init == "zero":
        S0 = np.zeros((batch, H, P, N), np.float32)
    else:
        S0 = np.stack([W.state_pair(seed, 1, b, H * P, N).reshape(H, P, N)
                       for b in range(batch)])
    st = O.state_from_f32(ocfg, S0)
    S_start = O.state_to_f32(st)
    slots = list(range(batch, 0, -1))                   # reversed, slot 0 unused
    pairs = [(slots[b], 1) for b in range(batch)]
    pool = upload(ssq, cfg, L, codec, st, pairs)
    slot_t = cuda(np.array(slots, np.int32), torch.int32)
    y = torch.empty((batch, T, H, P), device="cuda")
    ssq.ssq_prefill(cfg, pool, slot_t, batch, 1, T, cuda(inp["x"]), cuda(inp["B"]),
                    cuda(inp["C"]), cuda(inp["dt"]), cuda(inp["A"]), cuda(inp["D"]), y)
    y_ref = np.stack([O.prefill(ocfg, st, b, inp["x"][b], inp["B"][b], inp["C"][b],
                                inp["dt"][b], inp["A"], inp["D"]) for b in range(batch)])
    got = download(codec, pool, pairs, ocfg)
    stats = compare_states(ocfg, got, st, None, f"prefill {fmt}")
    assert stats["code_mismatch"] == 0
    # readout scale from the exact trajectory (the prefill's y comes from it)
    traj = np.zeros((batch, T, H, P, N))
    for b in range(batch):
        S = S_start[b].astype(np.float64)
        for t in range(T):
            S, _ = O.scan_f64(ocfg, S, inp["x"][b, t:t + 1], inp["B"][b, t:t + 1],
                              inp["C"][b, t:t + 1], inp["dt"][b, t:t + 1], inp["A"], inp["D"])
            traj[b, t] = S
    scale = prefill_scale(ocfg, inp["C"], inp["D"], inp["x"], traj)
    check_y(y.cpu().numpy(), y_ref, scale, f"prefill {fmt}")
    assert ssq.ssq_pool_error(cfg, pool) == 0
    return stats


@pytest.mark.parametrize("fmt", ALL_FMTS)
def test_prefill_tiny_parity(fmt):
    """2 heads x 8 x 16, T = 64, from the zero state."""
    run_prefill(fmt, H=2, P=8, N=16, G=1, batch=1, T=64, seed=0, init="zero")


@pytest.mark.parametrize("fmt", ALL_FMTS)
def test_prefill_groups_ragged_from_state(fmt):
    """6 heads x 12 rows (partial tiles) x 64, 3 groups, 3 requests, T = 19
    (a ragged last chunk), from an N(0,1) stored state."""
    run_prefill(fmt, H=6, P=12, N=64, G=3, batch=3, T=19, seed=4)


@pytest.mark.parametrize("mask", ["all", "mid"])
def test_prefill_370m_shape_reduced(mask):
    """The 370M head shape (32 heads in three decay bands x 64 x 128, int4
    asym), mid-band-only mask vs all heads, 2 requests, T = 21."""
    m = None if mask == "all" else W.mid_band_mask(32)
    run_prefill("i4a", H=32, P=64, N=128, G=1, batch=2, T=21, mask=m, seed=2, banded=True,
                init="zero")


def test_prefill_then_decode_continues_from_the_handoff():
    """A prefill of T tokens followed by decode steps: the decode reads the
    state the prefill quantized (what a serving engine does after the
    prompt).  Compared with the oracle doing the same two phases."""
    ssq = require_gpu()
    H, P, N, G, batch, T = 4, 16, 128, 1, 2, 9
    cfg, L, codec, ocfg = make_cfg(ssq, "i8a", 1, batch, H, P, N, G)
    wl = W.Scan("handoff", 7, batch, T, H, P, N, G, "i8a")
    inp = wl.inputs()
    st = O.State(ocfg, batch)
    pool = ssq.alloc_pool(cfg)
    y = torch.empty((batch, T, H, P), device="cuda")
    ssq.ssq_prefill(cfg, pool, None, batch, 0, T, cuda(inp["x"]), cuda(inp["B"]),
                    cuda(inp["C"]), cuda(inp["dt"]), cuda(inp["A"]), cuda(inp["D"]), y)
    for b in range(batch):
        O.prefill(ocfg, st, b, inp["x"][b], inp["B"][b], inp["C"][b], inp["dt"][b],
                  inp["A"], inp["D"])
    dec = W.Decode("handoff", 8, 1, batch, H, P, N, G, "i8a").inputs()
    yd = torch.empty((1, batch, H, P), device="cuda")
    ssq.ssq_decode_step(cfg, pool, None, batch, 0, 1, cuda(dec["x"]), cuda(dec["B"]),
                        cuda(dec["C"]), cuda(dec["dt"]), cuda(inp["A"][None]),
                        cuda(inp["D"][None]), yd)
    pre = np.zeros((batch, H * P, N), np.float32)
    for b in range(batch):
        _, pre[b] = O.step(ocfg, st, b, dec["x"][0, b], dec["B"][0, b], dec["C"][0, b],
                           dec["dt"][0, b], inp["A"], inp["D"], want_pre=True)
    got = download(codec, pool, [(b, 0) for b in range(batch)], ocfg)
    stats = compare_states(ocfg, got, st, pre, "prefill then decode")
    assert stats["code_mismatch"] == 0
    assert ssq.ssq_pool_error(cfg, pool) == 0
