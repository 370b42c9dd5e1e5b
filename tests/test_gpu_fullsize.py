"""GPU parity at the workloads' full sizes, in the launch configuration the
benchmark times, on sampled outputs the oracle computes one (layer, request)
pair at a time.

  - Mamba-2 130M-shaped decode: 24 layers x batch 256 in one launch, heads
    24 x 64 x 128, int8 asym, initial state N(0, 1) written by
    ssq_quantize_rows (whose codes are checked bit-exact first);
  - Mamba-2 8B-shaped decode: 128 heads x 64 x 128 in 8 groups, batch 64 and
    256, int8 sym / int8 asym / fp32;
  - serving-scale format sweep: 30 layers x batch 256, 32 heads x 128 x 128,
    fp32 / bf16 / int8 asym / int4 asym, zero initial state, two steps;
  - Mamba-2 370M-shaped scan: batch 8 x T 2048, 32 heads in three decay
    bands, int4 asym, all heads vs the mid band only;
  - the DAMP mixed-tier step on the 130M decode shape (16 of 128 key
    channels in FP16), hand-off and one decode launch of 24 layers x 256;
  - the stochastic-rounding step on the 130M shape, and the prefill
    hand-off on the 370M shape (batch 8 x T 2048).
"""
import numpy as np
import pytest
import torch

import oracle as O
from gpu_harness import check_y, compare_states, make_cfg, require_gpu, y_scale
from quantized_recurrent_state_mamba_b200 import workloads as W

pytestmark = pytest.mark.gpu


def cuda(a, dtype=torch.float32):
    return torch.from_numpy(np.ascontiguousarray(a)).to(device="cuda", dtype=dtype)


def read_pairs(codec, pool, pairs, ocfg):
    """Read sampled (slot, layer) states, copying only their slots."""
    st = O.State(ocfg, len(pairs))
    for i, (slot, layer) in enumerate(pairs):
        off, n = codec.slot_range(slot)
        buf = pool[off:off + n].cpu().numpy()
        codec.buf_offset = off
        try:
            st.q[i], st.delta[i], st.zero[i], st.val[i] = codec.read(buf, slot, layer)
        finally:
            codec.buf_offset = 0
    return st


def init_pool_from_workload(ssq, cfg, wl, pool):
    """Quantize the workload's initial state into the pool, one layer per call
    (the fp32 state is drawn on the host pair by pair)."""
    rows, N = wl.rows, wl.d_state
    for l in range(wl.nl):
        S = np.empty((wl.batch, rows, N), np.float32)
        for b in range(wl.batch):
            S[b] = wl.state_pair(l, b)
        ssq.ssq_quantize_rows(cfg, pool, None, wl.batch, l, 1, cuda(S))
    torch.cuda.synchronize()


SR_SEED = 12345


def sampled_decode_check(ssq, wl, fmt, samples, steps=1, init_from_pool=True, sr=False):
    H, P, N, G = wl.nheads, wl.headdim, wl.d_state, wl.ngroups
    cfg, L, codec, ocfg = make_cfg(ssq, fmt, wl.nl, wl.batch, H, P, N, G)
    pool = ssq.alloc_pool(cfg)
    pairs = [(b, l) for (l, b) in samples]
    if wl.init == "zero":
        st = O.State(ocfg, len(samples))
    else:
        init_pool_from_workload(ssq, cfg, wl, pool)
        S0 = np.stack([wl.state_pair(l, b).reshape(H, P, N) for (l, b) in samples])
        st = O.state_from_f32(ocfg, S0)
        got0 = read_pairs(codec, pool, pairs, ocfg)
        s0 = compare_states(ocfg, got0, st, None, "initial quantize")
        assert s0["code_mismatch"] == 0
    report = []
    for k in range(steps):
        inp = (wl.inputs() if k == 0 else
               W.Decode(wl.name, wl.seed + 100 * k, wl.nl, wl.batch, H, P, N, G, fmt).inputs())
        y = torch.empty((wl.nl, wl.batch, H, P), device="cuda")
        args = (cfg, pool, None, wl.batch, 0, wl.nl, cuda(inp["x"]), cuda(inp["B"]),
                cuda(inp["C"]), cuda(inp["dt"]), cuda(inp["A"]), cuda(inp["D"]), y)
        if sr:
            ssq.ssq_decode_step_sr(*args, SR_SEED, k + 1)
        else:
            ssq.ssq_decode_step(*args)
        yh = y.cpu().numpy()
        pre = np.zeros((len(samples), H * P, N), np.float32)
        y_ref = np.zeros((len(samples), H, P), np.float32)
        for i, (l, b) in enumerate(samples):
            a = (inp["x"][l, b], inp["B"][l, b], inp["C"][l, b], inp["dt"][l, b], inp["A"][l],
                 inp["D"][l])
            if sr:
                # slot = request b (identity slots), layer l
                y_ref[i] = O.step_sr(ocfg, st, i, *a, SR_SEED, k + 1, l, b)
            else:
                y_ref[i], pre[i] = O.step(ocfg, st, i, *a, want_pre=True)
        got = read_pairs(codec, pool, pairs, ocfg)
        stats = compare_states(ocfg, got, st, None if sr else pre, f"{wl.name} step {k}")
        if sr:
            assert stats["code_mismatch"] == 0
        C = np.stack([inp["C"][l, b] for (l, b) in samples])
        D = np.stack([inp["D"][l] for (l, b) in samples])
        x = np.stack([inp["x"][l, b] for (l, b) in samples])
        ys = np.stack([yh[l, b] for (l, b) in samples])
        stats["y_err"] = check_y(ys, y_ref, y_scale(ocfg, st, C, D, x), wl.name)
        report.append(stats)
        assert np.all(np.isfinite(yh))
    assert ssq.ssq_pool_error(cfg, pool) == 0
    print(wl.name, report)
    del pool
    torch.cuda.empty_cache()
    return report


def test_decode_130m_full():
    ssq = require_gpu()
    wl = W.decode_130m("i8a")
    samples = [(0, 0), (0, 255), (11, 97), (23, 255), (23, 1), (17, 128)]
    sampled_decode_check(ssq, wl, "i8a", samples)


def test_decode_130m_sr_full():
    """The stochastic-rounding step as the benchmark runs it
    (decode_130m_sr): 24 layers x 256 in one launch, two steps with step
    counters 1 and 2; sampled pairs bit-exact in codes."""
    ssq = require_gpu()
    wl = W.decode_130m("i8a")
    samples = [(0, 0), (23, 255), (11, 97), (5, 200)]
    sampled_decode_check(ssq, wl, "i8a", samples, steps=2, sr=True)


@pytest.mark.parametrize("fmt", ["i8s", "i8a", "f32"])
@pytest.mark.parametrize("batch", [64, 256])
def test_decode_8b_full(fmt, batch):
    ssq = require_gpu()
    wl = W.decode_8b(fmt, batch)
    samples = [(0, 0), (0, batch // 2 + 1), (0, batch - 1)]
    sampled_decode_check(ssq, wl, fmt, samples)


@pytest.mark.parametrize("fmt", ["f32", "bf16", "i8a", "i4a"])
def test_decode_serving_sweep_full(fmt):
    ssq = require_gpu()
    wl = W.sweep_serving(fmt)
    wl.init = "zero"
    samples = [(0, 0), (29, 255), (14, 77)]
    sampled_decode_check(ssq, wl, fmt, samples, steps=2)


@pytest.mark.parametrize("mask", ["all", "mid"])
def test_scan_370m_full(mask):
    """Full launch (batch 8, T 2048); the oracle follows one request and one
    head from each decay band (heads are independent with one group)."""
    ssq = require_gpu()
    wl = W.scan_370m(mask)
    H, P, N, T, Bt = wl.nheads, wl.headdim, wl.d_state, wl.T, wl.batch
    inp = wl.inputs()
    cfg, L, codec, ocfg_full = make_cfg(ssq, "i4a", 1, Bt, H, P, N, 1, wl.head_mask)
    pool = ssq.alloc_pool(cfg)
    y = torch.empty((Bt, T, H, P), device="cuda")
    ssq.ssq_scan(cfg, pool, None, Bt, 0, T, cuda(inp["x"]), cuda(inp["B"]), cuda(inp["C"]),
                 cuda(inp["dt"]), cuda(inp["A"]), cuda(inp["D"]), y)
    yh = y.cpu().numpy()
    b = 5
    heads = [3, 15, 27]
    sub_mask = None if wl.head_mask is None else wl.head_mask[heads]
    ocfg = O.Cfg(O.I4_ASYM, len(heads), P, N, 1, sub_mask)
    st = O.State(ocfg, 1)
    scale = np.zeros((T, len(heads), P))
    y_ref = np.zeros((T, len(heads), P), np.float32)
    for t in range(T):
        y_ref[t] = O.step(ocfg, st, 0, inp["x"][b, t, heads], inp["B"][b, t], inp["C"][b, t],
                          inp["dt"][b, t, heads], inp["A"][heads], inp["D"][heads])
        scale[t] = y_scale(ocfg, st, inp["C"][b, t][None], inp["D"][heads][None],
                           inp["x"][b, t, heads][None])[0]
    check_y(yh[b][:, heads], y_ref, scale, f"scan 370m {mask}")
    gotb = read_pairs(codec, pool, [(b, 0)], ocfg_full)
    q, d, z, v = gotb.q[0], gotb.delta[0], gotb.zero[0], gotb.val[0]
    got = O.State(ocfg, 1)
    for i, h in enumerate(heads):
        rows = slice(h * P, (h + 1) * P)
        sub = slice(i * P, (i + 1) * P)
        got.q[0, sub], got.delta[0, sub], got.zero[0, sub], got.val[0, sub] = \
            q[rows], d[rows], z[rows], v[rows]
    stats = compare_states(ocfg, got, st, None, f"scan 370m {mask}")
    assert stats["code_mismatch"] == 0
    assert ssq.ssq_pool_error(cfg, pool) == 0


def test_fullsize_damp_130m():
    """The DAMP step as the benchmark runs it (decode_130m_damp): the pool
    written by ssq_damp_quantize from the N(0, 1) state, one launch of 24
    layers x 256 requests; sampled (layer, request) pairs compared with the
    oracle: FP16 bits, codes, steps and zero points equal after the hand-off
    and after the step, y within the readout tolerance."""
    from poolcodec import DampCodec
    ssq = require_gpu()
    wl = W.decode_130m_damp()
    H, P, N, G, K = wl.nheads, wl.headdim, wl.d_state, wl.ngroups, 16
    cfg = ssq.DampConfig(wl.nl, wl.batch, H, P, N, G, K)
    L = ssq.ssq_damp_pool_layout(cfg)
    codec = DampCodec(H, P, N, K, L)
    chan = W.damp_channels(wl.seed, wl.nl, H, N)
    chan_t = cuda(chan, torch.int32)
    pool = ssq.damp_alloc_pool(cfg)
    for l in range(wl.nl):
        S = np.stack([wl.state_pair(l, b).reshape(H, P, N) for b in range(wl.batch)])
        ssq.ssq_damp_quantize(cfg, pool, chan_t, None, wl.batch, l, 1, cuda(S))
    torch.cuda.synchronize()
    rng = np.random.default_rng(5)
    samples = [(0, 0), (wl.nl - 1, wl.batch - 1), (11, 128)] + \
        [(int(rng.integers(wl.nl)), int(rng.integers(wl.batch))) for _ in range(3)]

    def read(l, b):
        off, n = codec.layer_range(b, l)
        codec.buf_offset = off
        try:
            buf = pool[off:off + n].cpu().numpy()
            return codec.read(buf, b, l), codec.read_hi_bits(buf, b, l)
        finally:
            codec.buf_offset = 0

    def check(st, l, b, where):
        (hi, q, d, z), bits = read(l, b)
        assert np.array_equal(bits, st.hi[0].astype(np.float16).view(np.uint16)), where
        assert np.array_equal(q, st.q[0]), where
        assert np.array_equal(d.view(np.uint32), st.delta[0].view(np.uint32)), where
        assert np.array_equal(z.view(np.uint32), st.zero[0].view(np.uint32)), where

    sts = {}
    for (l, b) in samples:
        oc = O.DampCfg(H, P, N, G, K, chan[l])
        sts[(l, b)] = (oc, O.damp_from_f32(oc, wl.state_pair(l, b).reshape(H, P, N)))
        check(sts[(l, b)][1], l, b, f"hand-off pair ({l}, {b})")
    inp = wl.inputs()
    y = torch.full((wl.nl, wl.batch, H, P), float("nan"), device="cuda")
    ssq.ssq_damp_decode_step(cfg, pool, chan_t, None, wl.batch, 0, wl.nl, cuda(inp["x"]),
                             cuda(inp["B"]), cuda(inp["C"]), cuda(inp["dt"]), cuda(inp["A"]),
                             cuda(inp["D"]), y)
    torch.cuda.synchronize()
    assert ssq.ssq_damp_pool_error(cfg, pool) == 0
    yg = y.cpu().numpy()
    assert np.isfinite(yg).all()
    for (l, b) in samples:
        oc, st = sts[(l, b)]
        x, B, C, dt = (inp[n][l, b] for n in ("x", "B", "C", "dt"))
        y_ref = O.damp_step(oc, st, 0, x, B, C, dt, inp["A"][l], inp["D"][l])
        check(st, l, b, f"step pair ({l}, {b})")
        S1 = O.damp_to_f32(st)[0].astype(np.float64)          # stored state, rotated back
        sc = np.abs(S1) @ np.abs(C[0].astype(np.float64)) + np.abs(inp["D"][l][:, None] * x)
        assert np.all(np.abs(yg[l, b] - y_ref) <= 1e-4 * (sc + 1e-30)), f"y pair ({l}, {b})"


def test_prefill_370m_full():
    """The prefill hand-off as the benchmark runs it (prefill_370m_all):
    batch 8 x T 2048, 32 heads in three decay bands, int4 asym, from the zero
    state; the oracle follows one request and one head from each band
    through all 2048 tokens (heads are independent with one group): the
    final codes bit-exact, y within the readout tolerance."""
    ssq = require_gpu()
    wl = W.scan_370m("all")
    H, P, N, T, Bt = wl.nheads, wl.headdim, wl.d_state, wl.T, wl.batch
    inp = wl.inputs()
    cfg, L, codec, ocfg_full = make_cfg(ssq, "i4a", 1, Bt, H, P, N, 1)
    pool = ssq.alloc_pool(cfg)
    y = torch.empty((Bt, T, H, P), device="cuda")
    ssq.ssq_prefill(cfg, pool, None, Bt, 0, T, cuda(inp["x"]), cuda(inp["B"]), cuda(inp["C"]),
                    cuda(inp["dt"]), cuda(inp["A"]), cuda(inp["D"]), y)
    yh = y.cpu().numpy()
    assert np.all(np.isfinite(yh))
    b = 6
    heads = [2, 17, 30]
    ocfg = O.Cfg(O.I4_ASYM, len(heads), P, N, 1)
    st = O.State(ocfg, 1)
    y_ref = O.prefill(ocfg, st, 0, inp["x"][b][:, heads], inp["B"][b], inp["C"][b],
                      inp["dt"][b][:, heads], inp["A"][heads], inp["D"][heads])
    # readout scale from the exact (fp64) trajectory of the same heads
    S = np.zeros((len(heads), P, N))
    scale = np.zeros((T, len(heads), P))
    Cb = np.abs(inp["C"][b][:, 0].astype(np.float64))                 # [T][N]
    for t in range(T):
        S, _ = O.scan_f64(ocfg, S, inp["x"][b, t:t + 1][:, heads], inp["B"][b, t:t + 1],
                          inp["C"][b, t:t + 1], inp["dt"][b, t:t + 1][:, heads],
                          inp["A"][heads], inp["D"][heads])
        scale[t] = np.abs(S) @ Cb[t] + np.abs(inp["D"][heads][:, None] * inp["x"][b, t][heads])
    check_y(yh[b][:, heads], y_ref, scale, "prefill 370m")
    gotb = read_pairs(codec, pool, [(b, 0)], ocfg_full)
    got = O.State(ocfg, 1)
    for i, h in enumerate(heads):
        rows = slice(h * P, (h + 1) * P)
        sub = slice(i * P, (i + 1) * P)
        got.q[0, sub], got.delta[0, sub], got.zero[0, sub], got.val[0, sub] = \
            gotb.q[0, rows], gotb.delta[0, rows], gotb.zero[0, rows], gotb.val[0, rows]
    stats = compare_states(ocfg, got, st, None, "prefill 370m")
    assert stats["code_mismatch"] == 0
    assert ssq.ssq_pool_error(cfg, pool) == 0
