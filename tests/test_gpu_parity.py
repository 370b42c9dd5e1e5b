"""GPU parity: libssq's CUDA kernels, called through the C ABI, against the
CPU oracle, element by element, on seeded inputs at sizes the oracle runs in
seconds that still span several tiles and a ragged tail.

The oracle's state is packed into the pool on the host and uploaded; the
GPU's pool is read back and unpacked; nothing flows from the GPU into the
oracle.  The acceptance rule is in gpu_harness.py.
"""
import numpy as np
import pytest
import torch

import oracle as O
from gpu_harness import (check_y, compare_states, download, make_cfg, require_gpu, upload,
                         y_scale)
from quantized_recurrent_state_mamba_b200 import workloads as W

pytestmark = pytest.mark.gpu

ALL_FMTS = ["f32", "bf16", "i8s", "i8a", "i4s", "i4a"]
QFMTS = ["i8s", "i8a", "i4s", "i4a"]


def cuda(a, dtype=torch.float32):
    return torch.from_numpy(np.ascontiguousarray(a)).to(device="cuda", dtype=dtype)


def zoo_state(rng, count, H, P, N):
    """States whose rows include the quantizer's hard cases: normal rows,
    all-positive / all-negative rows, constant rows, rows far from zero with a
    tiny spread (zero point beyond 2^22), outliers, subnormal rows."""
    S = rng.standard_normal((count, H, P, N)).astype(np.float32)
    flat = S.reshape(-1, N)
    R = flat.shape[0]
    kinds = rng.integers(0, 9, R)
    for r in range(R):
        k = kinds[r]
        if k == 1:
            flat[r] = np.abs(flat[r]) + 3.0
        elif k == 2:
            flat[r] = -np.abs(flat[r]) - 0.25
        elif k == 3:
            flat[r] = np.float32(rng.standard_normal())
        elif k == 4:
            flat[r] = 1000.0 + flat[r] * 1e-4
        elif k == 5:
            flat[r] *= 1e-3
            flat[r, rng.integers(0, N)] = 50.0
        elif k == 6:
            flat[r] = flat[r] * 1e-41
        elif k == 7:
            flat[r] = 0.0
    return S


def crafted_rows(N):
    """Rows that hit exact rounding ties, the top-code clamp, and huge zero
    points (the row quantizer's slow paths)."""
    rows = []
    base = np.zeros(N, np.float32)
    # tie on the max rounding up past the top code (asym), any bit width:
    # lo*inv = -1.5, hi*inv = top - 1.5
    for top in (15.0, 255.0):
        r = base.copy()
        r[:] = np.linspace(-1.5, top - 1.5, N).astype(np.float32)
        r[0], r[-1] = -1.5, top - 1.5
        rows.append(r)
    # exact half-integers everywhere on a unit grid
    r = (np.arange(N) % 16 - 7.5).astype(np.float32)
    rows.append(r)
    # near-constant far from zero
    rows.append((4096.0 + np.arange(N) * 2.0 ** -10).astype(np.float32))
    rows.append(np.full(N, -2.5, np.float32))
    return np.stack(rows)


# ---------------------------------------------------------------------------
# quantize / dequantize
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("fmt", ALL_FMTS)
@pytest.mark.parametrize("N", [16, 32, 64, 128, 256])
def test_quantize_rows_bit_exact(fmt, N):
    ssq = require_gpu()
    H, P, G, nl, batch = 5, 7, 1, 2, 3
    slots = [4, 0, 2]
    mask = [1, 0, 1, 1, 0] if fmt in QFMTS and N == 128 else None
    cfg, L, codec, ocfg = make_cfg(ssq, fmt, 3, 5, H, P, N, G, mask)
    rng = np.random.default_rng(N + 10 * len(fmt))
    S = zoo_state(rng, nl * batch, H, P, N)
    cr = crafted_rows(N)
    S.reshape(-1, N)[: cr.shape[0]] = cr
    ref = O.state_from_f32(ocfg, S)
    pool = ssq.alloc_pool(cfg)
    slot_t = cuda(np.array(slots, np.int32), torch.int32)
    ssq.ssq_quantize_rows(cfg, pool, slot_t, batch, 1, nl, cuda(S))
    pairs = [(slots[b], 1 + l) for l in range(nl) for b in range(batch)]
    got = download(codec, pool, pairs, ocfg)
    stats = compare_states(ocfg, got, ref, None, f"quantize {fmt} N{N}")
    assert stats["code_mismatch"] == 0
    assert stats.get("delta_ulp_max", 0) == 0        # the step is bit-exact too
    # untouched layer 0 and slots stay zero
    buf = pool.cpu().numpy()
    q0, d0, z0, v0 = codec.read(buf, 1, 0)
    assert not q0.any() and not d0.any() and not v0.any()
    assert ssq.ssq_pool_error(cfg, pool) == 0

    # dequantize reads back exactly what the oracle reconstructs
    out = torch.empty(nl * batch * H * P * N, device="cuda")
    ssq.ssq_dequantize_rows(cfg, pool, slot_t, batch, 1, nl, out)
    ref_f = O.state_to_f32(ref).reshape(-1)
    assert np.array_equal(out.cpu().numpy().view(np.uint32), ref_f.view(np.uint32))


# ---------------------------------------------------------------------------
# decode step
# ---------------------------------------------------------------------------

def run_decode(fmt, H, P, N, G, batch, nl, layer0, n_layers, slots, mask=None, seed=0,
               init="normal", steps=1, resync=True):
    """Run `steps` decode steps on the GPU and in the oracle; with resync the
    oracle state is re-uploaded before each step (single-step parity)."""
    ssq = require_gpu()
    n_slots = max(slots) + 1 if slots is not None else batch
    cfg, L, codec, ocfg = make_cfg(ssq, fmt, n_layers, n_slots, H, P, N, G, mask)
    slot_list = slots if slots is not None else list(range(batch))
    pairs = [(slot_list[b], layer0 + l) for l in range(nl) for b in range(batch)]
    wl0 = W.Decode("case", seed, nl, batch, H, P, N, G, fmt, init=init)
    S0 = np.stack([wl0.state_pair(l, b).reshape(H, P, N)
                   for l in range(nl) for b in range(batch)])
    st = O.state_from_f32(ocfg, S0)
    pool = upload(ssq, cfg, L, codec, st, pairs)
    slot_t = None if slots is None else cuda(np.array(slots, np.int32), torch.int32)
    all_stats = []
    for k in range(steps):
        inp = W.Decode("case", seed * 1000 + k + 1, nl, batch, H, P, N, G, fmt).inputs()
        if resync and k > 0:
            pool = upload(ssq, cfg, L, codec, st, pairs)
        y = torch.full((nl, batch, H, P), float("nan"), device="cuda")
        ssq.ssq_decode_step(cfg, pool, slot_t, batch, layer0, nl, cuda(inp["x"]),
                            cuda(inp["B"]), cuda(inp["C"]), cuda(inp["dt"]), cuda(inp["A"]),
                            cuda(inp["D"]), y)
        y_ref = np.zeros((nl, batch, H, P), np.float32)
        pre = np.zeros((nl * batch, H * P, N), np.float32)
        for i in range(nl * batch):
            l, b = divmod(i, batch)
            y_ref[l, b], pre[i] = O.step(ocfg, st, i, inp["x"][l, b], inp["B"][l, b],
                                         inp["C"][l, b], inp["dt"][l, b], inp["A"][l],
                                         inp["D"][l], want_pre=True)
        got = download(codec, pool, pairs, ocfg)
        stats = compare_states(ocfg, got, st, pre, f"decode {fmt} step {k}")
        Dpair = np.repeat(inp["D"][:, None, :], batch, axis=1).reshape(nl * batch, H)
        scale = y_scale(ocfg, st, inp["C"].reshape(nl * batch, G, N), Dpair,
                        inp["x"].reshape(nl * batch, H, P))
        stats["y_err"] = check_y(y.cpu().numpy().reshape(nl * batch, H, P),
                                 y_ref.reshape(nl * batch, H, P), scale, f"decode {fmt}")
        all_stats.append(stats)
        assert ssq.ssq_pool_error(cfg, pool) == 0
    return all_stats


@pytest.mark.parametrize("fmt", ALL_FMTS)
@pytest.mark.parametrize("N", [16, 64, 128])
def test_decode_step_parity(fmt, N):
    """Several tiles per (layer, request) with a ragged tail (6 heads x 24 rows
    = 144 rows), 3 groups, 2 of 3 layers, permuted slots."""
    run_decode(fmt, H=6, P=24, N=N, G=3, batch=3, nl=2, layer0=1, n_layers=3,
               slots=[2, 0, 4], seed=N)


@pytest.mark.parametrize("fmt", QFMTS)
def test_decode_step_parity_masked(fmt):
    """Only some heads quantized (fp32 rows for the others), as when a single
    decay band is rounded."""
    run_decode(fmt, H=7, P=16, N=128, G=1, batch=2, nl=1, layer0=0, n_layers=1,
               slots=None, mask=[0, 1, 1, 0, 1, 0, 0], seed=5)


@pytest.mark.parametrize("fmt", QFMTS)
def test_decode_step_parity_zoo(fmt):
    """Stored states with constant, near-constant, all-positive/negative,
    subnormal and zero rows: the slow paths of the row engine."""
    ssq = require_gpu()
    H, P, N, G, batch = 4, 16, 128, 2, 2
    cfg, L, codec, ocfg = make_cfg(ssq, fmt, 1, batch, H, P, N, G)
    rng = np.random.default_rng(77)
    S0 = zoo_state(rng, batch, H, P, N)
    st = O.state_from_f32(ocfg, S0)
    pairs = [(b, 0) for b in range(batch)]
    pool = upload(ssq, cfg, L, codec, st, pairs)
    inp = W.Decode("zoo", 17, 1, batch, H, P, N, G, fmt).inputs()
    inp["dt"][0, 0, :] = 0.0          # lambda = 1, no input: a pure requantize
    inp["x"][0, 1, 1, :] = 0.0        # pure decay rows
    y = torch.empty((1, batch, H, P), device="cuda")
    ssq.ssq_decode_step(cfg, pool, None, batch, 0, 1, cuda(inp["x"]), cuda(inp["B"]),
                        cuda(inp["C"]), cuda(inp["dt"]), cuda(inp["A"]), cuda(inp["D"]), y)
    pre = np.zeros((batch, H * P, N), np.float32)
    y_ref = np.zeros((batch, H, P), np.float32)
    for b in range(batch):
        y_ref[b], pre[b] = O.step(ocfg, st, b, inp["x"][0, b], inp["B"][0, b], inp["C"][0, b],
                                  inp["dt"][0, b], inp["A"][0], inp["D"][0], want_pre=True)
    got = download(codec, pool, pairs, ocfg)
    compare_states(ocfg, got, st, pre, f"zoo {fmt}")
    scale = y_scale(ocfg, st, inp["C"][0], np.repeat(inp["D"], batch, 0), inp["x"][0])
    check_y(y.cpu().numpy()[0], y_ref, scale, f"zoo {fmt}")


@pytest.mark.parametrize("fmt", QFMTS)
@pytest.mark.parametrize("N", [64, 128])
def test_decode_crafted_updates(fmt, N):
    """Updated rows chosen exactly: from the zero state with dt = x = 1 the
    update is s' = B of the row's group, so each group's B is one of the
    crafted rows (the top code rounding past the grid, exact half-integer
    ties, a near-constant row far from zero, a constant row) or a normal
    row.  Heads of 8 rows put two groups in every warp, so warps mix rows
    that need the clamped rounding or the exact path with ordinary ones."""
    ssq = require_gpu()
    H, P, batch = 12, 8, 2
    cr = crafted_rows(N)
    G = 6
    cfg, L, codec, ocfg = make_cfg(ssq, fmt, 1, batch, H, P, N, G)
    rng = np.random.default_rng(31 + N)
    inp = W.Decode("crafted", 3, 1, batch, H, P, N, G, fmt).inputs()
    inp["dt"][:] = 1.0
    inp["x"][:] = 1.0
    for b in range(batch):
        for g in range(G):
            k = (g + b) % (cr.shape[0] + 1)
            inp["B"][0, b, g] = cr[k] if k < cr.shape[0] else \
                rng.standard_normal(N).astype(np.float32)
    st = O.State(ocfg, batch)
    pool = ssq.alloc_pool(cfg)
    y = torch.empty((1, batch, H, P), device="cuda")
    ssq.ssq_decode_step(cfg, pool, None, batch, 0, 1, cuda(inp["x"]), cuda(inp["B"]),
                        cuda(inp["C"]), cuda(inp["dt"]), cuda(inp["A"]), cuda(inp["D"]), y)
    pre = np.zeros((batch, H * P, N), np.float32)
    y_ref = np.zeros((batch, H, P), np.float32)
    for b in range(batch):
        y_ref[b], pre[b] = O.step(ocfg, st, b, inp["x"][0, b], inp["B"][0, b], inp["C"][0, b],
                                  inp["dt"][0, b], inp["A"][0], inp["D"][0], want_pre=True)
    got = download(codec, pool, [(b, 0) for b in range(batch)], ocfg)
    stats = compare_states(ocfg, got, st, pre, f"crafted {fmt} N{N}")
    assert stats["code_mismatch"] == 0
    scale = y_scale(ocfg, st, inp["C"][0], np.repeat(inp["D"], batch, 0), inp["x"][0])
    check_y(y.cpu().numpy()[0], y_ref, scale, f"crafted {fmt} N{N}")
    assert ssq.ssq_pool_error(cfg, pool) == 0


def test_decode_tiny_multistep_drift():
    """The tiny workload (1 layer, batch 1, 2 heads x 8 x 16, int8 asym, zero
    initial state) for 64 free-running steps: GPU and oracle advance their own
    states; the codes stay identical and y within the tolerance at every
    step.  Drift against the exact (unrounded, fp64) trajectory is reported."""
    ssq = require_gpu()
    wl = W.tiny()
    inp = wl.inputs()
    H, P, N, T = wl.nheads, wl.headdim, wl.d_state, wl.T
    cfg, L, codec, ocfg = make_cfg(ssq, "i8a", 1, 1, H, P, N, 1)
    st = O.State(ocfg, 1)
    pool = ssq.alloc_pool(cfg)
    S64 = np.zeros((H, P, N))
    drift = []
    for t in range(T):
        x, B, C, dt = (inp[k][0, t] for k in ("x", "B", "C", "dt"))
        y = torch.empty((1, 1, H, P), device="cuda")
        ssq.ssq_decode_step(cfg, pool, None, 1, 0, 1, cuda(x[None, None]), cuda(B[None, None]),
                            cuda(C[None, None]), cuda(dt[None, None]), cuda(inp["A"][None]),
                            cuda(inp["D"][None]), y)
        y_ref, pre = O.step(ocfg, st, 0, x, B, C, dt, inp["A"], inp["D"], want_pre=True)
        got = download(codec, pool, [(0, 0)], ocfg)
        stats = compare_states(ocfg, got, st, pre[None], f"tiny step {t}")
        assert stats["code_mismatch"] == 0
        scale = y_scale(ocfg, st, C[None], inp["D"][None], x[None])
        check_y(y.cpu().numpy()[0], y_ref[None], scale, f"tiny step {t}")
        S64, _ = O.scan_f64(ocfg, S64, x[None], B[None], C[None], dt[None], inp["A"], inp["D"])
        Sq = O.state_to_f32(got)[0]
        drift.append(float(np.linalg.norm(Sq - S64) / max(np.linalg.norm(S64), 1e-30)))
    print("tiny drift vs exact fp64 trajectory (relative state error by step):",
          " ".join(f"{d:.2e}" for d in drift[::8]))
    assert drift[-1] < 0.05


def test_decode_bad_slot_sets_error_and_skips():
    """A slot index outside the pool sets SSQ_DEVERR_SLOT; that request is
    skipped (state and y untouched) and the others are processed."""
    ssq = require_gpu()
    H, P, N = 2, 8, 64
    cfg, L, codec, ocfg = make_cfg(ssq, "i8a", 1, 2, H, P, N, 1)
    S0 = np.random.default_rng(1).standard_normal((2, H, P, N)).astype(np.float32)
    st = O.state_from_f32(ocfg, S0)
    pool = upload(ssq, cfg, L, codec, st, [(0, 0), (1, 0)])
    before = pool.clone()
    inp = W.Decode("bad", 3, 1, 2, H, P, N, 1, "i8a").inputs()
    slots = cuda(np.array([1, 7], np.int32), torch.int32)
    y = torch.full((1, 2, H, P), -123.0, device="cuda")
    ssq.ssq_decode_step(cfg, pool, slots, 2, 0, 1, cuda(inp["x"]), cuda(inp["B"]),
                        cuda(inp["C"]), cuda(inp["dt"]), cuda(inp["A"]), cuda(inp["D"]), y)
    assert ssq.ssq_pool_error(cfg, pool) & ssq.SSQ_DEVERR_SLOT
    assert ssq.ssq_pool_error(cfg, pool) == 0          # read clears it
    yh = y.cpu().numpy()
    assert np.all(yh[0, 1] == -123.0)
    # slot 0 untouched, slot 1 updated like request 0 in the oracle
    buf, buf0 = pool.cpu().numpy(), before.cpu().numpy()
    s0 = L["header_bytes"]
    assert np.array_equal(buf[s0:s0 + L["slot_bytes"]], buf0[s0:s0 + L["slot_bytes"]])
    ref = st.copy()
    y_ref, pre = O.step(ocfg, ref, 1, inp["x"][0, 0], inp["B"][0, 0], inp["C"][0, 0],
                        inp["dt"][0, 0], inp["A"][0], inp["D"][0], want_pre=True)
    got = download(codec, pool, [(1, 0)], ocfg)
    one = O.State(ocfg, 1)
    one.q[0], one.delta[0], one.zero[0], one.val[0] = ref.q[1], ref.delta[1], ref.zero[1], ref.val[1]
    compare_states(ocfg, got, one, pre[None], "bad-slot survivor")


def test_decode_nonfinite_sets_error():
    ssq = require_gpu()
    H, P, N = 2, 8, 32
    cfg, L, codec, ocfg = make_cfg(ssq, "i4a", 1, 1, H, P, N, 1)
    pool = ssq.alloc_pool(cfg)
    inp = W.Decode("nan", 4, 1, 1, H, P, N, 1, "i4a").inputs()
    inp["x"][0, 0, 1, 3] = np.inf
    y = torch.empty((1, 1, H, P), device="cuda")
    ssq.ssq_decode_step(cfg, pool, None, 1, 0, 1, cuda(inp["x"]), cuda(inp["B"]),
                        cuda(inp["C"]), cuda(inp["dt"]), cuda(inp["A"]), cuda(inp["D"]), y)
    assert ssq.ssq_pool_error(cfg, pool) & ssq.SSQ_DEVERR_NONFINITE


def test_empty_batch_and_zero_tokens_are_noops():
    ssq = require_gpu()
    cfg, L, codec, ocfg = make_cfg(ssq, "i8a", 1, 2, 2, 8, 32, 1)
    pool = ssq.alloc_pool(cfg)
    before = pool.clone()
    z = torch.zeros(1024, device="cuda")
    ssq.ssq_decode_step(cfg, pool, None, 0, 0, 1, z, z, z, z, z, z, z)
    ssq.ssq_scan(cfg, pool, None, 2, 0, 0, z, z, z, z, z, z, z)
    torch.cuda.synchronize()
    assert torch.equal(pool, before)


# ---------------------------------------------------------------------------
# scan
# ---------------------------------------------------------------------------

def run_scan(fmt, H, P, N, G, batch, T, mask=None, seed=0, banded=False, init="normal"):
    ssq = require_gpu()
    cfg, L, codec, ocfg = make_cfg(ssq, fmt, 2, batch + 1, H, P, N, G, mask)
    wl = W.Scan("scan", seed, batch, T, H, P, N, G, fmt, banded=banded, init=init)
    inp = wl.inputs()
    if init == "zero":
        S0 = np.zeros((batch, H, P, N), np.float32)
    else:
        S0 = np.stack([W.state_pair(seed, 1, b, H * P, N).reshape(H, P, N)
                       for b in range(batch)])
    st = O.state_from_f32(ocfg, S0)
    slots = list(range(batch, 0, -1))                   # reversed, slot 0 unused
    pairs = [(slots[b], 1) for b in range(batch)]
    pool = upload(ssq, cfg, L, codec, st, pairs)
    slot_t = cuda(np.array(slots, np.int32), torch.int32)
    y = torch.empty((batch, T, H, P), device="cuda")
    ssq.ssq_scan(cfg, pool, slot_t, batch, 1, T, cuda(inp["x"]), cuda(inp["B"]),
                 cuda(inp["C"]), cuda(inp["dt"]), cuda(inp["A"]), cuda(inp["D"]), y)
    # the oracle scan, token by token, keeping the per-token readout scale
    y_ref = np.zeros((batch, T, H, P), np.float32)
    scale = np.zeros((batch, T, H, P))
    for t in range(T):
        for b in range(batch):
            y_ref[b, t] = O.step(ocfg, st, b, inp["x"][b, t], inp["B"][b, t], inp["C"][b, t],
                                 inp["dt"][b, t], inp["A"], inp["D"])
        scale[:, t] = y_scale(ocfg, st, inp["C"][:, t], np.repeat(inp["D"][None], batch, 0),
                              inp["x"][:, t])
    got = download(codec, pool, pairs, ocfg)
    stats = compare_states(ocfg, got, st, None, f"scan {fmt}")
    assert stats["code_mismatch"] == 0
    check_y(y.cpu().numpy(), y_ref, scale, f"scan {fmt}")
    assert ssq.ssq_pool_error(cfg, pool) == 0
    return cfg, pool, inp, st, y


@pytest.mark.parametrize("fmt", ALL_FMTS)
def test_scan_tiny_parity(fmt):
    """The tiny workload's shape: 2 heads x 8 x 16, T = 64."""
    run_scan(fmt, H=2, P=8, N=16, G=1, batch=1, T=64, seed=0, init="zero")


@pytest.mark.parametrize("mask", ["all", "mid"])
def test_scan_370m_shape_reduced(mask):
    """The 370M scan's head shape (32 heads in three decay bands x 64 x 128,
    int4 asym, mid-band-only mask vs all heads) on 2 requests and T = 45
    tokens (a ragged last chunk)."""
    m = None if mask == "all" else W.mid_band_mask(32)
    run_scan("i4a", H=32, P=64, N=128, G=1, batch=2, T=45, mask=m, seed=2, banded=True,
             init="zero")


@pytest.mark.parametrize("fmt", ["i8a", "i4s", "bf16"])
def test_scan_groups_and_ragged_tiles(fmt):
    run_scan(fmt, H=6, P=12, N=64, G=3, batch=3, T=19, seed=8)


def _wide_scan_batch(H, P, N):
    """Requests that make the scan give each lane 64 entries of a row: at
    least one warp per SM sub-partition at 32 / (N / 64) rows per warp."""
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    rpw = 32 // (N // 64)
    per_request = H * -(-P // rpw)
    return -(-4 * sms // per_request)


@pytest.mark.parametrize("fmt,H,N", [("i8a", 32, 128), ("i4s", 32, 128), ("bf16", 32, 128),
                                     ("i8s", 16, 256), ("i4a", 32, 64), ("f32", 16, 256)])
def test_scan_wide_rows(fmt, H, N):
    """Batches large enough for 64 entries per lane (one lane per row at
    d_state 64, four at 256), over several staged chunks."""
    ssq = require_gpu()
    del ssq
    P = 64
    batch = _wide_scan_batch(H, P, N)
    run_scan(fmt, H=H, P=P, N=N, G=2, batch=batch, T=11, seed=12)


@pytest.mark.parametrize("fmt", ["i8a", "i4a", "i8s", "f32"])
def test_scan_equals_repeated_decode(fmt):
    """T tokens of the scan leave exactly the codes and metadata that T decode
    steps leave (the state carried on chip is the stored row's value)."""
    ssq = require_gpu()
    H, P, N, G, batch, T = 4, 16, 128, 2, 2, 21
    cfg, L, codec, ocfg = make_cfg(ssq, fmt, 1, batch, H, P, N, G)
    wl = W.Scan("eq", 31, batch, T, H, P, N, G, fmt)
    inp = wl.inputs()
    S0 = np.random.default_rng(9).standard_normal((batch, H * P * N)).astype(np.float32)
    pool_a = ssq.alloc_pool(cfg)
    ssq.ssq_quantize_rows(cfg, pool_a, None, batch, 0, 1, cuda(S0))
    pool_b = pool_a.clone()
    y_a = torch.empty((batch, T, H, P), device="cuda")
    ssq.ssq_scan(cfg, pool_a, None, batch, 0, T, cuda(inp["x"]), cuda(inp["B"]),
                 cuda(inp["C"]), cuda(inp["dt"]), cuda(inp["A"]), cuda(inp["D"]), y_a)
    A1, D1 = cuda(inp["A"][None]), cuda(inp["D"][None])
    y_b = torch.empty((batch, T, H, P), device="cuda")
    for t in range(T):
        yt = torch.empty((1, batch, H, P), device="cuda")
        ssq.ssq_decode_step(cfg, pool_b, None, batch, 0, 1, cuda(inp["x"][:, t][None]),
                            cuda(inp["B"][:, t][None]), cuda(inp["C"][:, t][None]),
                            cuda(inp["dt"][:, t][None]), A1, D1, yt)
        y_b[:, t] = yt[0]
    torch.cuda.synchronize()
    assert torch.equal(pool_a, pool_b)
    assert torch.allclose(y_a, y_b, rtol=1e-4, atol=1e-4)


@pytest.mark.parametrize("fmt", ["i8a", "i4s"])
def test_decode_many_one_tile_units(fmt):
    """Thousands of (layer, request, region) units of one tile each (3 heads x
    5 rows, one head kept fp32; head_dim 5, so x comes by one 4-byte copy per
    row): every tile starts a unit, so the producer builds a unit buffer and
    the consumer warps change unit buffers at every tile."""
    ssq = require_gpu()
    H, P, N, G, batch, nl = 3, 5, 128, 1, 256, 16
    mask = [1, 0, 1]
    cfg, L, codec, ocfg = make_cfg(ssq, fmt, nl, batch, H, P, N, G, mask)
    rng = np.random.default_rng(55)
    S0 = rng.standard_normal((nl * batch, H, P, N)).astype(np.float32)
    st = O.state_from_f32(ocfg, S0)
    pairs = [(b, l) for l in range(nl) for b in range(batch)]
    pool = upload(ssq, cfg, L, codec, st, pairs)
    inp = W.Decode("units", 61, nl, batch, H, P, N, G, fmt).inputs()
    y = torch.empty((nl, batch, H, P), device="cuda")
    ssq.ssq_decode_step(cfg, pool, None, batch, 0, nl, cuda(inp["x"]), cuda(inp["B"]),
                        cuda(inp["C"]), cuda(inp["dt"]), cuda(inp["A"]), cuda(inp["D"]), y)
    y_ref = np.zeros((nl * batch, H, P), np.float32)
    pre = np.zeros((nl * batch, H * P, N), np.float32)
    for i in range(nl * batch):
        l, b = divmod(i, batch)
        y_ref[i], pre[i] = O.step(ocfg, st, i, inp["x"][l, b], inp["B"][l, b], inp["C"][l, b],
                                  inp["dt"][l, b], inp["A"][l], inp["D"][l], want_pre=True)
    got = download(codec, pool, pairs, ocfg)
    compare_states(ocfg, got, st, pre, f"units {fmt}")
    Dpair = np.repeat(inp["D"][:, None, :], batch, axis=1).reshape(nl * batch, H)
    scale = y_scale(ocfg, st, inp["C"].reshape(nl * batch, G, N), Dpair,
                    inp["x"].reshape(nl * batch, H, P))
    check_y(y.cpu().numpy().reshape(nl * batch, H, P), y_ref, scale, f"units {fmt}")
    assert ssq.ssq_pool_error(cfg, pool) == 0
