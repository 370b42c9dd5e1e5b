"""GPU parity of stochastic rounding (ssq_decode_step_sr, ssq_scan_sr through
the C ABI) against the CPU oracle ("ssm-state-quantization" README,
Findings 9).  Both sides draw from Philox4x32-10 with the same key and
counters, and take the rounding decision floor(s'*inv + u) exactly, so the
codes must match bit for bit; y within the readout tolerance."""
import numpy as np
import pytest
import torch

import oracle as O
from gpu_harness import check_y, compare_states, download, make_cfg, require_gpu, upload, y_scale
from quantized_recurrent_state_mamba_b200 import workloads as W

pytestmark = pytest.mark.gpu

QFMTS = ["i8s", "i8a", "i4s", "i4a"]
SEED = 0x9E3779B97F4A7C15


def cuda(a, dtype=torch.float32):
    return torch.from_numpy(np.ascontiguousarray(a)).to(device="cuda", dtype=dtype)


def run_decode_sr(fmt, H, P, N, G, batch, nl, layer0, n_layers, slots, step, mask=None,
                  seed=0, init="normal"):
    ssq = require_gpu()
    n_slots = max(slots) + 1
    cfg, L, codec, ocfg = make_cfg(ssq, fmt, n_layers, n_slots, H, P, N, G, mask)
    pairs = [(slots[b], layer0 + l) for l in range(nl) for b in range(batch)]
    wl = W.Decode("sr", seed, nl, batch, H, P, N, G, fmt, init=init)
    S0 = np.stack([wl.state_pair(l, b).reshape(H, P, N) for l in range(nl) for b in range(batch)])
    st = O.state_from_f32(ocfg, S0)
    pool = upload(ssq, cfg, L, codec, st, pairs)
    inp = W.Decode("sr", seed * 1000 + 1, nl, batch, H, P, N, G, fmt).inputs()
    y = torch.full((nl, batch, H, P), float("nan"), device="cuda")
    slot_t = cuda(np.array(slots, np.int32), torch.int32)
    ssq.ssq_decode_step_sr(cfg, pool, slot_t, batch, layer0, nl, cuda(inp["x"]), cuda(inp["B"]),
                           cuda(inp["C"]), cuda(inp["dt"]), cuda(inp["A"]), cuda(inp["D"]), y,
                           SEED, step)
    y_ref = np.zeros((nl, batch, H, P), np.float32)
    for i in range(nl * batch):
        l, b = divmod(i, batch)
        y_ref[l, b] = O.step_sr(ocfg, st, i, inp["x"][l, b], inp["B"][l, b], inp["C"][l, b],
                                inp["dt"][l, b], inp["A"][l], inp["D"][l], SEED, step,
                                layer0 + l, slots[b])
    got = download(codec, pool, pairs, ocfg)
    stats = compare_states(ocfg, got, st, None, f"decode sr {fmt}")
    assert stats["code_mismatch"] == 0
    Dpair = np.repeat(inp["D"][:, None, :], batch, axis=1).reshape(nl * batch, H)
    scale = y_scale(ocfg, st, inp["C"].reshape(nl * batch, G, N), Dpair,
                    inp["x"].reshape(nl * batch, H, P))
    check_y(y.cpu().numpy().reshape(nl * batch, H, P), y_ref.reshape(nl * batch, H, P), scale,
            f"decode sr {fmt}")
    assert ssq.ssq_pool_error(cfg, pool) == 0
    return ssq, cfg, pool, st


@pytest.mark.parametrize("fmt", QFMTS)
@pytest.mark.parametrize("N", [16, 64, 128, 256])
def test_decode_sr_parity(fmt, N):
    """Partial tiles (6 heads x 24 rows), 3 groups, 2 of 3 layers, permuted
    slots, a step counter above 2^31."""
    run_decode_sr(fmt, H=6, P=24, N=N, G=3, batch=3, nl=2, layer0=1, n_layers=3,
                  slots=[2, 0, 4], step=0x80000011, seed=N)


@pytest.mark.parametrize("fmt", QFMTS)
def test_decode_sr_masked(fmt):
    """Masked heads keep fp32 rows; only the quantized rows draw."""
    run_decode_sr(fmt, H=7, P=16, N=128, G=1, batch=2, nl=1, layer0=0, n_layers=1,
                  slots=[1, 0], step=5, mask=[0, 1, 1, 0, 1, 0, 0], seed=5)


def test_decode_sr_differs_from_nearest_and_from_other_steps():
    """Stochastic rounding changes codes against nearest rounding, and two
    step counters give different codes (same inputs)."""
    ssq, cfg, pool_a, st_a = run_decode_sr("i8a", H=4, P=16, N=128, G=1, batch=2, nl=1,
                                           layer0=0, n_layers=1, slots=[0, 1], step=1)
    _, _, pool_b, st_b = run_decode_sr("i8a", H=4, P=16, N=128, G=1, batch=2, nl=1,
                                       layer0=0, n_layers=1, slots=[0, 1], step=2)
    assert not np.array_equal(st_a.q, st_b.q)
    assert not torch.equal(pool_a, pool_b)


@pytest.mark.parametrize("fmt", QFMTS)
def test_scan_sr_parity(fmt):
    """T = 13 tokens with stochastic rounding at every token, 2 requests,
    64 x 128 rows (the 370M head shape at a small batch)."""
    ssq = require_gpu()
    H, P, N, G, batch, T = 4, 64, 128, 1, 2, 13
    cfg, L, codec, ocfg = make_cfg(ssq, fmt, 2, batch + 1, H, P, N, G)
    wl = W.Scan("scan_sr", 3, batch, T, H, P, N, G, fmt, init="normal")
    inp = wl.inputs()
    S0 = np.stack([W.state_pair(3, 1, b, H * P, N).reshape(H, P, N) for b in range(batch)])
    st = O.state_from_f32(ocfg, S0)
    slots = [2, 1]
    pairs = [(slots[b], 1) for b in range(batch)]
    pool = upload(ssq, cfg, L, codec, st, pairs)
    y = torch.empty((batch, T, H, P), device="cuda")
    ssq.ssq_scan_sr(cfg, pool, cuda(np.array(slots, np.int32), torch.int32), batch, 1, T,
                    cuda(inp["x"]), cuda(inp["B"]), cuda(inp["C"]), cuda(inp["dt"]),
                    cuda(inp["A"]), cuda(inp["D"]), y, SEED, 1000)
    y_ref = np.zeros((batch, T, H, P), np.float32)
    scale = np.zeros((batch, T, H, P))
    for t in range(T):
        for b in range(batch):
            y_ref[b, t] = O.step_sr(ocfg, st, b, inp["x"][b, t], inp["B"][b, t], inp["C"][b, t],
                                    inp["dt"][b, t], inp["A"], inp["D"], SEED, 1000 + t, 1,
                                    slots[b])
        scale[:, t] = y_scale(ocfg, st, inp["C"][:, t], np.repeat(inp["D"][None], batch, 0),
                              inp["x"][:, t])
    got = download(codec, pool, pairs, ocfg)
    stats = compare_states(ocfg, got, st, None, f"scan sr {fmt}")
    assert stats["code_mismatch"] == 0
    check_y(y.cpu().numpy(), y_ref, scale, f"scan sr {fmt}")
    assert ssq.ssq_pool_error(cfg, pool) == 0


def test_scan_sr_equals_repeated_decode_sr():
    """T tokens of ssq_scan_sr leave exactly the codes and metadata of T
    ssq_decode_step_sr calls at steps step0 .. step0+T-1."""
    ssq = require_gpu()
    H, P, N, G, batch, T = 3, 20, 64, 1, 2, 9
    cfg, L, codec, ocfg = make_cfg(ssq, "i4a", 1, batch, H, P, N, G)
    wl = W.Scan("sr_eq", 4, batch, T, H, P, N, G, "i4a", init="normal")
    inp = wl.inputs()
    a = ssq.alloc_pool(cfg)
    b = ssq.alloc_pool(cfg)
    S0 = cuda(np.stack([W.state_pair(4, 0, r, H * P, N) for r in range(batch)]))
    ssq.ssq_quantize_rows(cfg, a, None, batch, 0, 1, S0)
    ssq.ssq_quantize_rows(cfg, b, None, batch, 0, 1, S0)
    y = torch.empty((batch, T, H, P), device="cuda")
    ssq.ssq_scan_sr(cfg, a, None, batch, 0, T, cuda(inp["x"]), cuda(inp["B"]), cuda(inp["C"]),
                    cuda(inp["dt"]), cuda(inp["A"]), cuda(inp["D"]), y, 77, 40)
    yd = torch.empty((1, batch, H, P), device="cuda")
    for t in range(T):
        ssq.ssq_decode_step_sr(cfg, b, None, batch, 0, 1, cuda(inp["x"][:, t][None]),
                               cuda(inp["B"][:, t][None]), cuda(inp["C"][:, t][None]),
                               cuda(inp["dt"][:, t][None]), cuda(inp["A"][None]),
                               cuda(inp["D"][None]), yd, 77, 40 + t)
    torch.cuda.synchronize()
    assert torch.equal(a, b)
