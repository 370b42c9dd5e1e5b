"""GPU parity of the step diagnostics (ssq_decode_diag) against the oracle.

"ssm-state-quantization" README, Findings 4 and 5: per row, the number of
entries whose change the rounding turns against the step's input, the rounding
error seen by the readout over the reversed entries and over all entries,
and the readout signal.  The reversal decision is taken in fp32 on both sides
from bit-equal operands (same update, same refit, same rounding), so the
counts must agree exactly; the three sums are fp32 on the GPU and double in
the oracle and must agree within fp32 summation error:
  |got - ref| <= 1e-5 * sum_n |C_n| |t_n| + 1e-37,
t_n the summed term (e_n or s'_n), the scale taken from the oracle's own
step.  The call must leave the pool untouched.
"""
import numpy as np
import pytest
import torch

import oracle as O
from gpu_harness import download, make_cfg, require_gpu, upload
from quantized_recurrent_state_mamba_b200 import workloads as W

pytestmark = pytest.mark.gpu

ALL_FMTS = ["f32", "bf16", "i8s", "i8a", "i4s", "i4a"]
QFMTS = ["i8s", "i8a", "i4s", "i4a"]
SUM_TOL = 1e-5


def cuda(a, dtype=torch.float32):
    return torch.from_numpy(np.ascontiguousarray(a)).to(device="cuda", dtype=dtype)


def oracle_diag(ocfg, st, inp, nl, batch, H, P, N, G):
    """Oracle diagnostics of every pair plus the tolerance scales
    sum_n |C_n||e_n| and sum_n |C_n||s'_n| per row."""
    ref = np.zeros((nl, batch, H, P, 4), np.float32)
    esc = np.zeros((nl, batch, H, P))
    ssc = np.zeros((nl, batch, H, P))
    hpg = H // G
    for i in range(nl * batch):
        l, b = divmod(i, batch)
        args = (inp["x"][l, b], inp["B"][l, b], inp["C"][l, b], inp["dt"][l, b],
                inp["A"][l], inp["D"][l])
        ref[l, b] = O.step_diag(ocfg, st, i, *args)
        # s' from the same stored values through the fp32 step (no rounding)
        cf = O.Cfg(O.F32, H, P, N, G)
        sf = O.state_from_f32(cf, O.state_to_f32(st)[i])
        O.step(cf, sf, 0, *args)
        pre = O.state_to_f32(sf)[0].reshape(H * P, N)
        one = st.copy()
        O.step(ocfg, one, i, *args)
        deq = O.state_to_f32(one)[i].reshape(H * P, N)
        Cabs = np.abs(inp["C"][l, b].astype(np.float64))          # [G][N]
        Crow = np.repeat(Cabs, hpg * P, axis=0)                     # [H*P][N]
        err = np.abs(deq.astype(np.float64) - pre.astype(np.float64))
        esc[l, b] = (Crow * err).sum(1).reshape(H, P)
        ssc[l, b] = (Crow * np.abs(pre.astype(np.float64))).sum(1).reshape(H, P)
    return ref, esc, ssc


def check_diag(got, ref, esc, ssc, quant_rows, where):
    got = got.reshape(ref.shape)
    np.testing.assert_array_equal(got[..., 0], ref[..., 0], err_msg=f"{where} reversal counts")
    for k, sc in ((1, esc), (2, esc), (3, ssc)):
        d = np.abs(got[..., k].astype(np.float64) - ref[..., k].astype(np.float64))
        lim = SUM_TOL * sc + 1e-37
        bad = d > lim
        assert not bad.any(), (f"{where} column {k}: {int(bad.sum())} rows off, worst "
                               f"{float((d / lim).max()):.3g}x the bound")
    # rows held as fp32 / bf16 are not rounded: no reversals, no error
    fp = ~quant_rows
    assert not got[..., 0:3][np.broadcast_to(fp[..., None], got[..., 0:3].shape)].any()


def run_diag(fmt, H, P, N, G, batch, nl, layer0, n_layers, slots, mask=None, seed=0,
             S0=None, tweak=None):
    ssq = require_gpu()
    n_slots = max(slots) + 1 if slots is not None else batch
    cfg, L, codec, ocfg = make_cfg(ssq, fmt, n_layers, n_slots, H, P, N, G, mask)
    slot_list = slots if slots is not None else list(range(batch))
    pairs = [(slot_list[b], layer0 + l) for l in range(nl) for b in range(batch)]
    if S0 is None:
        wl0 = W.Decode("case", seed, nl, batch, H, P, N, G, fmt)
        S0 = np.stack([wl0.state_pair(l, b).reshape(H, P, N)
                       for l in range(nl) for b in range(batch)])
    st = O.state_from_f32(ocfg, S0)
    pool = upload(ssq, cfg, L, codec, st, pairs)
    before = pool.clone()
    inp = W.Decode("case", seed * 1000 + 1, nl, batch, H, P, N, G, fmt).inputs()
    if tweak is not None:
        tweak(inp)
    slot_t = None if slots is None else cuda(np.array(slots, np.int32), torch.int32)
    diag = torch.full((nl, batch, H, P, 4), float("nan"), device="cuda")
    ssq.ssq_decode_diag(cfg, pool, slot_t, batch, layer0, nl, cuda(inp["x"]), cuda(inp["B"]),
                        cuda(inp["C"]), cuda(inp["dt"]), cuda(inp["A"]), diag)
    torch.cuda.synchronize()
    assert torch.equal(pool, before), "the diagnostics call changed the pool"
    assert ssq.ssq_pool_error(cfg, pool) == 0
    ref, esc, ssc = oracle_diag(ocfg, st, inp, nl, batch, H, P, N, G)
    quant_rows = np.array([ocfg.row_is_quant(h) for h in range(H)])
    quant_rows = np.broadcast_to(quant_rows[None, None, :, None], (nl, batch, H, P))
    check_diag(diag.cpu().numpy(), ref, esc, ssc, quant_rows, f"diag {fmt} N{N}")
    return diag.cpu().numpy(), ref


@pytest.mark.parametrize("fmt", ALL_FMTS)
@pytest.mark.parametrize("N", [16, 64, 128, 256])
def test_diag_parity(fmt, N):
    """Several tiles per (layer, request) with a ragged tail (6 heads x 24
    rows), 3 groups, 2 of 3 layers, permuted slots."""
    got, ref = run_diag(fmt, H=6, P=24, N=N, G=3, batch=3, nl=2, layer0=1, n_layers=3,
                        slots=[2, 0, 4], seed=N + 3)
    if fmt in QFMTS:
        # the workload's states do reverse entries: the test is not vacuous
        assert ref[..., 0].sum() > 0


@pytest.mark.parametrize("fmt", QFMTS)
def test_diag_masked(fmt):
    """Only some heads quantized; the fp heads report the signal only."""
    run_diag(fmt, H=7, P=16, N=128, G=1, batch=2, nl=1, layer0=0, n_layers=1, slots=None,
             mask=[0, 1, 1, 0, 1, 0, 0], seed=5)


@pytest.mark.parametrize("fmt", QFMTS)
def test_diag_zoo(fmt):
    """Constant, near-constant, one-signed, subnormal and zero stored rows
    (the refit's slow paths), a pure requantize (dt = 0: no input, so no
    entry can reverse) and pure-decay rows (x = 0)."""
    from test_gpu_parity import zoo_state
    H, P, N, G, batch = 4, 16, 128, 2, 2
    S0 = zoo_state(np.random.default_rng(78), batch, H, P, N)

    def tweak(inp):
        inp["dt"][0, 0, :] = 0.0
        inp["x"][0, 1, 1, :] = 0.0

    got, ref = run_diag(fmt, H, P, N, G, batch, nl=1, layer0=0, n_layers=1, slots=None,
                        seed=17, S0=S0, tweak=tweak)
    got = got.reshape(ref.shape)
    assert not got[0, 0, :, :, 0].any()       # w = 0 everywhere: nothing reverses
    assert not got[0, 1, 1, :, 0].any()


@pytest.mark.parametrize("fmt", ["i8s", "i4a"])
def test_diag_empty_batch(fmt):
    ssq = require_gpu()
    cfg, L, codec, ocfg = make_cfg(ssq, fmt, 1, 2, 2, 8, 16, 1)
    pool = ssq.alloc_pool(cfg)
    d = torch.zeros(16, device="cuda")
    ssq.ssq_decode_diag(cfg, pool, None, 0, 0, 1, d, d, d, d, d, d)
    torch.cuda.synchronize()
