"""GPU parity of the DAMP mixed-tier state (ssq_damp_*) against the oracle.

"Mamba state quantization for inference", "Mixed precision spends bits on
persistent channels": Hadamard rotation of each key channel's value vector,
protected channels in FP16, the rest INT8 with a scale and a zero point, the
recurrence in FP32, new quantization parameters every token.

Acceptance: the rotated input and the rotation of the hand-off are summed in
double in the same order on both sides and rounded once, and every later
operation that decides a stored value is one fp32 operation in the same
order, so codes, steps, zero points and FP16 bit patterns must be equal, and
so must the read-back fp32 state; y is accumulated in fp32 on the GPU and in
double in the oracle:
  |y - y_ref| <= 1e-4 * ((1/P) sum_k sum_m |C[chan[m]]| |t'_m[k]| + |D x|).
The oracle's state is packed into the pool on the host and uploaded; the
GPU's pool is read back and unpacked; nothing flows from the GPU into the
oracle.
"""
import numpy as np
import pytest
import torch

import oracle as O
from gpu_harness import require_gpu
from poolcodec import DampCodec
from quantized_recurrent_state_mamba_b200 import workloads as W

pytestmark = pytest.mark.gpu

Y_TOL = 1e-4


def cuda(a, dtype=torch.float32):
    return torch.from_numpy(np.ascontiguousarray(a)).to(device="cuda", dtype=dtype)


def setup(ssq, n_layers, n_slots, H, P, N, G, K, seed):
    cfg = ssq.DampConfig(n_layers, n_slots, H, P, N, G, K)
    L = ssq.ssq_damp_pool_layout(cfg)
    rng = np.random.default_rng(seed)
    chan = np.stack([np.stack([rng.permutation(N) for _ in range(H)])
                     for _ in range(n_layers)]).astype(np.int32)     # [layers][H][N]
    codec = DampCodec(H, P, N, K, L)
    return cfg, L, chan, codec


def states(seed, count, H, P, N, kinds=True):
    """Normal states with some hard groups: constant channels, channels far
    from zero, tiny channels, zeros."""
    rng = np.random.default_rng(seed)
    S = rng.standard_normal((count, H, P, N)).astype(np.float32)
    if kinds:
        for c in range(count):
            for h in range(H):
                n = rng.integers(0, N, 4)
                S[c, h, :, n[0]] = np.float32(rng.standard_normal())
                S[c, h, :, n[1]] = 500.0 + S[c, h, :, n[1]] * 1e-3
                S[c, h, :, n[2]] *= 1e-30
                S[c, h, :, n[3]] = 0.0
    return S


def ocfg_of(l, H, P, N, G, K, chan, layer):
    return O.DampCfg(H, P, N, G, K, chan[layer])


def upload(ssq, L, codec, pairs, sts):
    buf = np.zeros(L["pool_bytes"], np.uint8)
    for (slot, layer), st in zip(pairs, sts):
        codec.write(buf, slot, layer, st.hi[0], st.q[0], st.delta[0], st.zero[0])
    return torch.from_numpy(buf).cuda()


def check_pair(codec, buf, slot, layer, st, where):
    hi, q, d, z = codec.read(buf, slot, layer)
    bits = codec.read_hi_bits(buf, slot, layer)
    ref_bits = st.hi[0].astype(np.float16).view(np.uint16)
    assert np.array_equal(bits, ref_bits), f"{where}: FP16 tier differs"
    assert np.array_equal(q, st.q[0]), f"{where}: codes differ ({int((q != st.q[0]).sum())})"
    assert np.array_equal(d.view(np.uint32), st.delta[0].view(np.uint32)), f"{where}: steps differ"
    assert np.array_equal(z.view(np.uint32), st.zero[0].view(np.uint32)), f"{where}: zeros differ"


@pytest.mark.parametrize("P", [16, 32, 64, 128])
@pytest.mark.parametrize("K", [0, 16, "all"])
def test_damp_quantize_dequantize_bit_exact(P, K):
    ssq = require_gpu()
    H, N, G, nl, batch, n_layers, n_slots = 3, 48 if P == 128 else 128, 1, 2, 3, 3, 5
    K = N if K == "all" else K
    cfg, L, chan, codec = setup(ssq, n_layers, n_slots, H, P, N, G, K, seed=P + K)
    slots = [4, 0, 2]
    S = states(P * 7 + K, nl * batch, H, P, N)
    pool = ssq.damp_alloc_pool(cfg)
    chan_t = cuda(chan, torch.int32)
    slot_t = cuda(np.array(slots, np.int32), torch.int32)
    ssq.ssq_damp_quantize(cfg, pool, chan_t, slot_t, batch, 1, nl, cuda(S))
    out = torch.full((nl * batch, H, P, N), float("nan"), device="cuda")
    ssq.ssq_damp_dequantize(cfg, pool, chan_t, slot_t, batch, 1, nl, out)
    assert ssq.ssq_damp_pool_error(cfg, pool) == 0
    buf = pool.cpu().numpy()
    out = out.cpu().numpy()
    for i in range(nl * batch):
        l, b = divmod(i, batch)
        oc = ocfg_of(l, H, P, N, G, K, chan, 1 + l)
        st = O.damp_from_f32(oc, S[i])
        check_pair(codec, buf, slots[b], 1 + l, st, f"quantize P{P} K{K} pair {i}")
        back = O.damp_to_f32(st)[0]
        assert np.array_equal(out[i].view(np.uint32), back.view(np.uint32)), \
            f"dequantize P{P} K{K} pair {i}"
    # untouched layer 0 stays zero
    hi, q, d, z = codec.read(buf, slots[0], 0)
    assert not hi.any() and not q.any() and not d.any()


def run_step(P, K, N=128, H=4, G=2, batch=3, nl=2, layer0=1, n_layers=3, slots=(2, 0, 4),
             seed=0, steps=1, S=None, tweak=None):
    """`steps` chained decode steps on the GPU and in the oracle (no
    re-upload between steps: the GPU state must stay bit-equal)."""
    ssq = require_gpu()
    n_slots = max(slots) + 1
    cfg, L, chan, codec = setup(ssq, n_layers, n_slots, H, P, N, G, K, seed)
    if S is None:
        S = states(seed + 1, nl * batch, H, P, N)
    pairs = [(slots[b], layer0 + l) for l in range(nl) for b in range(batch)]
    ocs = [ocfg_of(l, H, P, N, G, K, chan, layer0 + l) for l in range(nl) for b in range(batch)]
    sts = [O.damp_from_f32(oc, S[i]) for i, oc in enumerate(ocs)]
    pool = upload(ssq, L, codec, pairs, sts)
    chan_t = cuda(chan, torch.int32)
    slot_t = cuda(np.array(slots, np.int32), torch.int32)
    worst = 0.0
    for k in range(steps):
        inp = W.Decode("damp", seed * 100 + k + 1, nl, batch, H, P, N, G, "i8a").inputs()
        if tweak is not None:
            tweak(inp)
        y = torch.full((nl, batch, H, P), float("nan"), device="cuda")
        ssq.ssq_damp_decode_step(cfg, pool, chan_t, slot_t, batch, layer0, nl, cuda(inp["x"]),
                                 cuda(inp["B"]), cuda(inp["C"]), cuda(inp["dt"]),
                                 cuda(inp["A"]), cuda(inp["D"]), y)
        y = y.cpu().numpy()
        buf = pool.cpu().numpy()
        for i in range(nl * batch):
            l, b = divmod(i, batch)
            x, B, C, dt = (inp[n][l, b] for n in ("x", "B", "C", "dt"))
            y_ref = O.damp_step(ocs[i], sts[i], 0, x, B, C, dt, inp["A"][l], inp["D"][l])
            check_pair(codec, buf, slots[b], layer0 + l, sts[i], f"step {k} P{P} K{K} pair {i}")
            # y tolerance from the stored state
            st = sts[i]
            t = np.zeros((H, N, P))
            t[:, :K] = st.hi[0]
            t[:, K:] = (st.q[0] - st.zero[0][..., None]).astype(np.float64) \
                * st.delta[0][..., None]
            hpg = H // G
            for h in range(H):
                cabs = np.abs(C[h // hpg][chan[layer0 + l, h]]).astype(np.float64)   # [N] by m
                sc = (cabs[:, None] * np.abs(t[h])).sum() / P + np.abs(inp["D"][l][h] * x[h])
                err = np.abs(y[l, b, h].astype(np.float64) - y_ref[h])
                assert np.all(err <= Y_TOL * sc), \
                    f"step {k} P{P} K{K} pair {i} head {h}: y off by {float((err / sc).max()):.3g}"
                worst = max(worst, float((err / sc).max()))
    assert ssq.ssq_damp_pool_error(cfg, pool) == 0
    return worst


@pytest.mark.parametrize("P", [16, 32, 64, 128])
@pytest.mark.parametrize("K", [0, 16, 128])
def test_damp_decode_parity(P, K):
    """2 of 3 layers, 3 requests on permuted slots, 2 groups, a random
    channel map per (layer, head)."""
    run_step(P, K, seed=P + 3 * K)


def test_damp_decode_chained_steps():
    """Five chained steps with no re-upload: the GPU state stays bit-equal to
    the oracle's."""
    run_step(64, 16, steps=5, seed=9)


@pytest.mark.parametrize("N", [16, 48, 256])
def test_damp_decode_d_state(N):
    """d_state below one warp's positions, ragged against the CTA, and 256
    (two passes at headdim 64)."""
    run_step(64, min(16, N), N=N, H=3, G=1, batch=2, nl=1, layer0=0, n_layers=1, slots=(1, 0),
             seed=N)


def test_damp_decode_special_inputs():
    """dt = 0 for one request (lambda = 1, no input: a pure requantize) and
    x = 0 on one head (pure decay)."""
    def tweak(inp):
        inp["dt"][0, 0, :] = 0.0
        inp["x"][0, 1, 2, :] = 0.0
    run_step(64, 16, seed=21, tweak=tweak)


def test_damp_from_zero_pool():
    """A zeroed pool is the zero state: the first step is the input alone."""
    ssq = require_gpu()
    H, P, N, G, K, batch = 2, 64, 128, 1, 16, 2
    cfg, L, chan, codec = setup(ssq, 1, batch, H, P, N, G, K, seed=3)
    pool = ssq.damp_alloc_pool(cfg)
    chan_t = cuda(chan, torch.int32)
    inp = W.Decode("zero", 3, 1, batch, H, P, N, G, "i8a").inputs()
    y = torch.empty((1, batch, H, P), device="cuda")
    ssq.ssq_damp_decode_step(cfg, pool, chan_t, None, batch, 0, 1, cuda(inp["x"]), cuda(inp["B"]),
                             cuda(inp["C"]), cuda(inp["dt"]), cuda(inp["A"]), cuda(inp["D"]), y)
    buf = pool.cpu().numpy()
    oc = O.DampCfg(H, P, N, G, K, chan[0])
    for b in range(batch):
        st = O.DampState(oc)
        O.damp_step(oc, st, 0, inp["x"][0, b], inp["B"][0, b], inp["C"][0, b], inp["dt"][0, b],
                    inp["A"][0], inp["D"][0])
        check_pair(codec, buf, b, 0, st, f"zero pool request {b}")


def test_damp_bad_channel_map_and_slot():
    """A channel index out of range marks that head and skips it; a slot
    index out of range skips the request; both are reported in the error
    word and nothing else changes."""
    ssq = require_gpu()
    H, P, N, G, K, batch = 3, 64, 128, 1, 16, 2
    cfg, L, chan, codec = setup(ssq, 1, 4, H, P, N, G, K, seed=5)
    S = states(6, batch, H, P, N)
    slots = [1, 3]
    pool = ssq.damp_alloc_pool(cfg)
    chan_t = cuda(chan, torch.int32)
    slot_t = cuda(np.array(slots, np.int32), torch.int32)
    ssq.ssq_damp_quantize(cfg, pool, chan_t, slot_t, batch, 0, 1, cuda(S))
    assert ssq.ssq_damp_pool_error(cfg, pool) == 0
    before = pool.cpu().numpy().copy()
    bad = chan.copy()
    bad[0, 1, 7] = N          # head 1 of layer 0
    inp = W.Decode("bad", 7, 1, batch, H, P, N, G, "i8a").inputs()
    y = torch.zeros((1, batch, H, P), device="cuda")
    ssq.ssq_damp_decode_step(cfg, pool, cuda(bad, torch.int32), slot_t, batch, 0, 1,
                             cuda(inp["x"]), cuda(inp["B"]), cuda(inp["C"]), cuda(inp["dt"]),
                             cuda(inp["A"]), cuda(inp["D"]), y)
    assert ssq.ssq_damp_pool_error(cfg, pool) == ssq.SSQ_DEVERR_CHANNEL
    after = pool.cpu().numpy()
    for s in slots:
        h1 = codec.read(before, s, 0)
        h2 = codec.read(after, s, 0)
        for a, b in zip(h1, h2):
            assert np.array_equal(a[1], b[1])          # head 1 untouched
            assert not np.array_equal(a[0], b[0])      # head 0 stepped
    assert not y[0, :, 1].any()                        # its y is not written
    slot_bad = cuda(np.array([1, 9], np.int32), torch.int32)
    ssq.ssq_damp_decode_step(cfg, pool, chan_t, slot_bad, batch, 0, 1, cuda(inp["x"]),
                             cuda(inp["B"]), cuda(inp["C"]), cuda(inp["dt"]), cuda(inp["A"]),
                             cuda(inp["D"]), y)
    assert ssq.ssq_damp_pool_error(cfg, pool) == ssq.SSQ_DEVERR_SLOT


def test_damp_empty_batch():
    ssq = require_gpu()
    cfg = ssq.DampConfig(1, 2, 2, 64, 128, 1, 16)
    pool = ssq.damp_alloc_pool(cfg)
    chan = torch.zeros(2 * 128, dtype=torch.int32, device="cuda")
    d = torch.zeros(16, device="cuda")
    ssq.ssq_damp_decode_step(cfg, pool, chan, None, 0, 0, 1, d, d, d, d, d, d, d)
    torch.cuda.synchronize()
