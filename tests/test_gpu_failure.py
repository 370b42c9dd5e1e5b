"""The decode step's failure path, made to happen without faulting the GPU.

A bounded pipeline wait is made to run out on purpose: through the test
hooks of the C ABI (ssq_test_hooks) the producer of the first thread block
issues no copy for its first tile, so the wait on that tile's barrier never
completes (nothing is in flight); with the wait bound shortened, the call
must return, set SSQ_DEVERR_TIMEOUT in the pool's error word, and leave the
context usable: the next call, hooks off, matches the oracle.
"""
import numpy as np
import pytest
import torch

import oracle as O
from gpu_harness import check_y, compare_states, download, make_cfg, require_gpu, upload, \
    y_scale
from quantized_recurrent_state_mamba_b200 import workloads as W

pytestmark = pytest.mark.gpu


def cuda(a, dtype=torch.float32):
    return torch.from_numpy(np.ascontiguousarray(a)).to(device="cuda", dtype=dtype)


def _run(ssq, cfg, pool, inp, batch, H, P):
    y = torch.empty((1, batch, H, P), device="cuda")
    ssq.ssq_decode_step(cfg, pool, None, batch, 0, 1, cuda(inp["x"]), cuda(inp["B"]),
                        cuda(inp["C"]), cuda(inp["dt"]), cuda(inp["A"]), cuda(inp["D"]), y)
    torch.cuda.synchronize()
    return y


@pytest.mark.parametrize("fmt", ["i8a", "f32"])
def test_wait_timeout_sets_error_and_returns(fmt):
    ssq = require_gpu()
    H, P, N, batch = 4, 64, 128, 16
    cfg, L, codec, ocfg = make_cfg(ssq, fmt, 1, batch, H, P, N, 1)
    S0 = np.random.default_rng(3).standard_normal((batch, H, P, N)).astype(np.float32)
    st = O.state_from_f32(ocfg, S0)
    inp = W.Decode("timeout", 4, 1, batch, H, P, N, 1, fmt).inputs()
    pool = upload(ssq, cfg, L, codec, st, [(b, 0) for b in range(batch)])
    try:
        # about 1 ms of SM clock cycles per wait
        ssq.ssq_test_hooks(True, 2_000_000)
        _run(ssq, cfg, pool, inp, batch, H, P)
    finally:
        ssq.ssq_test_hooks(False, 0)
    assert ssq.ssq_pool_error(cfg, pool) & ssq.SSQ_DEVERR_TIMEOUT
    # the context is usable: a fresh pool, hooks off, matches the oracle
    pool = upload(ssq, cfg, L, codec, st, [(b, 0) for b in range(batch)])
    y = _run(ssq, cfg, pool, inp, batch, H, P)
    assert ssq.ssq_pool_error(cfg, pool) == 0
    y_ref = np.stack([O.step(ocfg, st, b, inp["x"][0, b], inp["B"][0, b], inp["C"][0, b],
                             inp["dt"][0, b], inp["A"][0], inp["D"][0]) for b in range(batch)])
    got = download(codec, pool, [(b, 0) for b in range(batch)], ocfg)
    stats = compare_states(ocfg, got, st, None, f"after timeout {fmt}")
    assert stats["code_mismatch"] == 0
    scale = y_scale(ocfg, st, inp["C"][0], np.repeat(inp["D"], batch, 0), inp["x"][0])
    check_y(y.cpu().numpy()[0], y_ref, scale, f"after timeout {fmt}")

