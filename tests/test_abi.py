"""Host-only checks of the C ABI: the library loads, exports every symbol
include/ssq.h declares, computes the documented pool layout, and rejects bad
arguments before touching the GPU.  No compute call is made."""
import ctypes
import os
import re

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "ssq.h")
GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


@pytest.fixture(scope="module")
def ssq():
    from quantized_recurrent_state_mamba_b200 import build
    build.build()
    from quantized_recurrent_state_mamba_b200 import ssq as m
    return m


def declared_symbols():
    src = open(HEADER).read()
    return sorted(set(re.findall(r"SSQ_API\s+[\w\s\*]+?\b(ssq_\w+)\s*\(", src)))


def test_exports_every_declared_symbol(ssq):
    syms = declared_symbols()
    assert len(syms) == 19, syms
    lib = ctypes.CDLL(ssq.LIB_PATH)
    for s in syms:
        assert hasattr(lib, s), f"libssq.so does not export {s}"


def test_status_strings(ssq):
    assert ssq.ssq_status_string(0) == "SSQ_OK"
    assert ssq.ssq_status_string(4) == "SSQ_ERR_CUDA"


def _layout(ssq, **kw):
    return ssq.ssq_pool_layout(ssq.Config(**kw))


def expected_slot_bytes(fmt, L, H, P, N, mask=None):
    """Bytes per slot from the header's description, computed here."""
    quant = fmt in ("i8s", "i8a", "i4s", "i4a")
    hq = (sum(1 for m in mask if m) if mask is not None else H) if quant else 0
    hf = H - hq
    b = {"i8s": 8, "i8a": 8, "i4s": 4, "i4a": 4}.get(fmt, 0)
    meta = {"i8s": 4, "i4s": 4, "i8a": 8, "i4a": 8}.get(fmt, 0)
    eb = 2 if fmt == "bf16" else 4
    up = lambda v: (v + 255) // 256 * 256
    codes = L * up(hq * P * N * b // 8)
    metab = L * up(hq * P * meta)
    fp = L * up(hf * P * N * eb)
    return up(up(up(codes) + metab) + fp)


@pytest.mark.parametrize("fmt", ["f32", "bf16", "i8s", "i8a", "i4s", "i4a"])
@pytest.mark.parametrize("shape", [(24, 24, 64, 128, 1), (1, 128, 64, 128, 8),
                                   (30, 32, 128, 128, 1), (1, 2, 8, 16, 1), (3, 5, 7, 32, 5)])
def test_layout_matches_documentation(ssq, fmt, shape):
    L, H, P, N, G = shape
    d, perm = _layout(ssq, n_layers=L, n_slots=3, nheads=H, headdim=P, d_state=N,
                      ngroups=G, fmt=fmt)
    assert d["header_bytes"] == 256
    assert d["slot_bytes"] == expected_slot_bytes(fmt, L, H, P, N)
    assert d["pool_bytes"] == 256 + 3 * d["slot_bytes"]
    for k in ("codes_off", "meta_off", "fp_off", "slot_bytes"):
        assert d[k] % 256 == 0
    # regions do not overlap
    assert d["codes_off"] + L * d["codes_layer_bytes"] <= d["meta_off"]
    assert d["meta_off"] + L * d["meta_layer_bytes"] <= d["fp_off"]
    assert d["fp_off"] + L * d["fp_layer_bytes"] <= d["slot_bytes"]
    assert perm == list(range(H))


def test_mask_regions(ssq):
    mask = [0, 1, 1, 0, 1]
    d, perm = _layout(ssq, n_layers=2, n_slots=1, nheads=5, headdim=4, d_state=16,
                      fmt="i4a", head_mask=mask)
    assert d["n_quant_heads"] == 3 and d["n_fp_heads"] == 2
    assert perm == [1, 2, 4, 0, 3]
    assert d["slot_bytes"] == expected_slot_bytes("i4a", 2, 5, 4, 16, mask)
    # the mask is ignored by the fp formats
    d2, perm2 = _layout(ssq, n_layers=2, n_slots=1, nheads=5, headdim=4, d_state=16,
                        fmt="f32", head_mask=mask)
    assert d2["n_quant_heads"] == 0 and perm2 == list(range(5))


def _golden_pool_sizes():
    vals = {}
    for line in open(os.path.join(GOLDEN, "state_pool_sizes.txt")):
        line = line.strip()
        if line and not line.startswith("#"):
            k, v = line.split("=")
            vals[k.strip()] = float(v)
    return vals


def test_fp32_pool_matches_page_figure(ssq):
    """The serving-scale fp32 pool (30 layers, 32 heads x 128 x 128, batch
    256) is the 15 GB, ~60 MB per request that "Mamba state quantization for
    inference" reports ("Recurrent state is fixed per request, not free")."""
    g = _golden_pool_sizes()
    d, _ = _layout(ssq, n_layers=30, n_slots=256, nheads=32, headdim=128, d_state=128,
                   fmt="f32")
    per_req = d["slot_bytes"]
    total = d["pool_bytes"] - d["header_bytes"]
    assert abs(total / 2 ** 30 - g["pool_gib_batch256"]) / g["pool_gib_batch256"] < 0.01
    assert abs(per_req / 1e6 - g["mb_per_request"]) / g["mb_per_request"] < 0.06
    # proportional estimates the page gives at batch 32 and 96
    assert abs(32 * per_req / 1e9 - g["gb_batch32"]) / g["gb_batch32"] < 0.12
    assert abs(96 * per_req / 1e9 - g["gb_batch96"]) / g["gb_batch96"] < 0.12
    # bits per value of the quantized formats, metadata included
    for fmt, bpv in (("i8a", 8.5), ("i8s", 8.25), ("i4a", 4.5), ("i4s", 4.25), ("bf16", 16)):
        dq, _ = _layout(ssq, n_layers=30, n_slots=1, nheads=32, headdim=128, d_state=128,
                        fmt=fmt)
        assert abs(dq["slot_bytes"] * 8 / (30 * 32 * 128 * 128) - bpv) < 1e-3


@pytest.mark.parametrize("kw,status", [
    (dict(d_state=48), 2), (dict(d_state=0), 2), (dict(nheads=0), 2),
    (dict(nheads=513), 2), (dict(ngroups=3), 1), (dict(n_layers=0), 1),
    (dict(n_slots=0), 1), (dict(headdim=0), 1), (dict(fmt=9), 1)])
def test_layout_rejects_bad_configs(ssq, kw, status):
    base = dict(n_layers=2, n_slots=4, nheads=8, headdim=16, d_state=64, ngroups=2, fmt="i8a")
    base.update(kw)
    with pytest.raises(ssq.SsqError) as e:
        ssq.ssq_pool_layout(ssq.Config(**base))
    assert e.value.status == status


def test_entry_points_validate_before_launch(ssq):
    """Bad pointers, sizes and ranges are rejected on the host: the calls
    return an argument status without any CUDA call (no GPU here)."""
    lib = ssq.raw()
    cfg = ssq.Config(n_layers=2, n_slots=4, nheads=4, headdim=8, d_state=32, fmt="i8a")
    P = ctypes.c_void_p
    good = 0x10000000
    args = dict(pool=good, slots=None, batch=2, layer0=0, nl=1, x=good, B=good, C=good,
                dt=good, A=good, D=good, y=good)

    def call(**over):
        a = dict(args, **over)
        return lib.ssq_decode_step(cfg.ref, P(a["pool"]), P(a["slots"]), a["batch"],
                                   a["layer0"], a["nl"], P(a["x"]), P(a["B"]), P(a["C"]),
                                   P(a["dt"]), P(a["A"]), P(a["D"]), P(a["y"]), None)

    assert call(pool=good + 16) == ssq.SSQ_ERR_ALIGNMENT
    assert call(pool=0) == ssq.SSQ_ERR_INVALID_ARG
    assert call(x=good + 4) == ssq.SSQ_ERR_ALIGNMENT
    assert call(y=0) == ssq.SSQ_ERR_INVALID_ARG
    assert call(dt=good + 2) == ssq.SSQ_ERR_ALIGNMENT
    assert call(batch=-1) == ssq.SSQ_ERR_INVALID_ARG
    assert call(batch=5) == ssq.SSQ_ERR_INVALID_ARG        # > n_slots, identity slots
    assert call(layer0=1, nl=2) == ssq.SSQ_ERR_INVALID_ARG
    assert call(nl=0) == ssq.SSQ_ERR_INVALID_ARG
    assert call(slots=good + 2) == ssq.SSQ_ERR_ALIGNMENT
    assert "aligned" in ssq.ssq_last_error_detail()
    # an empty batch is a no-op that succeeds without a launch
    assert call(batch=0) == ssq.SSQ_OK
    r = lib.ssq_scan(cfg.ref, P(good), None, 2, 0, -1, P(good), P(good), P(good), P(good),
                     P(good), P(good), P(good), None)
    assert r == ssq.SSQ_ERR_INVALID_ARG
    r = lib.ssq_scan(cfg.ref, P(good), None, 2, 2, 4, P(good), P(good), P(good), P(good),
                     P(good), P(good), P(good), None)
    assert r == ssq.SSQ_ERR_INVALID_ARG                      # layer out of range
    r = lib.ssq_quantize_rows(cfg.ref, P(good), None, 2, 0, 1, P(good + 8), None)
    assert r == ssq.SSQ_ERR_ALIGNMENT


def test_no_cpu_fallback_in_product(ssq):
    """The product modules neither import nor name the oracle."""
    pkg = os.path.join(ROOT, "quantized_recurrent_state_mamba_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h", ".cpp")):
                src = open(os.path.join(dirpath, f)).read()
                assert "import oracle" not in src and "from oracle" not in src, f
                assert "oref_" not in src, f


def test_damp_layout_matches_page_figure(ssq):
    """"Mamba state quantization for inference", "Mixed precision spends bits
    on persistent channels": 16 of 128 key channels in FP16 (16 bits), the
    rest at 9 bits with metadata, 9.875 bits per value on average.  At
    headdim 64 the INT8 tier's {fp32 step, fp32 zero point} per channel is
    one bit per value."""
    cfg = ssq.DampConfig(n_layers=2, n_slots=3, nheads=4, headdim=64, d_state=128, ngroups=1,
                         n_protected=16)
    d = ssq.ssq_damp_pool_layout(cfg)
    assert d["bits_per_value"] == 9.875
    assert d["hi_off"] == 0 and d["codes_off"] == 16 * 64 * 2
    assert d["meta_off"] == d["codes_off"] + 112 * 64
    assert d["head_bytes"] == d["meta_off"] + 112 * 8
    assert d["head_bytes"] * 8 / (128 * 64) == 9.875       # no padding at this shape
    assert d["layer_bytes"] == 4 * d["head_bytes"]
    assert d["slot_bytes"] % ssq.SSQ_POOL_ALIGN == 0 and d["slot_bytes"] >= 2 * d["layer_bytes"]
    assert d["pool_bytes"] == ssq.SSQ_POOL_HEADER_BYTES + 3 * d["slot_bytes"]
    # the uniform controls: all INT8 (9 bits), all FP16 (16 bits)
    for K, bpv in ((0, 9.0), (128, 16.0)):
        c = ssq.DampConfig(1, 1, 4, 64, 128, 1, K)
        assert ssq.ssq_damp_pool_layout(c)["bits_per_value"] == bpv
    # the 130M-shaped pool at batch 256 against its fp32 size: 9.875 / 32
    c = ssq.DampConfig(24, 256, 24, 64, 128, 1, 16)
    f = ssq.Config(24, 256, 24, 64, 128, 1, "f32")
    ratio = (ssq.ssq_damp_pool_layout(c)["pool_bytes"] / ssq.ssq_pool_layout(f)[0]["pool_bytes"])
    assert abs(ratio - 9.875 / 32) < 1e-4


@pytest.mark.parametrize("kw,status", [
    (dict(headdim=48), 2), (dict(headdim=256), 2), (dict(d_state=40), 2), (dict(d_state=512), 2),
    (dict(n_protected=129), 1), (dict(n_protected=-1), 1), (dict(ngroups=3), 1),
    (dict(nheads=0), 1), (dict(n_layers=0), 1)])
def test_damp_layout_rejects_bad_configs(ssq, kw, status):
    base = dict(n_layers=2, n_slots=4, nheads=4, headdim=64, d_state=128, ngroups=2,
                n_protected=16)
    base.update(kw)
    with pytest.raises(ssq.SsqError) as e:
        ssq.ssq_damp_pool_layout(ssq.DampConfig(**base))
    assert e.value.status == status


def test_damp_entry_points_validate_before_launch(ssq):
    lib = ssq.raw()
    cfg = ssq.DampConfig(2, 4, 4, 64, 128, 1, 16)
    P = ctypes.c_void_p
    g = 0x10000000

    def step(pool=g, chan=g, slots=None, batch=2, layer0=0, nl=1, x=g):
        return lib.ssq_damp_decode_step(cfg.ref, P(pool), P(chan), P(slots), batch, layer0, nl,
                                        P(x), P(g), P(g), P(g), P(g), P(g), P(g), None)

    assert step(pool=g + 16) == ssq.SSQ_ERR_ALIGNMENT
    assert step(chan=0) == ssq.SSQ_ERR_INVALID_ARG
    assert step(chan=g + 2) == ssq.SSQ_ERR_ALIGNMENT
    assert step(x=0) == ssq.SSQ_ERR_INVALID_ARG
    assert step(batch=5) == ssq.SSQ_ERR_INVALID_ARG
    assert step(layer0=1, nl=2) == ssq.SSQ_ERR_INVALID_ARG
    assert step(batch=0) == ssq.SSQ_OK
    r = lib.ssq_damp_quantize(cfg.ref, P(g), P(g), None, 2, 0, 1, P(g + 8), None)
    assert r == ssq.SSQ_ERR_ALIGNMENT
    r = lib.ssq_damp_dequantize(cfg.ref, P(g), P(g), None, 2, 0, 3, P(g), None)
    assert r == ssq.SSQ_ERR_INVALID_ARG


def test_damp_codec_round_trip(ssq):
    """The tests' DAMP packer writes and reads back an oracle state exactly
    (host only)."""
    import oracle as O
    from poolcodec import DampCodec
    H, P, N, K = 3, 64, 128, 16
    cfg = ssq.DampConfig(2, 3, H, P, N, 1, K)
    L = ssq.ssq_damp_pool_layout(cfg)
    rng = np.random.default_rng(0)
    chan = np.stack([rng.permutation(N) for _ in range(H)]).astype(np.int32)
    st = O.damp_from_f32(O.DampCfg(H, P, N, 1, K, chan),
                         rng.standard_normal((H, P, N)).astype(np.float32))
    codec = DampCodec(H, P, N, K, L)
    buf = np.zeros(L["pool_bytes"], np.uint8)
    codec.write(buf, 2, 1, st.hi[0], st.q[0], st.delta[0], st.zero[0])
    hi, q, d, z = codec.read(buf, 2, 1)
    assert np.array_equal(hi, st.hi[0]) and np.array_equal(q, st.q[0])
    assert np.array_equal(d, st.delta[0]) and np.array_equal(z, st.zero[0])
    # the block sits where the layout says: nothing else written
    o = L["header_bytes"] + 2 * L["slot_bytes"] + 1 * L["layer_bytes"]
    assert not buf[:o].any() and not buf[o + H * L["head_bytes"]:].any()


def test_binding_constants_match_header(ssq):
    """The binding's copies of the header's constants (error-word bits, pool
    header and alignment, the head limit) equal the header's values."""
    src = open(HEADER).read()
    defs = dict(re.findall(r"#define\s+(SSQ_\w+)\s+(0x[0-9a-fA-F]+|\d+)u?\b", src))
    assert {"SSQ_DEVERR_SLOT", "SSQ_DEVERR_NONFINITE", "SSQ_DEVERR_TIMEOUT",
            "SSQ_DEVERR_CHANNEL", "SSQ_POOL_HEADER_BYTES", "SSQ_POOL_ALIGN",
            "SSQ_MAX_HEADS"} <= set(defs)
    for name, val in defs.items():
        assert getattr(ssq, name) == int(val, 0), name


def test_damp_channel_maps_are_permutations():
    """The seeded channel maps of the DAMP workloads are one permutation of
    0..d_state-1 per (layer, head), reproducible from the seed."""
    from quantized_recurrent_state_mamba_b200 import workloads as W
    c = W.damp_channels(7, 3, 5, 128)
    assert c.shape == (3, 5, 128) and c.dtype == np.int32
    for l in range(3):
        for h in range(5):
            assert np.array_equal(np.sort(c[l, h]), np.arange(128))
    assert np.array_equal(c, W.damp_channels(7, 3, 5, 128))
    assert not np.array_equal(c, W.damp_channels(8, 3, 5, 128))


def test_test_hooks_validate_on_the_host(ssq):
    """The failure-path test hooks are host-only: a negative wait bound is an
    argument error, (0, 0) restores normal behaviour."""
    with pytest.raises(ssq.SsqError):
        ssq.ssq_test_hooks(False, -5)
    ssq.ssq_test_hooks(True, 1000)
    ssq.ssq_test_hooks(False, 0)
