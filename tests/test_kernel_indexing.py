"""Host check of the decode kernel's index arithmetic, before any launch.

The decode kernel (csrc/ssq_decode_impl.cuh) addresses shared memory, tensor
memory and the pool with arithmetic that no GPU run can check for an
out-of-bounds access without risking a fault.  This test restates that
arithmetic on the CPU -- the stage geometry and stage count, the tile walk,
the tensor-copy boxes and their coordinates, the producer's x copies, each
lane's swizzled code address, its metadata, x, B and C reads, its TMEM
columns and the rows it copies back to the pool -- and checks every access
against its buffer for
each shape the tests and the benchmark use.  The pool layout comes from the
library itself (ssq_pool_layout), so global addresses are checked against
the sizes the library allocates.  It also checks the identity the consumer
relies on: a lane's piece sp of its row lies at swizzle(first byte) XOR
(sp * piece bytes).

The constants below mirror the kernel's (16 consumer warps, one row a lane,
512-row tiles, boxes of 128 rows, stage budget, TMEM columns); a change
there must be mirrored here.
"""
import numpy as np
import pytest


@pytest.fixture(scope="module")
def ssq():
    from quantized_recurrent_state_mamba_b200 import build
    build.build()
    from quantized_recurrent_state_mamba_b200 import ssq as m
    return m


C_WARPS = 16
SETS = 1                          # rows per lane in a tile
G_THREADS = C_WARPS * 32          # the consumer threads
BOX_ROWS = 128
MAX_STAGES = 8
SMEM_BUDGET = 226 * 1024          # one CTA per SM
SMEM_LIMIT = 227 * 1024
TMEM_COLS = 512
FMT_BITS = {"i8s": 8, "i8a": 8, "i4s": 4, "i4a": 4}


def r16(v):
    return (v + 15) & ~15


def r256(v):
    return (v + 255) & ~255


def r1024(v):
    return (v + 1023) & ~1023


def swz128(off):
    return off ^ (((off >> 7) & 7) << 4)


def shapes(fmt, N):
    quant = fmt in FMT_BITS
    bits = FMT_BITS.get(fmt, 0)
    EQ = min(N, 128)
    LQ = N // EQ
    EF = min(N, 32)
    LF = N // EF
    return dict(quant=quant, RB=N * bits // 8 if quant else 0,
                CB=EQ * bits // 8 if quant else 16,
                MB=(4 if fmt in ("i8s", "i4s") else 8) if quant else 0,
                FEB=2 if fmt == "bf16" else 4, EQ=EQ, LQ=LQ, EF=EF, LF=LF,
                NP=EQ // 16, PB=(16 * bits // 8) if quant else 4,
                RPTq=G_THREADS * SETS // LQ, RPTf=G_THREADS * SETS // LF)


def geom(S, sh, has_q, has_fp, N, H, G):
    g = {}
    g["x_bytes"] = r1024(max(sh["RPTq"], sh["RPTf"]) * 4)
    g["qcodes"] = r1024(sh["RPTq"] * sh["RB"]) if has_q else 0
    qpay = g["qcodes"] + r16(sh["RPTq"] * sh["MB"]) if has_q else 0
    fpay = sh["RPTf"] * N * sh["FEB"] if has_fp else 0
    g["pay"] = max(qpay, fpay)
    g["stage"] = r1024(g["x_bytes"] + g["pay"])
    g["Hpad"] = (H + 3) & ~3
    g["off_perm"] = 1024
    ub_C = 256 + G * N * 4
    ub_ht = r256(ub_C + G * N * 4)
    ub_gt = ub_ht + g["Hpad"] * 16
    g["unit"] = r256(ub_gt + g["Hpad"] * 4)
    g["off_units"] = r256(g["off_perm"] + g["Hpad"] * 4)
    g["off_stages"] = r1024(g["off_units"] + 2 * g["unit"])
    g["smem"] = g["off_stages"] + S * g["stage"] + 1024
    return g


def plan(sh, has_q, has_fp, N, H, G):
    g = geom(2, sh, has_q, has_fp, N, H, G)
    S = (SMEM_BUDGET - (g["smem"] - 2 * g["stage"])) // g["stage"]
    S = max(2, min(MAX_STAGES, S))
    return S, geom(S, sh, has_q, has_fp, N, H, G)


def check_decode(ssq, fmt, H, P, N, G, n_layers, n_slots, mask=None):
    cfg = ssq.Config(n_layers=n_layers, n_slots=n_slots, nheads=H, headdim=P, d_state=N,
                     ngroups=G, fmt=fmt, head_mask=mask)
    L, perm = ssq.ssq_pool_layout(cfg)
    sh = shapes(fmt, N)
    Hq, Hf = L["n_quant_heads"], L["n_fp_heads"]
    has_q, has_fp = sh["quant"] and Hq > 0, Hf > 0
    S, g = plan(sh, has_q, has_fp, N, H, G)
    assert g["smem"] <= SMEM_LIMIT, (fmt, H, P, N, G, g["smem"])
    assert g["off_stages"] % 1024 == 0 and g["stage"] % 1024 == 0 and g["x_bytes"] % 1024 == 0
    RB, CB, MB, LQ, EQ = sh["RB"], sh["CB"], sh["MB"], sh["LQ"], sh["EQ"]
    gtid = np.arange(G_THREADS)
    if has_q:
        box_lines = (BOX_ROWS * RB + 127) // 128
        region = Hq * P * RB
        lines = (region + 127) // 128
        assert lines * 128 <= L["codes_layer_bytes"]
        assert box_lines <= 256 and (box_lines * 128) % 1024 == 0
        nrows = Hq * P
        for k in range((nrows + sh["RPTq"] - 1) // sh["RPTq"]):
            rbase = k * sh["RPTq"]
            n = min(sh["RPTq"], nrows - rbase)
            assert (rbase * RB) % 128 == 0                     # whole lines
            nbox = (n + BOX_ROWS - 1) // BOX_ROWS
            # tensor-copy destinations inside the codes area
            assert nbox * box_lines * 128 <= g["qcodes"]
            # metadata copy: 16-byte aligned, inside the stage and the pool
            mb = r16(n * MB)
            assert (rbase * MB) % 16 == 0 and mb <= g["pay"] - g["qcodes"]
            assert rbase * MB + mb <= L["meta_layer_bytes"]
            lane, w = gtid % 32, gtid // 32
            RWQ = 32 // LQ
            wrow0 = w * SETS * RWQ                              # the warp's block
            j = lane % LQ
            check_x_copies(rbase, n, P, Hq * P, g)
            for s in range(SETS):
                grow = wrow0 + s * RWQ + lane // LQ
                active = grow < n
                rl = np.where(active, grow, 0)
                hr = (rbase + rl) // P
                assert hr.max() < Hq and hr.max() < g["Hpad"]
                cs0 = g["x_bytes"] + grow * RB + j * CB
                lane_base = swz128(cs0)
                for sp in range(sh["NP"]):
                    a = lane_base ^ (sp * sh["PB"])
                    assert np.array_equal(a, swz128(cs0 + sp * sh["PB"])), "piece address identity"
                    assert a.min() >= g["x_bytes"]
                    assert (a + sh["PB"]).max() <= g["x_bytes"] + g["qcodes"]
                    # B / C entries of the piece (group offset + lane offset)
                    assert (j * EQ + sp * 16 + 16).max() <= N
                ms = g["x_bytes"] + g["qcodes"] + grow * MB
                assert (ms + MB).max() <= g["stage"]
                assert (grow * 4 + 4).max() <= g["x_bytes"]           # x of the row
                # TMEM: warp w's lane quarter w % 4, columns 128 SETS (w // 4)
                # + 128 s, EQ of them used
                assert ((w // 4) * 128 * SETS + 128 * s + EQ).max() <= TMEM_COLS and EQ <= 128
            # the rows of the warps' blocks cover the tile once
            rows = np.sort(np.concatenate([(wrow0 + s * RWQ + lane // LQ)[j == 0]
                                           for s in range(SETS)]))
            assert np.array_equal(rows, np.arange(sh["RPTq"]))
            # copy-back of each warp's block: 16-byte chunk c = lane + 32 i,
            # read at A[i & 1] + 512 i with A[0] the swizzled first chunk of
            # the lane and A[1] = A[0] ^ 64
            WB = SETS * RWQ * RB
            WCH = WB // 16
            wrows = np.clip(n - wrow0, 0, SETS * RWQ)
            cl = g["x_bytes"] + wrow0 * RB + 16 * lane
            a0 = swz128(cl)
            a1 = a0 ^ 64
            for i in range((WCH + 31) // 32):
                c = lane + 32 * i
                addr = np.where(i & 1, a1, a0) + 512 * i
                live = 16 * c < wrows * RB
                full = (wrows == SETS * RWQ) & (WCH % 32 == 0)
                read = live | full
                assert np.array_equal(addr[read], swz128(cl + 512 * i)[read]), "copy-back address"
                assert (addr[read] + 16).max(initial=0) <= g["x_bytes"] + g["qcodes"]
                glob = (rbase + wrow0) * RB + 16 * c + 16
                assert np.all(glob[read] <= region)
    if has_fp:
        EF, LF, FEB = sh["EF"], sh["LF"], sh["FEB"]
        nrows = Hf * P
        for k in range((nrows + sh["RPTf"] - 1) // sh["RPTf"]):
            rbase = k * sh["RPTf"]
            n = min(sh["RPTf"], nrows - rbase)
            check_x_copies(rbase, n, P, Hf * P, g)
            assert n * N * FEB <= g["pay"] and (rbase * N * FEB) % 16 == 0
            assert (rbase + n) * N * FEB <= L["fp_layer_bytes"]
            grows = np.concatenate([s * (G_THREADS // LF) + gtid // LF for s in range(SETS)])
            assert np.array_equal(np.sort(grows[np.tile(gtid % LF, SETS) == 0]),
                                  np.arange(sh["RPTf"]))
            assert (grows * 4 + 4).max() <= g["x_bytes"]
            j = gtid % LF
            epc = 16 // FEB
            for c in range(EF // epc):
                m = LF * c + j
                assert ((m + 1) * 16).max() <= N * FEB               # inside the row
    return S, g


def check_x_copies(rbase, n, P, nrows, g):
    """The producer's x copies of a tile: one bulk copy per head the tile's
    rows fall in (when head_dim is a multiple of 4), each 16-byte aligned at
    both ends, a multiple of 16 bytes, inside the stage's x area and the
    head's x, together covering the tile's rows once."""
    if P % 4:
        return
    assert rbase % 4 == 0 and n % 4 == 0 and nrows % 4 == 0
    h0, h1 = rbase // P, (rbase + n - 1) // P
    covered = 0
    for hr in range(h0, h1 + 1):
        r0, r1 = max(rbase, hr * P), min(rbase + n, (hr + 1) * P)
        assert r1 > r0
        dst, src, size = 4 * (r0 - rbase), 4 * (r0 - hr * P), 4 * (r1 - r0)
        assert dst % 16 == 0 and src % 16 == 0 and size % 16 == 0
        assert dst + size <= g["x_bytes"] and src + size <= 4 * P
        covered += r1 - r0
    assert covered == n


TEST_SHAPES = [
    # the GPU parity tests' shapes (several tiles, ragged tails, groups, masks)
    (fmt, 6, 24, N, 3, 3, 5) for fmt in ("f32", "bf16", "i8s", "i8a", "i4s", "i4a")
    for N in (16, 64, 128)
] + [
    ("i8a", 2, 8, 16, 1, 1, 1),                   # tiny
    ("i8a", 24, 64, 128, 1, 24, 256),             # 130M decode
    ("i4a", 32, 64, 128, 1, 1, 8),                # 370M (decode of its pool)
    ("i8a", 128, 64, 128, 8, 1, 256),             # 8B
    ("i8s", 128, 64, 128, 8, 1, 64),
    ("f32", 128, 64, 128, 8, 1, 64),
    ("i8a", 32, 128, 128, 1, 30, 256),            # serving sweep
    ("i4a", 32, 128, 128, 1, 30, 256),
    ("bf16", 32, 128, 128, 1, 30, 256),
    ("i8a", 4, 64, 256, 2, 2, 3),                 # d_state 256: two lanes a row
    ("i4s", 4, 64, 256, 2, 2, 3),
    ("i8a", 5, 7, 32, 5, 1, 2),                   # odd head_dim
]


@pytest.mark.parametrize("fmt,H,P,N,G,L,slots", TEST_SHAPES)
def test_decode_indexing_in_bounds(ssq, fmt, H, P, N, G, L, slots):
    check_decode(ssq, fmt, H, P, N, G, L, slots)


@pytest.mark.parametrize("fmt", ["i8a", "i4a"])
def test_decode_indexing_masked_pool(ssq, fmt):
    """A mid-band mask: a quantized region and an fp region per layer."""
    from quantized_recurrent_state_mamba_b200 import workloads as W
    check_decode(ssq, fmt, 32, 64, 128, 1, 1, 8, W.mid_band_mask(32))


def test_swizzle_is_a_permutation_of_chunks():
    """The 128-byte swizzle permutes the 16-byte chunks of every 1024-byte
    block and leaves the byte within a chunk alone."""
    off = np.arange(4096)
    s = swz128(off)
    assert np.array_equal(s & 15, off & 15)
    assert np.array_equal(s >> 10, off >> 10)
    for blk in range(4):
        chunks = s[blk * 1024:(blk + 1) * 1024:16] >> 4
        assert sorted(chunks) == list(range(blk * 64, blk * 64 + 64))


def test_lanes_of_a_quarter_warp_hit_distinct_banks():
    """Eight consecutive lanes reading the same logical chunk of their rows
    (one row each, rows of 128 or 64 bytes) touch eight distinct 16-byte bank
    groups: the conflict-free read the swizzle is there for."""
    for RB, CB in ((128, 128), (64, 64)):
        for c in range(CB // 16):
            for q0 in range(0, 32, 8):
                lanes = np.arange(q0, q0 + 8)
                a = swz128(1024 + lanes * RB) ^ (c * 16)
                assert len(set(((a >> 4) & 7).tolist())) == 8, (RB, c, q0)
