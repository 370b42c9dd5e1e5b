// ssq_decode_impl.cuh -- the fused decode-step kernel (instantiated per state
// format in ssq_decode_<format>.cu; dispatched from ssq_decode.cu).
//
// One launch updates the state of nl layers x batch requests by one token:
// read the packed row, decode, apply the recurrence in fp32, refit the row
// scale, requantize, write the packed row and its metadata back, and read y
// from the newly stored row: one kernel does all of it, as "Mamba state
// quantization for inference" ("Mixed precision spends bits on persistent
// channels") lays out for a low-bit state (decode, fp32 update, new scale,
// packed write-back in one pass), with the quantizer of
// "ssm-state-quantization" README, Setup.
//
// Structure (persistent, warp-specialised, one CTA of 17 warps per SM):
//   - work is a sequence of tiles (up to 512 rows of the quantized region, or
//     128 fp rows at d_state 128, of one (layer, request)); each CTA owns a
//     contiguous range of that sequence;
//   - a producer warp streams each tile into a ring of shared-memory stages:
//     the packed codes with tensor copies (TMA, cp.async.bulk.tensor) laid
//     out in the 128-byte swizzle, so that the lanes of a warp, one row each,
//     read the same logical 16-byte chunk of their rows from distinct banks;
//     the metadata and fp rows with bulk copies; x with one bulk copy per
//     head the tile touches (cp.async per row when head_dim is not a
//     multiple of 4).  Once per (layer, request, region) "unit" it stages B
//     and C and builds a head table (lambda, dt, D, the y offset and the B/C
//     group of every head), reading the head order from shared memory;
//   - 16 consumer warps share each tile, 32 rows a warp.  A lane owns a
//     quantized row (two lanes at d_state 256): all lanes of a warp
//     walk their rows' entries in the same order, so B and C come from
//     shared memory as warp-wide broadcasts.  The updated row waits in the
//     warp's columns of tensor memory (TMEM, tcgen05.st / tcgen05.ld)
//     between the min/max pass and the rounding pass (the refit runs while
//     the stores complete; the rounding pass keeps the next piece's load in
//     flight), which keeps the kernel within the 96 registers a thread that
//     17 warps leave (the sub-partition holding the producer has 5 of them);
//   - a warp writes its rows' new codes back into the stage, in place, and
//     then copies its 32 rows from the stage to the pool with 16-byte stores
//     in row-major order (8 lanes per 128-byte line: every store instruction
//     writes whole lines); each row's metadata is stored straight from the
//     row's lane.  The producer only loads: no write-back is queued behind a
//     refill;
//   - fp rows (the fp32 / bf16 formats and the unmasked heads of the integer
//     formats) are streamed by N/32 lanes of 32 entries and stored straight
//     to global memory;
//   - every wait is bounded: one that runs out sets SSQ_DEVERR_TIMEOUT in the
//     pool's error word and the CTA winds down (the producer first waits for
//     its own copies in flight; TMEM is released on every path).
//
// The same kernel, in its diagnostics mode, evaluates the step a decode would
// take and writes per-row figures instead of the new state
// ("ssm-state-quantization" README, Findings 4 and 5): the pool is only
// read.
#pragma once

#include "ssq_common.cuh"
#include "ssq_params.h"
#include "ssq_pipe.cuh"

#include <cuda.h>
#include <cudaTypedefs.h>

#include <cstring>
#include <type_traits>
#include <utility>

namespace ssq {

namespace {

// Consumer warps.  All 16 share each 512-row tile: with two or four groups
// of warps on smaller tiles the single producer warp could not prepare tiles
// as fast as the consumers took them.
constexpr int kCWarps = 16;
constexpr int kCThreads = kCWarps * 32;
constexpr int kDThreads = kCThreads + 32;   // + 1 producer warp
constexpr int kMaxStages = 8;
constexpr int kBoxRows = 128;               // rows per tensor copy
constexpr unsigned kTmemCols = 512;         // all of TMEM: 128 columns per consumer warp

// ---- PTX wrappers: shared memory at 32-bit addresses --------------------
// Loads of data that stays put while it is read (a landed stage, the unit
// buffer): plain asm, free for the compiler to schedule.  Their addresses
// come from laundered bases (launder() after the wait that makes the data
// visible), so no load can be placed before that wait.
template <int OFF>
__device__ __forceinline__ uint4 lds128(unsigned a)
{
    uint4 v;
    asm("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4+%5];"
        : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(a), "n"(OFF));
    return v;
}
template <int OFF>
__device__ __forceinline__ uint2 lds64(unsigned a)
{
    uint2 v;
    asm("ld.shared.v2.b32 {%0, %1}, [%2+%3];" : "=r"(v.x), "=r"(v.y) : "r"(a), "n"(OFF));
    return v;
}
template <int OFF>
__device__ __forceinline__ float4 lds128f(unsigned a)
{
    float4 v;
    asm("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4+%5];"
        : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w) : "r"(a), "n"(OFF));
    return v;
}
__device__ __forceinline__ uint32_t lds32(unsigned a)
{
    uint32_t v;
    asm("ld.shared.b32 %0, [%1];" : "=r"(v) : "r"(a));
    return v;
}
// A load kept in program order with the shared-memory stores around it (the
// warp reading back what its lanes just wrote).
template <int OFF>
__device__ __forceinline__ uint4 lds128_ordered(unsigned a)
{
    uint4 v;
    asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4+%5];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(a), "n"(OFF) : "memory");
    return v;
}
template <int OFF>
__device__ __forceinline__ float4 lds128f_ordered(unsigned a)
{
    float4 v;
    asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4+%5];"
                 : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w) : "r"(a), "n"(OFF) : "memory");
    return v;
}
// A shared-memory address that the compiler sees as produced here: loads
// from it cannot be moved above this point (a wait before it).
__device__ __forceinline__ unsigned launder(unsigned a)
{
    unsigned r;
    asm volatile("mov.b32 %0, %1;" : "=r"(r) : "r"(a) : "memory");
    return r;
}
// Stores predicated inside the instruction, so the warp stays converged
// around the tcgen05 instructions that follow.
__device__ __forceinline__ void sts128u_if(unsigned a, uint4 v, bool pred)
{
    asm volatile("{\n .reg .pred p;\n setp.ne.u32 p, %5, 0;\n"
                 " @p st.shared.v4.b32 [%0], {%1, %2, %3, %4};\n}\n"
                 :: "r"(a), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w), "r"((unsigned)pred)
                 : "memory");
}
__device__ __forceinline__ void sts64u_if(unsigned a, uint2 v, bool pred)
{
    asm volatile("{\n .reg .pred p;\n setp.ne.u32 p, %3, 0;\n"
                 " @p st.shared.v2.b32 [%0], {%1, %2};\n}\n"
                 :: "r"(a), "r"(v.x), "r"(v.y), "r"((unsigned)pred) : "memory");
}

// ---- tensor copies (TMA) -------------------------------------------------
// Codes of a pool as a 4-d tensor of bytes: [slot][layer][line][128], a line
// being 128 bytes of a layer's code region.  The innermost coordinate is
// always 0.
__device__ __forceinline__ void tma_load_codes(void* dst, const CUtensorMap* map, int line,
                                               int layer, int slot, uint64_t* bar)
{
    asm volatile(
        "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3, %4, %5}], [%6];"
        :: "r"(saddr(dst)), "l"(map), "r"(0), "r"(line), "r"(layer), "r"(slot), "r"(saddr(bar))
        : "memory");
}
__device__ __forceinline__ void tma_prefetch_codes(const CUtensorMap* map, int line, int layer,
                                                   int slot)
{
    asm volatile(
        "cp.async.bulk.prefetch.tensor.4d.L2.global.tile [%0, {%1, %2, %3, %4}];"
        :: "l"(map), "r"(0), "r"(line), "r"(layer), "r"(slot) : "memory");
}

// The 128-byte swizzle of the tensor copies: the 16-byte chunk index of a
// shared-memory offset (bits 4..6) is XORed with its 128-byte line index
// (bits 7..9); offsets are from a 1024-byte aligned base.
__host__ __device__ inline unsigned swz128(unsigned off)
{
    return off ^ (((off >> 7) & 7u) << 4);
}

// ---- tensor memory (tcgen05) ---------------------------------------------
__device__ __forceinline__ void tmem_alloc(uint32_t* dst, unsigned ncols)
{
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                 :: "r"(saddr(dst)), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tmem_relinquish()
{
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, unsigned ncols)
{
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;"
                 :: "r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before()
{
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after()
{
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
// 16 fp32 values of this lane into 16 consecutive columns of its TMEM lane.
// (TMEM is not memory the compiler tracks: the tcgen05 wrappers are volatile,
// which keeps them in program order with one another, without a memory
// clobber, which leaves shared-memory loads free to move around them.)
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const float (&v)[16])
{
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10,"
        " %11, %12, %13, %14, %15, %16};"
        :: "r"(taddr), "f"(v[0]), "f"(v[1]), "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]),
           "f"(v[6]), "f"(v[7]), "f"(v[8]), "f"(v[9]), "f"(v[10]), "f"(v[11]), "f"(v[12]),
           "f"(v[13]), "f"(v[14]), "f"(v[15]));
}
__device__ __forceinline__ void tmem_wait_st()
{
    asm volatile("tcgen05.wait::st.sync.aligned;");
}
// ... and back.  The registers are written asynchronously until
// tmem_wait_ld(v), which takes them as operands: every use of v follows it.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&v)[16])
{
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10,"
        " %11, %12, %13, %14, %15}, [%16];"
        : "=f"(v[0]), "=f"(v[1]), "=f"(v[2]), "=f"(v[3]), "=f"(v[4]), "=f"(v[5]), "=f"(v[6]),
          "=f"(v[7]), "=f"(v[8]), "=f"(v[9]), "=f"(v[10]), "=f"(v[11]), "=f"(v[12]),
          "=f"(v[13]), "=f"(v[14]), "=f"(v[15])
        : "r"(taddr));
}
__device__ __forceinline__ void tmem_wait_ld(float (&v)[16])
{
    asm volatile("tcgen05.wait::ld.sync.aligned;"
                 : "+f"(v[0]), "+f"(v[1]), "+f"(v[2]), "+f"(v[3]), "+f"(v[4]), "+f"(v[5]),
                   "+f"(v[6]), "+f"(v[7]), "+f"(v[8]), "+f"(v[9]), "+f"(v[10]), "+f"(v[11]),
                   "+f"(v[12]), "+f"(v[13]), "+f"(v[14]), "+f"(v[15]));
}

// f(std::integral_constant<int, i>) for i = 0 .. N-1, unrolled.
template <typename Fn, int... I>
__device__ __forceinline__ void static_for_seq(Fn&& f, std::integer_sequence<int, I...>)
{
    (f(std::integral_constant<int, I>{}), ...);
}
template <int N, typename Fn>
__device__ __forceinline__ void static_for(Fn&& f)
{
    static_for_seq(f, std::make_integer_sequence<int, N>{});
}

// f(v, piece) for the NP 16-column pieces of this lane's TMEM row.  With
// PIPE the load of piece sp + 1 is in flight while f works on piece sp (16
// more registers); without, each load is waited for at once.
template <int NP, bool PIPE, typename Fn>
__device__ __forceinline__ void tmem_pieces(uint32_t tm, Fn&& f)
{
    if constexpr (PIPE) {
        float va[16], vb[16];
        tmem_ld16(tm, va);
        tmem_wait_ld(va);
        static_for<NP>([&](auto spc) {
            constexpr int sp = decltype(spc)::value;
            if constexpr (sp % 2 == 0) {
                if constexpr (sp + 1 < NP) tmem_ld16(tm + 16 * (sp + 1), vb);
                f(va, spc);
                if constexpr (sp + 1 < NP) tmem_wait_ld(vb);
            } else {
                if constexpr (sp + 1 < NP) tmem_ld16(tm + 16 * (sp + 1), va);
                f(vb, spc);
                if constexpr (sp + 1 < NP) tmem_wait_ld(va);
            }
        });
    } else {
        static_for<NP>([&](auto spc) {
            constexpr int sp = decltype(spc)::value;
            float v[16];
            tmem_ld16(tm + 16 * sp, v);
            tmem_wait_ld(v);
            f(v, spc);
        });
    }
}

// Named barrier of the consumer warps (the producer does not take part).
__device__ __forceinline__ void consumers_sync()
{
    asm volatile("bar.sync 1, %0;" :: "n"(kCThreads) : "memory");
}

__host__ __device__ inline int r16(int v) { return (v + 15) & ~15; }
__host__ __device__ inline int r256(int v) { return (v + 255) & ~255; }
__host__ __device__ inline int r1024(int v) { return (v + 1023) & ~1023; }

// ---- tile sequence -----------------------------------------------------
// Tiles are ordered (layer, request, region, row block).  Every warp walks
// the CTA's contiguous range of them with counters (one division at the
// start); the tiles loaded into the ring are numbered in that order, and
// loaded tile k goes to stage k % S.
struct TileWalk {
    long long lb;   // layer * batch + request
    int l, b, k;    // k: tile within (layer, request)
    bool quant;
    int rbase, n;   // first region row, rows in this tile

    __device__ __forceinline__ void fill(int Hq, int Hf, int P, const CallView& cv)
    {
        quant = k < cv.qtiles;
        const int rpt = quant ? cv.rows_per_tile : cv.rows_per_tile_f;
        rbase = (quant ? k : k - cv.qtiles) * rpt;
        const int nrows = (quant ? Hq : Hf) * P;
        n = min(rpt, nrows - rbase);
    }
    __device__ __forceinline__ void start(int Hq, int Hf, int P, const CallView& cv, long long t)
    {
        const int per_lb = cv.qtiles + cv.ftiles;
        lb = t / per_lb;
        k = (int)(t - lb * per_lb);
        l = (int)(lb / cv.batch);
        b = (int)(lb - (long long)l * cv.batch);
        fill(Hq, Hf, P, cv);
    }
    // Advance; true when the next tile starts a new unit.
    __device__ __forceinline__ bool next(int Hq, int Hf, int P, const CallView& cv)
    {
        const bool was_quant = quant;
        if (++k == cv.qtiles + cv.ftiles) {
            k = 0;
            ++lb;
            if (++b == cv.batch) {
                b = 0;
                ++l;
            }
            fill(Hq, Hf, P, cv);
            return true;
        }
        fill(Hq, Hf, P, cv);
        return quant != was_quant;
    }
};

// ---- shared-memory geometry (host and device agree on it) --------------
// Head order:  [H ints] (quantized heads first), after the barriers
// Unit buffer: [256 B header: slot, bad][B: G*N f32][C: G*N f32]
//              [head table: Hpad x float4 {lambda, dt, D, y offset}]
//              [group table: Hpad x int (g*N)]
// Stage:       [x: RPT f32, padded to 1024 B]
//              [codes: RPTq*RB bytes, swizzled, padded to 1024 B][meta: RPTq*MB]
//           or [x][fp rows: RPTf*N elements]
struct DecodeGeom {
    int S;            // stages
    int RPTq, RPTf;   // rows per tile in the quantized / fp region
    int x_bytes;      // x area of a stage (a multiple of 1024)
    int qcodes_bytes; // codes area of a quantized tile (a multiple of 1024)
    int pay_bytes;    // payload area of a stage
    int stage_bytes;
    int ub_B, ub_C, ub_ht, ub_gt, unit_bytes;  // unit buffer layout
    int Hpad;
    int off_perm, off_units, off_stages, smem_bytes;
};

// Offsets are from a 1024-byte aligned base inside the dynamic shared memory
// (the launch adds 1024 bytes of slack); every stage and its codes area start
// on a 1024-byte boundary (the 128-byte swizzle repeats every 1024 bytes).
__host__ __device__ inline DecodeGeom decode_geom(int S, int RPTq, int RPTf, int RB, int MB,
                                                  int fpEB, bool has_q, bool has_fp, int N,
                                                  int H, int G)
{
    DecodeGeom g;
    g.S = S;
    g.RPTq = RPTq;
    g.RPTf = RPTf;
    g.x_bytes = r1024((RPTq > RPTf ? RPTq : RPTf) * 4);
    g.qcodes_bytes = has_q ? r1024(RPTq * RB) : 0;
    const int qpay = has_q ? g.qcodes_bytes + r16(RPTq * MB) : 0;
    const int fpay = has_fp ? RPTf * N * fpEB : 0;
    g.pay_bytes = qpay > fpay ? qpay : fpay;
    g.stage_bytes = r1024(g.x_bytes + g.pay_bytes);
    g.Hpad = (H + 3) & ~3;
    g.ub_B = 256;                      // [0, 16): slot, bad flag
    g.ub_C = g.ub_B + G * N * 4;
    g.ub_ht = r256(g.ub_C + G * N * 4);
    g.ub_gt = g.ub_ht + g.Hpad * 16;
    g.unit_bytes = r256(g.ub_gt + g.Hpad * 4);
    g.off_perm = 1024;                 // barriers and the TMEM address before it
    g.off_units = r256(g.off_perm + g.Hpad * 4);
    g.off_stages = r1024(g.off_units + 2 * g.unit_bytes);
    g.smem_bytes = g.off_stages + S * g.stage_bytes + 1024;
    return g;
}

// Lane shapes.  A quantized row is held by one lane (two at d_state 256):
// up to 128 entries, streamed in pieces of 16.  An fp row is streamed by
// N/32 lanes of 32 entries.
constexpr int kQuantE = 128;
template <int N>
struct QShape {
    static constexpr int E = N >= kQuantE ? kQuantE : N;
    static constexpr int LPR = N / E;
    static constexpr int RPT = kCThreads / LPR;   // rows per tile
};
template <int N>
struct FShape {
    static constexpr int E = N >= 32 ? 32 : N;
    static constexpr int LPR = N / E;
    static constexpr int RPT = kCThreads / LPR;
};

// A whole quantized row by the formulas verbatim (every fp32 operation one
// IEEE rounding in the order of the definition), for warps where some row
// falls outside the magic-number paths: a zero point or scaled values of
// 2^22 or more in magnitude (rows far from zero relative to their range).
// Every lane of the warp calls it together (the row reductions are
// shuffles).  Codes are read from and written to the stage at their
// swizzled places (cs0: the lane's first code byte as an unswizzled offset
// from the 1024-aligned stage base sb); B and C in natural order; mrow is
// the row's metadata in the pool.
template <int FMT, int N, bool SR>
__device__ __noinline__ float row_exact(uint8_t* __restrict__ sb, unsigned cs0, float delta0,
                                        float z0, float lam, float dtx,
                                        const float* __restrict__ gB,
                                        const float* __restrict__ gC, int j, bool active,
                                        uint8_t* __restrict__ mrow, uint32_t* err, SrKey srk)
{
    using F = Fmt<FMT>;
    constexpr int E = QShape<N>::E, LPR = QShape<N>::LPR;
    constexpr int CB = E * F::bits / 8;
    float s[E];
    float lo = 0.0f, hi = 0.0f;
#pragma unroll 1
    for (int n = 0; n < E; ++n) {
        int q;
        if constexpr (F::bits == 8) {
            const uint32_t bb = sb[swz128(cs0 + n)];
            q = F::sym ? (int)(int8_t)bb : (int)bb;
        } else {
            const uint32_t bb = (sb[swz128(cs0 + n / 2)] >> (4 * (n % 2))) & 0xFu;
            q = F::sym ? (int)((bb ^ 8u) - 8u) : (int)bb;
        }
        const float v = __fmul_rn(__fsub_rn((float)q, z0), delta0);
        const float w = __fmul_rn(dtx, gB[j * E + n]);
        const float sv = __fmaf_rn(lam, v, w);
        s[n] = sv;
        lo = n == 0 ? sv : fminf(lo, sv);
        hi = n == 0 ? sv : fmaxf(hi, sv);
    }
    const RowParams rp = refit_from_minmax<FMT, LPR>(lo, hi);
    float acc = 0.0f;
    uint32_t words[CB / 4 > 0 ? CB / 4 : 1];
#pragma unroll
    for (int i = 0; i < (CB / 4 > 0 ? CB / 4 : 1); ++i) words[i] = 0u;
#pragma unroll 1
    for (int n = 0; n < E; ++n) {
        float c, r;
        if constexpr (SR) {
            const int ng = j * E + n;                   // entry within the row
            const uint4 w = philox4x32_10(
                make_uint4(srk.row_block + (uint32_t)(ng / 8), srk.layer, srk.slot, srk.step),
                srk.key);
            const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
            const uint32_t d = (ww[(ng % 8) / 2] >> (16 * (ng % 2))) & 0xFFFFu;
            c = round1_sr_exact<FMT>(s[n], rp.inv, rp.z, (float)d * (1.0f / 65536.0f), &r);
        } else {
            const float rr = rint_prod(s[n], rp.inv);
            if constexpr (F::sym) {
                c = fminf(fmaxf(rr, -F::qmax), F::qmax);
                r = c;
            } else {
                c = fminf(__fadd_rn(rr, rp.z), F::qmax);
                r = __fsub_rn(c, rp.z);
            }
        }
        const uint32_t code = (uint32_t)(int)c & ((1u << F::bits) - 1u);
        words[n * F::bits / 32] |= code << ((n * F::bits) % 32);
        acc = __fmaf_rn(gC[j * E + n], __fmul_rn(r, rp.delta), acc);
    }
    const float ysum = grp_sum<LPR>(acc);
    if (active) {
#pragma unroll
        for (int i = 0; i < CB / 4; ++i)
            *reinterpret_cast<uint32_t*>(sb + swz128(cs0 + 4 * i)) = words[i];
        if (j == 0) {
            if constexpr (F::sym) {
                __stcs(reinterpret_cast<float*>(mrow), rp.delta);
            } else {
                __stcs(reinterpret_cast<float2*>(mrow), make_float2(rp.delta, rp.z));
            }
            if (!rp.finite) atomicOr(err, SSQ_DEVERR_NONFINITE);
        }
    }
    return ysum;
}

// The diagnostics of a whole quantized row by the formulas verbatim (the
// warps where some row falls outside the magic-number paths): the step the
// decode would take, and per row {reversals, sum over reversed entries of
// C e, sum of C e, sum of C s'}, e = fl(deq - s') the rounding error and an
// entry reversed when w != 0 and fl(e + w) has the other sign than w.
// Every lane of the warp calls it together.
template <int FMT, int N>
__device__ __noinline__ float4 row_exact_diag(const uint8_t* __restrict__ sb, unsigned cs0,
                                              float delta0, float z0, float lam, float dtx,
                                              const float* __restrict__ gB,
                                              const float* __restrict__ gC, int j)
{
    using F = Fmt<FMT>;
    constexpr int E = QShape<N>::E, LPR = QShape<N>::LPR;
    float s[E];
    float lo = 0.0f, hi = 0.0f;
#pragma unroll 1
    for (int n = 0; n < E; ++n) {
        int q;
        if constexpr (F::bits == 8) {
            const uint32_t bb = sb[swz128(cs0 + n)];
            q = F::sym ? (int)(int8_t)bb : (int)bb;
        } else {
            const uint32_t bb = (sb[swz128(cs0 + n / 2)] >> (4 * (n % 2))) & 0xFu;
            q = F::sym ? (int)((bb ^ 8u) - 8u) : (int)bb;
        }
        const float v = __fmul_rn(__fsub_rn((float)q, z0), delta0);
        const float sv = __fmaf_rn(lam, v, __fmul_rn(dtx, gB[j * E + n]));
        s[n] = sv;
        lo = n == 0 ? sv : fminf(lo, sv);
        hi = n == 0 ? sv : fmaxf(hi, sv);
    }
    const RowParams rp = refit_from_minmax<FMT, LPR>(lo, hi);
    float rev = 0.0f, rev_err = 0.0f, tot = 0.0f, sig = 0.0f;
#pragma unroll 1
    for (int n = 0; n < E; ++n) {
        const float rr = rint_prod(s[n], rp.inv);
        float r;
        if constexpr (F::sym) {
            r = fminf(fmaxf(rr, -F::qmax), F::qmax);
        } else {
            r = __fsub_rn(fminf(__fadd_rn(rr, rp.z), F::qmax), rp.z);
        }
        const float w = __fmul_rn(dtx, gB[j * E + n]);
        const float e = __fsub_rn(__fmul_rn(r, rp.delta), s[n]);
        const float inc = __fadd_rn(e, w);
        const float c = gC[j * E + n];
        sig = __fmaf_rn(c, s[n], sig);
        tot = __fmaf_rn(c, e, tot);
        if ((w > 0.0f && inc < 0.0f) || (w < 0.0f && inc > 0.0f)) {
            rev += 1.0f;
            rev_err = __fmaf_rn(c, e, rev_err);
        }
    }
    return make_float4(grp_sum<LPR>(rev), grp_sum<LPR>(rev_err), grp_sum<LPR>(tot),
                       grp_sum<LPR>(sig));
}

struct CodesMap {
    CUtensorMap map;   // 64-byte aligned inside the kernel parameters
};

// Modes of the kernel: the decode step with nearest rounding, with
// stochastic rounding (draws keyed by cv.sr_seed and countered by row block,
// layer, slot and cv.sr_step), or its diagnostics (written to cv.diag; the
// pool is only read).
enum { kNearest = 0, kStochastic = 1, kDiagnostics = 2 };

template <int FMT, int N, int MODE>
__global__ void __launch_bounds__(kDThreads, 1)
decode_kernel(const __grid_constant__ PoolView pv, const __grid_constant__ CallView cv,
              const __grid_constant__ DecodeGeom geo, const __grid_constant__ CodesMap cm)
{
    using F = Fmt<FMT>;
    constexpr bool SR = MODE == kStochastic;
    constexpr bool DIAG = MODE == kDiagnostics;
    // quantized rows: EQ entries per lane, LQ lanes per row; fp rows: EF, LF
    constexpr int EQ = QShape<N>::E, LQ = QShape<N>::LPR;
    constexpr int EF = FShape<N>::E, LF = FShape<N>::LPR;
    constexpr bool kBf16 = (FMT == SSQ_BF16);
    constexpr int RB = F::quant ? N * F::bits / 8 : 0;      // code bytes per row
    constexpr int CB = F::quant ? EQ * F::bits / 8 : 16;    // code bytes per lane
    constexpr int MB = F::meta_bytes;
    constexpr int FEB = kBf16 ? 2 : 4;                       // fp element bytes
    constexpr int NP = EQ / 16;                              // 16-entry pieces per lane
    constexpr int PW = F::quant ? Piece<FMT>::words : 1;     // code words per piece
    constexpr int PB = PW * 4;                               // code bytes per piece
    constexpr int kBoxLines = F::quant ? (kBoxRows * RB + 127) / 128 : 1;
    constexpr int kBoxes = F::quant ? (QShape<N>::RPT + kBoxRows - 1) / kBoxRows : 1;

    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* const smem = smem_raw + ((1024u - (saddr(smem_raw) & 1023u)) & 1023u);
    uint64_t* full = reinterpret_cast<uint64_t*>(smem);
    uint64_t* empty = full + kMaxStages;
    uint64_t* ufull = empty + kMaxStages;
    uint64_t* uempty = ufull + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(uempty + 2);
    int* const sperm = reinterpret_cast<int*>(smem + geo.off_perm);
    uint32_t* err = reinterpret_cast<uint32_t*>(pv.pool);

    const int S = geo.S;
    const int H = pv.H, P = pv.P, G = pv.G, Hq = pv.Hq, Hf = pv.Hf;
    const long long wlim = cv.wait_limit > 0 ? cv.wait_limit : kWaitLimit;
    const long long total = cv.total_tiles;
    const long long t0 = total * blockIdx.x / gridDim.x;
    const long long t1 = total * (blockIdx.x + 1) / gridDim.x;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const bool use_tmem = F::quant && Hq > 0;

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kCWarps);
        }
        for (int u = 0; u < 2; ++u) {
            mbar_init(&ufull[u], 1);
            mbar_init(&uempty[u], kCWarps);
        }
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    // the head order (quantized heads first) in shared memory, for the producer
    for (int h = threadIdx.x; h < H; h += kDThreads) sperm[h] = pv.perm[h];
    if (use_tmem && warp == 0) {
        tmem_alloc(tmem_slot, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    uint8_t* const units = smem + geo.off_units;
    uint8_t* const stages = smem + geo.off_stages;

    if (warp == kCWarps) {
        // ================= producer warp =================
        int k = 0, uk = -1;
        int si = 0;          // stage of loaded tile k
        unsigned eph = 0;    // parity of the release of that stage's previous tile
        bool bad = false, ok = true, newunit = true;
        int cur_slot = 0, cur_layer = 0;
        const uint8_t* meta_u = nullptr;
        const uint8_t* fp_u = nullptr;
        const float* x_u = nullptr;
        // x of a tile by bulk copies, one per head the tile touches, when
        // every copy is 16-byte aligned (head_dim a multiple of 4, x aligned);
        // else one 4-byte cp.async per row
        const bool x_bulk = (P & 3) == 0 && (reinterpret_cast<uintptr_t>(cv.x) & 15) == 0;
        TileWalk ti;
        ti.start(Hq, Hf, P, cv, t0);
        for (long long t = t0; t < t1; ++t, newunit = ti.next(Hq, Hf, P, cv)) {
            const int regbase = ti.quant ? 0 : Hq;
            if (newunit) {
                ++uk;
                const int u = uk & 1;
                if (!mbar_wait_suspend(&uempty[u], ((uk >> 1) & 1) ^ 1, wlim)) { ok = false; break; }
                const int slot = cv.slot_idx ? __ldg(cv.slot_idx + ti.b) : ti.b;
                bad = slot < 0 || slot >= pv.n_slots;
                uint8_t* ub = units + u * geo.unit_bytes;
                cur_slot = slot;
                cur_layer = cv.layer0 + ti.l;
                if (!bad) {
                    const uint8_t* sb = pv.pool + pv.header_bytes + (long long)slot * pv.slot_bytes;
                    meta_u = sb + pv.meta_off + (long long)cur_layer * pv.meta_layer_bytes;
                    fp_u = sb + pv.fp_off + (long long)cur_layer * pv.fp_layer_bytes;
                    x_u = cv.x + ti.lb * H * P;
                    // head table of the region: lambda = exp(dt*A) once per
                    // head, dt, D, the head's y offset and B/C group
                    float4* ht = reinterpret_cast<float4*>(ub + geo.ub_ht);
                    int* gtab = reinterpret_cast<int*>(ub + geo.ub_gt);
                    const int nreg = ti.quant ? Hq : Hf;
                    for (int hr = lane; hr < nreg; hr += 32) {
                        const int h = sperm[regbase + hr];
                        const float dtv = __ldg(cv.dt + ti.lb * H + h);
                        const float Av = __ldg(cv.A + (long long)ti.l * H + h);
                        const float Dv = cv.D ? __ldg(cv.D + (long long)ti.l * H + h) : 0.0f;
                        ht[hr] = make_float4(decay(dtv, Av), dtv, Dv, __int_as_float(h * P));
                        gtab[hr] = fdiv(h, pv.mHpg) * N;
                    }
                }
                __syncwarp();
                if (lane == 0) {
                    reinterpret_cast<int*>(ub)[0] = slot;
                    reinterpret_cast<int*>(ub)[1] = bad ? 1 : 0;
                    if (bad) {
                        atomicOr(err, SSQ_DEVERR_SLOT);
                        mbar_arrive(&ufull[u]);
                    } else {
                        // B and C of every group, in natural order
                        const unsigned gb = (unsigned)(G * N * 4);
                        mbar_arrive_tx(&ufull[u], 2 * gb);
                        bulk_g2s(ub + geo.ub_B, cv.B + ti.lb * G * N, gb, &ufull[u]);
                        bulk_g2s(ub + geo.ub_C, cv.C + ti.lb * G * N, gb, &ufull[u]);
                    }
                }
            }
            if (bad) continue;
            // start the tile's HBM reads into L2 now; the copy into the stage,
            // issued once a stage is free, then reads from L2
            if (lane == 0) {
                if (F::quant && ti.quant) {
                    const int line0 = ti.rbase * RB / 128;
#pragma unroll 1
                    for (int bx = 0; bx < kBoxes && bx * kBoxRows < ti.n; ++bx)
                        tma_prefetch_codes(&cm.map, line0 + bx * kBoxLines, cur_layer, cur_slot);
                    bulk_prefetch_l2(meta_u + (long long)ti.rbase * MB, (unsigned)r16(ti.n * MB));
                } else {
                    bulk_prefetch_l2(fp_u + (long long)ti.rbase * N * FEB, (unsigned)(ti.n * N * FEB));
                }
            }
            // the stage's previous tile (k - S) must have been released
            if (k >= S && !mbar_wait_suspend(&empty[si], eph, wlim)) {
                ok = false;
                break;
            }
            // test support: CTA 0 leaves its first stage unfilled, so its
            // consumers' bounded waits run out (ssq_test_hooks)
            if (!(cv.test_withhold && blockIdx.x == 0 && k == 0)) {
                uint8_t* st = stages + si * geo.stage_bytes;
                float* sx = reinterpret_cast<float*>(st);
                uint8_t* pay = st + geo.x_bytes;
                unsigned pay_bytes;
                if (F::quant && ti.quant) {
                    const int nbox = (ti.n + kBoxRows - 1) / kBoxRows;
                    pay_bytes = (unsigned)(nbox * kBoxLines * 128) + (unsigned)r16(ti.n * MB);
                } else {
                    pay_bytes = (unsigned)(ti.n * N * FEB);
                }
                if (x_bulk) {
                    // the heads [h0, h1] the tile's rows fall in, a copy each
                    const int h0 = fdiv(ti.rbase, pv.mP);
                    const int h1 = fdiv(ti.rbase + ti.n - 1, pv.mP);
                    if (lane == 0) mbar_arrive_tx(&full[si], pay_bytes + (unsigned)(ti.n * 4));
                    __syncwarp();
                    for (int hr = h0 + lane; hr <= h1; hr += 32) {
                        const int r0 = max(ti.rbase, hr * P);
                        const int r1 = min(ti.rbase + ti.n, (hr + 1) * P);
                        const int hh = sperm[regbase + hr];
                        bulk_g2s(sx + (r0 - ti.rbase), x_u + hh * P + (r0 - hr * P),
                                 (unsigned)((r1 - r0) * 4), &full[si]);
                    }
                } else {
                    for (int i = lane; i < ti.n; i += 32) {
                        const int rr = ti.rbase + i;
                        const int hr = fdiv(rr, pv.mP);
                        const int hh = sperm[regbase + hr];
                        cpa4(sx + i, x_u + hh * P + (rr - hr * P));
                    }
                    cpa_arrive(&full[si]);
                    __syncwarp();
                    if (lane == 0) mbar_arrive_tx(&full[si], pay_bytes);
                }
                if (lane == 0) {
                    if (F::quant && ti.quant) {
                        const int line0 = ti.rbase * RB / 128;
                        const int nbox = (ti.n + kBoxRows - 1) / kBoxRows;
#pragma unroll 1
                        for (int bx = 0; bx < nbox; ++bx)
                            tma_load_codes(pay + bx * kBoxLines * 128, &cm.map, line0 + bx * kBoxLines,
                                           cur_layer, cur_slot, &full[si]);
                        bulk_g2s(pay + geo.qcodes_bytes, meta_u + (long long)ti.rbase * MB,
                                 (unsigned)r16(ti.n * MB), &full[si]);
                    } else {
                        bulk_g2s(pay, fp_u + (long long)ti.rbase * N * FEB, pay_bytes, &full[si]);
                    }
                }
            }
            ++k;
            if (++si == S) {
                // tiles [k, k + S) wait for the releases of tiles [k - S, k)
                si = 0;
                if (k >= 2 * S) eph ^= 1u;
            }
        }
        if (!ok && lane == 0) atomicOr(err, SSQ_DEVERR_TIMEOUT);
        // No copy may still be writing shared memory when the CTA exits.
        asm volatile("cp.async.wait_all;" ::: "memory");
        if (lane == 0) {
            for (int kk = (k > S ? k - S : 0); kk < k; ++kk)
                mbar_wait<kConsumerSleep>(&full[kk % S], (kk / S) & 1, wlim);
        }
        return;
    }

    // ================= consumer warps =================
    const int gtid = threadIdx.x;    // thread within the consumers
    int uk = -1;
    int si = 0;            // stage of the next tile
    unsigned fph = 0;      // its fill parity
    bool bad = false, newunit = true, ok = true;
    unsigned ub_a = 0;     // unit buffer, laundered shared address
    const uint8_t* ub = units;
    uint8_t* codes_u = nullptr;
    uint8_t* meta_u = nullptr;
    uint8_t* fp_u = nullptr;
    float* y_u = nullptr;
    int cur_slot = 0;
    // this warp's TMEM: lanes 32*(warp%4) .., columns 128*(warp/4) ..
    const uint32_t tm = use_tmem
        ? *tmem_slot + ((uint32_t)(32 * (warp & 3)) << 16) + (uint32_t)(128 * (warp >> 2))
        : 0u;

    TileWalk ti;
    ti.start(Hq, Hf, P, cv, t0);
    for (long long t = t0; t < t1; ++t, newunit = ti.next(Hq, Hf, P, cv)) {
        if (newunit) {
            if (uk >= 0) {
                __syncwarp();
                mbar_arrive_if(&uempty[uk & 1], lane == 0);
            }
            ++uk;
            const int u = uk & 1;
            if (!mbar_wait_suspend(&ufull[u], (uk >> 1) & 1, wlim)) { ok = false; break; }
            ub = units + u * geo.unit_bytes;
            ub_a = launder(saddr(ub));
            const int slot = reinterpret_cast<const int*>(ub)[0];
            cur_slot = slot;
            bad = reinterpret_cast<const int*>(ub)[1] != 0;
            if (!bad) {
                const int layer = cv.layer0 + ti.l;
                uint8_t* sb = pv.pool + pv.header_bytes + (long long)slot * pv.slot_bytes;
                codes_u = sb + pv.codes_off + (long long)layer * pv.codes_layer_bytes;
                meta_u = sb + pv.meta_off + (long long)layer * pv.meta_layer_bytes;
                fp_u = sb + pv.fp_off + (long long)layer * pv.fp_layer_bytes;
                y_u = cv.y + ti.lb * H * P;
            }
        }
        if (bad) continue;
        const int tsi = si;
        if (!mbar_wait_suspend(&full[tsi], fph, wlim)) { ok = false; break; }
        if (++si == S) {
            si = 0;
            fph ^= 1u;
        }
        uint8_t* const st = stages + tsi * geo.stage_bytes;
        const unsigned st_a = launder(saddr(st));
        uint8_t* const pay = st + geo.x_bytes;
        // row within the tile and lane within the row, by the region's shape
        const int grow = ti.quant ? gtid / LQ : gtid / LF;
        const int j = ti.quant ? gtid % LQ : gtid % LF;
        const bool active = grow < ti.n;
        // Rows past the end of a partial tile compute on a zero row with the
        // head parameters of the tile's row 0 and store nothing.
        const int rl = active ? grow : 0;
        const int rr = ti.rbase + rl;
        const int hr = fdiv(rr, pv.mP);
        const int p = rr - hr * P;
        const float4 hti = lds128f<0>(ub_a + geo.ub_ht + 16 * hr);
        const int gN = (int)lds32(ub_a + geo.ub_gt + 4 * hr);
        const float xv = active ? __uint_as_float(lds32(st_a + 4 * grow)) : 0.0f;
        const float lamv = hti.x;
        const float dtx = __fmul_rn(hti.y, xv);
        const float* gB = reinterpret_cast<const float*>(ub + geo.ub_B) + gN;
        const float* gC = reinterpret_cast<const float*>(ub + geo.ub_C) + gN;
        float ysum = 0.0f;
        bool done = false;
        float4 dres = make_float4(0.0f, 0.0f, 0.0f, 0.0f);   // diagnostics of the row

        if constexpr (F::quant) {
            if (ti.quant) {
                done = true;
                // this lane's codes in the stage (piece sp of the lane at
                // cs_x ^ (sp * PB) under the swizzle) and the row's metadata
                const unsigned cs0 = (unsigned)(geo.x_bytes + grow * RB + j * CB);
                const unsigned cs_x = st_a + swz128(cs0);
                const unsigned ms_a = st_a + (unsigned)(geo.x_bytes + geo.qcodes_bytes + grow * MB);
                // (a row past the end of the tile reads its stage slot and
                // decodes zeros instead)
                float delta0, z0 = 0.0f;
                if constexpr (F::sym) {
                    delta0 = __uint_as_float(lds32(ms_a));
                } else {
                    const uint2 m = lds64<0>(ms_a);
                    delta0 = __uint_as_float(m.x);
                    z0 = __uint_as_float(m.y);
                }
                delta0 = active ? delta0 : 0.0f;
                z0 = active ? z0 : 0.0f;
                const unsigned bxa = ub_a + geo.ub_B + 4 * gN + j * EQ * 4;
                const unsigned cxa = ub_a + geo.ub_C + 4 * gN + j * EQ * 4;
                // decode + update, one 16-entry piece at a time, with
                // per-piece min / max; the updated pieces wait in TMEM.  The
                // decode is exact for |z| < 2^22; rows beyond take the exact
                // path below.
                float lo = 0.0f, hi = 0.0f;
                {
                    const float c0 = __fadd_rn(kTwo23, __fadd_rn(z0, F::bias));
                    const float2 nc02 = make_float2(-c0, -c0);
                    const float2 d2 = make_float2(delta0, delta0);
                    const float2 l2 = make_float2(lamv, lamv);
                    const float2 x2 = make_float2(dtx, dtx);
                    static_for<NP>([&](auto spc) {
                        constexpr int sp = decltype(spc)::value;
                        uint32_t w[PW];
                        if constexpr (PW == 4) {
                            const uint4 v = lds128<0>(cs_x ^ (sp * PB));
                            w[0] = v.x; w[1] = v.y; w[2] = v.z; w[3] = v.w;
                        } else {
                            const uint2 v = lds64<0>(cs_x ^ (sp * PB));
                            w[0] = v.x; w[1] = v.y;
                        }
                        float f[16];
                        unpack16_biased<FMT>(w, f);
                        float v16[16];
                        static_for<4>([&](auto ic) {
                            constexpr int i = decltype(ic)::value;
                            const float4 bv = lds128f<sp * 64 + i * 16>(bxa);
                            const float2 v0 = mul2(add2(make_float2(f[4 * i], f[4 * i + 1]), nc02), d2);
                            const float2 v1 = mul2(add2(make_float2(f[4 * i + 2], f[4 * i + 3]), nc02), d2);
                            const float2 u0 = fma2(l2, v0, mul2(x2, make_float2(bv.x, bv.y)));
                            const float2 u1 = fma2(l2, v1, mul2(x2, make_float2(bv.z, bv.w)));
                            v16[4 * i] = u0.x; v16[4 * i + 1] = u0.y;
                            v16[4 * i + 2] = u1.x; v16[4 * i + 3] = u1.y;
                        });
                        // (a symmetric grid needs only max |s'|: lo = -hi)
                        if constexpr (F::sym) {
                            if constexpr (sp == 0) {
                                absmax16(v16, hi);
                            } else {
                                absmax16_acc(v16, hi);
                            }
                        } else if constexpr (sp == 0) {
                            minmax16(v16, lo, hi);
                        } else {
                            minmax16_acc(v16, lo, hi);
                        }
                        tmem_st16(tm + sp * 16, v16);
                    });
                }
                if constexpr (F::sym) lo = -hi;
                const RowParams rp = refit_from_minmax<FMT, LQ>(lo, hi);
                // the magic-number paths are exact for every row of the warp;
                // rows whose top code must be capped take the clamped loop
                const bool fast = __all_sync(0xffffffffu, (F::sym || fabsf(z0) < kFastLimit)
                                                          && rp.fast);
                // the refit above ran while the TMEM stores completed
                tmem_wait_st();
                // the stochastic-rounding key of this row (unused for RTN)
                SrKey srk{};
                if constexpr (SR) {
                    srk.key = make_uint2((uint32_t)cv.sr_seed, (uint32_t)(cv.sr_seed >> 32));
                    srk.layer = (uint32_t)(cv.layer0 + ti.l);
                    srk.slot = (uint32_t)cur_slot;
                    srk.step = cv.sr_step;
                    srk.row_block = (uint32_t)(__float_as_int(hti.w) + p) * (uint32_t)(N / 8);
                }
                if (DIAG && fast) {
                    // the rounding of the step, then per entry e = fl(fl(r
                    // Delta) - s'), w = fl(dtx B), the reversal test on fl(e +
                    // w) in fp32, and the sums of C e (all, reversed) and C s'
                    const float2 inv2 = make_float2(rp.inv, rp.inv);
                    const float2 z2 = make_float2(rp.z, rp.z);
                    const float mz = F::sym ? -kMagic : -__fadd_rn(kMagic, rp.z);
                    const float2 mz2 = make_float2(mz, mz);
                    const float2 dl2 = make_float2(rp.delta, rp.delta);
                    const float2 m1 = make_float2(-1.0f, -1.0f);
                    const float2 x2 = make_float2(dtx, dtx);
                    float2 sig = make_float2(0.0f, 0.0f), tot = make_float2(0.0f, 0.0f);
                    float2 rve = make_float2(0.0f, 0.0f);
                    int nrev = 0;
                    auto dpiece = [&](auto clamp_tag, float (&v16)[16], auto spc) {
                        constexpr int sp = decltype(spc)::value;
                        float r[16];
                        uint32_t kq[16];
                        round16_carry<FMT, decltype(clamp_tag)::value>(inv2, z2, mz2, v16, r, kq);
                        static_for<4>([&](auto ic) {
                            constexpr int i = decltype(ic)::value;
                            // (loads in program order: scheduled freely they
                            // raise the live registers of this pass past 96)
                            const float4 bv = lds128f_ordered<sp * 64 + i * 16>(bxa);
                            const float4 c4 = lds128f_ordered<sp * 64 + i * 16>(cxa);
#pragma unroll
                            for (int h2 = 0; h2 < 2; ++h2) {
                                const int n = 4 * i + 2 * h2;
                                const float2 sn = make_float2(v16[n], v16[n + 1]);
                                const float2 cc = h2 ? make_float2(c4.z, c4.w) : make_float2(c4.x, c4.y);
                                const float2 w = mul2(x2, h2 ? make_float2(bv.z, bv.w) : make_float2(bv.x, bv.y));
                                // s' * (-1) + fl(r Delta): one rounding, the difference
                                const float2 e = fma2(sn, m1, mul2(make_float2(r[n], r[n + 1]), dl2));
                                const float2 inc = add2(e, w);
                                sig = fma2(cc, sn, sig);
                                tot = fma2(cc, e, tot);
                                const bool rx = (w.x > 0.0f && inc.x < 0.0f) || (w.x < 0.0f && inc.x > 0.0f);
                                const bool ry = (w.y > 0.0f && inc.y < 0.0f) || (w.y < 0.0f && inc.y > 0.0f);
                                rve = fma2(cc, make_float2(rx ? e.x : 0.0f, ry ? e.y : 0.0f), rve);
                                nrev += (int)rx + (int)ry;
                            }
                        });
                    };
                    if (F::sym || !__any_sync(0xffffffffu, rp.clamp)) {
                        tmem_pieces<NP, false>(tm, [&](float (&v)[16], auto spc) { dpiece(std::false_type{}, v, spc); });
                    } else {
                        tmem_pieces<NP, false>(tm, [&](float (&v)[16], auto spc) { dpiece(std::true_type{}, v, spc); });
                    }
                    dres = make_float4(grp_sum<LQ>((float)nrev),
                                       grp_sum<LQ>(__fadd_rn(rve.x, rve.y)),
                                       grp_sum<LQ>(__fadd_rn(tot.x, tot.y)),
                                       grp_sum<LQ>(__fadd_rn(sig.x, sig.y)));
                } else if (DIAG) {
                    dres = row_exact_diag<FMT, N>(st, cs0, delta0, z0, lamv, dtx, gB, gC, j);
                } else if (fast) {
                    const float2 inv2 = make_float2(rp.inv, rp.inv);
                    const float2 z2 = make_float2(rp.z, rp.z);
                    const float mz = F::sym ? -kMagic : -__fadd_rn(kMagic, rp.z);
                    const float2 mz2 = make_float2(mz, mz);
                    // round, pack, write back and read out, piece by piece
                    // (the next piece's TMEM load in flight); the readout sums
                    // C (q - z) and scales by Delta once
                    float2 acc = make_float2(0.0f, 0.0f), acc1 = make_float2(0.0f, 0.0f);
                    auto piece = [&](auto clamp_tag, float (&v16)[16], auto spc) {
                        constexpr int sp = decltype(spc)::value;
                        float r[16];
                        uint32_t kq[16];
                        if constexpr (SR) {
                            float u[16];
                            sr_draws16(srk, j * EQ + 16 * sp, u);
                            round16_sr<FMT>(inv2, z2, mz2, v16, u, r, kq);
                        } else {
                            round16_carry<FMT, decltype(clamp_tag)::value>(inv2, z2, mz2, v16, r, kq);
                        }
                        uint32_t w[PW];
                        pack16<FMT>(kq, w);
                        if constexpr (PW == 4)
                            sts128u_if(cs_x ^ (sp * PB), make_uint4(w[0], w[1], w[2], w[3]), active);
                        else
                            sts64u_if(cs_x ^ (sp * PB), make_uint2(w[0], w[1]), active);
                        static_for<4>([&](auto ic) {
                            constexpr int i = decltype(ic)::value;
                            const float4 cv4 = lds128f<sp * 64 + i * 16>(cxa);
                            acc = fma2(make_float2(cv4.x, cv4.y), make_float2(r[4 * i], r[4 * i + 1]), acc);
                            acc1 = fma2(make_float2(cv4.z, cv4.w), make_float2(r[4 * i + 2], r[4 * i + 3]), acc1);
                        });
                    };
                    if (SR || F::sym || !__any_sync(0xffffffffu, rp.clamp)) {
                        tmem_pieces<NP, true>(tm, [&](float (&v)[16], auto spc) { piece(std::false_type{}, v, spc); });
                    } else {
                        tmem_pieces<NP, true>(tm, [&](float (&v)[16], auto spc) { piece(std::true_type{}, v, spc); });
                    }
                    acc = add2(acc, acc1);
                    ysum = __fmul_rn(rp.delta, grp_sum<LQ>(__fadd_rn(acc.x, acc.y)));
                    if (active && j == 0) {
                        uint8_t* mg = meta_u + (long long)rr * MB;
                        if constexpr (F::sym) {
                            __stcs(reinterpret_cast<float*>(mg), rp.delta);
                        } else {
                            __stcs(reinterpret_cast<float2*>(mg), make_float2(rp.delta, rp.z));
                        }
                    }
                    if (__any_sync(0xffffffffu, active && !rp.finite) && lane == 0)
                        atomicOr(err, SSQ_DEVERR_NONFINITE);
                } else {
                    ysum = row_exact<FMT, N, SR>(st, cs0, delta0, z0, lamv, dtx, gB, gC, j,
                                                 active, meta_u + (long long)rr * MB, err, srk);
                }
                // This warp's rows, from the stage to the pool: the warp's
                // contiguous block of 32/LQ rows, 16-byte chunk c = lane + 32 i
                // by lane `lane`, so every store instruction covers whole lines.
                __syncwarp();
                if constexpr (!DIAG) {
                    constexpr int WB = (32 / LQ) * RB;              // bytes of the block
                    constexpr int WCH = WB / 16;                    // its 16-byte chunks
                    constexpr int NI = (WCH + 31) / 32;             // chunks per lane
                    const int wrow0 = warp * (32 / LQ);             // first row of the block
                    const int wrows = min(ti.n - wrow0, 32 / LQ);   // live rows (may be <= 0)
                    // chunk c at swizzle(cb + 16 c) = A[i & 1] + 512 i, cb the
                    // block's stage offset: 512 i moves bit 9 and up, and the
                    // swizzle's XOR term takes bits 7..9
                    const unsigned cl = (unsigned)(geo.x_bytes + wrow0 * RB + 16 * lane);
                    const unsigned a0 = st_a + swz128(cl);
                    const unsigned a1 = a0 ^ 64u;
                    uint8_t* const gdst = codes_u + (long long)(ti.rbase + wrow0) * RB + 16 * lane;
                    if (wrows == 32 / LQ && WCH % 32 == 0) {
                        uint4 v[NI];
                        static_for<NI>([&](auto ic) {
                            constexpr int i = decltype(ic)::value;
                            v[i] = lds128_ordered<i * 512>((i & 1) ? a1 : a0);
                        });
                        static_for<NI>([&](auto ic) {
                            constexpr int i = decltype(ic)::value;
                            __stcs(reinterpret_cast<uint4*>(gdst + i * 512), v[i]);
                        });
                    } else {
                        static_for<NI>([&](auto ic) {
                            constexpr int i = decltype(ic)::value;
                            if (16 * (lane + 32 * i) < max(wrows, 0) * RB)
                                __stcs(reinterpret_cast<uint4*>(gdst + i * 512),
                                       lds128_ordered<i * 512>((i & 1) ? a1 : a0));
                        });
                    }
                }
            }
        }
        if (!done) {
            // fp row (fp32, or bf16 for the bf16 format), streamed one 16-byte
            // storage chunk at a time.  Lane j owns chunks LF*c + j; a lane
            // starts at chunk `rot` so a warp's reads of one step spread over
            // every bank group while B and C stay within one 128-byte line.
            constexpr int EPC = 16 / FEB;           // elements per chunk
            constexpr int NCH = EF / EPC;            // chunks per lane
            constexpr int RW = (8 / LF) < NCH ? (8 / LF) : NCH;   // rotation width
            const int rot = RW > 1 ? grow % RW : 0;
            const uint8_t* fs = pay + (long long)rl * N * FEB;
            uint8_t* frow = fp_u + (long long)rr * N * FEB;
            const float2 l2 = make_float2(lamv, lamv);
            const float2 x2 = make_float2(dtx, dtx);
            float2 acc = make_float2(0.0f, 0.0f), acc1 = make_float2(0.0f, 0.0f);
#pragma unroll
            for (int c0 = 0; c0 < NCH; ++c0) {
                const int c = RW > 1 ? ((c0 + rot) & (NCH - 1)) : c0;
                const int m = LF * c + j;
                const uint4 v = reinterpret_cast<const uint4*>(fs)[m];
                uint32_t w[4] = {v.x, v.y, v.z, v.w};
                float sv[EPC];
                if constexpr (kBf16) {
#pragma unroll
                    for (int n = 0; n < EPC; ++n)
                        sv[n] = __uint_as_float((w[n / 2] >> (16 * (n % 2))) << 16);
                } else {
#pragma unroll
                    for (int n = 0; n < EPC; ++n) sv[n] = __uint_as_float(w[n]);
                }
#pragma unroll
                for (int q = 0; q < EPC / 4; ++q) {
                    const float4 vb = reinterpret_cast<const float4*>(gB)[m * (EPC / 4) + q];
                    const float4 vc = reinterpret_cast<const float4*>(gC)[m * (EPC / 4) + q];
                    float2 a = fma2(l2, make_float2(sv[4 * q], sv[4 * q + 1]),
                                    mul2(x2, make_float2(vb.x, vb.y)));
                    float2 b = fma2(l2, make_float2(sv[4 * q + 2], sv[4 * q + 3]),
                                    mul2(x2, make_float2(vb.z, vb.w)));
                    if constexpr (DIAG) {
                        // the readout signal of the unrounded update
                        acc = fma2(make_float2(vc.x, vc.y), a, acc);
                        acc1 = fma2(make_float2(vc.z, vc.w), b, acc1);
                        continue;
                    }
                    if constexpr (kBf16) {
                        a = make_float2(__bfloat162float(__float2bfloat16_rn(a.x)),
                                        __bfloat162float(__float2bfloat16_rn(a.y)));
                        b = make_float2(__bfloat162float(__float2bfloat16_rn(b.x)),
                                        __bfloat162float(__float2bfloat16_rn(b.y)));
                    }
                    sv[4 * q] = a.x; sv[4 * q + 1] = a.y; sv[4 * q + 2] = b.x; sv[4 * q + 3] = b.y;
                    acc = fma2(make_float2(vc.x, vc.y), a, acc);
                    acc1 = fma2(make_float2(vc.z, vc.w), b, acc1);
                }
                if constexpr (kBf16) {
#pragma unroll
                    for (int n = 0; n < EPC; n += 2)
                        w[n / 2] = (__float_as_uint(sv[n]) >> 16) | (__float_as_uint(sv[n + 1]) & 0xffff0000u);
                } else {
#pragma unroll
                    for (int n = 0; n < EPC; ++n) w[n] = __float_as_uint(sv[n]);
                }
                if (!DIAG && active)
                    __stcs(reinterpret_cast<uint4*>(frow) + m, make_uint4(w[0], w[1], w[2], w[3]));
            }
            acc = add2(acc, acc1);
            ysum = grp_sum<LF>(__fadd_rn(acc.x, acc.y));
            dres.w = ysum;
        }
        // every lane of the row writes the same y (after the row sum all
        // hold it); a row past the end of the tile writes nothing
        if constexpr (DIAG) {
            if (active && j == 0)
                __stcs(reinterpret_cast<float4*>(cv.diag) + ti.lb * H * P + __float_as_int(hti.w) + p,
                       dres);
        } else if (active) {
            __stcs(y_u + __float_as_int(hti.w) + p, __fadd_rn(ysum, __fmul_rn(hti.z, xv)));
        }
        // this warp's shared-memory writes are ordered before the tensor
        // copy that refills the stage
        if (!DIAG && F::quant && ti.quant) fence_proxy_async();
        __syncwarp();
        mbar_arrive_if(&empty[tsi], lane == 0);
    }
    if (!ok && lane == 0) atomicOr(err, SSQ_DEVERR_TIMEOUT);
    // release TMEM once every consumer warp's TMEM accesses are complete
    if (use_tmem) {
        tc_fence_before();
        consumers_sync();
        tc_fence_after();
        if (warp == 0) tmem_dealloc(*tmem_slot, kTmemCols);
    }
}

// The driver's tensor-map encoder, looked up once through the runtime.
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder()
{
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static bool looked = false;
    if (!looked) {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess && q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
        looked = true;
    }
    return fn;
}

// The codes of every (slot, layer) of the pool as [slot][layer][line][128 B],
// boxes of kBoxRows rows' lines, 128-byte swizzle.
cudaError_t make_codes_map(const PoolView& pv, int RB, CodesMap* cm)
{
    std::memset(cm, 0, sizeof(*cm));
    PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
    if (!enc) return cudaErrorNotSupported;
    const long long region = (long long)pv.Hq * pv.P * RB;
    const cuuint64_t lines = (cuuint64_t)((region + 127) / 128);
    cuuint64_t dims[4] = {128, lines, (cuuint64_t)pv.n_layers, (cuuint64_t)pv.n_slots};
    cuuint64_t strides[3] = {128, (cuuint64_t)pv.codes_layer_bytes, (cuuint64_t)pv.slot_bytes};
    const int box_lines = (kBoxRows * RB + 127) / 128;
    cuuint32_t box[4] = {128, (cuuint32_t)box_lines, 1, 1};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    void* base = pv.pool + pv.header_bytes + pv.codes_off;
    const CUresult r = enc(&cm->map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 4, base, dims, strides, box,
                           estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                           CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

template <int FMT, int N, int MODE>
cudaError_t launch_n(const PoolView& pv, const CallView& cv, cudaStream_t st)
{
    using F = Fmt<FMT>;
    constexpr int RPTq = QShape<N>::RPT, RPTf = FShape<N>::RPT;
    constexpr int RB = F::quant ? N * F::bits / 8 : 0;
    const bool has_q = F::quant && pv.Hq > 0, has_fp = pv.Hf > 0;
    const int fpEB = FMT == SSQ_BF16 ? 2 : 4;
    // stages: as many as fit one CTA per SM
    const int budget = 226 * 1024;
    DecodeGeom g = decode_geom(2, RPTq, RPTf, RB, F::meta_bytes, fpEB, has_q, has_fp, N, pv.H, pv.G);
    int S = (budget - (g.smem_bytes - 2 * g.stage_bytes)) / g.stage_bytes;
    if (S > kMaxStages) S = kMaxStages;
    if (S < 2) S = 2;
    g = decode_geom(S, RPTq, RPTf, RB, F::meta_bytes, fpEB, has_q, has_fp, N, pv.H, pv.G);
    if (g.smem_bytes > 227 * 1024) return cudaErrorInvalidConfiguration;
    CodesMap cm;
    std::memset(&cm, 0, sizeof(cm));
    if (has_q) {
        const cudaError_t e = make_codes_map(pv, RB, &cm);
        if (e != cudaSuccess) return e;
    }
    auto kern = decode_kernel<FMT, N, MODE>;
    // per-device launch facts, looked up once per kernel instantiation and device
    thread_local int s_dev = -1, s_grid = 0, s_smem = 0;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (s_dev != dev || s_smem != g.smem_bytes) {
        if ((e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      g.smem_bytes)) != cudaSuccess)
            return e;
        int sms = 0, occ = 0;
        if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
            return e;
        if ((e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, kDThreads,
                                                               g.smem_bytes)) != cudaSuccess)
            return e;
        // one CTA per SM (its shared memory alone rules out a second); it
        // owns all of the SM's TMEM
        if (occ != 1) return cudaErrorInvalidConfiguration;
        s_dev = dev;
        s_smem = g.smem_bytes;
        s_grid = sms;
    }
    long long grid = s_grid;
    if (grid > cv.total_tiles) grid = cv.total_tiles;
    kern<<<(int)grid, kDThreads, g.smem_bytes, st>>>(pv, cv, g, cm);
    return cudaGetLastError();
}

template <int FMT, int MODE>
cudaError_t launch_fmt(const PoolView& pv, const CallView& cv, cudaStream_t st)
{
    switch (pv.N) {
    case 16: return launch_n<FMT, 16, MODE>(pv, cv, st);
    case 32: return launch_n<FMT, 32, MODE>(pv, cv, st);
    case 64: return launch_n<FMT, 64, MODE>(pv, cv, st);
    case 128: return launch_n<FMT, 128, MODE>(pv, cv, st);
    case 256: return launch_n<FMT, 256, MODE>(pv, cv, st);
    default: return cudaErrorInvalidValue;
    }
}

// Every mode of one format (stochastic rounding only for the integer formats).
template <int FMT>
cudaError_t launch_mode(const PoolView& pv, const CallView& cv, int mode, cudaStream_t st)
{
    if constexpr (Fmt<FMT>::quant) {
        if (mode == kStochastic) return launch_fmt<FMT, kStochastic>(pv, cv, st);
    }
    if (mode == kDiagnostics) return launch_fmt<FMT, kDiagnostics>(pv, cv, st);
    return launch_fmt<FMT, kNearest>(pv, cv, st);
}

}  // namespace

}  // namespace ssq
