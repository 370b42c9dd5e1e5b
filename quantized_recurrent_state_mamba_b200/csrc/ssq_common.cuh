// ssq_common.cuh -- device building blocks shared by the libssq kernels.
//
// The row engine below implements one step of the quantized recurrent-state
// update for one state row (head h, head_dim index p, d_state entries), as
// specified by "ssm-state-quantization" README, Setup (lambda = exp(dt*A);
// one scale per (head, head_dim) row over the d_state entries, refit every
// step; symmetric grid [-amax, amax], step amax/(2^(b-1)-1); asymmetric grid
// [min, max], integer zero point, step (max-min)/(2^b-1); output read from
// the quantized state) and Findings 1 (nearest rounding), with the FP32
// update of "Mamba state quantization for inference" (mixed-precision
// section).  Every fp32 operation that decides a stored value is a single
// correctly rounded IEEE operation in a fixed order (the library is built
// with -fmad=false; FMAs are explicit), so codes and metadata are identical
// to a plain scalar evaluation of the same formulas.
//
// Thread mapping: a row of N entries is owned by LPR = N/E consecutive lanes
// of a warp, each holding E consecutive entries in registers.  Row-wide
// min/max and the C.S readout are warp-shuffle butterflies inside the group.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "ssq.h"

namespace ssq {

constexpr int kThreads = 256;

// x + 1.5*2^23 rounds x (|x| < 2^22) to the nearest integer, ties to even,
// and leaves that integer in the low mantissa bits of the sum.
constexpr float kMagic = 12582912.0f;
constexpr float kTwo23 = 8388608.0f;
// Below 2^22 in magnitude the magic-number decode is exact; the rounding
// path checks its scaled values against 2^21 (a margin for the fp32 product
// that the check uses).
constexpr float kFastLimit = 4194304.0f;
constexpr float kRoundLimit = 2097152.0f;

// ---------------------------------------------------------------------------
// Format traits
// ---------------------------------------------------------------------------
template <int FMT>
struct Fmt {
    static constexpr bool quant = (FMT >= SSQ_I8_SYM);
    static constexpr bool sym = (FMT == SSQ_I8_SYM || FMT == SSQ_I4_SYM);
    static constexpr int bits =
        (FMT == SSQ_I8_SYM || FMT == SSQ_I8_ASYM) ? 8
        : (FMT == SSQ_I4_SYM || FMT == SSQ_I4_ASYM) ? 4
        : (FMT == SSQ_BF16) ? 16 : 32;
    // qs = 2^(b-1)-1 (sym) or qa = 2^b-1 (asym)
    static constexpr float qmax =
        quant ? (sym ? float((1 << (bits - 1)) - 1) : float((1 << bits) - 1))
              : 0.0f;
    // Sym codes are stored two's complement; flipping the sign bit of each
    // code gives q + 2^(b-1) as an unsigned field.
    static constexpr float bias = sym ? float(1 << (bits - 1)) : 0.0f;
    static constexpr int meta_bytes = quant ? (sym ? 4 : 8) : 0;
};

template <int N>
struct Shape {
    static constexpr int E = (N >= 32) ? 32 : N;  // entries per lane
    static constexpr int LPR = N / E;             // lanes per row
    static constexpr int RPW = 32 / LPR;          // rows per warp
    static_assert(N == 16 || N == 32 || N == 64 || N == 128 || N == 256,
                  "d_state must be 16, 32, 64, 128 or 256");
};

// ---------------------------------------------------------------------------
// Packed fp32 pairs (f32x2, sm_100a): one instruction for two lanes of work,
// each component rounded like the scalar operation.
// ---------------------------------------------------------------------------
__device__ __forceinline__ float2 mul2(float2 a, float2 b) { return __fmul2_rn(a, b); }
__device__ __forceinline__ float2 add2(float2 a, float2 b) { return __fadd2_rn(a, b); }
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) { return __ffma2_rn(a, b, c); }

// ---------------------------------------------------------------------------
// Small helpers
// ---------------------------------------------------------------------------
__device__ __forceinline__ float fmin3(float a, float b, float c)
{
    float r;
    asm("min.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}
__device__ __forceinline__ float fmax3(float a, float b, float c)
{
    float r;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}

template <int LPR>
__device__ __forceinline__ float grp_min(float v)
{
#pragma unroll
    for (int o = LPR / 2; o > 0; o >>= 1)
        v = fminf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}
template <int LPR>
__device__ __forceinline__ float grp_max(float v)
{
#pragma unroll
    for (int o = LPR / 2; o > 0; o >>= 1)
        v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}
template <int LPR>
__device__ __forceinline__ float grp_sum(float v)
{
#pragma unroll
    for (int o = LPR / 2; o > 0; o >>= 1)
        v = __fadd_rn(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

// lambda = exp(dt*A): the fp32 product, exponentiated in double and rounded
// once to fp32 ("ssm-state-quantization", Setup).
__device__ __forceinline__ float decay(float dt, float A)
{
    return (float)exp((double)__fmul_rn(dt, A));
}

// Vector loads / stores of a lane's contiguous chunk.
template <int BYTES>
struct Chunk {
    static_assert(BYTES % 4 == 0, "chunk must be whole words");
    uint32_t w[BYTES / 4];
};

template <int BYTES>
__device__ __forceinline__ void load_chunk(Chunk<BYTES>& c, const void* p)
{
    if constexpr (BYTES % 16 == 0) {
#pragma unroll
        for (int i = 0; i < BYTES / 16; ++i) {
            uint4 v = __ldcs(reinterpret_cast<const uint4*>(p) + i);
            c.w[4 * i + 0] = v.x; c.w[4 * i + 1] = v.y;
            c.w[4 * i + 2] = v.z; c.w[4 * i + 3] = v.w;
        }
    } else if constexpr (BYTES == 8) {
        uint2 v = __ldcs(reinterpret_cast<const uint2*>(p));
        c.w[0] = v.x; c.w[1] = v.y;
    } else {
#pragma unroll
        for (int i = 0; i < BYTES / 4; ++i)
            c.w[i] = __ldcs(reinterpret_cast<const uint32_t*>(p) + i);
    }
}

template <int BYTES>
__device__ __forceinline__ void store_chunk(void* p, const Chunk<BYTES>& c)
{
    if constexpr (BYTES % 16 == 0) {
#pragma unroll
        for (int i = 0; i < BYTES / 16; ++i)
            __stcs(reinterpret_cast<uint4*>(p) + i,
                   make_uint4(c.w[4 * i], c.w[4 * i + 1], c.w[4 * i + 2],
                              c.w[4 * i + 3]));
    } else if constexpr (BYTES == 8) {
        __stcs(reinterpret_cast<uint2*>(p), make_uint2(c.w[0], c.w[1]));
    } else {
#pragma unroll
        for (int i = 0; i < BYTES / 4; ++i)
            __stcs(reinterpret_cast<uint32_t*>(p) + i, c.w[i]);
    }
}

// E consecutive fp32 values from (cached) global memory, 16-byte vectors.
template <int E>
__device__ __forceinline__ void load_f32(float (&v)[E], const float* p)
{
    static_assert(E % 4 == 0, "");
#pragma unroll
    for (int i = 0; i < E / 4; ++i) {
        float4 t = __ldg(reinterpret_cast<const float4*>(p) + i);
        v[4 * i] = t.x; v[4 * i + 1] = t.y; v[4 * i + 2] = t.z; v[4 * i + 3] = t.w;
    }
}

// ---------------------------------------------------------------------------
// Code (un)packing.
//
// Entry n of a row: 8-bit formats keep it in byte n; 4-bit formats keep
// entries 2k and 2k+1 in the low and high nibble of byte k.  Sym codes are
// two's complement.  Within a lane's chunk word i holds entries 4i..4i+3
// (8-bit) or 8i..8i+7 (4-bit).
// ---------------------------------------------------------------------------

// f[n] = 2^23 + u_n where u_n is the unsigned code field (sym: q + 2^(b-1)).
template <int FMT, int E>
__device__ __forceinline__ void unpack_biased(const Chunk<E * Fmt<FMT>::bits / 8>& c,
                                              float (&f)[E])
{
    constexpr bool sym = Fmt<FMT>::sym;
    constexpr uint32_t kExp = 0x4B000000u;  // bits of 2^23
    if constexpr (Fmt<FMT>::bits == 8) {
#pragma unroll
        for (int i = 0; i < E / 4; ++i) {
            const uint32_t v = sym ? (c.w[i] ^ 0x80808080u) : c.w[i];
            f[4 * i + 0] = __uint_as_float(__byte_perm(v, kExp, 0x7540));
            f[4 * i + 1] = __uint_as_float(__byte_perm(v, kExp, 0x7541));
            f[4 * i + 2] = __uint_as_float(__byte_perm(v, kExp, 0x7542));
            f[4 * i + 3] = __uint_as_float(__byte_perm(v, kExp, 0x7543));
        }
    } else {
#pragma unroll
        for (int i = 0; i < E / 8; ++i) {
            const uint32_t v = sym ? (c.w[i] ^ 0x88888888u) : c.w[i];
            const uint32_t lo = v & 0x0F0F0F0Fu;          // entries 8i+0,2,4,6
            const uint32_t hi = (v >> 4) & 0x0F0F0F0Fu;   // entries 8i+1,3,5,7
            f[8 * i + 0] = __uint_as_float(__byte_perm(lo, kExp, 0x7540));
            f[8 * i + 1] = __uint_as_float(__byte_perm(hi, kExp, 0x7540));
            f[8 * i + 2] = __uint_as_float(__byte_perm(lo, kExp, 0x7541));
            f[8 * i + 3] = __uint_as_float(__byte_perm(hi, kExp, 0x7541));
            f[8 * i + 4] = __uint_as_float(__byte_perm(lo, kExp, 0x7542));
            f[8 * i + 5] = __uint_as_float(__byte_perm(hi, kExp, 0x7542));
            f[8 * i + 6] = __uint_as_float(__byte_perm(lo, kExp, 0x7543));
            f[8 * i + 7] = __uint_as_float(__byte_perm(hi, kExp, 0x7543));
        }
    }
}

// Integer codes (sign-extended for sym), for the exact slow path.
template <int FMT, int E>
__device__ __forceinline__ void unpack_int(const Chunk<E * Fmt<FMT>::bits / 8>& c,
                                           int (&q)[E])
{
    if constexpr (Fmt<FMT>::bits == 8) {
#pragma unroll
        for (int n = 0; n < E; ++n) {
            const uint32_t b = (c.w[n / 4] >> (8 * (n % 4))) & 0xFFu;
            q[n] = Fmt<FMT>::sym ? (int)(int8_t)b : (int)b;
        }
    } else {
#pragma unroll
        for (int n = 0; n < E; ++n) {
            const uint32_t b = (c.w[n / 8] >> (4 * (n % 8))) & 0xFu;
            q[n] = Fmt<FMT>::sym ? (int)((b ^ 8u) - 8u) : (int)b;
        }
    }
}

// Pack code carriers (the code sits in the low 8 or 4 bits of each carrier)
// into the row's byte layout.
template <int FMT, int E>
__device__ __forceinline__ void pack_codes(const uint32_t (&k)[E],
                                           Chunk<E * Fmt<FMT>::bits / 8>& c)
{
    if constexpr (Fmt<FMT>::bits == 8) {
#pragma unroll
        for (int i = 0; i < E / 4; ++i) {
            const uint32_t a = __byte_perm(k[4 * i + 0], k[4 * i + 1], 0x0040);
            const uint32_t b = __byte_perm(k[4 * i + 2], k[4 * i + 3], 0x0040);
            c.w[i] = __byte_perm(a, b, 0x5410);
        }
    } else {
#pragma unroll
        for (int i = 0; i < E / 8; ++i) {
            const uint32_t e01 = __byte_perm(k[8 * i + 0], k[8 * i + 2], 0x0040);
            const uint32_t e23 = __byte_perm(k[8 * i + 4], k[8 * i + 6], 0x0040);
            const uint32_t o01 = __byte_perm(k[8 * i + 1], k[8 * i + 3], 0x0040);
            const uint32_t o23 = __byte_perm(k[8 * i + 5], k[8 * i + 7], 0x0040);
            const uint32_t ev = __byte_perm(e01, e23, 0x5410);
            const uint32_t od = __byte_perm(o01, o23, 0x5410);
            c.w[i] = (ev & 0x0F0F0F0Fu) | ((od << 4) & 0xF0F0F0F0u);
        }
    }
}

// ---------------------------------------------------------------------------
// 16-entry pieces of a lane's codes (4 words of 8-bit codes, 2 words of
// 4-bit codes), for kernels that stream a row through registers.
// ---------------------------------------------------------------------------
template <int FMT>
struct Piece {
    static constexpr int words = 16 * Fmt<FMT>::bits / 32;  // 4 or 2
};

// f[n] = 2^23 + u_n for the 16 entries held in w[0 .. words).
template <int FMT>
__device__ __forceinline__ void unpack16_biased(const uint32_t* w, float (&f)[16])
{
    constexpr bool sym = Fmt<FMT>::sym;
    constexpr uint32_t kExp = 0x4B000000u;
    if constexpr (Fmt<FMT>::bits == 8) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const uint32_t v = sym ? (w[i] ^ 0x80808080u) : w[i];
            f[4 * i + 0] = __uint_as_float(__byte_perm(v, kExp, 0x7540));
            f[4 * i + 1] = __uint_as_float(__byte_perm(v, kExp, 0x7541));
            f[4 * i + 2] = __uint_as_float(__byte_perm(v, kExp, 0x7542));
            f[4 * i + 3] = __uint_as_float(__byte_perm(v, kExp, 0x7543));
        }
    } else {
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            const uint32_t v = sym ? (w[i] ^ 0x88888888u) : w[i];
            const uint32_t lo = v & 0x0F0F0F0Fu;
            const uint32_t hi = (v >> 4) & 0x0F0F0F0Fu;
            f[8 * i + 0] = __uint_as_float(__byte_perm(lo, kExp, 0x7540));
            f[8 * i + 1] = __uint_as_float(__byte_perm(hi, kExp, 0x7540));
            f[8 * i + 2] = __uint_as_float(__byte_perm(lo, kExp, 0x7541));
            f[8 * i + 3] = __uint_as_float(__byte_perm(hi, kExp, 0x7541));
            f[8 * i + 4] = __uint_as_float(__byte_perm(lo, kExp, 0x7542));
            f[8 * i + 5] = __uint_as_float(__byte_perm(hi, kExp, 0x7542));
            f[8 * i + 6] = __uint_as_float(__byte_perm(lo, kExp, 0x7543));
            f[8 * i + 7] = __uint_as_float(__byte_perm(hi, kExp, 0x7543));
        }
    }
}

template <int FMT>
__device__ __forceinline__ void unpack16_int(const uint32_t* w, int (&q)[16])
{
#pragma unroll
    for (int n = 0; n < 16; ++n) {
        if constexpr (Fmt<FMT>::bits == 8) {
            const uint32_t b = (w[n / 4] >> (8 * (n % 4))) & 0xFFu;
            q[n] = Fmt<FMT>::sym ? (int)(int8_t)b : (int)b;
        } else {
            const uint32_t b = (w[n / 8] >> (4 * (n % 8))) & 0xFu;
            q[n] = Fmt<FMT>::sym ? (int)((b ^ 8u) - 8u) : (int)b;
        }
    }
}

template <int FMT>
__device__ __forceinline__ void pack16(const uint32_t (&k)[16], uint32_t* w)
{
    if constexpr (Fmt<FMT>::bits == 8) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const uint32_t a = __byte_perm(k[4 * i + 0], k[4 * i + 1], 0x0040);
            const uint32_t b = __byte_perm(k[4 * i + 2], k[4 * i + 3], 0x0040);
            w[i] = __byte_perm(a, b, 0x5410);
        }
    } else {
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            const uint32_t e01 = __byte_perm(k[8 * i + 0], k[8 * i + 2], 0x0040);
            const uint32_t e23 = __byte_perm(k[8 * i + 4], k[8 * i + 6], 0x0040);
            const uint32_t o01 = __byte_perm(k[8 * i + 1], k[8 * i + 3], 0x0040);
            const uint32_t o23 = __byte_perm(k[8 * i + 5], k[8 * i + 7], 0x0040);
            const uint32_t ev = __byte_perm(e01, e23, 0x5410);
            const uint32_t od = __byte_perm(o01, o23, 0x5410);
            w[i] = (ev & 0x0F0F0F0Fu) | ((od << 4) & 0xF0F0F0F0u);
        }
    }
}

// ---------------------------------------------------------------------------
// Row decode: s_n = (q_n - z)*Delta (asym) or q_n*Delta (sym).
// ---------------------------------------------------------------------------
template <int FMT, int E>
__device__ __forceinline__ void decode_row(const Chunk<E * Fmt<FMT>::bits / 8>& c,
                                           float delta, float z, float (&s)[E])
{
    using F = Fmt<FMT>;
    // Warp-uniform choice (every lane of the warp calls this): the exact
    // scalar path serves the whole warp when any of its rows needs it.
    if (F::sym || __all_sync(0xffffffffu, fabsf(z) < kFastLimit)) {
        // (2^23 + u) - (2^23 + z + bias) = q - z exactly; one rounding in
        // the product, as in the scalar formula.
        float f[E];
        unpack_biased<FMT, E>(c, f);
        const float c0 = __fadd_rn(kTwo23, __fadd_rn(z, F::bias));
        const float2 nc02 = make_float2(-c0, -c0);
        const float2 d2 = make_float2(delta, delta);
#pragma unroll
        for (int n = 0; n < E; n += 2) {
            float2 v = add2(make_float2(f[n], f[n + 1]), nc02);
            v = mul2(v, d2);
            s[n] = v.x; s[n + 1] = v.y;
        }
    } else {
        int q[E];
        unpack_int<FMT, E>(c, q);
#pragma unroll
        for (int n = 0; n < E; ++n)
            s[n] = __fmul_rn(__fsub_rn((float)q[n], z), delta);
    }
}

// rint(a*b) with the product exact: formed in double, where the product of
// two floats is exact, and rounded once to the nearest integer (ties to
// even).  The magic-number paths below compute the same value in one fp32
// FMA, fma(a, b, 1.5*2^23) - 1.5*2^23, for |a*b| < 2^21.
__device__ __forceinline__ float rint_prod(float a, float b)
{
    return (float)rint((double)a * (double)b);
}

// ---------------------------------------------------------------------------
// Row refit + round.
//
// Given the updated row s' (E entries per lane, LPR lanes per row), compute
// Delta, inv = 1/Delta and z, round every entry, and produce
//   r[n]  = q_n - z as fp32 (what the stored row decodes to, before * Delta)
//   k[n]  = a carrier whose low bits are the stored code.
// Reading of the pages' silent points: ties to even on the exact product
// s'*inv (one rounding); z =
// rint(-lo*inv) unclamped (negative zero stored as +0); a constant row takes
// Delta = |lo|; Delta below FLT_MIN flushes the row to zero; asym codes
// clamp at qa (the minimum maps to 0 by construction); the sym clamp never
// binds because |fl(amax*inv)| rounds to qs.
// ---------------------------------------------------------------------------
// a / qmax, correctly rounded, for every non-negative finite a: the product
// by the rounded reciprocal corrected once with two FMAs (Brisebarre,
// Muller, Raina, "Accelerating correctly rounded floating-point division
// when the divisor is known in advance", IEEE Trans. Computers 2004).  For
// qmax in {255, 15, 127, 7} the identity was checked against IEEE division on
// every non-negative finite fp32 value; tests/test_host_math.py re-checks a
// large sample of it on each run.
template <int FMT>
__device__ __forceinline__ float div_qmax(float a)
{
    constexpr float d = Fmt<FMT>::qmax;
    constexpr float r = 1.0f / Fmt<FMT>::qmax;
    const float q0 = __fmul_rn(a, r);
    const float rem = __fmaf_rn(-q0, d, a);
    return __fmaf_rn(rem, r, q0);
}

struct RowParams {
    float delta, inv, z;
    bool fast;    // magic-number rounding is exact for this row
    bool clamp;   // some entry rounds above qa (asym)
    bool finite;
};

// Refit from the lane's partial min and max of the updated row: reduce them
// over the row's LPR lanes, then derive Delta, inv and z.
template <int FMT, int LPR>
__device__ __forceinline__ RowParams refit_from_minmax(float lo, float hi)
{
    using F = Fmt<FMT>;
    lo = grp_min<LPR>(lo);
    hi = grp_max<LPR>(hi);

    RowParams rp;
    rp.finite = isfinite(lo) && isfinite(hi);
    float delta;
    if constexpr (F::sym) {
        const float amax = fmaxf(-lo, hi);
        delta = div_qmax<FMT>(amax);
    } else {
        delta = div_qmax<FMT>(__fsub_rn(hi, lo));
        if (delta == 0.0f) delta = fabsf(lo);
    }
    if (delta < 1.17549435e-38f) delta = 0.0f;  // FLT_MIN
    const float inv = (delta == 0.0f) ? 0.0f : __frcp_rn(delta);
    float z = 0.0f;
    const float plo = __fmul_rn(lo, inv), phi = __fmul_rn(hi, inv);
    // Below 2^21 the exact-product rounding is one FMA with the magic
    // number; rows beyond it (rare: far from zero relative to their range)
    // take it in double.
    const bool small = fmaxf(fabsf(plo), fabsf(phi)) < kRoundLimit;
    float rhi;
    if (small) {
        if constexpr (!F::sym) z = __fadd_rn(__fsub_rn(__fmaf_rn(-lo, inv, kMagic), kMagic), 0.0f);
        rhi = __fsub_rn(__fmaf_rn(hi, inv, kMagic), kMagic);
    } else {
        if constexpr (!F::sym) z = __fadd_rn(rint_prod(-lo, inv), 0.0f);
        rhi = rint_prod(hi, inv);
    }
    rp.delta = delta;
    rp.inv = inv;
    rp.z = z;
    rp.fast = small && fabsf(z) < kRoundLimit;
    rp.clamp = (!F::sym) && (__fadd_rn(rhi, z) > F::qmax);
    return rp;
}

// Lane-local min / max of n values, folded into (lo, hi).
template <int M>
__device__ __forceinline__ void minmax_acc(const float* v, float& lo, float& hi)
{
#pragma unroll
    for (int n = 0; n + 1 < M; n += 2) {
        lo = fmin3(lo, v[n], v[n + 1]);
        hi = fmax3(hi, v[n], v[n + 1]);
    }
    if constexpr (M % 2 == 1) {
        lo = fminf(lo, v[M - 1]);
        hi = fmaxf(hi, v[M - 1]);
    }
}

// Min and max of 16 values as shallow trees (depth 3) rather than one long
// dependent chain, so the scheduler can overlap them.
__device__ __forceinline__ void minmax16(const float* v, float& lo, float& hi)
{
    const float a = fmin3(v[0], v[1], v[2]), b = fmin3(v[3], v[4], v[5]);
    const float c = fmin3(v[6], v[7], v[8]), d = fmin3(v[9], v[10], v[11]);
    const float e = fmin3(v[12], v[13], v[14]);
    lo = fminf(fmin3(a, b, c), fmin3(d, e, v[15]));
    const float A = fmax3(v[0], v[1], v[2]), B = fmax3(v[3], v[4], v[5]);
    const float C = fmax3(v[6], v[7], v[8]), D = fmax3(v[9], v[10], v[11]);
    const float E = fmax3(v[12], v[13], v[14]);
    hi = fmaxf(fmax3(A, B, C), fmax3(D, E, v[15]));
}

// ... and folded into a running (lo, hi): eight 3-input operations each.
__device__ __forceinline__ void minmax16_acc(const float* v, float& lo, float& hi)
{
    const float a = fmin3(v[0], v[1], v[2]), b = fmin3(v[3], v[4], v[5]);
    const float c = fmin3(v[6], v[7], v[8]), d = fmin3(v[9], v[10], v[11]);
    const float e = fmin3(v[12], v[13], v[14]);
    lo = fmin3(lo, fmin3(a, b, c), fmin3(d, e, v[15]));
    const float A = fmax3(v[0], v[1], v[2]), B = fmax3(v[3], v[4], v[5]);
    const float C = fmax3(v[6], v[7], v[8]), D = fmax3(v[9], v[10], v[11]);
    const float E = fmax3(v[12], v[13], v[14]);
    hi = fmax3(hi, fmax3(A, B, C), fmax3(D, E, v[15]));
}

// max |v| of 16 values (the absolute values are operand modifiers of the
// 3-input max) ...
__device__ __forceinline__ void absmax16(const float* v, float& am)
{
    const float a = fmax3(fabsf(v[0]), fabsf(v[1]), fabsf(v[2]));
    const float b = fmax3(fabsf(v[3]), fabsf(v[4]), fabsf(v[5]));
    const float c = fmax3(fabsf(v[6]), fabsf(v[7]), fabsf(v[8]));
    const float d = fmax3(fabsf(v[9]), fabsf(v[10]), fabsf(v[11]));
    const float e = fmax3(fabsf(v[12]), fabsf(v[13]), fabsf(v[14]));
    am = fmax3(fmax3(a, b, c), fmax3(d, e, fabsf(v[15])), 0.0f);
}
// ... and folded into a running max.
__device__ __forceinline__ void absmax16_acc(const float* v, float& am)
{
    const float a = fmax3(fabsf(v[0]), fabsf(v[1]), fabsf(v[2]));
    const float b = fmax3(fabsf(v[3]), fabsf(v[4]), fabsf(v[5]));
    const float c = fmax3(fabsf(v[6]), fabsf(v[7]), fabsf(v[8]));
    const float d = fmax3(fabsf(v[9]), fabsf(v[10]), fabsf(v[11]));
    const float e = fmax3(fabsf(v[12]), fabsf(v[13]), fabsf(v[14]));
    am = fmax3(am, fmax3(a, b, c), fmax3(d, e, fabsf(v[15])));
}

template <int FMT, int E, int LPR>
__device__ __forceinline__ RowParams refit_row(const float (&s)[E])
{
    float lo = s[0], hi = s[0];
    minmax_acc<E - 1>(s + 1, lo, hi);
    return refit_from_minmax<FMT, LPR>(lo, hi);
}

// Fast rounding of 16 entries (valid when the warp's rows all passed the
// fast test): r = rint(s*inv) (exact product) exactly, k carries the stored code.
template <int FMT>
__device__ __forceinline__ void round16_fast(const RowParams& rp, const float* s, float* r,
                                             uint32_t (&k)[16])
{
    using F = Fmt<FMT>;
    const float2 inv2 = make_float2(rp.inv, rp.inv);
    const float2 m2 = make_float2(kMagic, kMagic);
    const float2 nm2 = make_float2(-kMagic, -kMagic);
    const float2 z2 = make_float2(rp.z, rp.z);
#pragma unroll
    for (int n = 0; n < 16; n += 2) {
        float2 t = fma2(make_float2(s[n], s[n + 1]), inv2, m2);   // 1.5*2^23 + rint(s*inv)
        float2 rr = add2(t, nm2);
        r[n] = rr.x; r[n + 1] = rr.y;
        if constexpr (F::sym) {
            k[n] = __float_as_uint(t.x);
            k[n + 1] = __float_as_uint(t.y);
        } else {
            float2 u = add2(t, z2);
            k[n] = __float_as_uint(u.x);
            k[n + 1] = __float_as_uint(u.y);
        }
    }
}

// Fast rounding of 16 entries for the decode step: r = q - z (asym) or q
// (sym) exactly, k carries the stored code.  With CLAMP the asymmetric code
// is capped at qa first (min(rint(p) + z, qa): the top code of a row whose
// largest entry rounds one step past the grid).  mz2 holds -(1.5*2^23 + z),
// nm2 -1.5*2^23; both sums are exact because every operand is an integer
// below 2^24 in magnitude.
template <int FMT, bool CLAMP>
__device__ __forceinline__ void round16_carry(float2 inv2, float2 z2, float2 mz2, float* s,
                                              float* r, uint32_t (&k)[16])
{
    using F = Fmt<FMT>;
    const float2 m2 = make_float2(kMagic, kMagic);
    const float2 nm2 = make_float2(-kMagic, -kMagic);
    constexpr float kTop = kMagic + F::qmax;   // carrier of code qa
#pragma unroll
    for (int n = 0; n < 16; n += 2) {
        // 1.5*2^23 + rint(s*inv): the exact product and the magic number
        // rounded together, once
        const float2 t = fma2(make_float2(s[n], s[n + 1]), inv2, m2);
        if constexpr (F::sym) {
            const float2 rr = add2(t, mz2);            // rint(p), exact
            r[n] = rr.x; r[n + 1] = rr.y;
            k[n] = __float_as_uint(t.x);
            k[n + 1] = __float_as_uint(t.y);
        } else {
            float2 u = add2(t, z2);                    // 1.5*2^23 + q
            float2 rr;
            if constexpr (CLAMP) {
                u.x = fminf(u.x, kTop);
                u.y = fminf(u.y, kTop);
                rr = add2(u, mz2);                     // q - z, exact
            } else {
                rr = add2(t, nm2);                     // rint(p) = q - z, exact, beside u
            }
            r[n] = rr.x; r[n + 1] = rr.y;
            k[n] = __float_as_uint(u.x);
            k[n + 1] = __float_as_uint(u.y);
        }
    }
}

// ---------------------------------------------------------------------------
// Stochastic rounding ("ssm-state-quantization" README, Findings 9).
//
// An entry rounds to floor(s*inv + u) (plus z, clamped to the code range),
// u = d * 2^-16 with d a 16-bit draw of Philox4x32-10 (Salmon, Moraes, Dror,
// Shaw, SC 2011) keyed by the caller's seed, counter (r*(N/8) + n/8, layer,
// slot, step) for entry n of row r = h*P + p: word (n%8)/2 of the output,
// low half for even n.  floor of the exact s*inv + u is formed as
// fma rounded toward -inf (floor of that float is floor of the exact sum)
// and an add of 1.5*2^23 rounded toward -inf.
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint4 philox4x32_10(uint4 c, uint2 k)
{
#pragma unroll
    for (int round = 0; round < 10; ++round) {
        const uint32_t hi0 = __umulhi(0xD2511F53u, c.x), lo0 = 0xD2511F53u * c.x;
        const uint32_t hi1 = __umulhi(0xCD9E8D57u, c.z), lo1 = 0xCD9E8D57u * c.z;
        c = make_uint4(hi1 ^ c.y ^ k.x, lo1, hi0 ^ c.w ^ k.y, lo0);
        k.x += 0x9E3779B9u;
        k.y += 0xBB67AE85u;
    }
    return c;
}

// Counter words of a stochastic-rounding draw: y = layer, z = slot, w = step;
// x is set per 8-entry block.
struct SrKey {
    uint2 key;
    uint32_t layer, slot, step;
    uint32_t row_block;   // r * (N/8): the first block of this row
};

// u = d * 2^-16 for the 16 entries [n0, n0 + 16) of a row (n0 a multiple of
// 16): two Philox blocks.
__device__ __forceinline__ void sr_draws16(const SrKey& k, int n0, float (&u)[16])
{
#pragma unroll
    for (int b = 0; b < 2; ++b) {
        const uint4 w = philox4x32_10(
            make_uint4(k.row_block + (uint32_t)(n0 / 8 + b), k.layer, k.slot, k.step), k.key);
        const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            // 1 + d*2^-16 has the 16 draw bits on top of the mantissa
            u[8 * b + 2 * i] = __uint_as_float(0x3F800000u | ((ww[i] & 0xFFFFu) << 7)) - 1.0f;
            u[8 * b + 2 * i + 1] = __uint_as_float(0x3F800000u | ((ww[i] >> 16) << 7)) - 1.0f;
        }
    }
}

__device__ __forceinline__ float2 fma2_rm(float2 a, float2 b, float2 c)
{
    unsigned long long d;
    asm("fma.rm.f32x2 %0, %1, %2, %3;" : "=l"(d)
        : "l"(*reinterpret_cast<unsigned long long*>(&a)),
          "l"(*reinterpret_cast<unsigned long long*>(&b)),
          "l"(*reinterpret_cast<unsigned long long*>(&c)));
    return *reinterpret_cast<float2*>(&d);
}
__device__ __forceinline__ float2 add2_rm(float2 a, float2 b)
{
    unsigned long long d;
    asm("add.rm.f32x2 %0, %1, %2;" : "=l"(d)
        : "l"(*reinterpret_cast<unsigned long long*>(&a)),
          "l"(*reinterpret_cast<unsigned long long*>(&b)));
    return *reinterpret_cast<float2*>(&d);
}

// Stochastic rounding of 16 entries on the fast path (|s*inv| < 2^21):
// r = q - z (asym) or q (sym) exactly, k carries the stored code.  mz2 holds
// -(1.5*2^23 + z) (asym) or -1.5*2^23 (sym).
template <int FMT>
__device__ __forceinline__ void round16_sr(float2 inv2, float2 z2, float2 mz2, const float* s,
                                           const float (&u)[16], float* r, uint32_t (&k)[16])
{
    using F = Fmt<FMT>;
    const float2 m2 = make_float2(kMagic, kMagic);
    constexpr float kLo = F::sym ? kMagic - F::qmax : kMagic;
    constexpr float kHi = kMagic + F::qmax;
#pragma unroll
    for (int n = 0; n < 16; n += 2) {
        const float2 v = fma2_rm(make_float2(s[n], s[n + 1]), inv2, make_float2(u[n], u[n + 1]));
        float2 t = add2_rm(v, m2);                     // 1.5*2^23 + floor(s*inv + u)
        if constexpr (!F::sym) t = add2(t, z2);        // 1.5*2^23 + q before the clamp
        t.x = fminf(fmaxf(t.x, kLo), kHi);
        t.y = fminf(fmaxf(t.y, kLo), kHi);
        const float2 rr = add2(t, mz2);
        r[n] = rr.x; r[n + 1] = rr.y;
        k[n] = __float_as_uint(t.x);
        k[n + 1] = __float_as_uint(t.y);
    }
}

// The same by the formulas verbatim (exact sum in double), for rows outside
// the fast range.
template <int FMT>
__device__ __forceinline__ float round1_sr_exact(float s, float inv, float z, float u,
                                                 float* r)
{
    using F = Fmt<FMT>;
    const double kf = floor((double)s * (double)inv + (double)u);
    float c = (float)kf;
    if constexpr (F::sym) {
        c = fminf(fmaxf(c, -F::qmax), F::qmax);
        *r = c;
    } else {
        c = fminf(fmaxf(__fadd_rn(c, z), 0.0f), F::qmax);
        *r = __fsub_rn(c, z);
    }
    return c;
}

// Exact scalar rounding of 16 entries (the definition verbatim).
template <int FMT>
__device__ __forceinline__ void round16_slow(const RowParams& rp, const float* s, float* r,
                                             uint32_t (&k)[16])
{
    using F = Fmt<FMT>;
#pragma unroll
    for (int n = 0; n < 16; ++n) {
        const float rr = rint_prod(s[n], rp.inv);
        float c;
        if constexpr (F::sym) {
            c = fminf(fmaxf(rr, -F::qmax), F::qmax);
            r[n] = c;
        } else {
            c = fminf(__fadd_rn(rr, rp.z), F::qmax);
            r[n] = __fsub_rn(c, rp.z);
        }
        k[n] = (uint32_t)(int)c;
    }
}

// Returns true when the magic-number path ran (then r holds exact q - z);
// the choice is warp-uniform and every lane of the warp must call this.
template <int FMT, int E>
__device__ __forceinline__ bool round_row(const RowParams& rp, const float (&s)[E],
                                          float (&r)[E], uint32_t (&k)[E])
{
    using F = Fmt<FMT>;
    const bool fast = __all_sync(0xffffffffu, rp.fast && !rp.clamp);
    if (fast) {
        const float2 inv2 = make_float2(rp.inv, rp.inv);
        const float2 m2 = make_float2(kMagic, kMagic);
        const float2 nm2 = make_float2(-kMagic, -kMagic);
        const float2 z2 = make_float2(rp.z, rp.z);
#pragma unroll
        for (int n = 0; n < E; n += 2) {
            float2 t = fma2(make_float2(s[n], s[n + 1]), inv2, m2);   // 1.5*2^23 + rint(s*inv)
            float2 rr = add2(t, nm2);          // rint(p), exact
            r[n] = rr.x; r[n + 1] = rr.y;
            if constexpr (F::sym) {
                k[n] = __float_as_uint(t.x);         // low bits: rint(p) two's complement
                k[n + 1] = __float_as_uint(t.y);
            } else {
                float2 u = add2(t, z2);        // 1.5*2^23 + q, exact
                k[n] = __float_as_uint(u.x);
                k[n + 1] = __float_as_uint(u.y);
            }
        }
    } else {
        // The scalar formulas verbatim.
#pragma unroll
        for (int n = 0; n < E; ++n) {
            const float rr = rint_prod(s[n], rp.inv);
            float c;
            if constexpr (F::sym) {
                c = fminf(fmaxf(rr, -F::qmax), F::qmax);
                r[n] = c;
            } else {
                c = fminf(__fadd_rn(rr, rp.z), F::qmax);
                r[n] = __fsub_rn(c, rp.z);
            }
            k[n] = (uint32_t)(int)c;
        }
    }
    return fast;
}

// The stored row as fp32: fl(r_n * Delta).
template <int E>
__device__ __forceinline__ void scale_row(float delta, const float (&r)[E], float (&s)[E])
{
    const float2 d2 = make_float2(delta, delta);
#pragma unroll
    for (int n = 0; n < E; n += 2) {
        float2 v = mul2(make_float2(r[n], r[n + 1]), d2);
        s[n] = v.x; s[n + 1] = v.y;
    }
}

// s'_n = fma(lambda, s_n, fl(dtx * B_n)).
template <int E>
__device__ __forceinline__ void update_row(float lam, float dtx, const float (&Bv)[E],
                                           float (&s)[E])
{
    const float2 l2 = make_float2(lam, lam);
    const float2 x2 = make_float2(dtx, dtx);
#pragma unroll
    for (int n = 0; n < E; n += 2) {
        float2 w = mul2(x2, make_float2(Bv[n], Bv[n + 1]));
        float2 v = fma2(l2, make_float2(s[n], s[n + 1]), w);
        s[n] = v.x; s[n + 1] = v.y;
    }
}

// sum_n C_n * v_n over the lane's entries (fp32, paired accumulators).
template <int E>
__device__ __forceinline__ float dot_row(const float (&Cv)[E], const float (&v)[E])
{
    float2 acc = make_float2(0.0f, 0.0f);
#pragma unroll
    for (int n = 0; n < E; n += 2)
        acc = fma2(make_float2(Cv[n], Cv[n + 1]), make_float2(v[n], v[n + 1]), acc);
    return __fadd_rn(acc.x, acc.y);
}

}  // namespace ssq
