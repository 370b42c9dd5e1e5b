// ssq_quant.cu -- writing fp32 states into the packed pool and reading them
// back.
//
// ssq_quantize_rows is the hand-off point of "Mamba state quantization for
// inference" ("Mamba state quantization needs phase-aware benchmarks": the
// state a prefill ends with, kept in fp32, enters the packed cache
// once): each row gets its scale fitted and
// is rounded exactly as a decode step would round it ("ssm-state-quantization"
// README, Setup).  ssq_dequantize_rows decodes rows back to fp32.
#include "ssq_common.cuh"
#include "ssq_params.h"

namespace ssq {

namespace {

struct QTile {
    int l, b, slot;
    bool quant;
    int rbase, nrows;
};

__device__ __forceinline__ QTile make_qtile(const PoolView& pv, const CallView& cv,
                                            long long t)
{
    QTile tl;
    const int per_lb = cv.qtiles + cv.ftiles;
    const long long lb = t / per_lb;
    const int k = (int)(t - lb * per_lb);
    tl.l = (int)(lb / cv.batch);
    tl.b = (int)(lb - (long long)tl.l * cv.batch);
    tl.quant = k < cv.qtiles;
    tl.rbase = (tl.quant ? k : k - cv.qtiles) * cv.rows_per_tile;
    tl.nrows = (tl.quant ? pv.Hq : pv.Hf) * pv.P;
    tl.slot = cv.slot_idx ? __ldg(cv.slot_idx + tl.b) : tl.b;
    return tl;
}

template <int FMT, int N, bool kQuantize>
__global__ void __launch_bounds__(kThreads)
rows_kernel(const __grid_constant__ PoolView pv, const __grid_constant__ CallView cv)
{
    using S = Shape<N>;
    using F = Fmt<FMT>;
    constexpr int E = S::E, LPR = S::LPR;
    constexpr int CB = F::quant ? E * F::bits / 8 : 4;
    constexpr bool kBf16 = (FMT == SSQ_BF16);

    uint32_t* err = reinterpret_cast<uint32_t*>(pv.pool);
    const int tid = threadIdx.x;
    const int grow = tid / LPR;
    const int j = tid % LPR;
    const int P = pv.P, H = pv.H;

    for (long long t = blockIdx.x; t < cv.total_tiles; t += gridDim.x) {
        const QTile tl = make_qtile(pv, cv, t);
        if (tl.slot < 0 || tl.slot >= pv.n_slots) {
            if (tid == 0) atomicOr(err, SSQ_DEVERR_SLOT);
            continue;
        }
        const long long lb = (long long)tl.l * cv.batch + tl.b;
        const int layer = cv.layer0 + tl.l;
        const int r = tl.rbase + grow;
        const bool active = r < tl.nrows;
        const int rr = active ? r : tl.rbase;
        const int hrl = rr / P;
        const int p = rr - hrl * P;
        const int h = pv.perm[(tl.quant ? 0 : pv.Hq) + hrl];
        const long long srow = ((lb * H + h) * P + p) * N + j * E;  // natural order
        uint8_t* slot_base = pv.pool + pv.header_bytes + (long long)tl.slot * pv.slot_bytes;

        bool done = false;
        if constexpr (F::quant) {
          if (tl.quant) {
            done = true;
            uint8_t* crow = slot_base + pv.codes_off + (long long)layer * pv.codes_layer_bytes
                            + (long long)rr * (N * F::bits / 8) + j * CB;
            uint8_t* mrow = slot_base + pv.meta_off + (long long)layer * pv.meta_layer_bytes
                            + (long long)rr * F::meta_bytes;
            float s[E];
            Chunk<CB> c;
            if constexpr (kQuantize) {
                load_f32<E>(s, cv.S_in + srow);
                const RowParams rp = refit_row<FMT, E, LPR>(s);
                float rq[E];
                uint32_t k[E];
                round_row<FMT, E>(rp, s, rq, k);
                pack_codes<FMT, E>(k, c);
                if (active) {
                    store_chunk<CB>(crow, c);
                    if (j == 0) {
                        if constexpr (F::sym) {
                            *reinterpret_cast<float*>(mrow) = rp.delta;
                        } else {
                            *reinterpret_cast<float2*>(mrow) = make_float2(rp.delta, rp.z);
                        }
                        if (!rp.finite) atomicOr(err, SSQ_DEVERR_NONFINITE);
                    }
                }
            } else {
                load_chunk<CB>(c, crow);
                float delta0, z0 = 0.0f;
                if constexpr (F::sym) {
                    delta0 = *reinterpret_cast<const float*>(mrow);
                } else {
                    const float2 m = *reinterpret_cast<const float2*>(mrow);
                    delta0 = m.x;
                    z0 = m.y;
                }
                decode_row<FMT, E>(c, delta0, z0, s);
                if (active) {
#pragma unroll
                    for (int i = 0; i < E / 4; ++i)
                        reinterpret_cast<float4*>(cv.S_out + srow)[i] =
                            make_float4(s[4 * i], s[4 * i + 1], s[4 * i + 2], s[4 * i + 3]);
                }
            }
          }
        }
        if (!done && active) {  // fp rows: no shuffles on this path
            constexpr int EB = kBf16 ? 2 : 4;
            uint8_t* frow = slot_base + pv.fp_off + (long long)layer * pv.fp_layer_bytes
                            + ((long long)rr * N + j * E) * EB;
            float s[E];
            if constexpr (kQuantize) {
                load_f32<E>(s, cv.S_in + srow);
                if constexpr (kBf16) {
                    Chunk<E * 2> c;
#pragma unroll
                    for (int n = 0; n < E; n += 2) {
                        c.w[n / 2] = (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(s[n]))
                                     | ((uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(s[n + 1])) << 16);
                    }
                    store_chunk<E * 2>(frow, c);
                } else {
                    Chunk<E * 4> c;
#pragma unroll
                    for (int n = 0; n < E; ++n) c.w[n] = __float_as_uint(s[n]);
                    store_chunk<E * 4>(frow, c);
                }
            } else {
                if constexpr (kBf16) {
                    Chunk<E * 2> c;
                    load_chunk<E * 2>(c, frow);
#pragma unroll
                    for (int n = 0; n < E; ++n)
                        s[n] = __uint_as_float((c.w[n / 2] >> (16 * (n % 2))) << 16);
                } else {
                    Chunk<E * 4> c;
                    load_chunk<E * 4>(c, frow);
#pragma unroll
                    for (int n = 0; n < E; ++n) s[n] = __uint_as_float(c.w[n]);
                }
#pragma unroll
                for (int i = 0; i < E / 4; ++i)
                    reinterpret_cast<float4*>(cv.S_out + srow)[i] =
                        make_float4(s[4 * i], s[4 * i + 1], s[4 * i + 2], s[4 * i + 3]);
            }
        }
    }
}

template <int FMT, int N, bool Q>
cudaError_t launch_rows_n(const PoolView& pv, const CallView& cv, cudaStream_t st)
{
    auto kern = rows_kernel<FMT, N, Q>;
    const int grid = grid_for((const void*)kern, kThreads, cv.total_tiles);
    if (grid <= 0) return cudaErrorInvalidConfiguration;
    kern<<<grid, kThreads, 0, st>>>(pv, cv);
    return cudaGetLastError();
}

template <int FMT, bool Q>
cudaError_t launch_rows_fmt(const PoolView& pv, const CallView& cv, cudaStream_t st)
{
    switch (pv.N) {
    case 16: return launch_rows_n<FMT, 16, Q>(pv, cv, st);
    case 32: return launch_rows_n<FMT, 32, Q>(pv, cv, st);
    case 64: return launch_rows_n<FMT, 64, Q>(pv, cv, st);
    case 128: return launch_rows_n<FMT, 128, Q>(pv, cv, st);
    case 256: return launch_rows_n<FMT, 256, Q>(pv, cv, st);
    default: return cudaErrorInvalidValue;
    }
}

template <bool Q>
cudaError_t launch_rows(const PoolView& pv, const CallView& cv, int fmt, cudaStream_t st)
{
    switch (fmt) {
    case SSQ_F32: return launch_rows_fmt<SSQ_F32, Q>(pv, cv, st);
    case SSQ_BF16: return launch_rows_fmt<SSQ_BF16, Q>(pv, cv, st);
    case SSQ_I8_SYM: return launch_rows_fmt<SSQ_I8_SYM, Q>(pv, cv, st);
    case SSQ_I8_ASYM: return launch_rows_fmt<SSQ_I8_ASYM, Q>(pv, cv, st);
    case SSQ_I4_SYM: return launch_rows_fmt<SSQ_I4_SYM, Q>(pv, cv, st);
    case SSQ_I4_ASYM: return launch_rows_fmt<SSQ_I4_ASYM, Q>(pv, cv, st);
    default: return cudaErrorInvalidValue;
    }
}

}  // namespace

cudaError_t launch_quantize(const PoolView& pv, const CallView& cv, int fmt,
                            cudaStream_t st)
{
    return launch_rows<true>(pv, cv, fmt, st);
}

cudaError_t launch_dequantize(const PoolView& pv, const CallView& cv, int fmt,
                              cudaStream_t st)
{
    return launch_rows<false>(pv, cv, fmt, st);
}

}  // namespace ssq
