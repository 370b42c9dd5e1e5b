// ssq_decode.cu -- the fused decode-step kernel.
//
// One launch updates the state of nl layers x batch requests by one token:
// read the packed row, decode, apply the recurrence in fp32, refit the row
// scale, requantize, write the packed row and its metadata back, and read y
// from the newly stored row -- the single fused pass that "Mamba state
// quantization for inference" describes for a low-bit state ("reconstructs
// the low tier, computes the recurrence in FP32, derives new quantization
// parameters, and writes the packed state back"), with the quantizer of
// "ssm-state-quantization" README, Setup.
//
// Work decomposition: a tile is up to rows_per_tile consecutive rows of one
// region (quantized or fp) of one (layer, request); tiles are distributed
// over a grid-stride loop.  A row is owned by LPR lanes (E entries each).
// The decay lambda of each head in a tile is computed once (exp in double)
// and shared through shared memory.
#include "ssq_common.cuh"
#include "ssq_params.h"

namespace ssq {

namespace {

template <int N>
struct TileHeads {
    static constexpr int RPT = kThreads / Shape<N>::LPR;
    static constexpr int kMax = RPT + 2;
};

// Per-tile bookkeeping, identical in every thread of the block.
struct Tile {
    int l, b, slot;
    bool quant;      // quantized region
    int rbase;       // first region row of the tile
    int nrows;       // rows in the region (Hq*P or Hf*P)
    int hr0;         // first region head touched by the tile
};

__device__ __forceinline__ Tile make_tile(const PoolView& pv, const CallView& cv,
                                          long long t)
{
    Tile tl;
    const int per_lb = cv.qtiles + cv.ftiles;
    const long long lb = t / per_lb;
    const int k = (int)(t - lb * per_lb);
    tl.l = (int)(lb / cv.batch);
    tl.b = (int)(lb - (long long)tl.l * cv.batch);
    tl.quant = k < cv.qtiles;
    const int kk = tl.quant ? k : k - cv.qtiles;
    tl.rbase = kk * cv.rows_per_tile;
    tl.nrows = (tl.quant ? pv.Hq : pv.Hf) * pv.P;
    tl.hr0 = tl.rbase / pv.P;
    tl.slot = cv.slot_idx ? __ldg(cv.slot_idx + tl.b) : tl.b;
    return tl;
}

template <int FMT, int N>
__global__ void __launch_bounds__(kThreads)
decode_kernel(const __grid_constant__ PoolView pv,
              const __grid_constant__ CallView cv)
{
    using S = Shape<N>;
    using F = Fmt<FMT>;
    constexpr int E = S::E, LPR = S::LPR;
    constexpr int CB = F::quant ? E * F::bits / 8 : 4;  // code bytes per lane
    constexpr bool kBf16 = (FMT == SSQ_BF16);

    __shared__ float s_lam[TileHeads<N>::kMax];
    __shared__ float s_dt[TileHeads<N>::kMax];

    uint32_t* err = reinterpret_cast<uint32_t*>(pv.pool);
    const int tid = threadIdx.x;
    const int grow = tid / LPR;     // row within the tile
    const int j = tid % LPR;        // lane within the row group
    const int P = pv.P, H = pv.H, G = pv.G;

    for (long long t = blockIdx.x; t < cv.total_tiles; t += gridDim.x) {
        const Tile tl = make_tile(pv, cv, t);
        if (tl.slot < 0 || tl.slot >= pv.n_slots) {
            if (tid == 0) atomicOr(err, SSQ_DEVERR_SLOT);
            continue;  // block-uniform
        }
        const long long lb = (long long)tl.l * cv.batch + tl.b;
        const int layer = cv.layer0 + tl.l;
        const int regbase = tl.quant ? 0 : pv.Hq;

        // lambda and dt of every head this tile touches
        const int hr_last = min((tl.rbase + cv.rows_per_tile - 1) / P,
                                tl.nrows / P - 1);
        if (tid <= hr_last - tl.hr0) {
            const int h = pv.perm[regbase + tl.hr0 + tid];
            const float dtv = __ldg(cv.dt + lb * H + h);
            const float Av = __ldg(cv.A + (long long)tl.l * H + h);
            s_dt[tid] = dtv;
            s_lam[tid] = decay(dtv, Av);
        }
        __syncthreads();

        const int r = tl.rbase + grow;
        const bool active = r < tl.nrows;
        const int rr = active ? r : tl.rbase;     // inactive rows shadow a real one
        const int hrl = rr / P;
        const int p = rr - hrl * P;
        const int h = pv.perm[regbase + hrl];
        const int g = h / pv.hpg;
        const float lam = s_lam[hrl - tl.hr0];
        const float dtv = s_dt[hrl - tl.hr0];
        const float xv = __ldg(cv.x + lb * H * P + (long long)h * P + p);
        const float Dv = __ldg(cv.D + (long long)tl.l * H + h);
        const float dtx = __fmul_rn(dtv, xv);
        const float* Bp = cv.B + (lb * G + g) * N + j * E;
        const float* Cp = cv.C + (lb * G + g) * N + j * E;
        uint8_t* slot_base = pv.pool + pv.header_bytes + (long long)tl.slot * pv.slot_bytes;

        float Bv[E], s[E];
        load_f32<E>(Bv, Bp);

        float ysum;
        if constexpr (F::quant) {
            if (tl.quant) {
                uint8_t* crow = slot_base + pv.codes_off + (long long)layer * pv.codes_layer_bytes
                                + (long long)rr * (N * F::bits / 8) + j * CB;
                uint8_t* mrow = slot_base + pv.meta_off + (long long)layer * pv.meta_layer_bytes
                                + (long long)rr * F::meta_bytes;
                Chunk<CB> c;
                load_chunk<CB>(c, crow);
                float delta0, z0 = 0.0f;
                if constexpr (F::sym) {
                    delta0 = __ldcs(reinterpret_cast<const float*>(mrow));
                } else {
                    const float2 m = __ldcs(reinterpret_cast<const float2*>(mrow));
                    delta0 = m.x;
                    z0 = m.y;
                }
                decode_row<FMT, E>(c, delta0, z0, s);
                update_row<E>(lam, dtx, Bv, s);
                const RowParams rp = refit_row<FMT, E, LPR>(s);
                float rq[E];
                uint32_t k[E];
                round_row<FMT, E>(rp, s, rq, k, pv.neg_zero);
                pack_codes<FMT, E>(k, c);
                float Cv[E];
                load_f32<E>(Cv, Cp);
                if (rp.fast && !rp.clamp) {
                    // y = Delta * sum_n C_n (q_n - z): the stored row read back
                    ysum = __fmul_rn(rp.delta, grp_sum<LPR>(dot_row<E>(Cv, rq)));
                } else {
                    float sv[E];
                    scale_row<E>(rp.delta, rq, sv);
                    ysum = grp_sum<LPR>(dot_row<E>(Cv, sv));
                }
                if (active) {
                    store_chunk<CB>(crow, c);
                    if (j == 0) {
                        if constexpr (F::sym) {
                            __stcs(reinterpret_cast<float*>(mrow), rp.delta);
                        } else {
                            __stcs(reinterpret_cast<float2*>(mrow), make_float2(rp.delta, rp.z));
                        }
                        if (!rp.finite) atomicOr(err, SSQ_DEVERR_NONFINITE);
                    }
                }
            }
        }
        if (!F::quant || !tl.quant) {
            // fp row: fp32 state (bf16 for the bf16 format)
            constexpr int EB = kBf16 ? 2 : 4;
            uint8_t* frow = slot_base + pv.fp_off + (long long)layer * pv.fp_layer_bytes
                            + ((long long)rr * N + j * E) * EB;
            if constexpr (kBf16) {
                Chunk<E * 2> c;
                load_chunk<E * 2>(c, frow);
#pragma unroll
                for (int n = 0; n < E; ++n)
                    s[n] = __uint_as_float((c.w[n / 2] >> (16 * (n % 2))) << 16);
                update_row<E>(lam, dtx, Bv, s);
#pragma unroll
                for (int n = 0; n < E; n += 2) {
                    const __nv_bfloat16 a = __float2bfloat16_rn(s[n]);
                    const __nv_bfloat16 b2 = __float2bfloat16_rn(s[n + 1]);
                    c.w[n / 2] = (uint32_t)__bfloat16_as_ushort(a)
                                 | ((uint32_t)__bfloat16_as_ushort(b2) << 16);
                    s[n] = __bfloat162float(a);
                    s[n + 1] = __bfloat162float(b2);
                }
                if (active) store_chunk<E * 2>(frow, c);
            } else {
                Chunk<E * 4> c;
                load_chunk<E * 4>(c, frow);
#pragma unroll
                for (int n = 0; n < E; ++n) s[n] = __uint_as_float(c.w[n]);
                update_row<E>(lam, dtx, Bv, s);
#pragma unroll
                for (int n = 0; n < E; ++n) c.w[n] = __float_as_uint(s[n]);
                if (active) store_chunk<E * 4>(frow, c);
            }
            float Cv[E];
            load_f32<E>(Cv, Cp);
            ysum = grp_sum<LPR>(dot_row<E>(Cv, s));
        }
        if (active && j == 0) {
            const float yv = __fadd_rn(ysum, __fmul_rn(Dv, xv));
            __stcs(cv.y + lb * H * P + (long long)h * P + p, yv);
        }
        __syncthreads();  // s_lam / s_dt are rewritten by the next tile
    }
}

template <int FMT, int N>
cudaError_t launch_n(const PoolView& pv, const CallView& cv, cudaStream_t st)
{
    auto kern = decode_kernel<FMT, N>;
    const int grid = grid_for((const void*)kern, kThreads, cv.total_tiles);
    if (grid <= 0) return cudaErrorInvalidConfiguration;
    kern<<<grid, kThreads, 0, st>>>(pv, cv);
    return cudaGetLastError();
}

template <int FMT>
cudaError_t launch_fmt(const PoolView& pv, const CallView& cv, cudaStream_t st)
{
    switch (pv.N) {
    case 16: return launch_n<FMT, 16>(pv, cv, st);
    case 32: return launch_n<FMT, 32>(pv, cv, st);
    case 64: return launch_n<FMT, 64>(pv, cv, st);
    case 128: return launch_n<FMT, 128>(pv, cv, st);
    case 256: return launch_n<FMT, 256>(pv, cv, st);
    default: return cudaErrorInvalidValue;
    }
}

}  // namespace

cudaError_t launch_decode(const PoolView& pv, const CallView& cv, int fmt,
                          cudaStream_t st)
{
    switch (fmt) {
    case SSQ_F32: return launch_fmt<SSQ_F32>(pv, cv, st);
    case SSQ_BF16: return launch_fmt<SSQ_BF16>(pv, cv, st);
    case SSQ_I8_SYM: return launch_fmt<SSQ_I8_SYM>(pv, cv, st);
    case SSQ_I8_ASYM: return launch_fmt<SSQ_I8_ASYM>(pv, cv, st);
    case SSQ_I4_SYM: return launch_fmt<SSQ_I4_SYM>(pv, cv, st);
    case SSQ_I4_ASYM: return launch_fmt<SSQ_I4_ASYM>(pv, cv, st);
    default: return cudaErrorInvalidValue;
    }
}

}  // namespace ssq
