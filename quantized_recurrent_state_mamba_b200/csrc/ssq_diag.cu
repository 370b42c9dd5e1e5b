// ssq_diag.cu -- diagnostics of a decode step, without changing the state.
//
// "ssm-state-quantization" README, Findings 4 and 5: an entry reverses when
// the rounding turns its change in the opposite direction to the step's
// input; the page reports how often this happens per decay band and how
// much of the rounding error the readout sees.  For every row this kernel
// evaluates the step
// the decode kernel would take (the same update, refit and rounding) and
// writes, per row, without touching the pool:
//   reversals   entries whose applied increment e + w, e = fl(deq - s') the
//               rounding error and w = fl(dt x) B_n the new input, has the
//               other sign than w (decided in fp32);
//   rev_err     sum over the reversed entries of C_n e_n;
//   tot_err     sum over all entries of C_n e_n;
//   signal      sum over all entries of C_n s'_n.
// fp rows (fp32 / bf16 formats, unmasked heads) are not rounded: zeros but
// the signal.  A row group of LPR lanes holds E = 32 entries per lane.
#include "ssq_common.cuh"
#include "ssq_params.h"

namespace ssq {

namespace {

template <int FMT, int N>
__global__ void __launch_bounds__(kThreads, 2)
diag_kernel(const __grid_constant__ PoolView pv, const __grid_constant__ CallView cv,
            float4* __restrict__ diag)
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
    const int P = pv.P, H = pv.H, G = pv.G;
    const int per_lb = cv.qtiles + cv.ftiles;

    for (long long t = blockIdx.x; t < cv.total_tiles; t += gridDim.x) {
        const long long lb = t / per_lb;
        const int k = (int)(t - lb * per_lb);
        const int l = (int)(lb / cv.batch);
        const int b = (int)(lb - (long long)l * cv.batch);
        const bool quant = k < cv.qtiles;
        const int rbase = (quant ? k : k - cv.qtiles) * cv.rows_per_tile;
        const int nrows = (quant ? pv.Hq : pv.Hf) * P;
        const int slot = cv.slot_idx ? __ldg(cv.slot_idx + b) : b;
        if (slot < 0 || slot >= pv.n_slots) {
            if (tid == 0) atomicOr(err, SSQ_DEVERR_SLOT);
            continue;
        }
        const int layer = cv.layer0 + l;
        const int r = rbase + grow;
        const bool active = r < nrows;
        const int rr = active ? r : rbase;
        const int hrl = rr / P;
        const int p = rr - hrl * P;
        const int h = pv.perm[(quant ? 0 : pv.Hq) + hrl];
        const int g = h / pv.hpg;
        const uint8_t* slot_base = pv.pool + pv.header_bytes + (long long)slot * pv.slot_bytes;

        // the stored row
        float s[E];
        bool qrow = false;
        if constexpr (F::quant) {
            if (quant) {
                qrow = true;
                const uint8_t* crow = slot_base + pv.codes_off
                                      + (long long)layer * pv.codes_layer_bytes
                                      + (long long)rr * (N * F::bits / 8) + j * CB;
                const uint8_t* mrow = slot_base + pv.meta_off
                                      + (long long)layer * pv.meta_layer_bytes
                                      + (long long)rr * F::meta_bytes;
                Chunk<CB> c;
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
            }
        }
        if (!qrow) {
            constexpr int EB = kBf16 ? 2 : 4;
            const uint8_t* frow = slot_base + pv.fp_off + (long long)layer * pv.fp_layer_bytes
                                  + ((long long)rr * N + j * E) * EB;
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
        }

        // the update, as the decode step forms it (B is dead once w is formed)
        const float xv = __ldg(cv.x + (lb * H + h) * P + p);
        const float dtv = __ldg(cv.dt + lb * H + h);
        const float lam = decay(dtv, __ldg(cv.A + (long long)l * H + h));
        const float dtx = __fmul_rn(dtv, xv);
        float w[E];
        {
            float Bv[E];
            load_f32<E>(Bv, cv.B + (lb * G + g) * N + j * E);
#pragma unroll
            for (int n = 0; n < E; ++n) {
                w[n] = __fmul_rn(dtx, Bv[n]);
                s[n] = __fmaf_rn(lam, s[n], w[n]);
            }
        }
        // rounding error e_n = fl(deq_n - s'_n) and the reversal flags (bit
        // n), before C is read
        float e[E];
        uint32_t rev_mask = 0u;
#pragma unroll
        for (int n = 0; n < E; ++n) e[n] = 0.0f;
        if constexpr (F::quant) {
            if (qrow) {
                // the refit and rounding of the decode step (warp-uniform
                // choice of path inside round_row)
                const RowParams rp = refit_row<FMT, E, LPR>(s);
                float rq[E];
                uint32_t kq[E];
                round_row<FMT, E>(rp, s, rq, kq);
#pragma unroll
                for (int n = 0; n < E; ++n) {
                    const float deq = __fmul_rn(rq[n], rp.delta);
                    e[n] = __fsub_rn(deq, s[n]);
                    const float inc = __fadd_rn(e[n], w[n]);
                    const bool reversed = (w[n] > 0.0f && inc < 0.0f) || (w[n] < 0.0f && inc > 0.0f);
                    rev_mask |= (reversed ? 1u : 0u) << n;
                }
            }
        }
        float Cv[E];
        load_f32<E>(Cv, cv.C + (lb * G + g) * N + j * E);
        float signal = 0.0f, tot = 0.0f, rev_err = 0.0f;
#pragma unroll
        for (int n = 0; n < E; ++n) {
            signal = __fmaf_rn(Cv[n], s[n], signal);
            tot = __fmaf_rn(Cv[n], e[n], tot);
            if ((rev_mask >> n) & 1u) rev_err = __fmaf_rn(Cv[n], e[n], rev_err);
        }
        int rev = __popc(rev_mask);
        signal = grp_sum<LPR>(signal);
        tot = grp_sum<LPR>(tot);
        rev_err = grp_sum<LPR>(rev_err);
        rev = (int)grp_sum<LPR>((float)rev);
        if (active && j == 0)
            diag[(lb * H + h) * P + p] = make_float4((float)rev, rev_err, tot, signal);
    }
}

template <int FMT, int N>
cudaError_t launch_diag_n(const PoolView& pv, const CallView& cv, float4* diag,
                          cudaStream_t st)
{
    auto kern = diag_kernel<FMT, N>;
    const int grid = grid_for((const void*)kern, kThreads, cv.total_tiles);
    if (grid <= 0) return cudaErrorInvalidConfiguration;
    kern<<<grid, kThreads, 0, st>>>(pv, cv, diag);
    return cudaGetLastError();
}

template <int FMT>
cudaError_t launch_diag_fmt(const PoolView& pv, const CallView& cv, float4* diag,
                            cudaStream_t st)
{
    switch (pv.N) {
    case 16: return launch_diag_n<FMT, 16>(pv, cv, diag, st);
    case 32: return launch_diag_n<FMT, 32>(pv, cv, diag, st);
    case 64: return launch_diag_n<FMT, 64>(pv, cv, diag, st);
    case 128: return launch_diag_n<FMT, 128>(pv, cv, diag, st);
    case 256: return launch_diag_n<FMT, 256>(pv, cv, diag, st);
    default: return cudaErrorInvalidValue;
    }
}

}  // namespace

cudaError_t launch_diag(const PoolView& pv, const CallView& cv, int fmt, float* diag,
                        cudaStream_t st)
{
    float4* d = reinterpret_cast<float4*>(diag);
    switch (fmt) {
    case SSQ_F32: return launch_diag_fmt<SSQ_F32>(pv, cv, d, st);
    case SSQ_BF16: return launch_diag_fmt<SSQ_BF16>(pv, cv, d, st);
    case SSQ_I8_SYM: return launch_diag_fmt<SSQ_I8_SYM>(pv, cv, d, st);
    case SSQ_I8_ASYM: return launch_diag_fmt<SSQ_I8_ASYM>(pv, cv, d, st);
    case SSQ_I4_SYM: return launch_diag_fmt<SSQ_I4_SYM>(pv, cv, d, st);
    case SSQ_I4_ASYM: return launch_diag_fmt<SSQ_I4_ASYM>(pv, cv, d, st);
    default: return cudaErrorInvalidValue;
    }
}

}  // namespace ssq
