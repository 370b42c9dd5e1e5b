// ssq_decode.cu -- dispatch of the fused decode-step kernel (the kernel is in
// ssq_decode_impl.cuh, its instantiations in ssq_decode_<format>.cu) and the
// tile geometry the host checks against.
#include "ssq_decode_impl.cuh"

namespace ssq {

void decode_tile_rows(int fmt, int d_state, int* rows_q, int* rows_f)
{
    const int eq = d_state >= kQuantE ? kQuantE : d_state;
    const int ef = d_state >= 32 ? 32 : d_state;
    *rows_q = kCThreads / (d_state / eq);
    *rows_f = kCThreads / (d_state / ef);
    (void)fmt;
}

bool decode_fits(int fmt, int d_state, int nheads, int ngroups)
{
    // B and C of every group plus the head tables must leave room for two
    // pipeline stages (of either region) within one CTA's shared memory
    int rq = 0, rf = 0;
    decode_tile_rows(fmt, d_state, &rq, &rf);
    const bool q = fmt >= SSQ_I8_SYM;
    const DecodeGeom g = decode_geom(2, rq, rf, d_state, 8, 4, q, true, d_state, nheads, ngroups);
    return g.smem_bytes <= 227 * 1024;
}

static cudaError_t launch_any(const PoolView& pv, const CallView& cv, int fmt, int mode,
                              cudaStream_t st)
{
    switch (fmt) {
    case SSQ_F32: return launch_decode_fmt<SSQ_F32>(pv, cv, mode, st);
    case SSQ_BF16: return launch_decode_fmt<SSQ_BF16>(pv, cv, mode, st);
    case SSQ_I8_SYM: return launch_decode_fmt<SSQ_I8_SYM>(pv, cv, mode, st);
    case SSQ_I8_ASYM: return launch_decode_fmt<SSQ_I8_ASYM>(pv, cv, mode, st);
    case SSQ_I4_SYM: return launch_decode_fmt<SSQ_I4_SYM>(pv, cv, mode, st);
    case SSQ_I4_ASYM: return launch_decode_fmt<SSQ_I4_ASYM>(pv, cv, mode, st);
    default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_decode(const PoolView& pv, const CallView& cv, int fmt, bool sr,
                          cudaStream_t st)
{
    // stochastic rounding changes only the integer formats
    return launch_any(pv, cv, fmt, sr ? kStochastic : kNearest, st);
}

cudaError_t launch_decode_diag(const PoolView& pv, const CallView& cv, int fmt, cudaStream_t st)
{
    return launch_any(pv, cv, fmt, kDiagnostics, st);
}

}  // namespace ssq
