// ssq_decode_i4a.cu -- the decode kernel for the int4 asymmetric state format (one
// file per format, so the instantiations compile in parallel).
#include "ssq_decode_impl.cuh"

namespace ssq {

template <>
cudaError_t launch_decode_fmt<SSQ_I4_ASYM>(const PoolView& pv, const CallView& cv, int mode,
                                 cudaStream_t st)
{
    return launch_mode<SSQ_I4_ASYM>(pv, cv, mode, st);
}

}  // namespace ssq
