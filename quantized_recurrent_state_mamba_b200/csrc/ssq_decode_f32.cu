// ssq_decode_f32.cu -- the decode kernel for the fp32 state format (one
// file per format, so the instantiations compile in parallel).
#include "ssq_decode_impl.cuh"

namespace ssq {

template <>
cudaError_t launch_decode_fmt<SSQ_F32>(const PoolView& pv, const CallView& cv, int mode,
                                 cudaStream_t st)
{
    return launch_mode<SSQ_F32>(pv, cv, mode, st);
}

}  // namespace ssq
