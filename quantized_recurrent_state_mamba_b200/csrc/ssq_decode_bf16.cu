// ssq_decode_bf16.cu -- the decode kernel for the bf16 state format (one
// file per format, so the instantiations compile in parallel).
#include "ssq_decode_impl.cuh"

namespace ssq {

template <>
cudaError_t launch_decode_fmt<SSQ_BF16>(const PoolView& pv, const CallView& cv, int mode,
                                 cudaStream_t st)
{
    return launch_mode<SSQ_BF16>(pv, cv, mode, st);
}

}  // namespace ssq
