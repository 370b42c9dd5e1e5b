// ssq_decode_i8s.cu -- the decode kernel for the int8 symmetric state format (one
// file per format, so the instantiations compile in parallel).
#include "ssq_decode_impl.cuh"

namespace ssq {

template <>
cudaError_t launch_decode_fmt<SSQ_I8_SYM>(const PoolView& pv, const CallView& cv, int mode,
                                 cudaStream_t st)
{
    return launch_mode<SSQ_I8_SYM>(pv, cv, mode, st);
}

}  // namespace ssq
