// simt_fwd_f32.cu -- fwd instantiations of the FP32 CUDA-core path for float inputs.
#include "simt_impl.cuh"

namespace ent {
cudaError_t simt_fwd_f32(const FwdArgs& a, int d, int gm, cudaStream_t s) {
    return d == 32 ? simt_fwd_d<float, 32>(a, gm, s)
           : d == 64 ? simt_fwd_d<float, 64>(a, gm, s) : simt_fwd_d<float, 128>(a, gm, s);
}
}  // namespace ent
