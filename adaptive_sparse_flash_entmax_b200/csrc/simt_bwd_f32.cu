// simt_bwd_f32.cu -- bwd instantiations of the FP32 CUDA-core path for float inputs.
#include "simt_impl.cuh"

namespace ent {
cudaError_t simt_bwd_f32(const BwdArgs& a, int d, int gm, cudaStream_t s) {
    return d == 32 ? simt_bwd_d<float, 32>(a, gm, s)
           : d == 64 ? simt_bwd_d<float, 64>(a, gm, s) : simt_bwd_d<float, 128>(a, gm, s);
}
}  // namespace ent
