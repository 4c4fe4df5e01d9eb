// simt_fwd_bf16.cu -- fwd instantiations of the FP32 CUDA-core path for __nv_bfloat16 inputs.
#include "simt_impl.cuh"

namespace ent {
cudaError_t simt_fwd_bf16(const FwdArgs& a, int d, int gm, cudaStream_t s) {
    return d == 64 ? simt_fwd_d<__nv_bfloat16, 64>(a, gm, s) : simt_fwd_d<__nv_bfloat16, 128>(a, gm, s);
}
}  // namespace ent
