// NCHW tiled kernels with bfloat16 activations: instantiations of the kernels
// in dw_tiled_nchw.cuh (4-element vectors of 8 bytes along W, float32 sums,
// one rounding per result).
#include "dw_tiled_nchw.cuh"

namespace dw {
namespace nchw {

dw_status_t nchw_launch_bf16(const Problem& p, Op op, const void* in, const void* w,
                            const float* b, void* out, cudaStream_t stream, int32_t* err,
                            bool dry_run) {
    return nchw_launch_t<__nv_bfloat16>(p, op, in, w, b, out, stream, err, dry_run);
}

}  // namespace nchw
}  // namespace dw
