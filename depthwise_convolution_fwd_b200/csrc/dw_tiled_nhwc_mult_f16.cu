// NHWC tiled kernels with a channel multiplier and float16 activations
// (kernels and configurations in dw_tiled_nhwc_mult.cuh; elements widen to
// float32 out of shared memory, each result is rounded once).
#include "dw_tiled_nhwc_mult.cuh"

namespace dw {
namespace nhwc {

dw_status_t mult_launch_f16(const Problem& p, const void* in, const void* w, const float* b,
                          void* out, cudaStream_t stream, int32_t* err, bool dry_run) {
    return mult_launch_t<__half>(p, in, w, b, out, stream, err, dry_run);
}

dw_status_t mult_bwd_launch_f16(const Problem& p, const void* in, const void* w, void* out,
                              cudaStream_t stream, int32_t* err, bool dry_run) {
    return mult_bwd_launch_t<__half>(p, in, w, out, stream, err, dry_run);
}

}  // namespace nhwc
}  // namespace dw
