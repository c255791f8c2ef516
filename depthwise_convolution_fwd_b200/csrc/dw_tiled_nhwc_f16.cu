// NHWC tiled kernels with float16 activations: forward and input-gradient
// instantiations of the kernel in dw_tiled_nhwc.cuh.  Elements are widened
// to float32 on their way out of shared memory, every sum is the float32 sum
// of the float32 path, and each result is rounded once to float16 before its
// store; a pixel's 32 channels are 64 bytes, so a tile moves half the bytes.
#include "dw_tiled_nhwc.cuh"

namespace dw {
namespace nhwc {

dw_status_t fwd_launch_f16(const Problem& p, const void* in, const void* w, const float* b,
                           void* out, cudaStream_t stream, int32_t* err, bool dry_run) {
    return fwd_launch_t<__half>(p, in, w, b, out, stream, err, dry_run);
}

dw_status_t bwd_launch_f16(const Problem& p, const void* in, const void* w, void* out,
                           cudaStream_t stream, int32_t* err, bool dry_run) {
    return bwd_launch_t<__half>(p, in, w, out, stream, err, dry_run);
}

}  // namespace nhwc
}  // namespace dw
