// NHWC tiled kernels: float32 input-gradient instantiations (transposed mode
// of the kernel in dw_tiled_nhwc.cuh).
#include "dw_tiled_nhwc.cuh"

namespace dw {
namespace nhwc {

dw_status_t bwd_launch_f32(const Problem& p, const void* in, const void* w, void* out,
                           cudaStream_t stream, int32_t* err, bool dry_run) {
    return bwd_launch_t<float>(p, in, w, out, stream, err, dry_run);
}

}  // namespace nhwc
}  // namespace dw
