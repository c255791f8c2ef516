// NHWC tiled kernels with a channel multiplier: the float32 instantiations
// and the dispatch by activation type (kernels and configurations in
// dw_tiled_nhwc_mult.cuh).
#include "dw_tiled_nhwc_mult.cuh"

namespace dw {
namespace nhwc {

dw_status_t mult_bwd_launch(const Problem& p, const void* in, const void* w, void* out,
                            cudaStream_t stream, int32_t* err, bool dry_run) {
    if (p.atype == DW_F16) return mult_bwd_launch_f16(p, in, w, out, stream, err, dry_run);
    if (p.atype == DW_BF16) return mult_bwd_launch_bf16(p, in, w, out, stream, err, dry_run);
    return mult_bwd_launch_t<float>(p, in, w, out, stream, err, dry_run);
}

dw_status_t mult_launch(const Problem& p, const void* in, const void* w, const float* b,
                        void* out, cudaStream_t stream, int32_t* err, bool dry_run) {
    if (p.atype == DW_F16) return mult_launch_f16(p, in, w, b, out, stream, err, dry_run);
    if (p.atype == DW_BF16) return mult_launch_bf16(p, in, w, b, out, stream, err, dry_run);
    return mult_launch_t<float>(p, in, w, b, out, stream, err, dry_run);
}

}  // namespace nhwc
}  // namespace dw
