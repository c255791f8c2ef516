// NHWC tiled kernels: the family's dispatcher and the float32 forward
// instantiations.  The kernel, its configurations and the launch code are in
// dw_tiled_nhwc.cuh; the other instantiations live in their own translation
// units so they compile in parallel.
#include "dw_tiled_nhwc.cuh"

namespace dw {
namespace nhwc {

dw_status_t fwd_launch_f32(const Problem& p, const void* in, const void* w, const float* b,
                           void* out, cudaStream_t stream, int32_t* err, bool dry_run) {
    return fwd_launch_t<float>(p, in, w, b, out, stream, err, dry_run);
}

}  // namespace nhwc

dw_status_t tiled_nhwc_launch(const Problem& p, Op op, const void* in, const void* w,
                              const float* b, void* out, cudaStream_t stream, int32_t* err,
                              bool dry_run) {
    using namespace nhwc;
    if (p.layout != DW_NHWC) return DW_ERR_UNSUPPORTED;
    // TMA needs 16-byte aligned bases and row strides (C elements a multiple
    // of 16 bytes); vector stores need an aligned output.
    if ((p.C * act_bytes(p.atype)) % 16 != 0) return DW_ERR_UNSUPPORTED;
    if ((reinterpret_cast<uintptr_t>(in) | reinterpret_cast<uintptr_t>(out)) & 15)
        return DW_ERR_UNSUPPORTED;
    if (p.sh != p.sw || p.dh != p.dw) return DW_ERR_UNSUPPORTED;
    if (p.N >= INT_MAX || p.H >= INT_MAX || p.W >= INT_MAX || p.Co >= INT_MAX)
        return DW_ERR_UNSUPPORTED;
    const bool f = op == OP_FWD;
    if (p.M != 1) {
        // channel multiplier tiles (any activation type); the rest runs on the
        // direct kernels
        return f ? mult_launch(p, in, w, b, out, stream, err, dry_run)
                 : mult_bwd_launch(p, in, w, out, stream, err, dry_run);
    }
    if (p.atype == DW_F16)
        return f ? fwd_launch_f16(p, in, w, b, out, stream, err, dry_run)
                 : bwd_launch_f16(p, in, w, out, stream, err, dry_run);
    if (p.atype == DW_BF16)
        return f ? fwd_launch_bf16(p, in, w, b, out, stream, err, dry_run)
                 : bwd_launch_bf16(p, in, w, out, stream, err, dry_run);
    return f ? fwd_launch_f32(p, in, w, b, out, stream, err, dry_run)
             : bwd_launch_f32(p, in, w, out, stream, err, dry_run);
}

}  // namespace dw
