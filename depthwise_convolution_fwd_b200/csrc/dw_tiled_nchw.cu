// NCHW tiled kernels: the family's dispatcher and the float32 instantiations
// (the kernels, configurations and launch code are in dw_tiled_nchw.cuh).
#include "dw_tiled_nchw.cuh"

namespace dw {
namespace nchw {

dw_status_t nchw_launch_f32(const Problem& p, Op op, const void* in, const void* w,
                            const float* b, void* out, cudaStream_t stream, int32_t* err,
                            bool dry_run) {
    return nchw_launch_t<float>(p, op, in, w, b, out, stream, err, dry_run);
}

}  // namespace nchw

dw_status_t tiled_nchw_launch(const Problem& p, Op op, const void* in, const void* w,
                              const float* b, void* out, cudaStream_t stream, int32_t* err,
                              bool dry_run) {
    using namespace nchw;
    if (p.layout != DW_NCHW) return DW_ERR_UNSUPPORTED;
    const int64_t Win = op == OP_FWD ? p.W : p.Wo;
    // TMA row stride: a multiple of 16 bytes
    if ((Win * act_bytes(p.atype)) % 16 != 0) return DW_ERR_UNSUPPORTED;
    if ((reinterpret_cast<uintptr_t>(in) | reinterpret_cast<uintptr_t>(out)) & 15)
        return DW_ERR_UNSUPPORTED;
    if (p.N >= INT_MAX || p.H >= INT_MAX || p.W >= INT_MAX || p.C >= INT_MAX ||
        p.Ho >= INT_MAX || p.Wo >= INT_MAX)
        return DW_ERR_UNSUPPORTED;
    if (p.atype == DW_F16) return nchw_launch_f16(p, op, in, w, b, out, stream, err, dry_run);
    if (p.atype == DW_BF16) return nchw_launch_bf16(p, op, in, w, b, out, stream, err, dry_run);
    return nchw_launch_f32(p, op, in, w, b, out, stream, err, dry_run);
}

}  // namespace dw
