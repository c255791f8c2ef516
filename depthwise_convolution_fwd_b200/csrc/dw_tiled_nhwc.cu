// NHWC tiled kernels: forward instantiations and the family's dispatcher.
// The kernel, its configuration template and the launch code are in
// dw_tiled_nhwc.cuh; the input-gradient and channel-multiplier
// instantiations live in their own translation units so they compile in
// parallel.
#include "dw_tiled_nhwc.cuh"

namespace dw {
namespace nhwc {

// Instantiated configurations (KH KW S D TR | THT TWT WX WY NS [VEC NO MINB CB]);
// shared memory = NS input stages + NO output staging buffers <= 227 KB.
using F33s1 = Cfg<3, 3, 1, 1, false, 2, 4, 8, 4, 4, 4, 0, 2>;
using F33s1s = Cfg<3, 3, 1, 1, false, 2, 4, 4, 2, 4, 1, 2, 2>;
using F33s2 = Cfg<3, 3, 2, 1, false, 1, 2, 8, 4, 4, 4, 0, 2>;
using F33d2 = Cfg<3, 3, 1, 2, false, 2, 4, 8, 4, 2>;
using F33d3 = Cfg<3, 3, 1, 3, false, 2, 4, 8, 4, 2>;
using F55s1 = Cfg<5, 5, 1, 1, false, 2, 4, 8, 4, 2>;
using F55s1s = Cfg<5, 5, 1, 1, false, 2, 4, 4, 2, 4, 1, 2, 2>;
using F1x3 = Cfg<1, 3, 1, 1, false, 1, 8, 16, 1, 4>;
using F1x5 = Cfg<1, 5, 1, 1, false, 1, 8, 16, 1, 4>;
using F1x7 = Cfg<1, 7, 1, 1, false, 1, 8, 16, 1, 4>;
using F1x15 = Cfg<1, 15, 1, 1, false, 1, 16, 8, 1, 4, 1>;
using F1x31 = Cfg<1, 31, 1, 1, false, 1, 16, 2, 1, 4, 1, 2, 1, 128>;
using F77s1 = Cfg<7, 7, 1, 1, false, 2, 4, 4, 2, 3, 1>;

dw_status_t fwd_launch(const Problem& p, const float* in, const void* w, const float* b,
                       float* out, cudaStream_t stream, int32_t* err, bool dry_run) {
    const int S = p.sh, D = p.dh;
    const Op op = OP_FWD;
#define DW_ONE(FC) return launch<FC>(p, op, in, w, b, out, stream, err, dry_run);
#define DW_TWO(FC, FCS) return launch_pick<FC, FCS>(p, op, in, w, b, out, stream, err, dry_run);
    if (p.kH == 3 && p.kW == 3 && S == 1 && D == 1) DW_TWO(F33s1, F33s1s)
    if (p.kH == 3 && p.kW == 3 && S == 2 && D == 1) DW_ONE(F33s2)
    if (p.kH == 3 && p.kW == 3 && S == 1 && D == 2) DW_ONE(F33d2)
    if (p.kH == 3 && p.kW == 3 && S == 1 && D == 3) DW_ONE(F33d3)
    if (p.kH == 5 && p.kW == 5 && S == 1 && D == 1) DW_TWO(F55s1, F55s1s)
    if (p.kH == 7 && p.kW == 7 && S == 1 && D == 1) DW_ONE(F77s1)
    if (p.kH == 1 && S == 1 && D == 1) {
        if (p.kW == 3) DW_ONE(F1x3)
        if (p.kW == 5) DW_ONE(F1x5)
        if (p.kW == 7) DW_ONE(F1x7)
        if (p.kW == 15) DW_ONE(F1x15)
        if (p.kW == 31) DW_ONE(F1x31)
    }
#undef DW_ONE
#undef DW_TWO
    return DW_ERR_UNSUPPORTED;
}

}  // namespace nhwc

dw_status_t tiled_nhwc_launch(const Problem& p, Op op, const float* in, const void* w,
                              const float* b, float* out, cudaStream_t stream, int32_t* err,
                              bool dry_run) {
    if (p.layout != DW_NHWC) return DW_ERR_UNSUPPORTED;
    // TMA needs 16-byte aligned base and row strides; float4 stores need an
    // aligned output.
    if (p.C % 4 != 0) return DW_ERR_UNSUPPORTED;
    if ((reinterpret_cast<uintptr_t>(in) | reinterpret_cast<uintptr_t>(out)) & 15)
        return DW_ERR_UNSUPPORTED;
    if (p.sh != p.sw || p.dh != p.dw) return DW_ERR_UNSUPPORTED;
    if (p.N >= INT_MAX || p.H >= INT_MAX || p.W >= INT_MAX || p.Co >= INT_MAX)
        return DW_ERR_UNSUPPORTED;
    if (op == OP_FWD)
        return p.M == 1 ? nhwc::fwd_launch(p, in, w, b, out, stream, err, dry_run)
                        : nhwc::mult_launch(p, in, w, b, out, stream, err, dry_run);
    if (p.M != 1) return DW_ERR_UNSUPPORTED;  // multiplier input gradient: direct kernel
    return nhwc::bwd_launch(p, in, w, out, stream, err, dry_run);
}

}  // namespace dw
