// NHWC tiled kernels: input-gradient instantiations (transposed mode of the
// kernel in dw_tiled_nhwc.cuh).
#include "dw_tiled_nhwc.cuh"

namespace dw {
namespace nhwc {

// (KH KW S D TR | THT TWT WX WY NS [VEC NO MINB CB])
using B33s1 = Cfg<3, 3, 1, 1, true, 2, 4, 8, 4, 4, 4, 0, 2>;
using B33s1s = Cfg<3, 3, 1, 1, true, 2, 4, 4, 2, 4, 1, 2, 2>;
using B33s2 = Cfg<3, 3, 2, 1, true, 4, 4, 8, 4, 4>;
using B33s2s = Cfg<3, 3, 2, 1, true, 2, 2, 8, 4, 4>;
using B33d2 = Cfg<3, 3, 1, 2, true, 2, 4, 8, 4, 2>;
using B33d3 = Cfg<3, 3, 1, 3, true, 2, 4, 8, 4, 2>;
using B55s1 = Cfg<5, 5, 1, 1, true, 2, 4, 8, 4, 2>;
using B55s1s = Cfg<5, 5, 1, 1, true, 2, 4, 4, 2, 4, 1, 2, 2>;
using B1x3 = Cfg<1, 3, 1, 1, true, 1, 8, 16, 1, 4>;
using B1x5 = Cfg<1, 5, 1, 1, true, 1, 8, 16, 1, 4>;
using B1x7 = Cfg<1, 7, 1, 1, true, 1, 8, 16, 1, 4>;
using B1x15 = Cfg<1, 15, 1, 1, true, 1, 16, 8, 1, 4, 1>;
using B1x31 = Cfg<1, 31, 1, 1, true, 1, 16, 2, 1, 4, 1, 2, 1, 128>;
using B77s1 = Cfg<7, 7, 1, 1, true, 2, 4, 4, 2, 3, 1>;

dw_status_t bwd_launch(const Problem& p, const float* in, const void* w, float* out,
                       cudaStream_t stream, int32_t* err, bool dry_run) {
    const int S = p.sh, D = p.dh;
    const Op op = OP_BWD_INPUT;
#define DW_ONE(BC) return launch<BC>(p, op, in, w, nullptr, out, stream, err, dry_run);
#define DW_TWO(BC, BCS) return launch_pick<BC, BCS>(p, op, in, w, nullptr, out, stream, err, dry_run);
    if (p.kH == 3 && p.kW == 3 && S == 1 && D == 1) DW_TWO(B33s1, B33s1s)
    if (p.kH == 3 && p.kW == 3 && S == 2 && D == 1) DW_TWO(B33s2, B33s2s)
    if (p.kH == 3 && p.kW == 3 && S == 1 && D == 2) DW_ONE(B33d2)
    if (p.kH == 3 && p.kW == 3 && S == 1 && D == 3) DW_ONE(B33d3)
    if (p.kH == 5 && p.kW == 5 && S == 1 && D == 1) DW_TWO(B55s1, B55s1s)
    if (p.kH == 7 && p.kW == 7 && S == 1 && D == 1) DW_ONE(B77s1)
    if (p.kH == 1 && S == 1 && D == 1) {
        if (p.kW == 3) DW_ONE(B1x3)
        if (p.kW == 5) DW_ONE(B1x5)
        if (p.kW == 7) DW_ONE(B1x7)
        if (p.kW == 15) DW_ONE(B1x15)
        if (p.kW == 31) DW_ONE(B1x31)
    }
#undef DW_ONE
#undef DW_TWO
    return DW_ERR_UNSUPPORTED;
}

}  // namespace nhwc
}  // namespace dw
