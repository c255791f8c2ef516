// NHWC tiled kernels: forward with a channel multiplier M (page "Incorrect
// stableHLO for grouped convolution gradient": a conv from C to C*M channels
// with groups = C).  A tile holds 32 output channels and the 32/M input
// channels they read; each lane's 4 output channels take their input values
// from one (M >= 4) or two (M = 2) input channels of the staged window (the
// kernel in dw_tiled_nhwc.cuh).  Input gradient (transposed mode): a tile
// holds 32 dx channels and stages their 32*M dy channels; a lane owns 4/M
// dx channels, whose 4 dy channels form one float4 (conflict-free 16-byte
// shared loads), and sums each dx channel's M products at the store.
// Other multipliers and shapes use the direct kernels.  Activations are
// float32, float16 or bfloat16 (one instantiation unit per type).
#pragma once

#include "dw_tiled_nhwc.cuh"

namespace dw {
namespace nhwc {

// (KH KW S D TR | THT TWT WX WY NS | VEC NO MINB CB MULT TA)
// float32: one CTA per SM (the 2-CTA register budget spills); 16-bit: two
template <int M, class TA>
using M33s1 = Cfg<3, 3, 1, 1, false, 2, 4, 8, 4, 4, 4, 0, sizeof(TA) == 4 ? 1 : 2, 32, M, TA>;
template <int M, class TA>
using M33s2 = Cfg<3, 3, 2, 1, false, 1, 2, 8, 4, 4, 4, 0, 2, 32, M, TA>;
template <int M, class TA>
using M55s1 = Cfg<5, 5, 1, 1, false, 2, 4, 8, 4, 2, 4, 2, 1, 32, M, TA>;

// transposed mode: a lane owns 4 / M dx channels (VEC = 2 for M = 2, 1 for
// M = 4), their 4 dy channels one float4 against one float4 of filters per tap
template <class TA> using MB33s1m2 = Cfg<3, 3, 1, 1, true, 2, 4, 4, 4, 3, 2, 2, 1, 32, 2, TA>;
template <class TA> using MB33s2m2 = Cfg<3, 3, 2, 1, true, 2, 4, 4, 4, 4, 2, 0, 1, 32, 2, TA>;
template <class TA> using MB33s1m4 = Cfg<3, 3, 1, 1, true, 2, 4, 2, 4, 3, 1, 2, 1, 32, 4, TA>;
template <class TA> using MB33s2m4 = Cfg<3, 3, 2, 1, true, 2, 4, 2, 4, 4, 1, 0, 1, 32, 4, TA>;

template <class TA>
dw_status_t mult_bwd_launch_t(const Problem& p, const void* in, const void* w, void* out,
                              cudaStream_t stream, int32_t* err, bool dry_run) {
    const Op op = OP_BWD_INPUT;
    if (p.kH != 3 || p.kW != 3 || p.dh != 1) return DW_ERR_UNSUPPORTED;
    if (p.sh == 1 && p.M == 2)
        return launch<MB33s1m2<TA>>(p, op, in, w, nullptr, out, stream, err, dry_run);
    if (p.sh == 1 && p.M == 4)
        return launch<MB33s1m4<TA>>(p, op, in, w, nullptr, out, stream, err, dry_run);
    if (p.sh == 2 && p.M == 2)
        return launch<MB33s2m2<TA>>(p, op, in, w, nullptr, out, stream, err, dry_run);
    if (p.sh == 2 && p.M == 4)
        return launch<MB33s2m4<TA>>(p, op, in, w, nullptr, out, stream, err, dry_run);
    return DW_ERR_UNSUPPORTED;
}

template <int M, class TA>
dw_status_t mult_pick(const Problem& p, const void* in, const void* w, const float* b,
                      void* out, cudaStream_t stream, int32_t* err, bool dry_run) {
    const Op op = OP_FWD;
    if (p.kH == 3 && p.kW == 3 && p.sh == 1 && p.dh == 1)
        return launch<M33s1<M, TA>>(p, op, in, w, b, out, stream, err, dry_run);
    if (p.kH == 3 && p.kW == 3 && p.sh == 2 && p.dh == 1)
        return launch<M33s2<M, TA>>(p, op, in, w, b, out, stream, err, dry_run);
    if (p.kH == 5 && p.kW == 5 && p.sh == 1 && p.dh == 1)
        return launch<M55s1<M, TA>>(p, op, in, w, b, out, stream, err, dry_run);
    return DW_ERR_UNSUPPORTED;
}

template <class TA>
dw_status_t mult_launch_t(const Problem& p, const void* in, const void* w, const float* b,
                          void* out, cudaStream_t stream, int32_t* err, bool dry_run) {
    if (p.M == 2) return mult_pick<2, TA>(p, in, w, b, out, stream, err, dry_run);
    if (p.M == 4) return mult_pick<4, TA>(p, in, w, b, out, stream, err, dry_run);
    return DW_ERR_UNSUPPORTED;
}

}  // namespace nhwc
}  // namespace dw
