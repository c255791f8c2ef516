// Direct kernels: one thread per output element, any layout, stride,
// dilation, padding, channel count or pointer alignment.  They are the
// fallback behind the tiled kernels and the DW_ALGO_DIRECT choice.
//
// Forward (page "LeanMlir Proofs/Architectures/Depthwise", section
// "Depthwise conv2d forward"): y = (sum over taps in kh-major, kw-minor
// order of x*W, float32 FMA) + b, with the stride and dilation applied in the
// input index (no decimation pass).  Input gradient (sections "Closed-form
// input gradient ... direct formula" and the stride-2 input-VJP sections):
// each dx element gathers the taps whose forward read lands on it, i.e. kh
// with hi + pt - kh*dh a non-negative multiple of sh below Ho*sh.
// Channel multiplier M (page "Incorrect stableHLO for grouped convolution
// gradient": groups = C, C*M output channels): forward output o reads input
// channel o / M through filter o; dx of channel c gathers from the M output
// channels c*M .. c*M + M-1, one after another.
#include "dw_common.cuh"

namespace dw {
namespace {

struct DirectArgs {
    int64_t N, C, H, W, Ho, Wo;
    int64_t M, Co;  // output channels per input channel, output channels
    int kH, kW, sh, sw, dh, dw, pt, pl;
    int wtype;
    int64_t total;
    Epilogue epi;  // forward only
};

// I: index type (int32_t when every flat index fits, else int64_t; 64-bit
// division is several times the cost of 32-bit division).
template <int LAYOUT, class I>
__device__ __forceinline__ void decode(I i, I C, I Hx, I Wx, I& n, I& c, I& h, I& w) {
    if (LAYOUT == DW_NHWC) {
        c = i % C; i /= C;
        w = i % Wx; i /= Wx;
        h = i % Hx; n = i / Hx;
    } else {
        w = i % Wx; i /= Wx;
        h = i % Hx; i /= Hx;
        c = i % C; n = i / C;
    }
}

template <int LAYOUT, class I>
__device__ __forceinline__ I offset(I n, I c, I h, I w, I C, I Hx, I Wx) {
    return LAYOUT == DW_NHWC ? ((n * Hx + h) * Wx + w) * C + c : ((n * C + c) * Hx + h) * Wx + w;
}

template <int LAYOUT, class TA, class I>
__global__ void __launch_bounds__(256) direct_fwd_kernel(const TA* __restrict__ x,
                                                         const void* __restrict__ w,
                                                         const float* __restrict__ b,
                                                         TA* __restrict__ y, DirectArgs a) {
    grid_dependency_wait();
    allow_dependents();
    const I C = I(a.C), Co = I(a.Co), M = I(a.M), H = I(a.H), W = I(a.W), Ho = I(a.Ho),
            Wo = I(a.Wo);
    const int64_t stride = int64_t(gridDim.x) * blockDim.x;
    for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < a.total; i += stride) {
        I n, o, ho, wo;
        decode<LAYOUT, I>(I(i), Co, Ho, Wo, n, o, ho, wo);
        const I c = o / M;  // the input channel output o reads
        float acc = 0.f;
        const int64_t wbase = int64_t(o) * a.kH * a.kW;
        for (int kh = 0; kh < a.kH; ++kh) {
            const I hi = ho * I(a.sh) + I(kh) * I(a.dh) - I(a.pt);
            if (hi < 0 || hi >= H) continue;
            for (int kw = 0; kw < a.kW; ++kw) {
                const I wi = wo * I(a.sw) + I(kw) * I(a.dw) - I(a.pl);
                if (wi < 0 || wi >= W) continue;
                acc = fmaf(ActIO<TA>::load1(x + offset<LAYOUT, I>(n, c, hi, wi, C, H, W)),
                           load_weight(w, a.wtype, wbase + kh * a.kW + kw), acc);
            }
        }
        if (b) acc += __ldg(b + o);
        if (a.epi.on()) {
            float scale, shift;
            bn_scale_shift(a.epi, int(o), scale, shift);
            acc = epilogue_apply(acc, scale, shift, a.epi.act);
        }
        ActIO<TA>::store1(y + i, acc);
    }
}

template <int LAYOUT, class TA, class I>
__global__ void __launch_bounds__(256) direct_bwd_kernel(const TA* __restrict__ dy,
                                                         const void* __restrict__ w,
                                                         TA* __restrict__ dx, DirectArgs a) {
    grid_dependency_wait();
    allow_dependents();
    const I C = I(a.C), Co = I(a.Co), M = I(a.M), H = I(a.H), W = I(a.W), Ho = I(a.Ho),
            Wo = I(a.Wo), sh = I(a.sh), sw = I(a.sw);
    const int64_t stride = int64_t(gridDim.x) * blockDim.x;
    for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < a.total; i += stride) {
        I n, c, hi, wi;
        decode<LAYOUT, I>(I(i), C, H, W, n, c, hi, wi);
        float acc = 0.f;
        // every output channel of input channel c: o = c*M .. c*M + M-1
        for (I o = c * M; o < (c + 1) * M; ++o) {
            const int64_t wbase = int64_t(o) * a.kH * a.kW;
            for (int kh = 0; kh < a.kH; ++kh) {
                const I th = hi + I(a.pt) - I(kh) * I(a.dh);  // = ho * sh
                if (th < 0 || th % sh != 0) continue;
                const I ho = th / sh;
                if (ho >= Ho) continue;
                for (int kw = 0; kw < a.kW; ++kw) {
                    const I tw = wi + I(a.pl) - I(kw) * I(a.dw);  // = wo * sw
                    if (tw < 0 || tw % sw != 0) continue;
                    const I wo = tw / sw;
                    if (wo >= Wo) continue;
                    acc = fmaf(load_weight(w, a.wtype, wbase + kh * a.kW + kw),
                               ActIO<TA>::load1(dy + offset<LAYOUT, I>(n, o, ho, wo, Co, Ho, Wo)),
                               acc);
                }
            }
        }
        ActIO<TA>::store1(dx + i, acc);
    }
}

// Input gradient of a strided forward with the filter extent and the stride
// known at compile time (dilation 1, no multiplier): the same gather and the
// same tap order as direct_bwd_kernel, with 32-bit multiply-shift index
// decoding and the divisibility tests resolved to masks.  Serves the strided
// input gradients the tiled families leave to the direct path (NCHW).
struct StridedArgs {
    int C, H, W, Ho, Wo, pt, pl, wtype, total;
    FastDiv fC, fH, fW;
};

template <int LAYOUT, class TA, int KH, int KW, int S>
__global__ void __launch_bounds__(256) strided_bwd_kernel(const TA* __restrict__ dy,
                                                          const void* __restrict__ w,
                                                          TA* __restrict__ dx, StridedArgs a) {
    grid_dependency_wait();
    allow_dependents();
    const int stride = gridDim.x * blockDim.x;
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < a.total; i += stride) {
        int n, c, hi, wi;
        if (LAYOUT == DW_NHWC) {
            const int q = fast_div(i, a.fC);
            c = i - q * a.C;
            const int r = fast_div(q, a.fW);
            wi = q - r * a.W;
            n = fast_div(r, a.fH);
            hi = r - n * a.H;
        } else {
            const int q = fast_div(i, a.fW);
            wi = i - q * a.W;
            const int r = fast_div(q, a.fH);
            hi = q - r * a.H;
            n = fast_div(r, a.fC);
            c = r - n * a.C;
        }
        const int th0 = hi + a.pt, tw0 = wi + a.pl;
        const int wbase = c * (KH * KW);
        float acc = 0.f;
#pragma unroll
        for (int kh = 0; kh < KH; ++kh) {
            const int th = th0 - kh;  // = ho * S
            if (th < 0 || th % S != 0) continue;
            const int ho = th / S;
            if (ho >= a.Ho) continue;
#pragma unroll
            for (int kw = 0; kw < KW; ++kw) {
                const int tw = tw0 - kw;  // = wo * S
                if (tw < 0 || tw % S != 0) continue;
                const int wo = tw / S;
                if (wo >= a.Wo) continue;
                const int off = LAYOUT == DW_NHWC ? ((n * a.Ho + ho) * a.Wo + wo) * a.C + c
                                                  : ((n * a.C + c) * a.Ho + ho) * a.Wo + wo;
                acc = fmaf(load_weight(w, a.wtype, wbase + kh * KW + kw), ActIO<TA>::load1(dy + off),
                           acc);
            }
        }
        ActIO<TA>::store1(dx + i, acc);
    }
}

template <class TA, int KH, int KW, int S>
cudaError_t launch_strided_bwd(const Problem& p, const void* in, const void* w, void* out,
                               cudaStream_t stream, dim3 grid, dim3 block) {
    StridedArgs a;
    a.C = int(p.C); a.H = int(p.H); a.W = int(p.W); a.Ho = int(p.Ho); a.Wo = int(p.Wo);
    a.pt = p.pt; a.pl = p.pl; a.wtype = p.wtype;
    a.total = int(p.N * p.C * p.H * p.W);
    a.fC = make_fastdiv(a.C);
    a.fH = make_fastdiv(a.H);
    a.fW = make_fastdiv(a.W);
    const TA* src = static_cast<const TA*>(in);
    TA* dst = static_cast<TA*>(out);
    return p.layout == DW_NHWC
               ? launch_pdl(strided_bwd_kernel<DW_NHWC, TA, KH, KW, S>, grid, block, 0, stream, src,
                            w, dst, a)
               : launch_pdl(strided_bwd_kernel<DW_NCHW, TA, KH, KW, S>, grid, block, 0, stream, src,
                            w, dst, a);
}

// The strided input gradients with a compile-time kernel: 3x3, 5x5, 7x7 at
// stride 2, dilation 1, no multiplier, every index inside int32.
template <class TA>
bool try_strided_bwd(const Problem& p, const void* in, const void* w, void* out,
                     cudaStream_t stream, dim3 grid, dim3 block, cudaError_t* e) {
    if (p.M != 1 || p.dh != 1 || p.dw != 1 || p.sh != 2 || p.sw != 2 || p.kH != p.kW) return false;
    const int64_t big = p.N * p.C * (p.H > p.Ho ? p.H : p.Ho) * (p.W > p.Wo ? p.W : p.Wo);
    if (big >= (int64_t(1) << 30) || p.pt + p.H >= (1 << 29) || p.pl + p.W >= (1 << 29)) return false;
    if (p.kH == 3) *e = launch_strided_bwd<TA, 3, 3, 2>(p, in, w, out, stream, grid, block);
    else if (p.kH == 5) *e = launch_strided_bwd<TA, 5, 5, 2>(p, in, w, out, stream, grid, block);
    else if (p.kH == 7) *e = launch_strided_bwd<TA, 7, 7, 2>(p, in, w, out, stream, grid, block);
    else return false;
    return true;
}

template <class TA, class I>
cudaError_t launch_typed(const Problem& p, Op op, const void* in, const void* w, const float* b,
                         void* out, cudaStream_t stream, dim3 grid, dim3 block,
                         const DirectArgs& a) {
    const TA* src = static_cast<const TA*>(in);
    TA* dst = static_cast<TA*>(out);
    if (op == OP_FWD)
        return p.layout == DW_NHWC
                   ? launch_pdl(direct_fwd_kernel<DW_NHWC, TA, I>, grid, block, 0, stream, src, w,
                                b, dst, a)
                   : launch_pdl(direct_fwd_kernel<DW_NCHW, TA, I>, grid, block, 0, stream, src, w,
                                b, dst, a);
    return p.layout == DW_NHWC
               ? launch_pdl(direct_bwd_kernel<DW_NHWC, TA, I>, grid, block, 0, stream, src, w,
                            dst, a)
               : launch_pdl(direct_bwd_kernel<DW_NCHW, TA, I>, grid, block, 0, stream, src, w,
                            dst, a);
}

template <class TA>
cudaError_t launch_index(const Problem& p, Op op, const void* in, const void* w, const float* b,
                         void* out, cudaStream_t stream, dim3 grid, dim3 block,
                         const DirectArgs& a) {
    cudaError_t e;
    if (op == OP_BWD_INPUT && try_strided_bwd<TA>(p, in, w, out, stream, grid, block, &e)) return e;
    // every flat index and intermediate (with pads and taps) inside int32?
    const int64_t big = p.N * (p.Co > p.C ? p.Co : p.C) * (p.H > p.Ho ? p.H : p.Ho) *
                        (p.W > p.Wo ? p.W : p.Wo);
    const int64_t span = int64_t(p.kH) * p.dh + int64_t(p.kW) * p.dw + p.pt + p.pl +
                         (p.H + p.W) * (p.sh + p.sw);
    if (big < (int64_t(1) << 30) && span < (int64_t(1) << 30))
        return launch_typed<TA, int32_t>(p, op, in, w, b, out, stream, grid, block, a);
    return launch_typed<TA, int64_t>(p, op, in, w, b, out, stream, grid, block, a);
}

}  // namespace

dw_status_t direct_launch(const Problem& p, Op op, const void* in, const void* w, const float* b,
                          void* out, cudaStream_t stream) {
    DirectArgs a;
    a.N = p.N; a.C = p.C; a.H = p.H; a.W = p.W; a.Ho = p.Ho; a.Wo = p.Wo;
    a.M = p.M; a.Co = p.Co;
    a.kH = p.kH; a.kW = p.kW; a.sh = p.sh; a.sw = p.sw; a.dh = p.dh; a.dw = p.dw;
    a.pt = p.pt; a.pl = p.pl; a.wtype = p.wtype;
    a.epi = op == OP_FWD ? p.epi : Epilogue{};
    a.total = op == OP_FWD ? p.N * p.Co * p.Ho * p.Wo : p.N * p.C * p.H * p.W;
    const int threads = 256;
    const int dev = current_device();
    const int64_t max_blocks = int64_t(sm_count(dev)) * 8;
    int64_t blocks = (a.total + threads - 1) / threads;
    if (blocks > max_blocks) blocks = max_blocks;
    if (blocks < 1) blocks = 1;
    const dim3 grid(static_cast<unsigned>(blocks)), block(threads);
    cudaError_t e;
    if (p.atype == DW_F16)
        e = launch_index<__half>(p, op, in, w, b, out, stream, grid, block, a);
    else if (p.atype == DW_BF16)
        e = launch_index<__nv_bfloat16>(p, op, in, w, b, out, stream, grid, block, a);
    else
        e = launch_index<float>(p, op, in, w, b, out, stream, grid, block, a);
    if (e != cudaSuccess) return DW_ERR_CUDA;
    return cudaGetLastError() == cudaSuccess ? DW_OK : DW_ERR_CUDA;
}

}  // namespace dw
