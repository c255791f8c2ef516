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

template <int LAYOUT>
__device__ __forceinline__ void decode(int64_t i, int64_t C, int64_t Hx, int64_t Wx, int64_t& n,
                                       int64_t& c, int64_t& h, int64_t& w) {
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

template <int LAYOUT>
__device__ __forceinline__ int64_t offset(int64_t n, int64_t c, int64_t h, int64_t w,
                                          int64_t C, int64_t Hx, int64_t Wx) {
    return LAYOUT == DW_NHWC ? ((n * Hx + h) * Wx + w) * C + c : ((n * C + c) * Hx + h) * Wx + w;
}

template <int LAYOUT>
__global__ void __launch_bounds__(256) direct_fwd_kernel(const float* __restrict__ x,
                                                         const void* __restrict__ w,
                                                         const float* __restrict__ b,
                                                         float* __restrict__ y, DirectArgs a) {
    grid_dependency_wait();
    allow_dependents();
    const int64_t stride = int64_t(gridDim.x) * blockDim.x;
    for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < a.total; i += stride) {
        int64_t n, o, ho, wo;
        decode<LAYOUT>(i, a.Co, a.Ho, a.Wo, n, o, ho, wo);
        const int64_t c = o / a.M;  // the input channel output o reads
        float acc = 0.f;
        const int64_t wbase = o * a.kH * a.kW;
        for (int kh = 0; kh < a.kH; ++kh) {
            const int64_t hi = ho * a.sh + int64_t(kh) * a.dh - a.pt;
            if (hi < 0 || hi >= a.H) continue;
            for (int kw = 0; kw < a.kW; ++kw) {
                const int64_t wi = wo * a.sw + int64_t(kw) * a.dw - a.pl;
                if (wi < 0 || wi >= a.W) continue;
                acc = fmaf(__ldg(x + offset<LAYOUT>(n, c, hi, wi, a.C, a.H, a.W)),
                           load_weight(w, a.wtype, wbase + kh * a.kW + kw), acc);
            }
        }
        if (b) acc += __ldg(b + o);
        if (a.epi.on()) {
            float scale, shift;
            bn_scale_shift(a.epi, int(o), scale, shift);
            acc = epilogue_apply(acc, scale, shift, a.epi.act);
        }
        y[i] = acc;
    }
}

template <int LAYOUT>
__global__ void __launch_bounds__(256) direct_bwd_kernel(const float* __restrict__ dy,
                                                         const void* __restrict__ w,
                                                         float* __restrict__ dx, DirectArgs a) {
    grid_dependency_wait();
    allow_dependents();
    const int64_t stride = int64_t(gridDim.x) * blockDim.x;
    for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < a.total; i += stride) {
        int64_t n, c, hi, wi;
        decode<LAYOUT>(i, a.C, a.H, a.W, n, c, hi, wi);
        float acc = 0.f;
        // every output channel of input channel c: o = c*M .. c*M + M-1
        for (int64_t o = c * a.M; o < (c + 1) * a.M; ++o) {
            const int64_t wbase = o * a.kH * a.kW;
            for (int kh = 0; kh < a.kH; ++kh) {
                const int64_t th = hi + a.pt - int64_t(kh) * a.dh;  // = ho * sh
                if (th < 0 || th % a.sh != 0) continue;
                const int64_t ho = th / a.sh;
                if (ho >= a.Ho) continue;
                for (int kw = 0; kw < a.kW; ++kw) {
                    const int64_t tw = wi + a.pl - int64_t(kw) * a.dw;  // = wo * sw
                    if (tw < 0 || tw % a.sw != 0) continue;
                    const int64_t wo = tw / a.sw;
                    if (wo >= a.Wo) continue;
                    acc = fmaf(load_weight(w, a.wtype, wbase + kh * a.kW + kw),
                               __ldg(dy + offset<LAYOUT>(n, o, ho, wo, a.Co, a.Ho, a.Wo)), acc);
                }
            }
        }
        dx[i] = acc;
    }
}

}  // namespace

dw_status_t direct_launch(const Problem& p, Op op, const float* in, const void* w, const float* b,
                          float* out, cudaStream_t stream) {
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
    const dim3 grid(static_cast<unsigned>(blocks));
    cudaError_t e;
    const dim3 block(threads);
    if (op == OP_FWD) {
        e = p.layout == DW_NHWC
                ? launch_pdl(direct_fwd_kernel<DW_NHWC>, grid, block, 0, stream, in, w, b, out, a)
                : launch_pdl(direct_fwd_kernel<DW_NCHW>, grid, block, 0, stream, in, w, b, out, a);
    } else {
        e = p.layout == DW_NHWC
                ? launch_pdl(direct_bwd_kernel<DW_NHWC>, grid, block, 0, stream, in, w, out, a)
                : launch_pdl(direct_bwd_kernel<DW_NCHW>, grid, block, 0, stream, in, w, out, a);
    }
    if (e != cudaSuccess) return DW_ERR_CUDA;
    return cudaGetLastError() == cudaSuccess ? DW_OK : DW_ERR_CUDA;
}

}  // namespace dw
