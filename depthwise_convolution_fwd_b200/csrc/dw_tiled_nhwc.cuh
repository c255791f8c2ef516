// NHWC tiled kernels: channels innermost, TMA halo tiles, persistent CTAs.
//
// Layout and mapping (page "cubek_convolution kernels::forward::depthwise",
// module text: the channel axis is a batch axis, channels stay innermost and
// consecutive lanes read consecutive channels of one pixel; the pass is
// bandwidth-bound).  A CTA tile is TH x TW output pixels x 32 channels.  Each
// lane owns 4 consecutive channels (one float4), 8 lanes cover the 32
// channels of a pixel, so a quarter-warp reads or writes 128 contiguous
// bytes.  The input halo tile [IH][IW][32] of every output tile is fetched by
// one 4-D TMA load (zero fill outside the tensor == zero padding) into a ring
// of NS shared-memory stages.  One producer warp issues the loads; the
// consumer warps wait on a per-stage "full" mbarrier, compute, and release the
// stage on a per-stage "empty" mbarrier, so no block-wide barrier sits in the
// tile loop and NS-1 loads stay in flight.  Filter taps and bias of the CTA's
// 32 channels sit in registers.  Each consumer thread computes a THT x TWT
// block of outputs: it streams the input cells of its block's window once
// from shared memory and feeds every (output, tap) pair that reads that cell,
// a register sliding window in both directions resolved at compile time.
// Lane width VEC: 4 (a lane owns 4 channels as one float4; 8 lanes per pixel,
// the memory-bound small kernels) or 1 (a lane owns one channel, a warp covers
// the 32 channels of a pixel with 4-byte shared loads and 128-byte coalesced
// stores; a thread then holds only kH*kW taps, so long and large kernels keep
// many warps resident).
//
// Forward (LeanMlir Proofs/Architectures/Depthwise, "Depthwise conv2d
// forward"): output (ho,wo) reads input (ho*S + kh*D - pt, wo*S + kw*D - pl);
// stride and dilation are part of the index map (no decimation pass).
// Transposed mode = input gradient ("Closed-form input gradient ... direct
// formula" and the stride-2 input-VJP sections): dx tile rows start at
// hi0 = ty*TH - (pt mod S) so that hi + pt is a multiple of S at the tile
// origin; dx(hi) gathers W[kh] * dy((hi + pt - kh*D)/S) for the kh where the
// division is exact - the zero-upsampled, reversed-kernel correlation without
// the upsampled tensor.  At S = 1 this is the reversed kernel with the
// complementary pad (kH-1)*D - pt.
#pragma once

#include <climits>
#include <type_traits>

#include "dw_common.cuh"

namespace dw {
namespace nhwc {


template <int VEC>
struct VecOps;

template <>
struct VecOps<4> {
    using T = float4;
    static __device__ __forceinline__ T zero() { return make_float4(0.f, 0.f, 0.f, 0.f); }
    static __device__ __forceinline__ void fma(T& acc, const T& v, const T& w) { fma4(acc, v, w); }
    static __device__ __forceinline__ T add(const T& a, const T& b) {
        return make_float4(a.x + b.x, a.y + b.y, a.z + b.z, a.w + b.w);
    }
    template <class TA>
    static __device__ __forceinline__ void store(TA* p, const T& v) { ActIO<TA>::store4(p, v); }
    template <class WT>
    static __device__ __forceinline__ T load_w(const WT* w, int64_t o, int step) {
        return make_float4(float(w[o]), float(w[o + step]), float(w[o + 2 * step]),
                           float(w[o + 3 * step]));
    }
    static __device__ __forceinline__ T load_b(const float* b, int c) {
        return make_float4(__ldg(b + c), __ldg(b + c + 1), __ldg(b + c + 2), __ldg(b + c + 3));
    }
    static __device__ __forceinline__ void scale_shift(const Epilogue& e, int c, T& s, T& t) {
        bn_scale_shift(e, c, s.x, t.x);
        bn_scale_shift(e, c + 1, s.y, t.y);
        bn_scale_shift(e, c + 2, s.z, t.z);
        bn_scale_shift(e, c + 3, s.w, t.w);
    }
    static __device__ __forceinline__ T mul(const T& a, const T& b) {
        return make_float4(a.x * b.x, a.y * b.y, a.z * b.z, a.w * b.w);
    }
    static __device__ __forceinline__ T fma(const T& a, const T& b, const T& c, int) {
        return make_float4(fmaf(a.x, b.x, c.x), fmaf(a.y, b.y, c.y), fmaf(a.z, b.z, c.z),
                           fmaf(a.w, b.w, c.w));
    }
    template <int ACT>
    static __device__ __forceinline__ T act(const T& u) {
        return make_float4(activate<ACT>(u.x), activate<ACT>(u.y), activate<ACT>(u.z),
                           activate<ACT>(u.w));
    }
};

// two channels per lane: only the transposed multiplier-2 tiles (TR1 mode)
template <>
struct VecOps<2> {
    using T = float2;
    static __device__ __forceinline__ T zero() { return make_float2(0.f, 0.f); }
    template <class TA>
    static __device__ __forceinline__ void store(TA* p, const T& v) { ActIO<TA>::store2(p, v); }
    static __device__ __forceinline__ T load_b(const float* b, int c) {
        return make_float2(__ldg(b + c), __ldg(b + c + 1));
    }
};

template <>
struct VecOps<1> {
    using T = float;
    static __device__ __forceinline__ T zero() { return 0.f; }
    static __device__ __forceinline__ void fma(T& acc, const T& v, const T& w) {
        acc = fmaf(v, w, acc);
    }
    static __device__ __forceinline__ T add(const T& a, const T& b) { return a + b; }
    template <class TA>
    static __device__ __forceinline__ void store(TA* p, const T& v) { ActIO<TA>::store1(p, v); }
    template <class WT>
    static __device__ __forceinline__ T load_w(const WT* w, int64_t o, int) {
        return float(w[o]);
    }
    static __device__ __forceinline__ T load_b(const float* b, int c) { return __ldg(b + c); }
    static __device__ __forceinline__ void scale_shift(const Epilogue& e, int c, T& s, T& t) {
        bn_scale_shift(e, c, s, t);
    }
    static __device__ __forceinline__ T mul(const T& a, const T& b) { return a * b; }
    static __device__ __forceinline__ T fma(const T& a, const T& b, const T& c, int) {
        return fmaf(a, b, c);
    }
    template <int ACT>
    static __device__ __forceinline__ T act(const T& u) {
        return activate<ACT>(u);
    }
};

struct Args {
    const void* w;
    const float* b;
    void* out;  // elements of the configuration's activation type
    int32_t* err;
    int wtype;
    int C;
    int Hout, Wout;  // extents of the tensor written
    int pt, pl;      // forward low pads
    int org_y, org_x;
    FastDiv tiles_c, tiles_x, tiles_y;
    int ntiles;
    Epilogue epi;  // used by the EPI instantiations only
};

// NO: output staging buffers for the TMA-store epilogue (0 = results are
// stored straight from registers).  MINB: CTAs per SM the register budget is
// sized for.
template <int KH_, int KW_, int S_, int D_, bool TR_, int THT_, int TWT_, int WX_, int WY_, int NS_,
          int VEC_ = 4, int NO_ = 2, int MINB_ = 1, int CB_ = 32, int MULT_ = 1,
          class TA_ = float>
struct Cfg {
    using TA = TA_;  // activation element type (float, __half, __nv_bfloat16)
    static constexpr int ESZ = sizeof(TA);
    static constexpr int CB = CB_;  // channels per tile of the tensor written
    // channel multiplier (output channel o reads input channel o / MULT).
    // Forward: a tile's CB output channels read CB / MULT staged input
    // channels.  Transposed mode: a tile's CB dx channels gather from
    // CB * MULT staged dy channels, MT = MULT float4s per lane and cell.
    static constexpr int MULT = MULT_;
    static constexpr bool TR0 = TR_;
    static constexpr int SC = TR0 ? CB * MULT : CB / MULT;  // staged channels per pixel
    // transposed multiplier with VEC * MULT = 4 (one dx channel per lane for
    // M = 4, two for M = 2): the lane's 4 dy channels are one float4, against
    // one float4 of filters
    static constexpr bool TR1 = TR0 && VEC_ < 4 && VEC_ * MULT == 4;
    static constexpr int MT = TR0 && !TR1 ? MULT : 1;
    static constexpr int KH = KH_, KW = KW_, S = S_, D = D_;
    static constexpr bool TR = TR_;
    static constexpr int THT = THT_, TWT = TWT_, WX = WX_, WY = WY_, NS = NS_;
    static constexpr int VEC = VEC_;
    // transposed tiles with S > 1 may start at a negative row/column, where a
    // TMA store must not start: those keep register stores
    static constexpr int NO = (TR && S > 1) ? 0 : NO_;
    static constexpr int MINB = MINB_;
    static constexpr int CV = CB / VEC;  // lanes per pixel
    static constexpr int NCW = WX * WY * CV / 32;  // consumer warps
    static constexpr int NCT = NCW * 32;           // consumer threads
    static constexpr int NT = NCW * 32 + 32;       // + one producer warp
    static constexpr int TH = THT * WY, TW = TWT * WX;
    static constexpr int AH = TR ? ((KH - 1) * D + S - 1) / S : 0;
    static constexpr int AW = TR ? ((KW - 1) * D + S - 1) / S : 0;
    static constexpr int IH = TR ? AH + TH / S : (TH - 1) * S + (KH - 1) * D + 1;
    static constexpr int IW = TR ? AW + TW / S : (TW - 1) * S + (KW - 1) * D + 1;
    // rows / columns of the input window one thread reads
    static constexpr int RH = TR ? AH + (THT - 1) / S + 1 : (THT - 1) * S + (KH - 1) * D + 1;
    static constexpr int RW = TR ? AW + (TWT - 1) / S + 1 : (TWT - 1) * S + (KW - 1) * D + 1;
    static constexpr int STAGE_BYTES = IH * IW * SC * ESZ;  // one TMA load
    static constexpr int STAGE_PITCH = (STAGE_BYTES + 127) / 128 * 128;
    static constexpr int OUT_ELEMS = TH * TW * CB;  // output staging buffer
    static constexpr int OUT_BYTES = OUT_ELEMS * ESZ;
    static constexpr size_t SMEM =
        size_t(NS) * STAGE_PITCH + size_t(NO) * OUT_BYTES + size_t(2 * NS) * 8 + 16;
    static_assert((WX * WY * CV) % 32 == 0, "whole consumer warps");
    static_assert(IH <= 256 && IW <= 256, "TMA box dimension limit");
    // every stage starts on a 128-byte boundary (tensor-copy destination rule)
    static_assert(MULT > 1 || ESZ < 4 || STAGE_BYTES % 128 == 0, "TMA shared-memory alignment");
    static_assert(NO == 0 || OUT_BYTES % 128 == 0, "staging buffers on 128-byte boundaries");
    static_assert((SC * ESZ) % 16 == 0 && SC <= 256, "16-byte rows in the input box");
    static_assert(MULT == 1 || TR1 || (VEC == 4 && (TR || CB % MULT == 0)),
                  "multiplier tiles: 4-channel lanes");
    static_assert(!TR || (THT % S == 0 && TWT % S == 0), "transposed blocks are phase aligned");
    static_assert(SMEM <= 227 * 1024, "shared memory per CTA");
};


// Tap index that maps output offset j (within a thread block) to window
// row r, or -1.  Forward: r = j*S + k*D.  Transposed: r - A = (j - k*D)/S
// with exact division.
template <class K, bool ROW>
__host__ __device__ constexpr int tap_for(int r, int j) {
    constexpr int Kn = ROW ? K::KH : K::KW;
    constexpr int A = ROW ? K::AH : K::AW;
    if constexpr (!K::TR) {
        const int num = r - j * K::S;
        if (num < 0 || num % K::D != 0 || num / K::D >= Kn) return -1;
        return num / K::D;
    } else {
        for (int k = 0; k < Kn; ++k) {
            const int num = j - k * K::D;  // must be (r - A) * S
            if (num == (r - A) * K::S) return k;
        }
        return -1;
    }
}

struct Tile {
    int cb, n, oy0, ox0, iy0, ix0;
};

template <class K>
__device__ __forceinline__ Tile decode_tile(int t, const Args& a) {
    Tile T;
    int q = fast_div(t, a.tiles_c);
    T.cb = t - q * a.tiles_c.d;
    const int r = fast_div(q, a.tiles_x);
    const int tx = q - r * a.tiles_x.d;
    T.n = fast_div(r, a.tiles_y);
    const int ty = r - T.n * a.tiles_y.d;
    if constexpr (!K::TR) {
        T.oy0 = ty * K::TH;
        T.ox0 = tx * K::TW;
        T.iy0 = T.oy0 * K::S - a.pt;
        T.ix0 = T.ox0 * K::S - a.pl;
    } else {
        T.oy0 = ty * K::TH - a.org_y;
        T.ox0 = tx * K::TW - a.org_x;
        T.iy0 = (T.oy0 + a.pt) / K::S - K::AH;  // oy0 + pt >= 0 and divisible by S
        T.ix0 = (T.ox0 + a.pl) / K::S - K::AW;
    }
    return T;
}

// The lane vector of one window cell: the lane's VEC channels (MULT = 1), or
// for a channel multiplier the input channels its 4 output channels read,
// each repeated MULT times (MULT = 2: two channels, MULT >= 4: one).
template <class K>
__device__ __forceinline__ typename VecOps<K::VEC>::T load_cell(const typename K::TA* p) {
    using IO = ActIO<typename K::TA>;
    if constexpr (K::MULT == 1) {
        if constexpr (K::VEC == 4) return IO::load4(p);
        else return IO::load1(p);
    } else if constexpr (K::MULT == 2) {
        const float2 f = IO::load2(p);
        return make_float4(f.x, f.x, f.y, f.y);
    } else {
        const float f = IO::load1(p);
        return make_float4(f, f, f, f);
    }
}

// EPI: kNoEpilogue, or the activation of the fused batch-norm / activation
// epilogue of the forward.
template <class K, int EPI>
__global__ void __launch_bounds__(K::NT, K::MINB)
    tiled_kernel(const __grid_constant__ CUtensorMap tmap, const __grid_constant__ CUtensorMap omap,
                 const Args a) {
    static_assert(EPI == kNoEpilogue || !K::TR, "the epilogue belongs to the forward");
    using VO = VecOps<K::VEC>;
    using V = typename VO::T;
    constexpr int CV = K::CV;
    extern __shared__ __align__(128) unsigned char smem[];
    using TA = typename K::TA;
    TA* outbuf = reinterpret_cast<TA*>(smem + size_t(K::NS) * K::STAGE_PITCH);
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + size_t(K::NS) * K::STAGE_PITCH +
                                                 size_t(K::NO) * K::OUT_BYTES);
    uint64_t* empty = full + K::NS;
    volatile int* abort_flag = reinterpret_cast<volatile int*>(empty + K::NS);

    const int tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;
    const int G = gridDim.x;

    if (tid == 0) {
#pragma unroll
        for (int s = 0; s < K::NS; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], K::NCW);
        }
        *abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();
    grid_dependency_wait();
    allow_dependents();

    if (warp == K::NCW) {
        // ---------------- producer warp: one lane issues every TMA load ----
        if (lane == 0) {
            prefetch_tensor_map(&tmap);
            if constexpr (K::NO > 0) prefetch_tensor_map(&omap);
            int k = 0;
            bool ok = true;
            for (int t = blockIdx.x; t < a.ntiles; t += G, ++k) {
                const int s = k % K::NS;
                if (k >= K::NS && !mbar_wait_or_abort(&empty[s], ((k / K::NS) - 1) & 1, abort_flag)) {
                    ok = false;
                    break;
                }
                const Tile T = decode_tile<K>(t, a);
                mbar_arrive_expect_tx(&full[s], K::STAGE_BYTES);
                tma_load_4d(smem + size_t(s) * K::STAGE_PITCH, &tmap, &full[s], T.cb * K::SC, T.ix0,
                            T.iy0, T.n);
            }
            if (!ok) {
                *abort_flag = 1;
                atomicExch(a.err, DW_ERR_DEVICE_TIMEOUT);
                // let the loads already issued land before the CTA can exit
                for (int j = (k > K::NS ? k - K::NS : 0); j < k; ++j)
                    mbar_wait_bounded(&full[j % K::NS], (j / K::NS) & 1);
            }
        }
        return;
    }

    // -------------------------- consumer warps --------------------------------
    const int cv = tid % CV;
    const int xi = (tid / CV) % K::WX;
    const int yi = tid / (CV * K::WX);
    const int r0 = K::TR ? yi * (K::THT / K::S) : yi * K::THT * K::S;
    const int q0 = K::TR ? xi * (K::TWT / K::S) : xi * K::TWT * K::S;
    const int j0 = yi * K::THT, i0 = xi * K::TWT;
    const int64_t row_pitch = int64_t(a.Wout) * a.C;

    // filters and accumulators: float4 in the TR1 mode (4 dy channels per lane)
    using VOA = VecOps<K::TR1 ? 4 : K::VEC>;
    using VA = typename VOA::T;
    VA wr[K::KH][K::KW][K::MT];
    V bias = VO::zero();
    int cur_cb = -1;
    // the value stored for one output: acc (+ bias) (-> activation); with a
    // multiplier in transposed mode, dx channel c + e sums the MULT
    // consecutive products of output channels (c + e) * MULT ..
    auto finish = [&](const VA (&acc)[K::MT]) -> V {
        if constexpr (K::TR1 && K::VEC == 1) {
            return (acc[0].x + acc[0].y) + (acc[0].z + acc[0].w);
        } else if constexpr (K::TR1) {
            return make_float2(acc[0].x + acc[0].y, acc[0].z + acc[0].w);
        } else if constexpr (K::TR && K::MT == 2) {
            return make_float4(acc[0].x + acc[0].y, acc[0].z + acc[0].w, acc[1].x + acc[1].y,
                               acc[1].z + acc[1].w);
        } else if constexpr (K::TR && K::MT == 4) {
            return make_float4((acc[0].x + acc[0].y) + (acc[0].z + acc[0].w),
                               (acc[1].x + acc[1].y) + (acc[1].z + acc[1].w),
                               (acc[2].x + acc[2].y) + (acc[2].z + acc[2].w),
                               (acc[3].x + acc[3].y) + (acc[3].z + acc[3].w));
        } else if constexpr (K::TR) {
            return acc[0];
        } else if constexpr (EPI != kNoEpilogue) {
            return VO::template act<EPI>(VO::add(acc[0], bias));
        } else {
            return VO::add(acc[0], bias);
        }
    };
    static_assert(K::MT == 1 || K::MT == 2 || K::MT == 4, "transposed multiplier 2 or 4");

    int k = 0;
    for (int t = blockIdx.x; t < a.ntiles; t += G, ++k) {
        const int s = k % K::NS;
        const Tile T = decode_tile<K>(t, a);
        const int c = T.cb * K::CB + cv * K::VEC;
        if (T.cb != cur_cb) {
            cur_cb = T.cb;
            const bool live = c < a.C;
            constexpr int step = K::KH * K::KW;
            // filter rows: channel c (forward: the output channel), or in
            // transposed mode with a multiplier output channels c*MULT + 4m..
            // (TR1: the 4 output channels c*4 .. c*4+3)
            const int64_t o = int64_t(live ? c : 0) * (K::TR ? K::MULT : 1) * step;
            // one branch on the weight type, then straight loads
            if (a.wtype == DW_F16) {
                const __half* wp = static_cast<const __half*>(a.w);
#pragma unroll
                for (int m = 0; m < K::MT; ++m)
#pragma unroll
                    for (int kh = 0; kh < K::KH; ++kh)
#pragma unroll
                        for (int kw = 0; kw < K::KW; ++kw)
                            wr[kh][kw][m] = VOA::load_w(wp, o + 4 * m * step + kh * K::KW + kw, step);
            } else {
                const float* wp = static_cast<const float*>(a.w);
#pragma unroll
                for (int m = 0; m < K::MT; ++m)
#pragma unroll
                    for (int kh = 0; kh < K::KH; ++kh)
#pragma unroll
                        for (int kw = 0; kw < K::KW; ++kw)
                            wr[kh][kw][m] = VOA::load_w(wp, o + 4 * m * step + kh * K::KW + kw, step);
            }
            if (!live) {
#pragma unroll
                for (int m = 0; m < K::MT; ++m)
#pragma unroll
                    for (int kh = 0; kh < K::KH; ++kh)
#pragma unroll
                        for (int kw = 0; kw < K::KW; ++kw) wr[kh][kw][m] = VOA::zero();
            }
            if (!K::TR && a.b != nullptr && live) bias = VO::load_b(a.b, c);
            if constexpr (EPI != kNoEpilogue) {
                // fold the normalisation into the filter and the bias
                if (live) {
                    V sc, sh;
                    VO::scale_shift(a.epi, c, sc, sh);
#pragma unroll
                    for (int kh = 0; kh < K::KH; ++kh)
#pragma unroll
                        for (int kw = 0; kw < K::KW; ++kw) wr[kh][kw][0] = VO::mul(wr[kh][kw][0], sc);
                    bias = VO::fma(bias, sc, sh, 0);
                }
            }
        }

        const bool ok = mbar_wait_or_abort(&full[s], (k / K::NS) & 1, abort_flag);
        if constexpr (K::NO == 0) {
            if (!ok) {
                if (lane == 0) {
                    *abort_flag = 1;
                    atomicExch(a.err, DW_ERR_DEVICE_TIMEOUT);
                }
                break;
            }
        }
        // (with the TMA-store epilogue a failed wait is acted on at the
        // consumer barrier below, so every consumer leaves together; the
        // shared-memory reads in between stay inside the stage)

        VA acc[K::THT][K::TWT][K::MT];
#pragma unroll
        for (int j = 0; j < K::THT; ++j)
#pragma unroll
            for (int i = 0; i < K::TWT; ++i)
#pragma unroll
                for (int m = 0; m < K::MT; ++m) acc[j][i][m] = VOA::zero();

        // this thread's window: cell (r, q) holds SC staged channels.  The
        // lane's 4 channels cv*4.. read, in the forward, input channels
        // (cv*4)/MULT..; in transposed mode dy channels cv*4*MULT ..
        const TA* win = reinterpret_cast<const TA*>(smem + size_t(s) * K::STAGE_PITCH) +
                        (r0 * K::IW + q0) * K::SC +
                        (K::TR ? cv * K::VEC * K::MULT : (cv * K::VEC) / K::MULT);
        static_for<0, K::RH>([&](auto r_) {
            constexpr int r = decltype(r_)::value;
            static_for<0, K::RW>([&](auto q_) {
                constexpr int q = decltype(q_)::value;
                // does any (output, tap) pair of this thread read cell (r,q)?
                constexpr bool used = [] {
                    for (int j = 0; j < K::THT; ++j)
                        for (int i = 0; i < K::TWT; ++i)
                            if (tap_for<K, true>(r, j) >= 0 && tap_for<K, false>(q, i) >= 0)
                                return true;
                    return false;
                }();
                if constexpr (used) {
                    VA v[K::MT];
                    if constexpr (K::TR1) {
                        v[0] = ActIO<TA>::load4(win + (r * K::IW + q) * K::SC);
                    } else if constexpr (K::MT == 1) {
                        v[0] = load_cell<K>(win + (r * K::IW + q) * K::SC);
                    } else {
#pragma unroll
                        for (int m = 0; m < K::MT; ++m)
                            v[m] = ActIO<TA>::load4(win + (r * K::IW + q) * K::SC + 4 * m);
                    }
                    static_for<0, K::THT>([&](auto j_) {
                        constexpr int j = decltype(j_)::value;
                        constexpr int kh = tap_for<K, true>(r, j);
                        if constexpr (kh >= 0) {
                            static_for<0, K::TWT>([&](auto i_) {
                                constexpr int i = decltype(i_)::value;
                                constexpr int kw = tap_for<K, false>(q, i);
                                if constexpr (kw >= 0) {
#pragma unroll
                                    for (int m = 0; m < K::MT; ++m)
                                        VOA::fma(acc[j][i][m], v[m], wr[kh][kw][m]);
                                }
                            });
                        }
                    });
                }
            });
        });

        // every lane of this warp is done with stage s
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[s]);

        if constexpr (K::NO > 0) {
            // ------- epilogue: registers -> staging buffer -> TMA store ----
            const int ob = k % K::NO;
            if (k >= K::NO) {
                // the store issued NO tiles ago must be done reading buffer ob
                if (tid == 0) bulk_wait_group_read<K::NO - 1>();
                named_barrier_sync(1, K::NCT);
            }
            TA* o = outbuf + size_t(ob) * K::OUT_ELEMS + (j0 * K::TW + i0) * K::CB + cv * K::VEC;
#pragma unroll
            for (int j = 0; j < K::THT; ++j)
#pragma unroll
                for (int i = 0; i < K::TWT; ++i)
                    VO::store(o + (j * K::TW + i) * K::CB, finish(acc[j][i]));
            fence_proxy_async_smem();
            if (named_barrier_or(1, K::NCT, !ok)) {
                if (tid == 0) {
                    *abort_flag = 1;
                    atomicExch(a.err, DW_ERR_DEVICE_TIMEOUT);
                }
                break;
            }
            if (tid == 0) {
                tma_store_4d(&omap, outbuf + size_t(ob) * K::OUT_ELEMS, T.cb * K::CB, T.ox0, T.oy0,
                             T.n);
                bulk_commit_group();
            }
        } else if (c < a.C) {
            const int ho0 = T.oy0 + j0, wo0 = T.ox0 + i0;
            TA* base = static_cast<TA*>(a.out) + (int64_t(T.n) * a.Hout + ho0) * row_pitch +
                       int64_t(wo0) * a.C + c;
#pragma unroll
            for (int j = 0; j < K::THT; ++j) {
                const int ho = ho0 + j;
                if (ho < 0 || ho >= a.Hout) continue;
#pragma unroll
                for (int i = 0; i < K::TWT; ++i) {
                    const int wo = wo0 + i;
                    if (wo < 0 || wo >= a.Wout) continue;
                    VO::store(base + j * row_pitch + int64_t(i) * a.C, finish(acc[j][i]));
                }
            }
        }
    }
    // stores issued by this CTA complete before it exits
    if constexpr (K::NO > 0) {
        if (tid == 0) bulk_wait_group<0>();
    }
}

// Launch attributes and the tensor map; `grid_cap` caps resident CTAs.
template <class K>
dw_status_t launch(const Problem& p, Op op, const void* in, const void* w, const float* b,
                   void* out, cudaStream_t stream, int32_t* err, bool dry_run) {
    const bool tr = op == OP_BWD_INPUT;
    if (tr != K::TR) return DW_ERR_UNSUPPORTED;
    Args a;
    a.w = w;
    a.b = tr ? nullptr : b;
    a.out = out;
    a.err = err;
    a.wtype = p.wtype;
    if (p.M != K::MULT) return DW_ERR_UNSUPPORTED;
    a.C = static_cast<int>(tr ? p.C : p.Co);  // channels of the tensor written
    a.Hout = static_cast<int>(tr ? p.H : p.Ho);
    a.Wout = static_cast<int>(tr ? p.W : p.Wo);
    a.pt = p.pt;
    a.pl = p.pl;
    a.org_y = tr ? p.pt % K::S : 0;
    a.org_x = tr ? p.pl % K::S : 0;
    const int64_t ty = (a.Hout + a.org_y + K::TH - 1) / K::TH;
    const int64_t tx = (a.Wout + a.org_x + K::TW - 1) / K::TW;
    const int64_t tc = (a.C + K::CB - 1) / K::CB;
    const int64_t nt = ty * tx * tc * p.N;
    if (nt >= INT_MAX || ty >= INT_MAX || tx >= INT_MAX) return DW_ERR_UNSUPPORTED;
    a.tiles_y = make_fastdiv(static_cast<int>(ty));
    a.tiles_x = make_fastdiv(static_cast<int>(tx));
    a.tiles_c = make_fastdiv(static_cast<int>(tc));
    a.ntiles = static_cast<int>(nt);
    a.epi = tr ? Epilogue{} : p.epi;
    if (dry_run) return DW_OK;

    // the epilogue instantiations exist for the forward only
    const int ev = epilogue_variant(a.epi);
    void (*kern)(CUtensorMap, CUtensorMap, Args) = tiled_kernel<K, kNoEpilogue>;
    if constexpr (!K::TR) {
        if (ev == DW_ACT_NONE) kern = tiled_kernel<K, DW_ACT_NONE>;
        if (ev == DW_ACT_RELU) kern = tiled_kernel<K, DW_ACT_RELU>;
        if (ev == DW_ACT_RELU6) kern = tiled_kernel<K, DW_ACT_RELU6>;
        if (ev == DW_ACT_SILU) kern = tiled_kernel<K, DW_ACT_SILU>;
    }
    static LaunchCache cache[5];
    const int dev = current_device();
    const int occ = prepare_kernel(reinterpret_cast<const void*>(kern), K::NT, K::SMEM,
                                   cache[ev + 1], dev);
    if (occ < 1) return DW_ERR_CUDA;

    const int64_t Hin = tr ? p.Ho : p.H, Win = tr ? p.Wo : p.W;
    CUtensorMap map;
    constexpr cuuint64_t E = K::ESZ;
    constexpr CUtensorMapDataType dt = ActIO<typename K::TA>::kTma;
    const int64_t Cin = tr ? p.Co : p.C;  // channels of the tensor read (dy or x)
    const cuuint64_t dims[4] = {cuuint64_t(Cin), cuuint64_t(Win), cuuint64_t(Hin), cuuint64_t(p.N)};
    const cuuint64_t strides[3] = {cuuint64_t(Cin) * E, cuuint64_t(Cin * Win) * E,
                                   cuuint64_t(Cin * Win * Hin) * E};
    const cuuint32_t box[4] = {K::SC, K::IW, K::IH, 1};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    if (encode_tensor_map(&map, dt, 4, const_cast<void*>(in), dims, strides, box, estr) !=
        CUDA_SUCCESS)
        return DW_ERR_CUDA;
    // output map: the staging buffer is a [TH][TW][32] box of the output
    CUtensorMap omap = map;
    if constexpr (K::NO > 0) {
        const cuuint64_t odims[4] = {cuuint64_t(a.C), cuuint64_t(a.Wout), cuuint64_t(a.Hout),
                                     cuuint64_t(p.N)};
        const cuuint64_t ostrides[3] = {cuuint64_t(a.C) * E, cuuint64_t(a.C) * a.Wout * E,
                                        cuuint64_t(a.C) * a.Wout * a.Hout * E};
        const cuuint32_t obox[4] = {K::CB, K::TW, K::TH, 1};
        if (encode_tensor_map(&omap, dt, 4, out, odims, ostrides, obox, estr) != CUDA_SUCCESS)
            return DW_ERR_CUDA;
    }

    int64_t grid = int64_t(sm_count(dev)) * occ;
    // keep each CTA on one channel block (weights loaded once per CTA)
    if (grid >= tc) grid -= grid % tc;
    if (grid > nt) grid = nt;
    if (grid < 1) grid = 1;
    if (launch_pdl(kern, dim3(static_cast<unsigned>(grid)), dim3(K::NT), K::SMEM, stream, map,
                   omap, a) != cudaSuccess)
        return DW_ERR_CUDA;
    return cudaGetLastError() == cudaSuccess ? DW_OK : DW_ERR_CUDA;
}

// Tiles a configuration would cut the problem into (host side).
template <class K>
int64_t tile_count(const Problem& p, Op op) {
    const bool tr = op == OP_BWD_INPUT;
    const int64_t Hout = tr ? p.H : p.Ho, Wout = tr ? p.W : p.Wo;
    const int64_t oy = tr ? p.pt % K::S : 0, ox = tr ? p.pl % K::S : 0;
    return ((Hout + oy + K::TH - 1) / K::TH) * ((Wout + ox + K::TW - 1) / K::TW) *
           (((tr ? p.C : p.Co) + K::CB - 1) / K::CB) * p.N;
}

// Big tiles for large problems; small tiles when the big ones would leave
// most SMs idle.
template <class Big, class Small>
dw_status_t launch_pick(const Problem& p, Op op, const void* in, const void* w, const float* b,
                        void* out, cudaStream_t stream, int32_t* err, bool dry_run) {
    const int sms = dry_run ? 148 : sm_count(current_device());
    if (tile_count<Big>(p, op) >= 2 * int64_t(sms))
        return launch<Big>(p, op, in, w, b, out, stream, err, dry_run);
    return launch<Small>(p, op, in, w, b, out, stream, err, dry_run);
}

// Instantiated configurations, per activation type TA
// (KH KW S D TR | THT TWT WX WY NS [VEC NO MINB CB MULT TA]);
// shared memory = NS input stages + NO output staging buffers <= 227 KB.
template <class TA> using F33s1 = Cfg<3, 3, 1, 1, false, 2, 4, 8, 4, 4, 4, 0, 2, 32, 1, TA>;
template <class TA> using F33s1s = Cfg<3, 3, 1, 1, false, 2, 4, 4, 2, 4, 1, 2, 2, 32, 1, TA>;
template <class TA> using F33s2 = Cfg<3, 3, 2, 1, false, 1, 2, 8, 4, 4, 4, 0, 2, 32, 1, TA>;
template <class TA> using F33d2 = Cfg<3, 3, 1, 2, false, 2, 4, 8, 4, 2, 4, 2, 1, 32, 1, TA>;
template <class TA> using F33d3 = Cfg<3, 3, 1, 3, false, 2, 4, 8, 4, 2, 4, 2, 1, 32, 1, TA>;
template <class TA> using F55s1 = Cfg<5, 5, 1, 1, false, 2, 4, 8, 4, 2, 4, 2, 1, 32, 1, TA>;
template <class TA> using F55s1s = Cfg<5, 5, 1, 1, false, 2, 4, 4, 2, 4, 1, 2, 2, 32, 1, TA>;
template <class TA> using F1x3 = Cfg<1, 3, 1, 1, false, 1, 8, 16, 1, 4, 4, 2, 1, 32, 1, TA>;
template <class TA> using F1x5 = Cfg<1, 5, 1, 1, false, 1, 8, 16, 1, 4, 4, 2, 1, 32, 1, TA>;
template <class TA> using F1x7 = Cfg<1, 7, 1, 1, false, 1, 8, 16, 1, 4, 4, 2, 1, 32, 1, TA>;
template <class TA> using F1x15 = Cfg<1, 15, 1, 1, false, 1, 16, 8, 1, 4, 1, 2, 1, 32, 1, TA>;
template <class TA> using F1x31 = Cfg<1, 31, 1, 1, false, 1, 16, 2, 1, 4, 1, 2, 1, 128, 1, TA>;
template <class TA> using F77s1 = Cfg<7, 7, 1, 1, false, 2, 4, 4, 2, 3, 1, 2, 1, 32, 1, TA>;
template <class TA> using B33s1 = Cfg<3, 3, 1, 1, true, 2, 4, 8, 4, 4, 4, 0, 2, 32, 1, TA>;
template <class TA> using B33s1s = Cfg<3, 3, 1, 1, true, 2, 4, 4, 2, 4, 1, 2, 2, 32, 1, TA>;
template <class TA> using B33s2 = Cfg<3, 3, 2, 1, true, 4, 4, 8, 4, 4, 4, 2, 1, 32, 1, TA>;
template <class TA> using B33s2s = Cfg<3, 3, 2, 1, true, 2, 2, 8, 4, 4, 4, 2, 1, 32, 1, TA>;
template <class TA> using B33d2 = Cfg<3, 3, 1, 2, true, 2, 4, 8, 4, 2, 4, 2, 1, 32, 1, TA>;
template <class TA> using B33d3 = Cfg<3, 3, 1, 3, true, 2, 4, 8, 4, 2, 4, 2, 1, 32, 1, TA>;
template <class TA> using B55s1 = Cfg<5, 5, 1, 1, true, 2, 4, 8, 4, 2, 4, 2, 1, 32, 1, TA>;
template <class TA> using B55s1s = Cfg<5, 5, 1, 1, true, 2, 4, 4, 2, 4, 1, 2, 2, 32, 1, TA>;
template <class TA> using B1x3 = Cfg<1, 3, 1, 1, true, 1, 8, 16, 1, 4, 4, 2, 1, 32, 1, TA>;
template <class TA> using B1x5 = Cfg<1, 5, 1, 1, true, 1, 8, 16, 1, 4, 4, 2, 1, 32, 1, TA>;
template <class TA> using B1x7 = Cfg<1, 7, 1, 1, true, 1, 8, 16, 1, 4, 4, 2, 1, 32, 1, TA>;
template <class TA> using B1x15 = Cfg<1, 15, 1, 1, true, 1, 16, 8, 1, 4, 1, 2, 1, 32, 1, TA>;
template <class TA> using B1x31 = Cfg<1, 31, 1, 1, true, 1, 16, 2, 1, 4, 1, 2, 1, 128, 1, TA>;
template <class TA> using B77s1 = Cfg<7, 7, 1, 1, true, 2, 4, 4, 2, 3, 1, 2, 1, 32, 1, TA>;

template <class TA>
dw_status_t fwd_launch_t(const Problem& p, const void* in, const void* w, const float* b,
                         void* out, cudaStream_t stream, int32_t* err, bool dry_run) {
    const int S = p.sh, D = p.dh;
    const Op op = OP_FWD;
#define DW_ONE(FC) return launch<FC<TA>>(p, op, in, w, b, out, stream, err, dry_run);
#define DW_TWO(FC, FCS) \
    return launch_pick<FC<TA>, FCS<TA>>(p, op, in, w, b, out, stream, err, dry_run);
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

template <class TA>
dw_status_t bwd_launch_t(const Problem& p, const void* in, const void* w, void* out,
                         cudaStream_t stream, int32_t* err, bool dry_run) {
    const int S = p.sh, D = p.dh;
    const Op op = OP_BWD_INPUT;
#define DW_ONE(BC) return launch<BC<TA>>(p, op, in, w, nullptr, out, stream, err, dry_run);
#define DW_TWO(BC, BCS) \
    return launch_pick<BC<TA>, BCS<TA>>(p, op, in, w, nullptr, out, stream, err, dry_run);
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

// Instantiation units, each compiled on its own: the forward for float32
// (dw_tiled_nhwc.cu, also the family's dispatcher), the input gradient for
// float32 (dw_tiled_nhwc_bwd.cu), both calls for float16 and bfloat16
// activations (dw_tiled_nhwc_f16.cu, dw_tiled_nhwc_bf16.cu) and the forward
// with a channel multiplier (dw_tiled_nhwc_mult.cu).  Each returns
// DW_ERR_UNSUPPORTED for a shape it has no configuration for.
dw_status_t fwd_launch_f32(const Problem& p, const void* in, const void* w, const float* b,
                           void* out, cudaStream_t stream, int32_t* err, bool dry_run);
dw_status_t bwd_launch_f32(const Problem& p, const void* in, const void* w, void* out,
                           cudaStream_t stream, int32_t* err, bool dry_run);
dw_status_t fwd_launch_f16(const Problem& p, const void* in, const void* w, const float* b,
                           void* out, cudaStream_t stream, int32_t* err, bool dry_run);
dw_status_t bwd_launch_f16(const Problem& p, const void* in, const void* w, void* out,
                           cudaStream_t stream, int32_t* err, bool dry_run);
dw_status_t fwd_launch_bf16(const Problem& p, const void* in, const void* w, const float* b,
                            void* out, cudaStream_t stream, int32_t* err, bool dry_run);
dw_status_t bwd_launch_bf16(const Problem& p, const void* in, const void* w, void* out,
                            cudaStream_t stream, int32_t* err, bool dry_run);
dw_status_t mult_launch(const Problem& p, const void* in, const void* w, const float* b,
                        void* out, cudaStream_t stream, int32_t* err, bool dry_run);
dw_status_t mult_bwd_launch(const Problem& p, const void* in, const void* w, void* out,
                            cudaStream_t stream, int32_t* err, bool dry_run);
dw_status_t mult_launch_f16(const Problem& p, const void* in, const void* w, const float* b,
                          void* out, cudaStream_t stream, int32_t* err, bool dry_run);
dw_status_t mult_bwd_launch_f16(const Problem& p, const void* in, const void* w, void* out,
                              cudaStream_t stream, int32_t* err, bool dry_run);
dw_status_t mult_launch_bf16(const Problem& p, const void* in, const void* w, const float* b,
                          void* out, cudaStream_t stream, int32_t* err, bool dry_run);
dw_status_t mult_bwd_launch_bf16(const Problem& p, const void* in, const void* w, void* out,
                              cudaStream_t stream, int32_t* err, bool dry_run);

}  // namespace nhwc
}  // namespace dw
