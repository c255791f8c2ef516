// NCHW tiled kernels (stride 1): W innermost, TMA halo tiles, persistent CTAs.
//
// Each (n, c) plane is an independent image with its own filter (page
// "LeanMlir Proofs/Architectures/Depthwise", comparison with regular conv2d:
// no cross-channel mixing).  Lanes run along W: a thread owns 4 consecutive
// outputs of a row (one float4) and THT rows, so a warp covers 128 columns
// with 16-byte accesses on both the shared-memory reads and the global
// stores.  For kH > 1 a CTA tile is TH x 128 outputs of one plane and its
// input halo [TH + (kH-1)D][IWB] comes in one TMA load; for kH = 1 (the long
// 1-D kernels) a tile is one row of 128 outputs in WY consecutive channels and
// the TMA box spans those channels instead of rows.  TMA boxes must start on a
// 16-byte boundary, so the box starts (-pl) mod (16 bytes / element size)
// columns left of the first input column a tile needs: REM = that shift mod 4
// is a template parameter, the rest (0 or 4 columns, 16-bit elements only)
// a run-time offset of every thread's window; windows are read as aligned
// 4-element vectors and indexed at compile time.  Activations are float32,
// float16 or bfloat16 (template parameter TA): elements widen to float32 on
// their way out of shared memory and each result is rounded once.
// Taps sit in registers (per thread: the filter of its plane), streamed in
// kh-major, kw-minor order per output.
//
// Modes: forward (y from x, pads pt/pl); reversed (input gradient at stride
// 1: dx from dy with the reversed filter and the complementary pads
// (kH-1)D - pt, (kW-1)D - pl; "Closed-form input gradient", reversed-kernel
// form).
#pragma once

#include <climits>
#include <type_traits>

#include "dw_common.cuh"

namespace dw {
namespace nchw {

struct Args {
    const void* w;
    const float* b;
    void* out;   // elements of the configuration's activation type
    int32_t* err;
    int wtype;
    int N, C, Hout, Wout;  // C: channels the tiles run over
    int Cout;              // channels of the tensor written
    int M;                 // forward, one output plane per tile: it reads input plane c / M
    int pt, pl;  // effective low pads of the correlation this kernel runs
    int sh4;     // extra box shift beyond REM (0, or 4 for 16-bit elements)
    FastDiv tiles_x, tiles_y, tiles_c;
    int ntiles;
    Epilogue epi;  // used by the EPI instantiations only
};

template <int KH_, int KW_, int D_, bool REV_, int REM_, int THT_, int WX_, int WY_, int NS_,
          int MINB_ = 1, class TA_ = float, int S_ = 1, int PL_ = 1, int MP_ = 1>
struct Cfg {
    using TA = TA_;
    // planes per tile: small planes share a CTA tile, the WY thread rows
    // split into PL groups of YP rows, one (n, c) plane each
    static constexpr int PL = PL_;
    // channel multiplier inside a tile: in the forward one input plane c feeds
    // the MP output planes c*MP .. c*MP+MP-1 (NA accumulator sets per thread);
    // in the input gradient one box holds the MP dy planes c*MP .. whose
    // reversed correlations sum into dx plane c (NB planes per box)
    static constexpr int MP = MP_;
    static constexpr int NA = REV_ ? 1 : MP;
    static constexpr int NB = REV_ ? MP : 1;
    static constexpr int S = S_;  // stride (forward only: output (ho, wo) reads row ho*S.., col wo*S..)
    static constexpr int ESZ = sizeof(TA);
    static constexpr int ALIGN = 16 / ESZ;  // elements per 16 bytes
    static constexpr int MINB = MINB_;  // CTAs per SM the register budget is sized for
    static constexpr int KH = KH_, KW = KW_, D = D_, REM = REM_;
    static constexpr bool REV = REV_;
    static constexpr bool ROWS = KH == 1;  // 1-D: thread rows are channels
    static constexpr int THT = ROWS ? 1 : THT_, WX = WX_, WY = WY_, NS = NS_;
    static constexpr int NCW = WX * WY / 32;  // consumer warps
    static constexpr int NT = WX * WY + 32;   // + one producer warp
    static constexpr int TW = 4 * WX;
    static constexpr int YP = WY / PL;  // thread rows per plane
    static constexpr int TH = ROWS ? 1 : THT * YP;
    static constexpr int IH = ROWS ? 1 : (TH - 1) * S + (KH - 1) * D + 1;
    static constexpr int IWB =
        (REM + (ALIGN - 4) + (TW - 1) * S + (KW - 1) * D + 1 + ALIGN - 1) / ALIGN * ALIGN;
    static constexpr int BOXH = IH;
    static constexpr int BOXC = ROWS ? WY : PL * NB;
    // bytes one TMA box delivers, and the stage pitch: every stage must start
    // on a 128-byte boundary (shared-memory destination rule of tensor copies)
    static constexpr int STAGE_BYTES = IWB * IH * BOXC * ESZ;
    static constexpr int STAGE_PITCH = (STAGE_BYTES + 127) / 128 * 128;
    static constexpr int RH = (THT - 1) * S + (KH - 1) * D + 1;       // window rows
    static constexpr int NV = (REM + 3 * S + (KW - 1) * D) / 4 + 1;  // 4-vectors per window row
    static constexpr size_t SMEM = size_t(NS) * STAGE_PITCH + size_t(2 * NS) * 8 + 16;
    static_assert((WX * WY) % 32 == 0, "whole consumer warps");
    static_assert(IWB <= 256 && IH <= 256 && BOXC <= 256, "TMA box dimension limit");
    static_assert(STAGE_PITCH % 128 == 0 && (IWB * ESZ) % 16 == 0, "TMA alignment");
    static_assert(SMEM <= 227 * 1024, "shared memory per CTA");
    static_assert(S == 1 || (!REV && !ROWS), "strided tiles: 2-D forward only");
    static_assert(WY % PL == 0 && (PL == 1 || !ROWS), "whole thread rows per plane");
    static_assert(MP == 1 || (!ROWS && PL == 1), "multiplier planes: 2-D tiles of one plane");
};


// tile t -> (tx, ty or output row h, plane or channel group, n)
template <class K>
__device__ __forceinline__ void decode_tile(int t, const Args& a, int& tx, int& ty, int& c,
                                            int& n) {
    int q = fast_div(t, a.tiles_x);
    tx = t - q * a.tiles_x.d;
    int r = fast_div(q, a.tiles_y);
    ty = q - r * a.tiles_y.d;  // ROWS: output row h
    n = fast_div(r, a.tiles_c);
    c = r - n * a.tiles_c.d;   // ROWS: channel group; else channel
}

// EPI: kNoEpilogue, or the activation of the fused batch-norm / activation
// epilogue of the forward.
template <class K, int EPI>
__global__ void __launch_bounds__(K::NT, K::MINB)
    tiled_kernel(const __grid_constant__ CUtensorMap tmap, const Args a) {
    static_assert(EPI == kNoEpilogue || !K::REV, "the epilogue belongs to the forward");
    using TA = typename K::TA;
    using IO = ActIO<TA>;
    extern __shared__ __align__(128) unsigned char smem[];
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + size_t(K::NS) * K::STAGE_PITCH);
    uint64_t* empty = full + K::NS;
    volatile int* abort_flag = reinterpret_cast<volatile int*>(empty + K::NS);

    const int tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;
    // contiguous range of tiles for this CTA: neighbouring tiles share a
    // plane (filter stays in registers) and their halos (L2 hits)
    const int t_begin = int((int64_t(blockIdx.x) * a.ntiles) / gridDim.x);
    const int t_end = int((int64_t(blockIdx.x + 1) * a.ntiles) / gridDim.x);

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
            int k = 0;
            bool ok = true;
            for (int t = t_begin; t < t_end; ++t, ++k) {
                const int s = k % K::NS;
                if (k >= K::NS && !mbar_wait_or_abort(&empty[s], ((k / K::NS) - 1) & 1, abort_flag)) {
                    ok = false;
                    break;
                }
                int tx, ty, c, n;
                decode_tile<K>(t, a, tx, ty, c, n);
                const int ix0 = tx * K::TW * K::S - a.pl - K::REM - a.sh4;
                unsigned char* dst = smem + size_t(s) * K::STAGE_PITCH;
                mbar_arrive_expect_tx(&full[s], K::STAGE_BYTES);
                if constexpr (K::ROWS)
                    tma_load_4d(dst, &tmap, &full[s], ix0, ty - a.pt, c * K::WY, n);
                else
                    // input gradient: dy planes c*PL*MP..; forward: PL input planes
                    // c*PL.., or input plane c / M for one output plane c per tile
                    tma_load_4d(dst, &tmap, &full[s], ix0, ty * K::TH * K::S - a.pt,
                                K::REV ? c * K::PL * K::MP : (K::PL > 1 ? c * K::PL : c / a.M),
                                n);
            }
            if (!ok) {
                *abort_flag = 1;
                atomicExch(a.err, DW_ERR_DEVICE_TIMEOUT);
                for (int j = (k > K::NS ? k - K::NS : 0); j < k; ++j)
                    mbar_wait_bounded(&full[j % K::NS], (j / K::NS) & 1);
            }
        }
        return;
    }

    // -------------------------- consumer warps --------------------------------
    const int xi = tid % K::WX;
    const int yi = tid / K::WX;
    float wr[K::MP][K::KH][K::KW];
    float bias[K::NA];
    int cur_key = -1;
    bool live = false;
    // the value stored for output set q: acc + bias (-> epilogue)
    auto finish = [&](float v, int q) -> float {
        if constexpr (EPI != kNoEpilogue) return activate<EPI>(v + bias[q]);
        else return v + bias[q];
    };

    int k = 0;
    for (int t = t_begin; t < t_end; ++t, ++k) {
        const int s = k % K::NS;
        int tx, ty, cg, n;
        decode_tile<K>(t, a, tx, ty, cg, n);
        const int c = K::ROWS ? cg * K::WY + yi : cg * K::PL + yi / K::YP;
        const int key = cg + n * a.tiles_c.d;
        if (key != cur_key) {
            cur_key = key;
            live = c < a.C;
#pragma unroll
            for (int m = 0; m < K::MP; ++m) {
                // filter of channel c*MP + m (MP = 1: channel c)
                const int64_t base = (int64_t(live ? c : 0) * K::MP + m) * (K::KH * K::KW);
#pragma unroll
                for (int kh = 0; kh < K::KH; ++kh)
#pragma unroll
                    for (int kw = 0; kw < K::KW; ++kw) {
                        const int src = K::REV ? (K::KH - 1 - kh) * K::KW + (K::KW - 1 - kw)
                                               : kh * K::KW + kw;
                        wr[m][kh][kw] = live ? load_weight(a.w, a.wtype, base + src) : 0.f;
                    }
            }
#pragma unroll
            for (int q = 0; q < K::NA; ++q) {
                const int oc = c * K::NA + q;  // output channel of set q
                bias[q] = (!K::REV && a.b != nullptr && live) ? __ldg(a.b + oc) : 0.f;
                if constexpr (EPI != kNoEpilogue) {
                    // fold the normalisation into the filter and the bias
                    if (live) {
                        float sc, sh;
                        bn_scale_shift(a.epi, oc, sc, sh);
#pragma unroll
                        for (int kh = 0; kh < K::KH; ++kh)
#pragma unroll
                            for (int kw = 0; kw < K::KW; ++kw) wr[q][kh][kw] *= sc;
                        bias[q] = fmaf(bias[q], sc, sh);
                    }
                }
            }
        }

        if (!mbar_wait_or_abort(&full[s], (k / K::NS) & 1, abort_flag)) {
            if (lane == 0) {
                *abort_flag = 1;
                atomicExch(a.err, DW_ERR_DEVICE_TIMEOUT);
            }
            break;
        }

        float acc[K::NA][K::THT][4];
#pragma unroll
        for (int q = 0; q < K::NA; ++q)
#pragma unroll
            for (int j = 0; j < K::THT; ++j)
#pragma unroll
                for (int i = 0; i < 4; ++i) acc[q][j][i] = 0.f;

        const int row0 = K::ROWS ? yi : (yi % K::YP) * K::THT;  // first output row of this thread
        const int plane = K::ROWS ? 0 : yi / K::YP;            // the thread's plane in the box
        const TA* win0 = reinterpret_cast<const TA*>(smem + size_t(s) * K::STAGE_PITCH) +
                         size_t(plane * K::IH + row0 * K::S) * K::IWB + 4 * xi * K::S + a.sh4;
        static_for<0, K::NB>([&](auto b_) {
            constexpr int pb = decltype(b_)::value;
            const TA* win = win0 + size_t(pb) * K::IH * K::IWB;  // dy plane c*MP + pb
            static_for<0, K::RH>([&](auto r_) {
                constexpr int r = decltype(r_)::value;
                float v[4 * K::NV];
#pragma unroll
                for (int u = 0; u < K::NV; ++u) {
                    const float4 f = IO::load4(win + r * K::IWB + 4 * u);
                    v[4 * u] = f.x;
                    v[4 * u + 1] = f.y;
                    v[4 * u + 2] = f.z;
                    v[4 * u + 3] = f.w;
                }
                static_for<0, K::THT>([&](auto j_) {
                    constexpr int j = decltype(j_)::value;
                    constexpr int khn = r - j * K::S;
                    if constexpr (khn >= 0 && khn % K::D == 0 && khn / K::D < K::KH) {
                        constexpr int kh = khn / K::D;
#pragma unroll
                        for (int q = 0; q < K::NA; ++q)
#pragma unroll
                            for (int i = 0; i < 4; ++i)
#pragma unroll
                                for (int kw = 0; kw < K::KW; ++kw)
                                    acc[q][j][i] = fmaf(v[K::REM + i * K::S + kw * K::D],
                                                        wr[K::REV ? pb : q][kh][kw], acc[q][j][i]);
                    }
                });
            });
        });

        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[s]);

        if (live) {
            const int wo0 = tx * K::TW + 4 * xi;
#pragma unroll
            for (int q = 0; q < K::NA; ++q) {
                const int oc = c * K::NA + q;
#pragma unroll
                for (int j = 0; j < K::THT; ++j) {
                    const int ho = K::ROWS ? ty : ty * K::TH + row0 + j;
                    if (ho >= a.Hout) continue;
                    TA* dst = static_cast<TA*>(a.out) +
                              ((int64_t(n) * a.Cout + oc) * a.Hout + ho) * a.Wout + wo0;
                    const float4 v = make_float4(finish(acc[q][j][0], q), finish(acc[q][j][1], q),
                                                 finish(acc[q][j][2], q), finish(acc[q][j][3], q));
                    if ((a.Wout & 3) == 0 && wo0 + 3 < a.Wout) {
                        IO::store4(dst, v);
                    } else {
                        if (wo0 < a.Wout) IO::store1(dst, v.x);
                        if (wo0 + 1 < a.Wout) IO::store1(dst + 1, v.y);
                        if (wo0 + 2 < a.Wout) IO::store1(dst + 2, v.z);
                        if (wo0 + 3 < a.Wout) IO::store1(dst + 3, v.w);
                    }
                }
            }
        }
    }
}

template <class K>
dw_status_t launch(const Problem& p, const void* in, const void* w, const float* b, void* out,
                   cudaStream_t stream, int32_t* err, bool dry_run, int pt_eff, int pl_eff,
                   int sh4) {
    const int64_t Hin = K::REV ? p.Ho : p.H, Win = K::REV ? p.Wo : p.W;
    Args a;
    a.w = w;
    a.b = K::REV ? nullptr : b;
    a.out = out;
    a.err = err;
    a.wtype = p.wtype;
    a.N = static_cast<int>(p.N);
    // channel multiplier: MP = M planes inside a tile (forward fan-out, or
    // the input gradient's summed dy planes), or a forward with one output
    // plane per tile (MP = 1, PL = 1)
    if (K::MP > 1 ? p.M != K::MP : (p.M != 1 && (K::REV || K::ROWS || K::PL != 1)))
        return DW_ERR_UNSUPPORTED;
    a.M = K::MP > 1 ? 1 : static_cast<int>(p.M);
    a.C = static_cast<int>((K::REV || K::MP > 1) ? p.C : p.Co);
    a.Cout = static_cast<int>(K::REV ? p.C : p.Co);
    a.Hout = static_cast<int>(K::REV ? p.H : p.Ho);
    a.Wout = static_cast<int>(K::REV ? p.W : p.Wo);
    a.pt = pt_eff;
    a.pl = pl_eff;
    a.sh4 = sh4;
    const int64_t tx = (a.Wout + K::TW - 1) / K::TW;
    const int64_t ty = K::ROWS ? a.Hout : (a.Hout + K::TH - 1) / K::TH;
    const int64_t tc = K::ROWS ? (a.C + K::WY - 1) / K::WY : (a.C + K::PL - 1) / K::PL;
    const int64_t nt = tx * ty * tc * p.N;
    if (nt >= INT_MAX) return DW_ERR_UNSUPPORTED;
    a.tiles_x = make_fastdiv(static_cast<int>(tx));
    a.tiles_y = make_fastdiv(static_cast<int>(ty));
    a.tiles_c = make_fastdiv(static_cast<int>(tc));
    a.ntiles = static_cast<int>(nt);
    a.epi = K::REV ? Epilogue{} : p.epi;
    if (dry_run) return DW_OK;

    const int ev = epilogue_variant(a.epi);
    void (*kern)(CUtensorMap, Args) = tiled_kernel<K, kNoEpilogue>;
    if constexpr (!K::REV) {
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

    CUtensorMap map;
    const int64_t Cin = K::REV ? p.Co : p.C;  // planes of the tensor read (dy: C*M)
    const cuuint64_t dims[4] = {cuuint64_t(Win), cuuint64_t(Hin), cuuint64_t(Cin), cuuint64_t(p.N)};
    constexpr cuuint64_t E = K::ESZ;
    const cuuint64_t strides[3] = {cuuint64_t(Win) * E, cuuint64_t(Win * Hin) * E,
                                   cuuint64_t(Win * Hin * Cin) * E};
    const cuuint32_t box[4] = {K::IWB, K::BOXH, K::BOXC, 1};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    if (encode_tensor_map(&map, ActIO<typename K::TA>::kTma, 4, const_cast<void*>(in), dims,
                          strides, box, estr) != CUDA_SUCCESS)
        return DW_ERR_CUDA;
    int64_t grid = int64_t(sm_count(dev)) * occ;
    if (grid > a.ntiles) grid = a.ntiles;
    if (launch_pdl(kern, dim3(static_cast<unsigned>(grid)), dim3(K::NT), K::SMEM, stream, map,
                   a) != cudaSuccess)
        return DW_ERR_CUDA;
    return cudaGetLastError() == cudaSuccess ? DW_OK : DW_ERR_CUDA;
}

// ---------------------------------------------------------------------------
// Channel-lane kernel for 1 x kW filters (the long 1-D kernels): one TMA box
// is 32 channel rows x the W halo of one output row; lane = channel row,
// warp = W strip, each thread computes TWT consecutive outputs of its own
// channel with its kW taps in registers, streaming its window from shared
// memory once.  For float32 the stage row pitch IWB is chosen with IWB/4
// odd, so the 32 lanes' 16-byte reads (32 different rows, same column) fall
// in distinct bank groups and never conflict; 16-bit rows must be a multiple
// of 8 elements (16-byte box rows), which leaves 2-way conflicts.  Results leave through a per-warp TMA
// store: each warp stages its 32-row x TWT-column block in its own
// double-buffered slot and one lane issues the bulk store (the tensor engine
// does the 32-row scatter); when the output row pitch is not a multiple of
// 16 bytes they are stored from registers instead.
template <int KW_, bool REV_, int REM_, int TWT_, int NCW_, int NS_, class TA_ = float>
struct ClCfg {
    using TA = TA_;
    static constexpr int ESZ = sizeof(TA);
    static constexpr int ALIGN = 16 / ESZ;  // elements per 16 bytes
    static constexpr int KW = KW_, REM = REM_, TWT = TWT_, NCW = NCW_, NS = NS_;
    static constexpr bool REV = REV_;
    static constexpr int CH = 32;  // channel rows per tile (lanes)
    static constexpr int NT = NCW * 32 + 32;
    static constexpr int TW = TWT * NCW;
    static constexpr int IWB0 =
        (REM + (ALIGN - 4) + TW + (KW - 1) + ALIGN - 1) / ALIGN * ALIGN;
    static constexpr int IWB = (ESZ < 4 || (IWB0 / 4) % 2 == 1) ? IWB0 : IWB0 + 4;
    static constexpr int STAGE_BYTES = IWB * CH * ESZ;
    static constexpr int STAGE_PITCH = (STAGE_BYTES + 127) / 128 * 128;
    static constexpr int NV = (REM + TWT + KW - 1 + 3) / 4;  // 4-element chunks per window
    static constexpr int OUT_ELEMS = CH * TWT;  // one warp's staging slot
    static constexpr int OUT_BYTES = OUT_ELEMS * ESZ;
    static constexpr size_t SMEM = size_t(NS) * STAGE_PITCH + size_t(2 * NCW) * OUT_BYTES +
                                   size_t(2 * NS) * 8 + 16;
    static_assert(TWT % 4 == 0, "thread strips are whole 4-element vectors");
    static_assert(OUT_BYTES % 128 == 0, "staging slots on 128-byte boundaries");
    static_assert(IWB <= 256, "TMA box dimension limit");
    static_assert(ESZ < 4 || (IWB / 4) % 2 == 1, "conflict-free row pitch");
    static_assert((IWB * ESZ) % 16 == 0, "16-byte box rows");
    static_assert(SMEM <= 227 * 1024, "shared memory per CTA");
};

template <class K, int EPI>
__global__ void __launch_bounds__(K::NT, 1)
    chl_kernel(const __grid_constant__ CUtensorMap tmap, const __grid_constant__ CUtensorMap omap,
               const Args a, const int tma_store) {
    static_assert(EPI == kNoEpilogue || !K::REV, "the epilogue belongs to the forward");
    using TA = typename K::TA;
    using IO = ActIO<TA>;
    extern __shared__ __align__(128) unsigned char smem[];
    TA* outbuf = reinterpret_cast<TA*>(smem + size_t(K::NS) * K::STAGE_PITCH);
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + size_t(K::NS) * K::STAGE_PITCH +
                                                 size_t(2 * K::NCW) * K::OUT_BYTES);
    uint64_t* empty = full + K::NS;
    volatile int* abort_flag = reinterpret_cast<volatile int*>(empty + K::NS);

    const int tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;
    const int t_begin = int((int64_t(blockIdx.x) * a.ntiles) / gridDim.x);
    const int t_end = int((int64_t(blockIdx.x + 1) * a.ntiles) / gridDim.x);

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
        if (lane == 0) {
            prefetch_tensor_map(&tmap);
            int k = 0;
            bool ok = true;
            for (int t = t_begin; t < t_end; ++t, ++k) {
                const int s = k % K::NS;
                if (k >= K::NS && !mbar_wait_or_abort(&empty[s], ((k / K::NS) - 1) & 1, abort_flag)) {
                    ok = false;
                    break;
                }
                int tx, h, cg, n;
                decode_tile<K>(t, a, tx, h, cg, n);
                mbar_arrive_expect_tx(&full[s], K::STAGE_BYTES);
                tma_load_4d(smem + size_t(s) * K::STAGE_PITCH, &tmap, &full[s],
                            tx * K::TW - a.pl - K::REM - a.sh4, h - a.pt, cg * K::CH, n);
            }
            if (!ok) {
                *abort_flag = 1;
                atomicExch(a.err, DW_ERR_DEVICE_TIMEOUT);
                for (int j = (k > K::NS ? k - K::NS : 0); j < k; ++j)
                    mbar_wait_bounded(&full[j % K::NS], (j / K::NS) & 1);
            }
        }
        return;
    }

    float wr[K::KW];
    float bias = 0.f;
    int cur_key = -1;
    bool live = false;
    // the value stored for one output: acc + bias (-> epilogue)
    auto finish = [&](float v) -> float {
        if constexpr (EPI != kNoEpilogue) return activate<EPI>(v + bias);
        else return v + bias;
    };
    int k = 0;
    for (int t = t_begin; t < t_end; ++t, ++k) {
        const int s = k % K::NS;
        int tx, h, cg, n;
        decode_tile<K>(t, a, tx, h, cg, n);
        const int c = cg * K::CH + lane;
        const int key = cg + n * a.tiles_c.d;
        if (key != cur_key) {
            cur_key = key;
            live = c < a.C;
            const int64_t base = int64_t(live ? c : 0) * K::KW;
            if (a.wtype == DW_F16) {
                const __half* wp = static_cast<const __half*>(a.w) + base;
#pragma unroll
                for (int kw = 0; kw < K::KW; ++kw)
                    wr[kw] = __half2float(wp[K::REV ? K::KW - 1 - kw : kw]);
            } else {
                const float* wp = static_cast<const float*>(a.w) + base;
#pragma unroll
                for (int kw = 0; kw < K::KW; ++kw) wr[kw] = __ldg(wp + (K::REV ? K::KW - 1 - kw : kw));
            }
            bias = (!K::REV && a.b != nullptr && live) ? __ldg(a.b + c) : 0.f;
            if constexpr (EPI != kNoEpilogue) {
                // fold the normalisation into the filter and the bias
                if (live) {
                    float sc, sh;
                    bn_scale_shift(a.epi, c, sc, sh);
#pragma unroll
                    for (int kw = 0; kw < K::KW; ++kw) wr[kw] *= sc;
                    bias = fmaf(bias, sc, sh);
                }
            }
        }

        if (!mbar_wait_or_abort(&full[s], (k / K::NS) & 1, abort_flag)) {
            if (lane == 0) {
                *abort_flag = 1;
                atomicExch(a.err, DW_ERR_DEVICE_TIMEOUT);
            }
            break;
        }

        float acc[K::TWT];
#pragma unroll
        for (int i = 0; i < K::TWT; ++i) acc[i] = 0.f;
        const TA* win = reinterpret_cast<const TA*>(smem + size_t(s) * K::STAGE_PITCH) +
                        lane * K::IWB + warp * K::TWT + a.sh4;
        static_for<0, K::NV>([&](auto u_) {
            constexpr int u = decltype(u_)::value;
            const float4 f = IO::load4(win + 4 * u);
            const float e[4] = {f.x, f.y, f.z, f.w};
            static_for<0, 4>([&](auto m_) {
                constexpr int q = 4 * u + decltype(m_)::value - K::REM;  // window column
                static_for<0, K::TWT>([&](auto i_) {
                    constexpr int i = decltype(i_)::value;
                    constexpr int kw = q - i;
                    if constexpr (kw >= 0 && kw < K::KW)
                        acc[i] = fmaf(e[decltype(m_)::value], wr[kw], acc[i]);
                });
            });
        });
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[s]);

        if (tma_store) {
            // warp-private staging slot ob: the store issued two tiles ago
            // by this warp must have finished reading it
            const int ob = k & 1;
            if (k >= 2 && lane == 0) bulk_wait_group_read<1>();
            __syncwarp();
            TA* o = outbuf + size_t(2 * warp + ob) * K::OUT_ELEMS + lane * K::TWT;
#pragma unroll
            for (int u = 0; u < K::TWT / 4; ++u)
                IO::store4(o + 4 * u, make_float4(finish(acc[4 * u]), finish(acc[4 * u + 1]),
                                                  finish(acc[4 * u + 2]), finish(acc[4 * u + 3])));
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
                tma_store_4d(&omap, outbuf + size_t(2 * warp + ob) * K::OUT_ELEMS,
                             tx * K::TW + warp * K::TWT, h, cg * K::CH, n);
                bulk_commit_group();
            }
        } else if (live && h < a.Hout) {
            const int wo0 = tx * K::TW + warp * K::TWT;
            TA* dst = static_cast<TA*>(a.out) + ((int64_t(n) * a.C + c) * a.Hout + h) * a.Wout + wo0;
            const bool vec = (a.Wout & 3) == 0;
#pragma unroll
            for (int u = 0; u < K::TWT / 4; ++u) {
                const float4 v = make_float4(finish(acc[4 * u]), finish(acc[4 * u + 1]),
                                             finish(acc[4 * u + 2]), finish(acc[4 * u + 3]));
                const int wo = wo0 + 4 * u;
                if (vec && wo + 3 < a.Wout) {
                    IO::store4(dst + 4 * u, v);
                } else {
                    if (wo < a.Wout) IO::store1(dst + 4 * u, v.x);
                    if (wo + 1 < a.Wout) IO::store1(dst + 4 * u + 1, v.y);
                    if (wo + 2 < a.Wout) IO::store1(dst + 4 * u + 2, v.z);
                    if (wo + 3 < a.Wout) IO::store1(dst + 4 * u + 3, v.w);
                }
            }
        }
    }
    if (tma_store && lane == 0) bulk_wait_group<0>();
}

template <class K>
dw_status_t launch_chl(const Problem& p, const void* in, const void* w, const float* b,
                       void* out, cudaStream_t stream, int32_t* err, bool dry_run, int pt_eff,
                       int pl_eff, int sh4) {
    const int64_t Hin = K::REV ? p.Ho : p.H, Win = K::REV ? p.Wo : p.W;
    Args a;
    a.w = w;
    a.b = K::REV ? nullptr : b;
    a.out = out;
    a.err = err;
    a.wtype = p.wtype;
    a.N = static_cast<int>(p.N);
    if (p.M != 1) return DW_ERR_UNSUPPORTED;  // boxes of 32 consecutive channels
    a.M = 1;
    a.C = static_cast<int>(p.C);
    a.Hout = static_cast<int>(K::REV ? p.H : p.Ho);
    a.Wout = static_cast<int>(K::REV ? p.W : p.Wo);
    a.pt = pt_eff;
    a.pl = pl_eff;
    a.sh4 = sh4;
    const int64_t tx = (a.Wout + K::TW - 1) / K::TW;
    const int64_t ty = a.Hout;
    const int64_t tc = (p.C + K::CH - 1) / K::CH;
    const int64_t nt = tx * ty * tc * p.N;
    if (nt >= INT_MAX) return DW_ERR_UNSUPPORTED;
    a.tiles_x = make_fastdiv(static_cast<int>(tx));
    a.tiles_y = make_fastdiv(static_cast<int>(ty));
    a.tiles_c = make_fastdiv(static_cast<int>(tc));
    a.ntiles = static_cast<int>(nt);
    a.epi = K::REV ? Epilogue{} : p.epi;
    if (dry_run) return DW_OK;

    const int ev = epilogue_variant(a.epi);
    void (*kern)(CUtensorMap, CUtensorMap, Args, int) = chl_kernel<K, kNoEpilogue>;
    if constexpr (!K::REV) {
        if (ev == DW_ACT_NONE) kern = chl_kernel<K, DW_ACT_NONE>;
        if (ev == DW_ACT_RELU) kern = chl_kernel<K, DW_ACT_RELU>;
        if (ev == DW_ACT_RELU6) kern = chl_kernel<K, DW_ACT_RELU6>;
        if (ev == DW_ACT_SILU) kern = chl_kernel<K, DW_ACT_SILU>;
    }
    static LaunchCache cache[5];
    const int dev = current_device();
    const int occ = prepare_kernel(reinterpret_cast<const void*>(kern), K::NT, K::SMEM,
                                   cache[ev + 1], dev);
    if (occ < 1) return DW_ERR_CUDA;
    CUtensorMap map;
    const cuuint64_t dims[4] = {cuuint64_t(Win), cuuint64_t(Hin), cuuint64_t(p.C), cuuint64_t(p.N)};
    constexpr cuuint64_t E = K::ESZ;
    constexpr CUtensorMapDataType dt = ActIO<typename K::TA>::kTma;
    const cuuint64_t strides[3] = {cuuint64_t(Win) * E, cuuint64_t(Win * Hin) * E,
                                   cuuint64_t(Win * Hin * p.C) * E};
    const cuuint32_t box[4] = {K::IWB, 1, K::CH, 1};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    if (encode_tensor_map(&map, dt, 4, const_cast<void*>(in), dims, strides, box, estr) !=
        CUDA_SUCCESS)
        return DW_ERR_CUDA;
    // output map for the per-warp bulk stores (row pitch must be a multiple
    // of 16 bytes, as for every tensor map)
    CUtensorMap omap = map;
    int tma_store = 0;
    if ((int64_t(a.Wout) * K::ESZ) % 16 == 0) {
        const cuuint64_t odims[4] = {cuuint64_t(a.Wout), cuuint64_t(a.Hout), cuuint64_t(p.C),
                                     cuuint64_t(p.N)};
        const cuuint64_t ostrides[3] = {cuuint64_t(a.Wout) * E, cuuint64_t(a.Wout) * a.Hout * E,
                                        cuuint64_t(a.Wout) * a.Hout * p.C * E};
        const cuuint32_t obox[4] = {K::TWT, 1, K::CH, 1};
        if (encode_tensor_map(&omap, dt, 4, out, odims, ostrides, obox, estr) != CUDA_SUCCESS)
            return DW_ERR_CUDA;
        tma_store = 1;
    }
    int64_t grid = int64_t(sm_count(dev)) * occ;
    if (grid > a.ntiles) grid = a.ntiles;
    if (launch_pdl(kern, dim3(static_cast<unsigned>(grid)), dim3(K::NT), K::SMEM, stream, map,
                   omap, a, tma_store) != cudaSuccess)
        return DW_ERR_CUDA;
    return cudaGetLastError() == cudaSuccess ? DW_OK : DW_ERR_CUDA;
}

// ---------------------------------------------------------------------------
// Input gradient at stride 2 (stride-2 input-VJP sections): dx(hi, wi) gathers
// W[kh][kw] * dy((hi + pt - kh) / 2, (wi + pl - kw) / 2) over the taps for
// which both divisions are exact.  A tile is TH x TW dx values at the aligned
// origin (ty*TH, tx*TW); with PH = pt mod 2 and PW = pl mod 2 as template
// parameters, every (dx row, tap) and (dx column, tap) pairing is known at
// compile time.  A lane owns 8 consecutive dx columns, which read 6
// consecutive dy columns (2 or 3 aligned 4-vectors), and THT rows; results
// leave as two 4-vectors per row.  The dy box starts at the row
// ty*TH/2 + floor(pt/2) - AH and at the column tx*TW/2 + floor(pl/2) - AW,
// moved left by REM (compile time) + sh4 (run time) to a 16-byte boundary.
template <int KH_, int KW_, int PH_, int PW_, int REM_, int THT_, int WX_, int WY_, int NS_,
          class TA_, int MP_ = 1>
struct T2Cfg {
    using TA = TA_;
    // channel multiplier: the box holds the MP dy planes c*MP .. of dx plane c,
    // whose contributions are summed
    static constexpr int MP = MP_;
    static constexpr int ESZ = sizeof(TA), ALIGN = 16 / ESZ;
    static constexpr int KH = KH_, KW = KW_, PH = PH_, PW = PW_, REM = REM_;
    static constexpr int THT = THT_, WX = WX_, WY = WY_, NS = NS_;
    static constexpr int NCW = WX * WY / 32, NT = WX * WY + 32;
    static constexpr int TW = 8 * WX, TH = THT * WY;     // dx tile
    static constexpr int AH = KH / 2, AW = KW / 2;      // dy rows / columns before the tile's
    static constexpr int DMAX = (7 + PW) / 2;           // largest (e + PW - kw) / 2
    static constexpr int NV = (DMAX + AW + REM) / 4 + 1;  // 4-vectors per lane and dy row
    static constexpr int IH = AH + (TH - 1 + PH) / 2 + 1;
    static constexpr int IWB =
        ((TW / 2 - 4 + 4 * NV + (ALIGN - 4)) + ALIGN - 1) / ALIGN * ALIGN;
    static constexpr int RH = AH + (THT - 1 + PH) / 2 + 1;  // dy rows one thread reads
    static constexpr int STAGE_BYTES = IWB * IH * MP * ESZ;
    static constexpr int STAGE_PITCH = (STAGE_BYTES + 127) / 128 * 128;
    static constexpr size_t SMEM = size_t(NS) * STAGE_PITCH + size_t(2 * NS) * 8 + 16;
    static_assert(THT % 2 == 0 && (TW / 2) % ALIGN == 0, "even rows, aligned dy columns");
    static_assert((WX * WY) % 32 == 0, "whole consumer warps");
    static_assert(IWB <= 256 && IH <= 256, "TMA box dimension limit");
    static_assert(SMEM <= 227 * 1024, "shared memory per CTA");
};

template <class K>
__global__ void __launch_bounds__(K::NT, 1)
    t2_kernel(const __grid_constant__ CUtensorMap tmap, const Args a) {
    using TA = typename K::TA;
    using IO = ActIO<TA>;
    extern __shared__ __align__(128) unsigned char smem[];
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + size_t(K::NS) * K::STAGE_PITCH);
    uint64_t* empty = full + K::NS;
    volatile int* abort_flag = reinterpret_cast<volatile int*>(empty + K::NS);
    const int tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;
    const int t_begin = int((int64_t(blockIdx.x) * a.ntiles) / gridDim.x);
    const int t_end = int((int64_t(blockIdx.x + 1) * a.ntiles) / gridDim.x);

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

    // a.pt, a.pl hold floor(pt/2) and floor(pl/2)
    if (warp == K::NCW) {
        if (lane == 0) {
            prefetch_tensor_map(&tmap);
            int k = 0;
            bool ok = true;
            for (int t = t_begin; t < t_end; ++t, ++k) {
                const int s = k % K::NS;
                if (k >= K::NS && !mbar_wait_or_abort(&empty[s], ((k / K::NS) - 1) & 1, abort_flag)) {
                    ok = false;
                    break;
                }
                int tx, ty, c, n;
                decode_tile<K>(t, a, tx, ty, c, n);
                mbar_arrive_expect_tx(&full[s], K::STAGE_BYTES);
                tma_load_4d(smem + size_t(s) * K::STAGE_PITCH, &tmap, &full[s],
                            tx * (K::TW / 2) + a.pl - K::AW - K::REM - a.sh4,
                            ty * (K::TH / 2) + a.pt - K::AH, c * K::MP, n);
            }
            if (!ok) {
                *abort_flag = 1;
                atomicExch(a.err, DW_ERR_DEVICE_TIMEOUT);
                for (int j = (k > K::NS ? k - K::NS : 0); j < k; ++j)
                    mbar_wait_bounded(&full[j % K::NS], (j / K::NS) & 1);
            }
        }
        return;
    }

    const int xi = tid % K::WX;
    const int yi = tid / K::WX;
    const int row0 = yi * K::THT;  // first dx row of this thread in the tile (even)
    float wr[K::MP][K::KH][K::KW];
    int cur_key = -1;
    bool live = false;
    int k = 0;
    for (int t = t_begin; t < t_end; ++t, ++k) {
        const int s = k % K::NS;
        int tx, ty, c, n;
        decode_tile<K>(t, a, tx, ty, c, n);
        const int key = c + n * a.tiles_c.d;
        if (key != cur_key) {
            cur_key = key;
            live = c < a.C;
#pragma unroll
            for (int m = 0; m < K::MP; ++m) {
                // filter of output channel c*MP + m
                const int64_t base = (int64_t(live ? c : 0) * K::MP + m) * (K::KH * K::KW);
#pragma unroll
                for (int kh = 0; kh < K::KH; ++kh)
#pragma unroll
                    for (int kw = 0; kw < K::KW; ++kw)
                        wr[m][kh][kw] =
                            live ? load_weight(a.w, a.wtype, base + kh * K::KW + kw) : 0.f;
            }
        }
        if (!mbar_wait_or_abort(&full[s], (k / K::NS) & 1, abort_flag)) {
            if (lane == 0) {
                *abort_flag = 1;
                atomicExch(a.err, DW_ERR_DEVICE_TIMEOUT);
            }
            break;
        }
        float acc[K::THT][8];
#pragma unroll
        for (int j = 0; j < K::THT; ++j)
#pragma unroll
            for (int e = 0; e < 8; ++e) acc[j][e] = 0.f;
        // dy row (row0/2 + rr) of the box and the lane's dy columns from 4*xi
        const TA* win0 = reinterpret_cast<const TA*>(smem + size_t(s) * K::STAGE_PITCH) +
                         size_t(row0 / 2) * K::IWB + 4 * xi + a.sh4;
        static_for<0, K::MP>([&](auto m_) {
            constexpr int m = decltype(m_)::value;
            const TA* win = win0 + size_t(m) * K::IH * K::IWB;  // dy plane c*MP + m
            static_for<0, K::RH>([&](auto rr_) {
                constexpr int rr = decltype(rr_)::value;
                float v[4 * K::NV];
#pragma unroll
                for (int u = 0; u < K::NV; ++u) {
                    const float4 f = IO::load4(win + rr * K::IWB + 4 * u);
                    v[4 * u] = f.x; v[4 * u + 1] = f.y; v[4 * u + 2] = f.z; v[4 * u + 3] = f.w;
                }
                static_for<0, K::THT>([&](auto j_) {
                    constexpr int j = decltype(j_)::value;
                    static_for<0, K::KH>([&](auto kh_) {
                        constexpr int kh = decltype(kh_)::value;
                        // dx row row0 + j reads dy box row row0/2 + (j + PH - kh)/2 + AH
                        constexpr int num = j + K::PH - kh;
                        if constexpr (num % 2 == 0 && num / 2 + K::AH == rr) {
                            static_for<0, 8>([&](auto e_) {
                                constexpr int e = decltype(e_)::value;
                                static_for<0, K::KW>([&](auto kw_) {
                                    constexpr int kw = decltype(kw_)::value;
                                    constexpr int numw = e + K::PW - kw;
                                    if constexpr (((numw % 2) + 2) % 2 == 0)
                                        acc[j][e] = fmaf(wr[m][kh][kw],
                                                         v[numw / 2 + K::AW + K::REM], acc[j][e]);
                                });
                            });
                        }
                    });
                });
            });
        });
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[s]);

        if (live) {
            const int wi0 = tx * K::TW + 8 * xi;
#pragma unroll
            for (int j = 0; j < K::THT; ++j) {
                const int hi = ty * K::TH + row0 + j;
                if (hi >= a.Hout) continue;
                TA* dst = static_cast<TA*>(a.out) + ((int64_t(n) * a.C + c) * a.Hout + hi) * a.Wout + wi0;
                const float4 lo = make_float4(acc[j][0], acc[j][1], acc[j][2], acc[j][3]);
                const float4 hi4 = make_float4(acc[j][4], acc[j][5], acc[j][6], acc[j][7]);
                if ((a.Wout & 3) == 0 && wi0 + 7 < a.Wout) {
                    IO::store4(dst, lo);
                    IO::store4(dst + 4, hi4);
                } else {
                    const float vals[8] = {lo.x, lo.y, lo.z, lo.w, hi4.x, hi4.y, hi4.z, hi4.w};
#pragma unroll
                    for (int e = 0; e < 8; ++e)
                        if (wi0 + e < a.Wout) IO::store1(dst + e, vals[e]);
                }
            }
        }
    }
}

template <class K>
dw_status_t launch_t2(const Problem& p, const void* in, const void* w, void* out,
                      cudaStream_t stream, int32_t* err, bool dry_run, int sh4) {
    Args a;
    a.w = w;
    a.b = nullptr;
    a.out = out;
    a.err = err;
    a.wtype = p.wtype;
    if (p.M != K::MP) return DW_ERR_UNSUPPORTED;
    a.M = 1;
    a.N = int(p.N);
    a.C = int(p.C);
    a.Cout = int(p.C);
    a.Hout = int(p.H);
    a.Wout = int(p.W);
    a.pt = p.pt / 2;  // floor(pt/2), floor(pl/2): the parities are template parameters
    a.pl = p.pl / 2;
    a.sh4 = sh4;
    const int64_t tx = (p.W + K::TW - 1) / K::TW, ty = (p.H + K::TH - 1) / K::TH;
    const int64_t nt = tx * ty * p.C * p.N;
    if (nt >= INT_MAX) return DW_ERR_UNSUPPORTED;
    a.tiles_x = make_fastdiv(int(tx));
    a.tiles_y = make_fastdiv(int(ty));
    a.tiles_c = make_fastdiv(int(p.C));
    a.ntiles = int(nt);
    if (dry_run) return DW_OK;
    static LaunchCache cache;
    const int dev = current_device();
    const int occ = prepare_kernel(reinterpret_cast<const void*>(&t2_kernel<K>), K::NT, K::SMEM,
                                   cache, dev);
    if (occ < 1) return DW_ERR_CUDA;
    CUtensorMap map;
    constexpr cuuint64_t E = K::ESZ;
    // dy: Co = C*MP planes
    const cuuint64_t dims[4] = {cuuint64_t(p.Wo), cuuint64_t(p.Ho), cuuint64_t(p.Co), cuuint64_t(p.N)};
    const cuuint64_t strides[3] = {cuuint64_t(p.Wo) * E, cuuint64_t(p.Wo * p.Ho) * E,
                                   cuuint64_t(p.Wo * p.Ho * p.Co) * E};
    const cuuint32_t box[4] = {K::IWB, K::IH, K::MP, 1};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    if (encode_tensor_map(&map, ActIO<typename K::TA>::kTma, 4, const_cast<void*>(in), dims,
                          strides, box, estr) != CUDA_SUCCESS)
        return DW_ERR_CUDA;
    int64_t grid = int64_t(sm_count(dev)) * occ;
    if (grid > a.ntiles) grid = a.ntiles;
    if (launch_pdl(t2_kernel<K>, dim3(unsigned(grid)), dim3(K::NT), K::SMEM, stream, map, a) !=
        cudaSuccess)
        return DW_ERR_CUDA;
    return cudaGetLastError() == cudaSuccess ? DW_OK : DW_ERR_CUDA;
}

// dispatch on the pad parities and the box remainder
template <int KH, int KW, int THT, int WX, int WY, int NS, class TA, int MP = 1>
dw_status_t launch_t2_any(const Problem& p, const void* in, const void* w, void* out,
                          cudaStream_t stream, int32_t* err, bool dry_run) {
    constexpr int align = 16 / int(sizeof(TA));
    const int full = ((p.pl / 2 - KW / 2) % align + align) % align;  // box start mod 16 bytes
    const int rem = full % 4, sh4 = full - rem;
    const int par = (p.pt & 1) * 2 + (p.pl & 1);
#define DW_T2(PH, PW, R) \
    return launch_t2<T2Cfg<KH, KW, PH, PW, R, THT, WX, WY, NS, TA, MP>>(p, in, w, out, stream, err, dry_run, sh4);
#define DW_T2R(PH, PW) \
    switch (rem) { case 0: DW_T2(PH, PW, 0) case 1: DW_T2(PH, PW, 1) case 2: DW_T2(PH, PW, 2) default: DW_T2(PH, PW, 3) }
    switch (par) {
        case 0: DW_T2R(0, 0)
        case 1: DW_T2R(0, 1)
        case 2: DW_T2R(1, 0)
        default: DW_T2R(1, 1)
    }
#undef DW_T2R
#undef DW_T2
}

// Box shift (-pl) mod (16 bytes / element size): its part mod 4 is the
// configuration's REM, the rest (0 or 4) the run-time sh4.
template <class TA>
void box_shift(int pl_eff, int& rem, int& sh4) {
    constexpr int align = 16 / int(sizeof(TA));
    const int full = ((-pl_eff) % align + align) % align;
    rem = full % 4;
    sh4 = full - rem;
}

template <int KW, bool REV, int TWT, int NCW, int NS, class TA>
dw_status_t launch_chl_rem(const Problem& p, const void* in, const void* w, const float* b,
                           void* out, cudaStream_t stream, int32_t* err, bool dry_run,
                           int pt_eff, int pl_eff) {
    int rem, sh4;
    box_shift<TA>(pl_eff, rem, sh4);
#define DW_CHL(R) \
    return launch_chl<ClCfg<KW, REV, R, TWT, NCW, NS, TA>>(p, in, w, b, out, stream, err, \
                                                           dry_run, pt_eff, pl_eff, sh4);
    switch (rem) {
        case 0: DW_CHL(0)
        case 1: DW_CHL(1)
        case 2: DW_CHL(2)
        default: DW_CHL(3)
    }
#undef DW_CHL
}

template <int KW, int TWT, int NCW, int NS, class TA>
dw_status_t launch_chl_op(const Problem& p, Op op, const void* in, const void* w, const float* b,
                          void* out, cudaStream_t stream, int32_t* err, bool dry_run) {
    if (op == OP_FWD)
        return launch_chl_rem<KW, false, TWT, NCW, NS, TA>(p, in, w, b, out, stream, err, dry_run,
                                                           p.pt, p.pl);
    return launch_chl_rem<KW, true, TWT, NCW, NS, TA>(p, in, w, b, out, stream, err, dry_run,
                                                      -p.pt, (KW - 1) - p.pl);
}

template <int KH, int KW, bool REV, int THT, int WX, int WY, int NS, int MINB, class TA, int PL = 1,
          int MP = 1>
dw_status_t launch_rem(const Problem& p, const void* in, const void* w, const float* b,
                       void* out, cudaStream_t stream, int32_t* err, bool dry_run, int pt_eff,
                       int pl_eff) {
    int rem, sh4;
    box_shift<TA>(pl_eff, rem, sh4);
#define DW_2D(R) \
    return launch<Cfg<KH, KW, 1, REV, R, THT, WX, WY, NS, MINB, TA, 1, PL, MP>>(     \
        p, in, w, b, out, stream, err, dry_run, pt_eff, pl_eff, sh4);
    switch (rem) {
        case 0: DW_2D(0)
        case 1: DW_2D(1)
        case 2: DW_2D(2)
        default: DW_2D(3)
    }
#undef DW_2D
}

template <int KH, int KW, int THT, int WX, int WY, int NS, class TA, int MINB = 1, int PL = 1>
dw_status_t launch_op(const Problem& p, Op op, const void* in, const void* w, const float* b,
                      void* out, cudaStream_t stream, int32_t* err, bool dry_run) {
    if (op == OP_FWD)
        return launch_rem<KH, KW, false, THT, WX, WY, NS, MINB, TA, PL>(p, in, w, b, out, stream,
                                                                        err, dry_run, p.pt, p.pl);
    return launch_rem<KH, KW, true, THT, WX, WY, NS, MINB, TA, PL>(p, in, w, b, out, stream, err,
                                                                   dry_run, (KH - 1) - p.pt,
                                                                   (KW - 1) - p.pl);
}

// Channel multiplier MP inside a tile (stride 1): the forward computes the MP
// output planes of one input plane, the input gradient sums the MP dy planes
// of one dx plane (one box).  OPS: 1 = forward only, 2 = input gradient only,
// 3 = both.
template <int KH, int KW, int THT, int WX, int WY, int NS, class TA, int MP, int OPS = 3>
dw_status_t launch_mult(const Problem& p, Op op, const void* in, const void* w, const float* b,
                        void* out, cudaStream_t stream, int32_t* err, bool dry_run) {
    if (op == OP_FWD) {
        if constexpr ((OPS & 1) != 0)
            return launch_rem<KH, KW, false, THT, WX, WY, NS, 1, TA, 1, MP>(
                p, in, w, b, out, stream, err, dry_run, p.pt, p.pl);
        return DW_ERR_UNSUPPORTED;
    }
    if constexpr ((OPS & 2) != 0)
        return launch_rem<KH, KW, true, THT, WX, WY, NS, 1, TA, 1, MP>(
            p, in, w, nullptr, out, stream, err, dry_run, (KH - 1) - p.pt, (KW - 1) - p.pl);
    return DW_ERR_UNSUPPORTED;
}

// Stride-2 forward (2-D kernel with S = 2): a tile is TH x 4*WX outputs, its
// box the (TH-1)*2 + kH rows and (TW-1)*2 + kW columns they read.
template <int KH, int KW, int THT, int WX, int WY, int NS, class TA, int PL = 1, int MP = 1>
dw_status_t launch_s2_fwd(const Problem& p, const void* in, const void* w, const float* b,
                          void* out, cudaStream_t stream, int32_t* err, bool dry_run) {
    int rem, sh4;
    box_shift<TA>(p.pl, rem, sh4);
#define DW_S2(R) \
    return launch<Cfg<KH, KW, 1, false, R, THT, WX, WY, NS, 1, TA, 2, PL, MP>>(        \
        p, in, w, b, out, stream, err, dry_run, p.pt, p.pl, sh4);
    switch (rem) {
        case 0: DW_S2(0)
        case 1: DW_S2(1)
        case 2: DW_S2(2)
        default: DW_S2(3)
    }
#undef DW_S2
}

// The configurations of one activation type.
template <class TA>
dw_status_t nchw_launch_t(const Problem& p, Op op, const void* in, const void* w, const float* b,
                          void* out, cudaStream_t stream, int32_t* err, bool dry_run) {
    if (p.dh != 1 || p.dw != 1) return DW_ERR_UNSUPPORTED;
    if (p.sh == 2 && p.sw == 2) {
        // strided: the forward of 3x3 filters (input gradients on the direct kernel)
        if (op == OP_FWD && p.kH == 3 && p.kW == 3) {
            // small planes (at most 32 output columns): 4 planes of 32 x 32 outputs per tile
            if (p.Wo <= 32 && p.M == 1)
                return launch_s2_fwd<3, 3, 4, 8, 32, 3, TA, 4>(p, in, w, b, out, stream, err, dry_run);
            if (p.M == 2)  // both output planes of an input plane per tile
                return launch_s2_fwd<3, 3, 2, 16, 16, 4, TA, 1, 2>(p, in, w, b, out, stream, err, dry_run);
            return launch_s2_fwd<3, 3, 2, 16, 16, 4, TA>(p, in, w, b, out, stream, err, dry_run);
        }
        if (op == OP_BWD_INPUT && p.kH == 3 && p.kW == 3 && (p.M == 1 || p.M == 2)) {
            //                                           KH KW THT WX WY NS
            if (p.M == 2 && p.W <= 64) return launch_t2_any<3, 3, 4, 8, 16, 4, TA, 2>(p, in, w, out, stream, err, dry_run);
            if (p.M == 2) return launch_t2_any<3, 3, 4, 16, 16, 4, TA, 2>(p, in, w, out, stream, err, dry_run);
            if (p.W <= 64) return launch_t2_any<3, 3, 4, 8, 16, 4, TA>(p, in, w, out, stream, err, dry_run);
            return launch_t2_any<3, 3, 4, 16, 16, 4, TA>(p, in, w, out, stream, err, dry_run);
        }
        return DW_ERR_UNSUPPORTED;
    }
    if (p.sh != 1 || p.sw != 1) return DW_ERR_UNSUPPORTED;
    if (p.M != 1) {
        // the input gradient's box of M dy planes (M = 4: half the rows per tile)
        const bool fw = op == OP_FWD;
        //                                                          KH KW THT WX WY NS     MP OPS
        if (p.kH == 3 && p.kW == 3 && p.M == 2) return launch_mult<3, 3, 4, 32, 8, 4, TA, 2>(p, op, in, w, b, out, stream, err, dry_run);
        if (p.kH == 3 && p.kW == 3 && p.M == 4 && fw) return launch_mult<3, 3, 4, 32, 8, 4, TA, 4, 1>(p, op, in, w, b, out, stream, err, dry_run);
        if (p.kH == 3 && p.kW == 3 && p.M == 4) return launch_mult<3, 3, 2, 32, 8, 4, TA, 4, 2>(p, op, in, w, b, out, stream, err, dry_run);
        if (p.kH == 5 && p.kW == 5 && p.M == 2) return launch_mult<5, 5, 4, 32, 8, 4, TA, 2>(p, op, in, w, b, out, stream, err, dry_run);
        if (p.kH == 7 && p.kW == 7 && p.M == 2 && !fw) return launch_mult<7, 7, 4, 32, 4, 4, TA, 2, 2>(p, op, in, w, b, out, stream, err, dry_run);
        if (op == OP_BWD_INPUT) return DW_ERR_UNSUPPORTED;
        // other multipliers: one output plane per tile (below)
    }
    // small planes (at most 64 columns, the 3x3 and 5x5 filters): 2 planes of
    // 32 x 64 per tile instead of one plane in a 32 x 128 tile
    const int64_t wmax = p.W > p.Wo ? p.W : p.Wo;
    //                                                                    KH KW THT WX WY NS     MINB PL
    const bool small = wmax <= 64 && p.M == 1;  // several planes per tile need M = 1
    if (small && p.kH == 3 && p.kW == 3) return launch_op<3, 3, 4, 16, 16, 4, TA, 1, 2>(p, op, in, w, b, out, stream, err, dry_run);
    if (small && p.kH == 5 && p.kW == 5) return launch_op<5, 5, 4, 16, 16, 4, TA, 1, 2>(p, op, in, w, b, out, stream, err, dry_run);
    //                                                       KH  KW THT WX  WY NS
    if (p.kH == 3 && p.kW == 3) return launch_op<3, 3, 4, 32, 8, 4, TA>(p, op, in, w, b, out, stream, err, dry_run);
    if (p.kH == 5 && p.kW == 5) return launch_op<5, 5, 4, 32, 8, 4, TA>(p, op, in, w, b, out, stream, err, dry_run);
    if (p.kH == 7 && p.kW == 7) return launch_op<7, 7, 4, 32, 4, 4, TA>(p, op, in, w, b, out, stream, err, dry_run);
    //                                               KW TWT NCW NS
    if (p.kH == 1 && p.kW == 15) return launch_chl_op<15, 16, 8, 4, TA>(p, op, in, w, b, out, stream, err, dry_run);
    if (p.kH == 1 && p.kW == 31) return launch_chl_op<31, 16, 8, 4, TA>(p, op, in, w, b, out, stream, err, dry_run);
    return DW_ERR_UNSUPPORTED;
}

// Instantiation units: dw_tiled_nchw.cu (float32 and the family's
// dispatcher), dw_tiled_nchw_f16.cu, dw_tiled_nchw_bf16.cu.
dw_status_t nchw_launch_f32(const Problem& p, Op op, const void* in, const void* w,
                            const float* b, void* out, cudaStream_t stream, int32_t* err,
                            bool dry_run);
dw_status_t nchw_launch_f16(const Problem& p, Op op, const void* in, const void* w,
                            const float* b, void* out, cudaStream_t stream, int32_t* err,
                            bool dry_run);
dw_status_t nchw_launch_bf16(const Problem& p, Op op, const void* in, const void* w,
                             const float* b, void* out, cudaStream_t stream, int32_t* err,
                             bool dry_run);

}  // namespace nchw
}  // namespace dw
