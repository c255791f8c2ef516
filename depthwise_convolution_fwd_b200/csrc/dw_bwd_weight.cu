// Weight and bias gradients (page "LeanMlir Proofs/Architectures/Depthwise",
// sections "Depthwise weight-VJP", "Depthwise bias gradient - closed-form
// formula" and the stride-2 / XLA-SAME weight and bias VJP sections):
//
//   dW[c,kh,kw] = sum_{n,ho,wo} dy[n,ho,wo,c] * X(n, ho*sh + kh*dh - pt,
//                                                 wo*sw + kw*dw - pl, c)
//   db[c]       = sum_{n,ho,wo} dy[n,ho,wo,c]
//
// A per-channel reduction over every output position, done in two levels
// with a deterministic order (no atomics):
//   1. partial kernels write one float64 partial per (block of work, tap,
//      channel) into the caller's workspace.  Inside a thread, products are
//      summed in float32 over at most a handful of outputs and then folded
//      into float64, so the result is accurate to well below float32
//      rounding of the final value.
//   2. a finalize kernel sums each channel's partials in a fixed order and
//      writes dW / db as float32.
// The tiled partial kernels load, per tile, the input halo box and the
// matching dy box into one pipeline stage (TMA).  NHWC: lane = channel (a
// warp covers the 32 channels of a pixel), each thread owns THT x TWT outputs
// and streams its input window once, feeding every (output, tap) pair at
// compile-time offsets.  NCHW (stride 1): lanes run along W, 4 outputs per
// lane; a CTA works through whole units (one row band of one (n, c) plane)
// and reduces each unit to one float64 partial per tap.  The direct partial
// kernels cover every other shape.
#include <climits>

#include "dw_common.cuh"

namespace dw {
namespace wgrad {

constexpr int kLanes = 32;          // channels per tiled work block
constexpr int kMaxTiledCtas = 1024; // cap on the tiled grid (sizes the workspace)
constexpr int kMaxChunks = 128;     // direct kernels: position chunks per (tap, channel)
constexpr int64_t kMinChunk = 256;  // direct kernels: positions per chunk at least
constexpr int kFold = 16;           // direct kernels: float32 terms per float64 fold

// ----------------------------------------------------------- direct kernels --

struct DArgs {
    int64_t N, C, H, W, Ho, Wo;
    int64_t M, Co;   // output channels per input channel, output channels
    int kH, kW, sh, sw, dh, dw, pt, pl;
    int T;           // taps + 1 (the last slot is the bias)
    int64_t P;       // output positions per channel = N*Ho*Wo
    int64_t chunk;   // positions per chunk
    int64_t chunks;  // number of chunks
    int64_t items;   // chunks * T * C
};

// NHWC: one thread per (chunk, tap, channel), channel fastest, so a warp reads
// 32 consecutive channels of one pixel.
template <class TA>
__global__ void __launch_bounds__(256) partial_direct_nhwc(const TA* __restrict__ x,
                                                           const TA* __restrict__ dy,
                                                           double* __restrict__ part, DArgs a) {
    grid_dependency_wait();
    allow_dependents();
    const int64_t stride = int64_t(gridDim.x) * blockDim.x;
    for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < a.items; i += stride) {
        const int64_t o = i % a.Co;  // output channel; it reads input channel o / M
        const int64_t c = o / a.M;
        const int64_t r = i / a.Co;
        const int t = int(r % a.T);
        const int64_t j = r / a.T;
        const bool bias = t == a.T - 1;
        const int kh = bias ? 0 : t / a.kW, kw = bias ? 0 : t % a.kW;
        const int64_t p0 = j * a.chunk;
        const int64_t p1 = p0 + a.chunk < a.P ? p0 + a.chunk : a.P;
        int64_t wo = p0 % a.Wo, q = p0 / a.Wo;
        int64_t ho = q % a.Ho, n = q / a.Ho;
        double acc = 0.0;
        float part32 = 0.f;
        int cnt = 0;
        for (int64_t pp = p0; pp < p1; ++pp) {
            const float g = ActIO<TA>::load1(dy + ((n * a.Ho + ho) * a.Wo + wo) * a.Co + o);
            if (bias) {
                part32 += g;
            } else {
                const int64_t hi = ho * a.sh + int64_t(kh) * a.dh - a.pt;
                const int64_t wi = wo * a.sw + int64_t(kw) * a.dw - a.pl;
                if (hi >= 0 && hi < a.H && wi >= 0 && wi < a.W)
                    part32 = fmaf(g, ActIO<TA>::load1(x + ((n * a.H + hi) * a.W + wi) * a.C + c),
                                  part32);
            }
            if (++cnt == kFold) {
                acc += double(part32);
                part32 = 0.f;
                cnt = 0;
            }
            if (++wo == a.Wo) {
                wo = 0;
                if (++ho == a.Ho) {
                    ho = 0;
                    ++n;
                }
            }
        }
        part[i] = acc + double(part32);
    }
}

// NCHW: one warp per (chunk, tap, channel); lanes walk consecutive output
// positions (W innermost), then the warp sums its lanes.
template <class TA>
__global__ void __launch_bounds__(256) partial_direct_nchw(const TA* __restrict__ x,
                                                           const TA* __restrict__ dy,
                                                           double* __restrict__ part, DArgs a) {
    grid_dependency_wait();
    allow_dependents();
    const int lane = threadIdx.x & 31;
    const int64_t warps = int64_t(gridDim.x) * (blockDim.x >> 5);
    for (int64_t i = (int64_t(blockIdx.x) * blockDim.x + threadIdx.x) >> 5; i < a.items;
         i += warps) {
        const int64_t o = i % a.Co;  // output channel; it reads input channel o / M
        const int64_t c = o / a.M;
        const int64_t r = i / a.Co;
        const int t = int(r % a.T);
        const int64_t j = r / a.T;
        const bool bias = t == a.T - 1;
        const int kh = bias ? 0 : t / a.kW, kw = bias ? 0 : t % a.kW;
        const int64_t p0 = j * a.chunk;
        const int64_t p1 = p0 + a.chunk < a.P ? p0 + a.chunk : a.P;
        double acc = 0.0;
        float part32 = 0.f;
        int cnt = 0;
        for (int64_t pp = p0 + lane; pp < p1; pp += 32) {
            const int64_t wo = pp % a.Wo, q = pp / a.Wo;
            const int64_t ho = q % a.Ho, n = q / a.Ho;
            const float g = ActIO<TA>::load1(dy + ((n * a.Co + o) * a.Ho + ho) * a.Wo + wo);
            if (bias) {
                part32 += g;
            } else {
                const int64_t hi = ho * a.sh + int64_t(kh) * a.dh - a.pt;
                const int64_t wi = wo * a.sw + int64_t(kw) * a.dw - a.pl;
                if (hi >= 0 && hi < a.H && wi >= 0 && wi < a.W)
                    part32 = fmaf(g, ActIO<TA>::load1(x + ((n * a.C + c) * a.H + hi) * a.W + wi),
                                  part32);
            }
            if (++cnt == kFold) {
                acc += double(part32);
                part32 = 0.f;
                cnt = 0;
            }
        }
        acc += double(part32);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
        if (lane == 0) part[i] = acc;
    }
}

// NCHW with the filter extent known at compile time: one warp per (chunk,
// output channel) forms every tap's sum at once, so each dy value is read
// once (not once per tap) and the x values a position's taps share come from
// L1.  Partials in the layout of partial_direct_nchw, same finalize.
template <class TA, int KH, int KW>
__global__ void __launch_bounds__(256) partial_direct_nchw_taps(const TA* __restrict__ x,
                                                                const TA* __restrict__ dy,
                                                                double* __restrict__ part, DArgs a) {
    grid_dependency_wait();
    allow_dependents();
    constexpr int T = KH * KW + 1;
    const int lane = threadIdx.x & 31;
    const int64_t warps = int64_t(gridDim.x) * (blockDim.x >> 5);
    const int64_t n_items = a.chunks * a.Co;
    for (int64_t i = (int64_t(blockIdx.x) * blockDim.x + threadIdx.x) >> 5; i < n_items;
         i += warps) {
        const int64_t o = i % a.Co;  // output channel; it reads input channel o / M
        const int64_t c = o / a.M;
        const int64_t j = i / a.Co;
        const int64_t p0 = j * a.chunk;
        const int64_t p1 = p0 + a.chunk < a.P ? p0 + a.chunk : a.P;
        double acc64[T];
        float acc[T];
#pragma unroll
        for (int t = 0; t < T; ++t) {
            acc64[t] = 0.0;
            acc[t] = 0.f;
        }
        int cnt = 0;
        const TA* xc = x + c * a.H * a.W;  // plane of (n = 0, c); n added below
        for (int64_t pp = p0 + lane; pp < p1; pp += 32) {
            const int64_t wo = pp % a.Wo, q = pp / a.Wo;
            const int64_t ho = q % a.Ho, n = q / a.Ho;
            const float g = ActIO<TA>::load1(dy + ((n * a.Co + o) * a.Ho + ho) * a.Wo + wo);
            const TA* xp = xc + n * a.C * a.H * a.W;
#pragma unroll
            for (int kh = 0; kh < KH; ++kh) {
                const int64_t hi = ho * a.sh + int64_t(kh) * a.dh - a.pt;
                const bool hin = hi >= 0 && hi < a.H;
#pragma unroll
                for (int kw = 0; kw < KW; ++kw) {
                    const int64_t wi = wo * a.sw + int64_t(kw) * a.dw - a.pl;
                    if (hin && wi >= 0 && wi < a.W)
                        acc[kh * KW + kw] = fmaf(g, ActIO<TA>::load1(xp + hi * a.W + wi),
                                                 acc[kh * KW + kw]);
                }
            }
            acc[T - 1] += g;
            if (++cnt == kFold) {
#pragma unroll
                for (int t = 0; t < T; ++t) {
                    acc64[t] += double(acc[t]);
                    acc[t] = 0.f;
                }
                cnt = 0;
            }
        }
#pragma unroll
        for (int t = 0; t < T; ++t) {
            double v = acc64[t] + double(acc[t]);
#pragma unroll
            for (int s = 16; s > 0; s >>= 1) v += __shfl_xor_sync(0xffffffffu, v, s);
            if (lane == 0) part[(j * T + t) * a.Co + o] = v;
        }
    }
}

// Fixed-order sum of `count` float64 terms by one warp: lane l adds terms
// l, l+32, ... in order, then a fixed butterfly combines the lanes; lane 0's
// value is the result (the same bits on every run).  32 independent load
// streams hide the latency a single thread's sequential sum would expose.
template <class F>
__device__ __forceinline__ double warp_ordered_sum(int64_t count, F&& term) {
    const int lane = threadIdx.x & 31;
    double s = 0.0;
#pragma unroll 4
    for (int64_t j = lane; j < count; j += 32) s += term(j);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    return s;
}

// Writes item i = t*C + c of the result: dW[c, t] for t < T-1, db[c] for t = T-1.
__device__ __forceinline__ void store_item(float* dw, float* db, int64_t C, int T, int64_t c,
                                           int t, double v) {
    if (t == T - 1) {
        if (db) db[c] = float(v);
    } else {
        dw[c * (T - 1) + t] = float(v);
    }
}

// Finalize kernels: one warp per (channel, tap) item, grid-stride over items.
constexpr int kFinalizeThreads = 256;

int64_t finalize_blocks(int64_t items, int sms) {
    int64_t fb = (items * 32 + kFinalizeThreads - 1) / kFinalizeThreads;
    const int64_t cap = int64_t(sms) * 8;
    if (fb > cap) fb = cap;
    return fb < 1 ? 1 : fb;
}

// part[(j*T + t)*C + c] summed over j (C: the output channels).
__global__ void __launch_bounds__(256) finalize_direct(const double* __restrict__ part,
                                                       float* __restrict__ dw,
                                                       float* __restrict__ db, int64_t C, int T,
                                                       int64_t chunks) {
    grid_dependency_wait();
    allow_dependents();
    const int64_t n = C * T;
    const int64_t warps = int64_t(gridDim.x) * (blockDim.x / 32);
    for (int64_t i = (int64_t(blockIdx.x) * blockDim.x + threadIdx.x) / 32; i < n; i += warps) {
        const int64_t c = i % C;
        const int t = int(i / C);
        const double s =
            warp_ordered_sum(chunks, [&](int64_t j) { return part[(j * T + t) * C + c]; });
        if ((threadIdx.x & 31) == 0) store_item(dw, db, C, T, c, t, s);
    }
}

// ------------------------------------------------------------ tiled kernel --

struct TArgs {
    double* part;
    int32_t* err;
    int C;
    int pt, pl;
    FastDiv tiles_c, tiles_x, tiles_y;
    int ntiles;
};

template <int KH_, int KW_, int S_, int D_, int THT_, int TWT_, int WX_, int WY_, int NS_,
          class TA_ = float, int MULT_ = 1>
struct WCfg {
    using TA = TA_;  // activation element type of x and dy
    static constexpr int ESZ = sizeof(TA);
    // channel multiplier: lane = output channel o of a 32-channel block, which
    // reads input channel o / MULT; the x box holds the XC = 32 / MULT input
    // channels of the block
    static constexpr int MULT = MULT_;
    static constexpr int XC = kLanes / MULT;
    static constexpr int KH = KH_, KW = KW_, S = S_, D = D_;
    static constexpr int THT = THT_, TWT = TWT_, WX = WX_, WY = WY_, NS = NS_;
    static constexpr int T = KH * KW + 1;
    static constexpr int NCW = WX * WY;  // consumer warps (one 32-channel pixel row each)
    static constexpr int NCT = NCW * 32;
    static constexpr int NT = NCT + 32;  // + producer warp
    static constexpr int TH = THT * WY, TW = TWT * WX;
    static constexpr int IH = (TH - 1) * S + (KH - 1) * D + 1;
    static constexpr int IW = (TW - 1) * S + (KW - 1) * D + 1;
    static constexpr int RH = (THT - 1) * S + (KH - 1) * D + 1;
    static constexpr int RW = (TWT - 1) * S + (KW - 1) * D + 1;
    static constexpr int XBYTES = IH * IW * XC * ESZ;
    static constexpr int GBYTES = TH * TW * kLanes * ESZ;
    static constexpr int XPITCH = (XBYTES + 127) / 128 * 128;  // dy box on a 128-byte boundary
    static constexpr int STAGE_TX = XBYTES + GBYTES;           // bytes the two loads bring
    static constexpr int STAGE_BYTES = (XPITCH + GBYTES + 127) / 128 * 128;
    static constexpr int RED_BYTES = NCW * T * kLanes * 8;
    static constexpr int AREA = NS * STAGE_BYTES > RED_BYTES ? NS * STAGE_BYTES : RED_BYTES;
    static constexpr size_t SMEM = size_t(AREA) + size_t(2 * NS) * 8 + 16;
    static_assert((XC * ESZ) % 16 == 0 && kLanes % MULT == 0, "16-byte rows in the x box");
    static_assert(IH <= 256 && IW <= 256 && TW <= 256 && TH <= 256, "TMA box limit");
    static_assert(SMEM <= 227 * 1024, "shared memory per CTA");
};

template <class K>
__host__ __device__ constexpr int tap_of(int r, int j) {  // tap reading window cell r for output j
    const int num = r - j * K::S;
    if (num < 0 || num % K::D != 0) return -1;
    return num / K::D;
}

struct WTile {
    int cb, n, oy0, ox0, iy0, ix0;
};

template <class K>
__device__ __forceinline__ WTile decode(int t, const TArgs& a) {
    WTile T;
    const int q = fast_div(t, a.tiles_c);
    T.cb = t - q * a.tiles_c.d;
    const int r = fast_div(q, a.tiles_x);
    const int tx = q - r * a.tiles_x.d;
    T.n = fast_div(r, a.tiles_y);
    const int ty = r - T.n * a.tiles_y.d;
    T.oy0 = ty * K::TH;
    T.ox0 = tx * K::TW;
    T.iy0 = T.oy0 * K::S - a.pt;
    T.ix0 = T.ox0 * K::S - a.pl;
    return T;
}

template <class K>
__global__ void __launch_bounds__(K::NT, 1)
    partial_tiled(const __grid_constant__ CUtensorMap xmap, const __grid_constant__ CUtensorMap gmap,
                  const TArgs a) {
    extern __shared__ __align__(128) unsigned char smem[];
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + K::AREA);
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
        if (lane == 0) {
            prefetch_tensor_map(&xmap);
            prefetch_tensor_map(&gmap);
            int k = 0;
            bool ok = true;
            for (int t = blockIdx.x; t < a.ntiles; t += G, ++k) {
                const int s = k % K::NS;
                if (k >= K::NS && !mbar_wait_or_abort(&empty[s], ((k / K::NS) - 1) & 1, abort_flag)) {
                    ok = false;
                    break;
                }
                const WTile T = decode<K>(t, a);
                unsigned char* st = smem + size_t(s) * K::STAGE_BYTES;
                mbar_arrive_expect_tx(&full[s], K::STAGE_TX);
                tma_load_4d(st, &xmap, &full[s], T.cb * K::XC, T.ix0, T.iy0, T.n);
                tma_load_4d(st + K::XPITCH, &gmap, &full[s], T.cb * kLanes, T.ox0, T.oy0, T.n);
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

    const int xi = warp % K::WX, yi = warp / K::WX;
    const int j0 = yi * K::THT, i0 = xi * K::TWT;
    double acc64[K::T];
#pragma unroll
    for (int t = 0; t < K::T; ++t) acc64[t] = 0.0;

    int k = 0;
    for (int t = blockIdx.x; t < a.ntiles; t += G, ++k) {
        const int s = k % K::NS;
        if (!mbar_wait_or_abort(&full[s], (k / K::NS) & 1, abort_flag)) {
            if (lane == 0) {
                *abort_flag = 1;
                atomicExch(a.err, DW_ERR_DEVICE_TIMEOUT);
            }
            break;
        }
        using TA = typename K::TA;
        const TA* xb = reinterpret_cast<const TA*>(smem + size_t(s) * K::STAGE_BYTES);
        const TA* gb = reinterpret_cast<const TA*>(smem + size_t(s) * K::STAGE_BYTES + K::XPITCH);
        float g[K::THT][K::TWT];
#pragma unroll
        for (int j = 0; j < K::THT; ++j)
#pragma unroll
            for (int i = 0; i < K::TWT; ++i)
                g[j][i] = ActIO<TA>::load1(gb + ((j0 + j) * K::TW + i0 + i) * kLanes + lane);
        float acc[K::KH][K::KW];
#pragma unroll
        for (int kh = 0; kh < K::KH; ++kh)
#pragma unroll
            for (int kw = 0; kw < K::KW; ++kw) acc[kh][kw] = 0.f;
        const TA* win = xb + ((j0 * K::S) * K::IW + i0 * K::S) * K::XC + lane / K::MULT;
        static_for<0, K::RH>([&](auto r_) {
            constexpr int r = decltype(r_)::value;
            static_for<0, K::RW>([&](auto q_) {
                constexpr int q = decltype(q_)::value;
                const float v = ActIO<TA>::load1(win + (r * K::IW + q) * K::XC);
                static_for<0, K::THT>([&](auto j_) {
                    constexpr int j = decltype(j_)::value;
                    constexpr int kh = tap_of<K>(r, j);
                    if constexpr (kh >= 0 && kh < K::KH) {
                        static_for<0, K::TWT>([&](auto i_) {
                            constexpr int i = decltype(i_)::value;
                            constexpr int kw = tap_of<K>(q, i);
                            if constexpr (kw >= 0 && kw < K::KW)
                                acc[kh][kw] = fmaf(g[j][i], v, acc[kh][kw]);
                        });
                    }
                });
            });
        });
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[s]);
        float gs = 0.f;
#pragma unroll
        for (int j = 0; j < K::THT; ++j)
#pragma unroll
            for (int i = 0; i < K::TWT; ++i) gs += g[j][i];
#pragma unroll
        for (int kh = 0; kh < K::KH; ++kh)
#pragma unroll
            for (int kw = 0; kw < K::KW; ++kw) acc64[kh * K::KW + kw] += double(acc[kh][kw]);
        acc64[K::T - 1] += double(gs);
    }

    // every consumer is past its last tile (no copy in flight any more): sum
    // the warps' float64 partials through shared memory, in warp order
    named_barrier_sync(1, K::NCT);
    double* red = reinterpret_cast<double*>(smem);
#pragma unroll
    for (int t = 0; t < K::T; ++t) red[(warp * K::T + t) * kLanes + lane] = acc64[t];
    named_barrier_sync(1, K::NCT);
    for (int t = warp; t < K::T; t += K::NCW) {
        double sum = 0.0;
        for (int w = 0; w < K::NCW; ++w) sum += red[(w * K::T + t) * kLanes + lane];
        a.part[(int64_t(blockIdx.x) * K::T + t) * kLanes + lane] = sum;
    }
}

// part[(b*T + t)*32 + lane], b = cb, cb + tiles_c, ... < G, summed in order.
__global__ void __launch_bounds__(256) finalize_tiled(const double* __restrict__ part,
                                                      float* __restrict__ dw,
                                                      float* __restrict__ db, int C, int T,
                                                      int tiles_c, int G) {
    grid_dependency_wait();
    allow_dependents();
    const int64_t n = int64_t(C) * T;
    const int64_t warps = int64_t(gridDim.x) * (blockDim.x / 32);
    for (int64_t i = (int64_t(blockIdx.x) * blockDim.x + threadIdx.x) / 32; i < n; i += warps) {
        const int c = int(i % C);
        const int t = int(i / C);
        const int cb = c / kLanes, lane = c % kLanes;
        // the CTAs of channel block cb are cb, cb + tiles_c, ... < G
        const int64_t count = (G - cb + tiles_c - 1) / tiles_c;
        const double s = warp_ordered_sum(count, [&](int64_t j) {
            return part[((cb + j * tiles_c) * T + t) * kLanes + lane];
        });
        if ((threadIdx.x & 31) == 0) store_item(dw, db, C, T, c, t, s);
    }
}

// ------------------------------------------------------------------- host --

int64_t direct_chunks(const Problem& p, int64_t& chunk) {
    const int64_t P = p.N * p.Ho * p.Wo;
    int64_t chunks = (P + kMinChunk - 1) / kMinChunk;
    if (chunks > kMaxChunks) chunks = kMaxChunks;
    if (chunks < 1) chunks = 1;
    chunk = (P + chunks - 1) / chunks;
    chunks = (P + chunk - 1) / chunk;
    return chunks;
}

size_t direct_workspace(const Problem& p) {
    int64_t chunk;
    const int64_t chunks = direct_chunks(p, chunk);
    return size_t(chunks) * size_t(p.kH * p.kW + 1) * size_t(p.Co) * sizeof(double);
}

size_t tiled_workspace(const Problem& p) {
    const int64_t tc = (p.Co + kLanes - 1) / kLanes;
    const int64_t g = tc >= kMaxTiledCtas ? tc : (kMaxTiledCtas / tc) * tc;
    return size_t(g) * size_t(p.kH * p.kW + 1) * kLanes * sizeof(double);
}

template <class TA>
cudaError_t launch_direct_partial(const Problem& p, const void* x, const void* dy, double* part,
                                  const DArgs& a, int64_t blocks, cudaStream_t stream) {
    const TA* xt = static_cast<const TA*>(x);
    const TA* gt = static_cast<const TA*>(dy);
    if (p.layout == DW_NCHW && p.kH == p.kW && (p.kH == 3 || p.kH == 5)) {
        // one warp per (chunk, output channel) with every tap in registers
        int64_t nb = (a.chunks * a.Co * 32 + 255) / 256;
        const int64_t cap = int64_t(sm_count(current_device())) * 8;
        if (nb > cap) nb = cap;
        if (nb < 1) nb = 1;
        if (p.kH == 3)
            return launch_pdl(partial_direct_nchw_taps<TA, 3, 3>, dim3(unsigned(nb)), dim3(256), 0,
                              stream, xt, gt, part, a);
        return launch_pdl(partial_direct_nchw_taps<TA, 5, 5>, dim3(unsigned(nb)), dim3(256), 0,
                          stream, xt, gt, part, a);
    }
    return p.layout == DW_NHWC ? launch_pdl(partial_direct_nhwc<TA>, dim3(unsigned(blocks)),
                                            dim3(256), 0, stream, xt, gt, part, a)
                               : launch_pdl(partial_direct_nchw<TA>, dim3(unsigned(blocks)),
                                            dim3(256), 0, stream, xt, gt, part, a);
}

dw_status_t launch_direct(const Problem& p, const void* x, const void* dy, float* dw, float* db,
                          void* ws, cudaStream_t stream) {
    DArgs a;
    a.N = p.N; a.C = p.C; a.H = p.H; a.W = p.W; a.Ho = p.Ho; a.Wo = p.Wo;
    a.M = p.M; a.Co = p.Co;
    a.kH = p.kH; a.kW = p.kW; a.sh = p.sh; a.sw = p.sw; a.dh = p.dh; a.dw = p.dw;
    a.pt = p.pt; a.pl = p.pl;
    a.T = p.kH * p.kW + 1;
    a.P = p.N * p.Ho * p.Wo;
    a.chunks = direct_chunks(p, a.chunk);
    a.items = a.chunks * a.T * p.Co;
    double* part = static_cast<double*>(ws);
    const int dev = current_device();
    const int64_t cap = int64_t(sm_count(dev)) * 8;
    const int64_t threads_needed = p.layout == DW_NHWC ? a.items : a.items * 32;
    int64_t blocks = (threads_needed + 255) / 256;
    if (blocks > cap) blocks = cap;
    if (blocks < 1) blocks = 1;
    cudaError_t e =
        p.atype == DW_F16    ? launch_direct_partial<__half>(p, x, dy, part, a, blocks, stream)
        : p.atype == DW_BF16 ? launch_direct_partial<__nv_bfloat16>(p, x, dy, part, a, blocks, stream)
                             : launch_direct_partial<float>(p, x, dy, part, a, blocks, stream);
    if (e != cudaSuccess) return DW_ERR_CUDA;
    const int64_t fb = finalize_blocks(p.Co * a.T, sm_count(dev));
    e = launch_pdl(finalize_direct, dim3(unsigned(fb)), dim3(kFinalizeThreads), 0, stream,
                   static_cast<const double*>(part), dw, db, int64_t(p.Co), a.T, a.chunks);
    if (e != cudaSuccess) return DW_ERR_CUDA;
    return cudaGetLastError() == cudaSuccess ? DW_OK : DW_ERR_CUDA;
}

template <class K>
dw_status_t launch_tiled(const Problem& p, const void* x, const void* dy, float* dw, float* db,
                         void* ws, cudaStream_t stream, int32_t* err, bool dry_run) {
    TArgs a;
    a.part = static_cast<double*>(ws);
    a.err = err;
    if (p.M != K::MULT) return DW_ERR_UNSUPPORTED;
    a.C = static_cast<int>(p.Co);  // output channels: the lanes
    a.pt = p.pt;
    a.pl = p.pl;
    const int64_t ty = (p.Ho + K::TH - 1) / K::TH;
    const int64_t tx = (p.Wo + K::TW - 1) / K::TW;
    const int64_t tc = (p.Co + kLanes - 1) / kLanes;
    const int64_t spatial = ty * tx * p.N;
    const int64_t nt = spatial * tc;
    if (nt >= INT_MAX) return DW_ERR_UNSUPPORTED;
    a.tiles_y = make_fastdiv(int(ty));
    a.tiles_x = make_fastdiv(int(tx));
    a.tiles_c = make_fastdiv(int(tc));
    a.ntiles = int(nt);
    if (dry_run) return DW_OK;

    static LaunchCache cache;
    const int dev = current_device();
    const int occ = prepare_kernel(reinterpret_cast<const void*>(&partial_tiled<K>), K::NT,
                                   K::SMEM, cache, dev);
    if (occ < 1) return DW_ERR_CUDA;
    // every CTA keeps one channel block: the grid is a multiple of tiles_c,
    // at most kMaxTiledCtas (the bound the workspace size assumes)
    int64_t reps = (int64_t(sm_count(dev)) * occ) / tc;
    const int64_t reps_cap = tc >= kMaxTiledCtas ? 1 : kMaxTiledCtas / tc;
    if (reps > reps_cap) reps = reps_cap;
    if (reps > spatial) reps = spatial;
    if (reps < 1) reps = 1;
    const int64_t G = reps * tc;

    const cuuint32_t estr[4] = {1, 1, 1, 1};
    CUtensorMap xmap, gmap;
    constexpr cuuint64_t E = K::ESZ;
    const cuuint64_t xd[4] = {cuuint64_t(p.C), cuuint64_t(p.W), cuuint64_t(p.H), cuuint64_t(p.N)};
    const cuuint64_t xs[3] = {cuuint64_t(p.C) * E, cuuint64_t(p.C * p.W) * E,
                              cuuint64_t(p.C * p.W * p.H) * E};
    const cuuint32_t xbox[4] = {K::XC, K::IW, K::IH, 1};
    const cuuint64_t gd[4] = {cuuint64_t(p.Co), cuuint64_t(p.Wo), cuuint64_t(p.Ho), cuuint64_t(p.N)};
    const cuuint64_t gs[3] = {cuuint64_t(p.Co) * E, cuuint64_t(p.Co * p.Wo) * E,
                              cuuint64_t(p.Co * p.Wo * p.Ho) * E};
    const cuuint32_t gbox[4] = {kLanes, K::TW, K::TH, 1};
    constexpr CUtensorMapDataType dt = ActIO<typename K::TA>::kTma;
    if (encode_tensor_map(&xmap, dt, 4, const_cast<void*>(x), xd, xs, xbox, estr) != CUDA_SUCCESS ||
        encode_tensor_map(&gmap, dt, 4, const_cast<void*>(dy), gd, gs, gbox, estr) != CUDA_SUCCESS)
        return DW_ERR_CUDA;
    if (launch_pdl(partial_tiled<K>, dim3(unsigned(G)), dim3(K::NT), K::SMEM, stream, xmap, gmap,
                   a) != cudaSuccess)
        return DW_ERR_CUDA;
    const int64_t fb = finalize_blocks(p.Co * K::T, sm_count(dev));
    if (launch_pdl(finalize_tiled, dim3(unsigned(fb)), dim3(kFinalizeThreads), 0, stream,
                   static_cast<const double*>(a.part), dw, db, int(p.Co), K::T, int(tc),
                   int(G)) != cudaSuccess)
        return DW_ERR_CUDA;
    return cudaGetLastError() == cudaSuccess ? DW_OK : DW_ERR_CUDA;
}

// ------------------------------------------------- tiled kernel, NCHW ------

struct NArgs {
    double* part;
    int32_t* err;
    int C, pt, pl;         // C: output channels (planes of dy); x plane of o is o / M
    int M;
    int sh4;               // extra x-box shift beyond REM (0, or 4 for 16-bit elements)
    int tiles_x, tiles_y;  // tiles per plane
    int bands, band_rows;  // row bands per plane, tile rows per band
    int units;             // N * C * bands
};

template <int KH_, int KW_, int REM_, int THT_, int WY_, int NS_, int S_ = 1, class TA_ = float>
struct NWCfg {
    using TA = TA_;  // activation element type of x and dy
    static constexpr int ESZ = sizeof(TA);
    // x boxes start on 16-byte boundaries: REM = the start shift mod 4 (compile
    // time), plus 0 or 4 more elements at run time for 16-bit elements
    static constexpr int ALIGN = 16 / ESZ;
    static constexpr int KH = KH_, KW = KW_, REM = REM_, THT = THT_, WY = WY_, NS = NS_;
    // stride S (1 or 2): a lane owns OPL = 4 / S consecutive outputs, whose
    // input window starts 4 columns after its neighbour's in both cases
    static constexpr int S = S_, OPL = 4 / S_;
    static constexpr int T = KH * KW + 1;
    static constexpr int NCW = WY;  // consumer warps, one row strip of 32 * OPL outputs each
    static constexpr int NCT = NCW * 32;
    static constexpr int NT = NCT + 32;
    static constexpr int TW = 32 * OPL, TH = THT * WY;
    static constexpr int IH = (TH - 1) * S + KH;
    static constexpr int IWB = (REM + (ALIGN - 4) + (TW - 1) * S + KW + ALIGN - 1) / ALIGN * ALIGN;
    static constexpr int NV = (REM + (OPL - 1) * S + KW - 1) / 4 + 1;  // float4 per window row
    static_assert(S == 1 || S == 2, "stride 1 or 2");
    static constexpr int XBYTES = IWB * IH * ESZ;
    static constexpr int XPITCH = (XBYTES + 127) / 128 * 128;
    static constexpr int GBYTES = TW * TH * ESZ;
    static constexpr int STAGE_BYTES = XPITCH + GBYTES;
    static constexpr int RED_BYTES = NCW * T * 8;
    static constexpr size_t SMEM = size_t(NS) * STAGE_BYTES + RED_BYTES + size_t(2 * NS) * 8 + 16;
    static_assert(GBYTES % 128 == 0 && (IWB * ESZ) % 16 == 0, "TMA shared-memory alignment");
    static_assert(IWB <= 256 && IH <= 256, "TMA box limit");
    static_assert(SMEM <= 227 * 1024, "shared memory per CTA");
};

template <class K>
__global__ void __launch_bounds__(K::NT, 1)
    partial_tiled_nchw(const __grid_constant__ CUtensorMap xmap,
                       const __grid_constant__ CUtensorMap gmap, const NArgs a) {
    extern __shared__ __align__(128) unsigned char smem[];
    double* red = reinterpret_cast<double*>(smem + size_t(K::NS) * K::STAGE_BYTES);
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + size_t(K::NS) * K::STAGE_BYTES + K::RED_BYTES);
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

    // unit u = (n*C + c) * bands + band; its tiles: rows of the band x all columns
    auto unit_tiles = [&](int u, int& plane, int& ty0, int& rows) {
        plane = u / a.bands;
        const int band = u - plane * a.bands;
        ty0 = band * a.band_rows;
        rows = a.tiles_y - ty0 < a.band_rows ? a.tiles_y - ty0 : a.band_rows;
    };

    if (warp == K::NCW) {
        if (lane == 0) {
            prefetch_tensor_map(&xmap);
            prefetch_tensor_map(&gmap);
            int k = 0;
            bool ok = true;
            for (int u = blockIdx.x; u < a.units && ok; u += G) {
                int plane, ty0, rows;
                unit_tiles(u, plane, ty0, rows);
                const int c = plane % a.C, n = plane / a.C;  // c: output channel
                for (int r = 0; r < rows && ok; ++r)
                    for (int tx = 0; tx < a.tiles_x; ++tx, ++k) {
                        const int s = k % K::NS;
                        if (k >= K::NS &&
                            !mbar_wait_or_abort(&empty[s], ((k / K::NS) - 1) & 1, abort_flag)) {
                            ok = false;
                            break;
                        }
                        const int ty = ty0 + r;
                        unsigned char* st = smem + size_t(s) * K::STAGE_BYTES;
                        mbar_arrive_expect_tx(&full[s], K::XBYTES + K::GBYTES);
                        tma_load_4d(st, &xmap, &full[s],
                                    tx * K::TW * K::S - a.pl - K::REM - a.sh4,
                                    ty * K::TH * K::S - a.pt, c / a.M, n);
                        tma_load_4d(st + K::XPITCH, &gmap, &full[s], tx * K::TW, ty * K::TH, c, n);
                    }
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

    const int row0 = warp * K::THT;
    int k = 0;
    bool failed = false;
    for (int u = blockIdx.x; u < a.units; u += G) {
        int plane, ty0, rows;
        unit_tiles(u, plane, ty0, rows);
        double acc64[K::T];
#pragma unroll
        for (int t = 0; t < K::T; ++t) acc64[t] = 0.0;
        const int ntile = rows * a.tiles_x;
        for (int i = 0; i < ntile && !failed; ++i, ++k) {
            const int s = k % K::NS;
            if (!mbar_wait_or_abort(&full[s], (k / K::NS) & 1, abort_flag)) {
                if (lane == 0) {
                    *abort_flag = 1;
                    atomicExch(a.err, DW_ERR_DEVICE_TIMEOUT);
                }
                failed = true;
                break;
            }
            using TA = typename K::TA;
            using IO = ActIO<TA>;
            const unsigned char* st = smem + size_t(s) * K::STAGE_BYTES;
            // lane window: 4-element vectors from column 4*lane (+ the run-time shift)
            const TA* xw = reinterpret_cast<const TA*>(st) + row0 * K::S * K::IWB + 4 * lane + a.sh4;
            const TA* gw = reinterpret_cast<const TA*>(st + K::XPITCH) + row0 * K::TW +
                           lane * K::OPL;
            float g[K::THT][K::OPL];
#pragma unroll
            for (int j = 0; j < K::THT; ++j) {
                if constexpr (K::OPL == 4) {
                    const float4 f = IO::load4(gw + j * K::TW);
                    g[j][0] = f.x; g[j][1] = f.y; g[j][2] = f.z; g[j][3] = f.w;
                } else {
                    const float2 f = IO::load2(gw + j * K::TW);
                    g[j][0] = f.x; g[j][1] = f.y;
                }
            }
            float acc[K::KH][K::KW];
#pragma unroll
            for (int kh = 0; kh < K::KH; ++kh)
#pragma unroll
                for (int kw = 0; kw < K::KW; ++kw) acc[kh][kw] = 0.f;
            static_for<0, (K::THT - 1) * K::S + K::KH>([&](auto r_) {
                constexpr int r = decltype(r_)::value;
                float v[4 * K::NV];
#pragma unroll
                for (int q = 0; q < K::NV; ++q) {
                    const float4 f = IO::load4(xw + r * K::IWB + 4 * q);
                    v[4 * q] = f.x; v[4 * q + 1] = f.y; v[4 * q + 2] = f.z; v[4 * q + 3] = f.w;
                }
                static_for<0, K::THT>([&](auto j_) {
                    constexpr int j = decltype(j_)::value;
                    constexpr int kh = r - j * K::S;
                    if constexpr (kh >= 0 && kh < K::KH) {
#pragma unroll
                        for (int ii = 0; ii < K::OPL; ++ii)
#pragma unroll
                            for (int kw = 0; kw < K::KW; ++kw)
                                acc[kh][kw] = fmaf(g[j][ii], v[K::REM + ii * K::S + kw], acc[kh][kw]);
                    }
                });
            });
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[s]);
            float gs = 0.f;
#pragma unroll
            for (int j = 0; j < K::THT; ++j) {
                if constexpr (K::OPL == 4) gs += (g[j][0] + g[j][1]) + (g[j][2] + g[j][3]);
                else gs += g[j][0] + g[j][1];
            }
#pragma unroll
            for (int kh = 0; kh < K::KH; ++kh)
#pragma unroll
                for (int kw = 0; kw < K::KW; ++kw) acc64[kh * K::KW + kw] += double(acc[kh][kw]);
            acc64[K::T - 1] += double(gs);
        }
        // the unit's partial: warp sums, then the warps in order
#pragma unroll
        for (int t = 0; t < K::T; ++t) {
            double v = acc64[t];
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
            if (lane == 0) red[warp * K::T + t] = v;
        }
        named_barrier_sync(1, K::NCT);
        if (tid < K::T) {
            double sum = 0.0;
            for (int w = 0; w < K::NCW; ++w) sum += red[w * K::T + tid];
            a.part[int64_t(u) * K::T + tid] = sum;
        }
        named_barrier_sync(1, K::NCT);
        if (failed) break;
    }
}

// part[u*T + t], u = (n*C + c)*bands + band, summed over n and band in order.
__global__ void __launch_bounds__(256) finalize_tiled_nchw(const double* __restrict__ part,
                                                           float* __restrict__ dw,
                                                           float* __restrict__ db, int N, int C,
                                                           int T, int bands) {
    grid_dependency_wait();
    allow_dependents();
    const int64_t n_items = int64_t(C) * T;
    const int64_t warps = int64_t(gridDim.x) * (blockDim.x / 32);
    for (int64_t i = (int64_t(blockIdx.x) * blockDim.x + threadIdx.x) / 32; i < n_items;
         i += warps) {
        const int c = int(i % C);
        const int t = int(i / C);
        // term j = (n, band) = (j / bands, j % bands)
        const double s = warp_ordered_sum(int64_t(N) * bands, [&](int64_t j) {
            const int64_t n = j / bands, b = j - n * bands;
            return part[((n * C + c) * bands + b) * T + t];
        });
        if ((threadIdx.x & 31) == 0) store_item(dw, db, C, T, c, t, s);
    }
}

// ------------------------------------- tiled kernel, NCHW, 1 x kW filters --
// With kH = 1 every row is an independent 1-D correlation.  A unit is (block
// of n, group of 8 channels): consumer warp w owns channel cg*8 + w and walks,
// for every n of the block, every output row and every 128-column strip; one
// pipeline stage holds that row of the 8 channels' planes (a 4-D TMA box of
// one row by 8 channels, zero-filled past C).  Lanes run along W with 4
// outputs each, the kW taps at compile-time offsets of a register window.
// A lane accumulates float32 sums over kRowsFold strips (16 products per
// tap), then a warp reduce-scatter (fixed butterfly order) leaves tap t's sum
// on lane t, which adds it to its float64 total; each warp's totals over its
// unit become one partial per (n block, tap, channel), laid out as the
// direct partials are, so the same fixed-order finalize sums the n blocks.

constexpr int kRowsFold = 4;  // strips per float32 partial sum

// Warp reduce-scatter of NP (a power of two, <= 32) per-lane values: on
// return lane l holds the sum over all 32 lanes of value l % NP.  The lane
// bits above NP are summed first (every lane keeps all NP values), then each
// round halves the values a lane keeps, the lane's bit choosing the half.
template <int NP>
__device__ __forceinline__ float warp_reduce_scatter(float (&v)[NP], int lane) {
    static_assert(NP >= 1 && NP <= 32 && (NP & (NP - 1)) == 0, "power of two up to 32");
#pragma unroll
    for (int o = 16; o >= NP; o >>= 1)
#pragma unroll
        for (int i = 0; i < NP; ++i) v[i] += __shfl_xor_sync(0xffffffffu, v[i], o);
#pragma unroll
    for (int h = NP / 2; h >= 1; h >>= 1) {
        const bool up = (lane & h) != 0;
#pragma unroll
        for (int i = 0; i < h; ++i) {
            const float send = up ? v[i] : v[i + h];
            const float keep = up ? v[i + h] : v[i];
            v[i] = keep + __shfl_xor_sync(0xffffffffu, send, h);
        }
    }
    return v[0];
}

struct RArgs {
    double* part;
    int32_t* err;
    int N, C, Ho, pt, pl;
    int sh4;       // extra x-box shift beyond REM (0, or 4 for 16-bit elements)
    int tiles_x;   // 128-column strips per row
    int cgroups;   // groups of 8 channels
    int nper;      // n per block
    int units;     // n blocks * cgroups
};

template <int KW_, int REM_, int NS_, class TA_ = float>
struct RCfg {
    using TA = TA_;  // activation element type of x and dy
    static constexpr int ESZ = sizeof(TA);
    static constexpr int ALIGN = 16 / ESZ;  // x boxes start on 16-byte columns
    static constexpr int KW = KW_, REM = REM_, NS = NS_;
    static constexpr int T = KW + 1;
    static constexpr int NP = T <= 4 ? 4 : T <= 8 ? 8 : T <= 16 ? 16 : 32;  // T rounded up to 2^k
    static_assert(T <= 32, "taps + bias fit one warp");
    static constexpr int NCW = 8;  // consumer warps = channels per unit
    static constexpr int NT = NCW * 32 + 32;
    static constexpr int TW = 128;
    static constexpr int IWB = (REM + (ALIGN - 4) + TW + KW - 1 + ALIGN - 1) / ALIGN * ALIGN;
    static constexpr int NV = (REM + 3 + KW - 1) / 4 + 1;  // 4-vectors per window
    static constexpr int XBYTES = IWB * NCW * ESZ;
    static constexpr int XPITCH = (XBYTES + 127) / 128 * 128;
    static constexpr int GBYTES = TW * NCW * ESZ;
    static constexpr int STAGE_BYTES = XPITCH + GBYTES;
    static constexpr size_t SMEM = size_t(NS) * STAGE_BYTES + size_t(2 * NS) * 8 + 16;
    static_assert(GBYTES % 128 == 0, "TMA shared-memory alignment");
    static_assert(IWB <= 256, "TMA box limit");
    static_assert(SMEM <= 227 * 1024, "shared memory per CTA");
};

template <class K>
__global__ void __launch_bounds__(K::NT, 1)
    partial_rows_nchw(const __grid_constant__ CUtensorMap xmap,
                      const __grid_constant__ CUtensorMap gmap, const RArgs a) {
    extern __shared__ __align__(128) unsigned char smem[];
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + size_t(K::NS) * K::STAGE_BYTES);
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
        if (lane == 0) {
            prefetch_tensor_map(&xmap);
            prefetch_tensor_map(&gmap);
            int k = 0;
            bool ok = true;
            for (int u = blockIdx.x; u < a.units && ok; u += G) {
                const int nb = u / a.cgroups, cg = u - nb * a.cgroups;
                const int n0 = nb * a.nper;
                const int n1 = a.N - n0 < a.nper ? a.N : n0 + a.nper;
                for (int n = n0; n < n1 && ok; ++n)
                    for (int h = 0; h < a.Ho && ok; ++h)
                        for (int tx = 0; tx < a.tiles_x; ++tx, ++k) {
                            const int s = k % K::NS;
                            if (k >= K::NS &&
                                !mbar_wait_or_abort(&empty[s], ((k / K::NS) - 1) & 1, abort_flag)) {
                                ok = false;
                                break;
                            }
                            unsigned char* st = smem + size_t(s) * K::STAGE_BYTES;
                            mbar_arrive_expect_tx(&full[s], K::XBYTES + K::GBYTES);
                            tma_load_4d(st, &xmap, &full[s], tx * K::TW - a.pl - K::REM - a.sh4,
                                        h - a.pt, cg * K::NCW, n);
                            tma_load_4d(st + K::XPITCH, &gmap, &full[s], tx * K::TW, h,
                                        cg * K::NCW, n);
                        }
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

    int k = 0;
    bool failed = false;
    for (int u = blockIdx.x; u < a.units && !failed; u += G) {
        const int nb = u / a.cgroups, cg = u - nb * a.cgroups;
        const int n0 = nb * a.nper;
        const int n1 = a.N - n0 < a.nper ? a.N : n0 + a.nper;
        const int c = cg * K::NCW + warp;
        float acc[K::NP];  // float32 sums since the last fold (taps, then the bias)
#pragma unroll
        for (int t = 0; t < K::NP; ++t) acc[t] = 0.f;
        double total = 0.0;  // lane t: the unit's sum of tap t
        const int ntile = (n1 - n0) * a.Ho * a.tiles_x;
        for (int i = 0; i < ntile; ++i, ++k) {
            const int s = k % K::NS;
            // warp-uniform outcome: the fold below shuffles across the warp
            const bool got = mbar_wait_or_abort(&full[s], (k / K::NS) & 1, abort_flag);
            if (!__all_sync(0xffffffffu, got)) {
                if (lane == 0) {
                    *abort_flag = 1;
                    atomicExch(a.err, DW_ERR_DEVICE_TIMEOUT);
                }
                failed = true;
                break;
            }
            using IO = ActIO<typename K::TA>;
            const unsigned char* st = smem + size_t(s) * K::STAGE_BYTES;
            const typename K::TA* xw =
                reinterpret_cast<const typename K::TA*>(st) + warp * K::IWB + 4 * lane + a.sh4;
            const float4 gf = IO::load4(reinterpret_cast<const typename K::TA*>(st + K::XPITCH) +
                                        warp * K::TW + 4 * lane);
            const float g[4] = {gf.x, gf.y, gf.z, gf.w};
            float v[4 * K::NV];
#pragma unroll
            for (int q = 0; q < K::NV; ++q) {
                const float4 f = IO::load4(xw + 4 * q);
                v[4 * q] = f.x; v[4 * q + 1] = f.y; v[4 * q + 2] = f.z; v[4 * q + 3] = f.w;
            }
#pragma unroll
            for (int kw = 0; kw < K::KW; ++kw) {
                float t0 = fmaf(g[0], v[K::REM + kw], acc[kw]);
                t0 = fmaf(g[1], v[K::REM + 1 + kw], t0);
                t0 = fmaf(g[2], v[K::REM + 2 + kw], t0);
                acc[kw] = fmaf(g[3], v[K::REM + 3 + kw], t0);
            }
            acc[K::T - 1] += (g[0] + g[1]) + (g[2] + g[3]);
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[s]);
            if ((i + 1) % kRowsFold == 0 || i + 1 == ntile) {
                total += double(warp_reduce_scatter<K::NP>(acc, lane));
#pragma unroll
                for (int t = 0; t < K::NP; ++t) acc[t] = 0.f;
            }
        }
        if (failed) break;
        // lane t (t < T) holds the unit's total of tap t
        if (lane < K::T && c < a.C) a.part[(int64_t(nb) * K::T + lane) * a.C + c] = total;
    }
}

// n blocks of the rows kernel: enough units to cover the SMs twice over (a
// fixed count, so the workspace depends on the problem alone).
constexpr int kRowsUnits = 296;

int rows_nblocks(const Problem& p, int& nper) {
    const int64_t cgroups = (p.C + 7) / 8;
    int64_t nb = (kRowsUnits + cgroups - 1) / cgroups;
    if (nb > p.N) nb = p.N;
    if (nb < 1) nb = 1;
    nper = int((p.N + nb - 1) / nb);
    return int((p.N + nper - 1) / nper);
}

size_t rows_nchw_workspace(const Problem& p) {
    if (p.layout != DW_NCHW || p.kH != 1 || p.M != 1) return 0;
    int nper;
    const int nb = rows_nblocks(p, nper);
    return size_t(nb) * size_t(p.kW + 1) * size_t(p.C) * sizeof(double);
}

template <class K>
dw_status_t launch_rows_nchw(const Problem& p, const void* x, const void* dy, float* dw,
                             float* db, void* ws, cudaStream_t stream, int32_t* err,
                             bool dry_run) {
    RArgs a;
    a.part = static_cast<double*>(ws);
    a.err = err;
    a.N = int(p.N);
    a.C = int(p.C);
    a.Ho = int(p.Ho);
    a.pt = p.pt;
    a.pl = p.pl;
    a.sh4 = ((-p.pl) % K::ALIGN + K::ALIGN) % K::ALIGN - K::REM;  // 0 or 4
    const int64_t tx = (p.Wo + K::TW - 1) / K::TW;
    const int64_t cgroups = (p.C + K::NCW - 1) / K::NCW;
    int nper;
    const int nb = rows_nblocks(p, nper);
    const int64_t units = int64_t(nb) * cgroups;
    if (units >= INT_MAX || tx >= INT_MAX || int64_t(nper) * p.Ho * tx >= INT_MAX)
        return DW_ERR_UNSUPPORTED;
    a.tiles_x = int(tx);
    a.cgroups = int(cgroups);
    a.nper = nper;
    a.units = int(units);
    if (dry_run) return DW_OK;

    static LaunchCache cache;
    const int dev = current_device();
    const int occ = prepare_kernel(reinterpret_cast<const void*>(&partial_rows_nchw<K>), K::NT,
                                   K::SMEM, cache, dev);
    if (occ < 1) return DW_ERR_CUDA;
    int64_t G = int64_t(sm_count(dev)) * occ;
    if (G > units) G = units;
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    CUtensorMap xmap, gmap;
    constexpr cuuint64_t E = K::ESZ;
    const cuuint64_t xd[4] = {cuuint64_t(p.W), cuuint64_t(p.H), cuuint64_t(p.C), cuuint64_t(p.N)};
    const cuuint64_t xs[3] = {cuuint64_t(p.W) * E, cuuint64_t(p.W * p.H) * E,
                              cuuint64_t(p.W * p.H * p.C) * E};
    const cuuint32_t xbox[4] = {K::IWB, 1, K::NCW, 1};
    const cuuint64_t gd[4] = {cuuint64_t(p.Wo), cuuint64_t(p.Ho), cuuint64_t(p.C), cuuint64_t(p.N)};
    const cuuint64_t gs[3] = {cuuint64_t(p.Wo) * E, cuuint64_t(p.Wo * p.Ho) * E,
                              cuuint64_t(p.Wo * p.Ho * p.C) * E};
    const cuuint32_t gbox[4] = {K::TW, 1, K::NCW, 1};
    constexpr CUtensorMapDataType dt = ActIO<typename K::TA>::kTma;
    if (encode_tensor_map(&xmap, dt, 4, const_cast<void*>(x), xd, xs, xbox, estr) != CUDA_SUCCESS ||
        encode_tensor_map(&gmap, dt, 4, const_cast<void*>(dy), gd, gs, gbox, estr) != CUDA_SUCCESS)
        return DW_ERR_CUDA;
    if (launch_pdl(partial_rows_nchw<K>, dim3(unsigned(G)), dim3(K::NT), K::SMEM, stream, xmap,
                   gmap, a) != cudaSuccess)
        return DW_ERR_CUDA;
    const int64_t fb = finalize_blocks(p.C * K::T, sm_count(dev));
    if (launch_pdl(finalize_direct, dim3(unsigned(fb)), dim3(kFinalizeThreads), 0, stream,
                   static_cast<const double*>(a.part), dw, db, int64_t(p.C), K::T,
                   int64_t(nb)) != cudaSuccess)
        return DW_ERR_CUDA;
    return cudaGetLastError() == cudaSuccess ? DW_OK : DW_ERR_CUDA;
}

template <int KW, int NS, class TA>
dw_status_t launch_rows_rem(const Problem& p, const void* x, const void* dy, float* dw,
                            float* db, void* ws, cudaStream_t stream, int32_t* err, bool dry_run) {
#define DW_R(R) return launch_rows_nchw<RCfg<KW, R, NS, TA>>(p, x, dy, dw, db, ws, stream, err, dry_run);
    switch (((-p.pl) % 4 + 4) % 4) {
        case 0: DW_R(0)
        case 1: DW_R(1)
        case 2: DW_R(2)
        default: DW_R(3)
    }
#undef DW_R
}

template <class TA>
dw_status_t rows_pick(const Problem& p, const void* x, const void* dy, float* dw, float* db,
                      void* ws, cudaStream_t stream, int32_t* err, bool dry_run) {
    if (p.kW == 3) return launch_rows_rem<3, 8, TA>(p, x, dy, dw, db, ws, stream, err, dry_run);
    if (p.kW == 5) return launch_rows_rem<5, 8, TA>(p, x, dy, dw, db, ws, stream, err, dry_run);
    if (p.kW == 7) return launch_rows_rem<7, 8, TA>(p, x, dy, dw, db, ws, stream, err, dry_run);
    if (p.kW == 15) return launch_rows_rem<15, 8, TA>(p, x, dy, dw, db, ws, stream, err, dry_run);
    if (p.kW == 31) return launch_rows_rem<31, 8, TA>(p, x, dy, dw, db, ws, stream, err, dry_run);
    return DW_ERR_UNSUPPORTED;
}

constexpr int kNchwUnitsCap = 2048;  // bands are added until N*C*bands reaches this

int nchw_bands_cap(const Problem& p) {
    const int64_t planes = p.N * p.Co;
    int64_t r = (kNchwUnitsCap + planes - 1) / planes;
    return int(r < 1 ? 1 : r);
}

size_t tiled_nchw_workspace(const Problem& p) {
    if (p.layout != DW_NCHW) return 0;
    return size_t(p.N) * size_t(p.Co) * size_t(nchw_bands_cap(p)) * size_t(p.kH * p.kW + 1) *
           sizeof(double);
}

template <class K>
dw_status_t launch_tiled_nchw(const Problem& p, const void* x, const void* dy, float* dw,
                              float* db, void* ws, cudaStream_t stream, int32_t* err,
                              bool dry_run) {
    NArgs a;
    a.part = static_cast<double*>(ws);
    a.err = err;
    a.C = int(p.Co);
    a.M = int(p.M);
    a.pt = p.pt;
    a.pl = p.pl;
    a.sh4 = ((-p.pl) % K::ALIGN + K::ALIGN) % K::ALIGN - K::REM;  // 0 or 4
    const int64_t ty = (p.Ho + K::TH - 1) / K::TH, tx = (p.Wo + K::TW - 1) / K::TW;
    if (ty >= INT_MAX || tx >= INT_MAX) return DW_ERR_UNSUPPORTED;
    a.tiles_x = int(tx);
    a.tiles_y = int(ty);
    const int64_t planes = p.N * p.Co;
    // enough units to spread over every SM, never more bands than tile rows
    int64_t bands = (2 * 148 + planes - 1) / planes;
    if (bands > nchw_bands_cap(p)) bands = nchw_bands_cap(p);
    if (bands > ty) bands = ty;
    if (bands < 1) bands = 1;
    a.band_rows = int((ty + bands - 1) / bands);
    a.bands = int((ty + a.band_rows - 1) / a.band_rows);
    const int64_t units = planes * a.bands;
    if (units >= INT_MAX) return DW_ERR_UNSUPPORTED;
    a.units = int(units);
    if (dry_run) return DW_OK;

    static LaunchCache cache;
    const int dev = current_device();
    const int occ = prepare_kernel(reinterpret_cast<const void*>(&partial_tiled_nchw<K>), K::NT,
                                   K::SMEM, cache, dev);
    if (occ < 1) return DW_ERR_CUDA;
    int64_t G = int64_t(sm_count(dev)) * occ;
    if (G > units) G = units;
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    CUtensorMap xmap, gmap;
    constexpr cuuint64_t E = K::ESZ;
    const cuuint64_t xd[4] = {cuuint64_t(p.W), cuuint64_t(p.H), cuuint64_t(p.C), cuuint64_t(p.N)};
    const cuuint64_t xs[3] = {cuuint64_t(p.W) * E, cuuint64_t(p.W * p.H) * E,
                              cuuint64_t(p.W * p.H * p.C) * E};
    const cuuint32_t xbox[4] = {K::IWB, K::IH, 1, 1};
    const cuuint64_t gd[4] = {cuuint64_t(p.Wo), cuuint64_t(p.Ho), cuuint64_t(p.Co), cuuint64_t(p.N)};
    const cuuint64_t gs[3] = {cuuint64_t(p.Wo) * E, cuuint64_t(p.Wo * p.Ho) * E,
                              cuuint64_t(p.Wo * p.Ho * p.Co) * E};
    const cuuint32_t gbox[4] = {K::TW, K::TH, 1, 1};
    constexpr CUtensorMapDataType dt = ActIO<typename K::TA>::kTma;
    if (encode_tensor_map(&xmap, dt, 4, const_cast<void*>(x), xd, xs, xbox, estr) != CUDA_SUCCESS ||
        encode_tensor_map(&gmap, dt, 4, const_cast<void*>(dy), gd, gs, gbox, estr) != CUDA_SUCCESS)
        return DW_ERR_CUDA;
    if (launch_pdl(partial_tiled_nchw<K>, dim3(unsigned(G)), dim3(K::NT), K::SMEM, stream, xmap,
                   gmap, a) != cudaSuccess)
        return DW_ERR_CUDA;
    const int64_t fb = finalize_blocks(p.Co * K::T, sm_count(dev));
    if (launch_pdl(finalize_tiled_nchw, dim3(unsigned(fb)), dim3(kFinalizeThreads), 0, stream,
                   static_cast<const double*>(a.part), dw, db, int(p.N), int(p.Co), K::T,
                   a.bands) != cudaSuccess)
        return DW_ERR_CUDA;
    return cudaGetLastError() == cudaSuccess ? DW_OK : DW_ERR_CUDA;
}

template <int KH, int KW, int THT, int WY, int NS, int S, class TA>
dw_status_t launch_nchw_rem(const Problem& p, const void* x, const void* dy, float* dw,
                            float* db, void* ws, cudaStream_t stream, int32_t* err, bool dry_run) {
#define DW_N(R) return launch_tiled_nchw<NWCfg<KH, KW, R, THT, WY, NS, S, TA>>(p, x, dy, dw, db, ws, stream, err, dry_run);
    switch (((-p.pl) % 4 + 4) % 4) {
        case 0: DW_N(0)
        case 1: DW_N(1)
        case 2: DW_N(2)
        default: DW_N(3)
    }
#undef DW_N
}

template <class TA>
dw_status_t tiled_pick_nchw_2d(const Problem& p, const void* x, const void* dy, float* dw,
                               float* db, void* ws, cudaStream_t stream, int32_t* err,
                               bool dry_run) {
    if (p.sh == 2) {
        //                                                          KH KW THT WY NS S
        if (p.kH == 3 && p.kW == 3) return launch_nchw_rem<3, 3, 4, 8, 3, 2, TA>(p, x, dy, dw, db, ws, stream, err, dry_run);
        return DW_ERR_UNSUPPORTED;
    }
    //                                                          KH KW THT WY NS S
    if (p.kH == 3 && p.kW == 3) return launch_nchw_rem<3, 3, 4, 8, 3, 1, TA>(p, x, dy, dw, db, ws, stream, err, dry_run);
    if (p.kH == 5 && p.kW == 5) return launch_nchw_rem<5, 5, 4, 8, 3, 1, TA>(p, x, dy, dw, db, ws, stream, err, dry_run);
    if (p.kH == 7 && p.kW == 7) return launch_nchw_rem<7, 7, 2, 8, 3, 1, TA>(p, x, dy, dw, db, ws, stream, err, dry_run);
    return DW_ERR_UNSUPPORTED;
}

dw_status_t tiled_pick_nchw(const Problem& p, const void* x, const void* dy, float* dw,
                            float* db, void* ws, cudaStream_t stream, int32_t* err,
                            bool dry_run) {
    if (p.layout != DW_NCHW) return DW_ERR_UNSUPPORTED;
    if (p.dh != 1 || p.dw != 1 || p.sh != p.sw || p.sh > 2) return DW_ERR_UNSUPPORTED;
    const int esz = act_bytes(p.atype);
    if ((p.W * esz) % 16 != 0 || (p.Wo * esz) % 16 != 0) return DW_ERR_UNSUPPORTED;  // TMA row pitches
    if ((reinterpret_cast<uintptr_t>(x) | reinterpret_cast<uintptr_t>(dy)) & 15)
        return DW_ERR_UNSUPPORTED;
    if (p.N >= INT_MAX || p.C >= INT_MAX || p.H >= INT_MAX || p.W >= INT_MAX) return DW_ERR_UNSUPPORTED;
    if (p.kH == 1) {
        // rows of 1 x kW filters
        if (p.sh != 1) return DW_ERR_UNSUPPORTED;
        if (p.atype == DW_F16) return rows_pick<__half>(p, x, dy, dw, db, ws, stream, err, dry_run);
        if (p.atype == DW_BF16)
            return rows_pick<__nv_bfloat16>(p, x, dy, dw, db, ws, stream, err, dry_run);
        return rows_pick<float>(p, x, dy, dw, db, ws, stream, err, dry_run);
    }
    if (p.atype == DW_F16) return tiled_pick_nchw_2d<__half>(p, x, dy, dw, db, ws, stream, err, dry_run);
    if (p.atype == DW_BF16)
        return tiled_pick_nchw_2d<__nv_bfloat16>(p, x, dy, dw, db, ws, stream, err, dry_run);
    return tiled_pick_nchw_2d<float>(p, x, dy, dw, db, ws, stream, err, dry_run);
}

//                         KH KW  S  D THT TWT WX WY NS
template <class TA> using W33s1 = WCfg<3, 3, 1, 1, 2, 4, 4, 2, 4, TA>;
template <int M, class TA> using W33s1m = WCfg<3, 3, 1, 1, 2, 4, 4, 2, 4, TA, M>;
template <int M, class TA> using W33s2m = WCfg<3, 3, 2, 1, 2, 4, 4, 2, 4, TA, M>;
template <int M, class TA> using W55s1m = WCfg<5, 5, 1, 1, 2, 4, 4, 2, 3, TA, M>;
template <class TA> using W33s2 = WCfg<3, 3, 2, 1, 2, 4, 4, 2, 4, TA>;
template <class TA> using W55s1 = WCfg<5, 5, 1, 1, 2, 4, 4, 2, 3, TA>;
template <class TA> using W77s1 = WCfg<7, 7, 1, 1, 1, 4, 4, 2, 3, TA>;
template <class TA> using W1x15 = WCfg<1, 15, 1, 1, 1, 8, 8, 1, 4, TA>;
template <class TA> using W1x31 = WCfg<1, 31, 1, 1, 1, 8, 8, 1, 4, TA>;

template <class TA>
dw_status_t tiled_pick_nhwc(const Problem& p, const void* x, const void* dy, float* dw, float* db,
                            void* ws, cudaStream_t stream, int32_t* err, bool dry_run) {
    // TMA row strides: C elements a multiple of 16 bytes
    if ((p.C * int64_t(sizeof(TA))) % 16 != 0) return DW_ERR_UNSUPPORTED;
    const int S = p.sh;
#define DW_W(CFG) return launch_tiled<CFG<TA>>(p, x, dy, dw, db, ws, stream, err, dry_run);
    if (p.kH == 3 && p.kW == 3 && S == 1) DW_W(W33s1)
    if (p.kH == 3 && p.kW == 3 && S == 2) DW_W(W33s2)
    if (p.kH == 5 && p.kW == 5 && S == 1) DW_W(W55s1)
    if (p.kH == 7 && p.kW == 7 && S == 1) DW_W(W77s1)
    if (p.kH == 1 && p.kW == 15 && S == 1) DW_W(W1x15)
    if (p.kH == 1 && p.kW == 31 && S == 1) DW_W(W1x31)
#undef DW_W
    return DW_ERR_UNSUPPORTED;
}

// Channel multiplier (NHWC, M = 2 or 4): 3x3, 3x3 stride 2, 5x5.
template <int M, class TA>
dw_status_t tiled_pick_mult(const Problem& p, const void* x, const void* dy, float* dw,
                            float* db, void* ws, cudaStream_t stream, int32_t* err, bool dry_run) {
    const int S = p.sh;
#define DW_W(CFG) return launch_tiled<CFG<M, TA>>(p, x, dy, dw, db, ws, stream, err, dry_run);
    if (p.kH == 3 && p.kW == 3 && S == 1) DW_W(W33s1m)
    if (p.kH == 3 && p.kW == 3 && S == 2) DW_W(W33s2m)
    if (p.kH == 5 && p.kW == 5 && S == 1) DW_W(W55s1m)
#undef DW_W
    return DW_ERR_UNSUPPORTED;
}

dw_status_t tiled_pick(const Problem& p, const void* x, const void* dy, float* dw, float* db,
                       void* ws, cudaStream_t stream, int32_t* err, bool dry_run) {
    if (p.M != 1 && p.layout == DW_NCHW) {
        // channel multiplier, NCHW: the plane-per-unit tiles (2-D filters)
        if (p.kH == 1) return DW_ERR_UNSUPPORTED;
        return tiled_pick_nchw(p, x, dy, dw, db, ws, stream, err, dry_run);
    }
    if (p.M != 1) {
        // channel multiplier: NHWC tiles for M = 2, 4; else the direct kernels
        if (p.layout != DW_NHWC || (p.M != 2 && p.M != 4)) return DW_ERR_UNSUPPORTED;
        // TMA row strides: C elements a multiple of 16 bytes
        if ((p.C * act_bytes(p.atype)) % 16 != 0 ||
            ((reinterpret_cast<uintptr_t>(x) | reinterpret_cast<uintptr_t>(dy)) & 15))
            return DW_ERR_UNSUPPORTED;
        if (p.sh != p.sw || p.dh != 1 || p.dw != 1) return DW_ERR_UNSUPPORTED;
        if (p.N >= INT_MAX || p.H >= INT_MAX || p.W >= INT_MAX || p.Co >= INT_MAX)
            return DW_ERR_UNSUPPORTED;
#define DW_M(TA)                                                                        \
    return p.M == 2 ? tiled_pick_mult<2, TA>(p, x, dy, dw, db, ws, stream, err, dry_run) \
                    : tiled_pick_mult<4, TA>(p, x, dy, dw, db, ws, stream, err, dry_run);
        if (p.atype == DW_F16) DW_M(__half)
        if (p.atype == DW_BF16) DW_M(__nv_bfloat16)
        DW_M(float)
#undef DW_M
    }
    if (p.layout == DW_NCHW) return tiled_pick_nchw(p, x, dy, dw, db, ws, stream, err, dry_run);
    if (p.layout != DW_NHWC) return DW_ERR_UNSUPPORTED;
    if ((reinterpret_cast<uintptr_t>(x) | reinterpret_cast<uintptr_t>(dy)) & 15)
        return DW_ERR_UNSUPPORTED;
    if (p.sh != p.sw || p.dh != 1 || p.dw != 1) return DW_ERR_UNSUPPORTED;
    if (p.N >= INT_MAX || p.H >= INT_MAX || p.W >= INT_MAX || p.C >= INT_MAX) return DW_ERR_UNSUPPORTED;
    if (p.atype == DW_F16) return tiled_pick_nhwc<__half>(p, x, dy, dw, db, ws, stream, err, dry_run);
    if (p.atype == DW_BF16)
        return tiled_pick_nhwc<__nv_bfloat16>(p, x, dy, dw, db, ws, stream, err, dry_run);
    return tiled_pick_nhwc<float>(p, x, dy, dw, db, ws, stream, err, dry_run);
}

}  // namespace wgrad

size_t bwd_weight_workspace_bytes(const Problem& p) {
    size_t m = wgrad::direct_workspace(p);
    const size_t b = wgrad::tiled_workspace(p), c = wgrad::tiled_nchw_workspace(p);
    const size_t r = wgrad::rows_nchw_workspace(p);
    if (b > m) m = b;
    if (r > m) m = r;
    if (c > m) m = c;
    return m;
}

dw_status_t bwd_weight_launch(const Problem& p, int algo, const void* x, const void* dy,
                              float* dw, float* db, void* ws, cudaStream_t stream, int32_t* err,
                              bool dry_run, int32_t* chosen) {
    if (algo == DW_ALGO_AUTO || algo == DW_ALGO_TILED) {
        const dw_status_t t = wgrad::tiled_pick(p, x, dy, dw, db, ws, stream, err, dry_run);
        if (t == DW_OK) {
            if (chosen) *chosen = DW_ALGO_TILED;
            return DW_OK;
        }
        if (t != DW_ERR_UNSUPPORTED || algo == DW_ALGO_TILED) return t;
    }
    if (chosen) *chosen = DW_ALGO_DIRECT;
    if (dry_run) return DW_OK;
    return wgrad::launch_direct(p, x, dy, dw, db, ws, stream);
}

}  // namespace dw
