/*
 * Depthwise 2-D convolution: float64 CPU oracle.
 *
 * TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and the
 * cpu_baseline / reference legs of bench.py may load this library.  It shares
 * no code, header, table or helper with the CUDA path: it is written from the
 * source pages' definitions, in plain loops, and is deliberately slow.
 *
 * Definitions followed (page "LeanMlir Proofs/Architectures/Depthwise",
 * lean.brettkoonce.com):
 *   - forward, section "Depthwise conv2d forward (SAME padding, stride 1)":
 *       y[c,h,w] = (sum_{kh,kw} x[c, h+kh-p, w+kw-p] * W[c,kh,kw]) + b[c]
 *     generalised to a batch axis n, stride s, dilation d and per-side pads:
 *       y[n,ho,wo,c] = sum_{kh<kH,kw<kW} X(n, ho*sh + kh*dh - pt,
 *                                            wo*sw + kw*dw - pl, c) * W[c,kh,kw]
 *                      + b[c]
 *     with X = x inside [0,H)x[0,W) and 0 outside (the "pad-cond" of the
 *     input-VJP section).  Cross-correlation: the kernel is not flipped.
 *   - "no cross-channel mixing" (comparison with regular conv2d): channel c
 *     of y reads only channel c of x and filter c.
 *   - input gradient, section "Depthwise conv input-VJP": the map is affine in
 *     x, so its VJP is the transpose of the linear part.  dwo_bwd_input()
 *     applies that transpose literally (each output cotangent is sent back
 *     along the same index map the forward reads through); dwo_bwd_input_at()
 *     evaluates the section's closed-form "direct formula", a sum over output
 *     positions (ho,wo) with the kernel offset reconstructed from
 *     hi + pt = ho*sh + kh*dh.
 *   - weight and bias gradients, sections "Depthwise weight-VJP" and "Depthwise
 *     bias gradient - closed-form formula": the forward is affine in W and in b,
 *     so dW[c,kh,kw] = sum_{n,ho,wo} dy[n,ho,wo,c] * X(n, ho*sh + kh*dh - pt,
 *     wo*sw + kw*dw - pl, c) (the x_pad term that multiplies W[c,kh,kw]) and
 *     db[c] = sum_{n,ho,wo} dy[n,ho,wo,c]; the strided and XLA-SAME variants
 *     are the same sums with the strided index map (dwo_bwd_weight()).
 *   - stride-2 "SAME" and "XLA-SAME" (sections "Stride-2 SAME depthwise conv"
 *     and "Stride-2 XLA-SAME depthwise conv") fix which input rows a strided
 *     output reads; dwo_same_pads() implements the XLA rule
 *     (Ho = ceil(H/s), total pad = max((Ho-1)s + d(k-1) + 1 - H, 0), the odd
 *     half at the bottom/right), which reproduces the odd-position decimation.
 *
 *   - channel multiplier M (page "Incorrect stableHLO for grouped convolution
 *     gradient", the Reactant.jl issue: a 3x3 conv from 4 to 8 channels with
 *     groups = 4): C input channels, C*M output channels, output channel
 *     o = c*M + j (j < M) reads only input channel c = o / M through its own
 *     filter W[o] - a grouped convolution with one input channel per group.
 *     The forward, input gradient (dx[c] sums over the M output channels of
 *     c) and weight gradient (dW[o] pairs dy[o] with x[o / M]) follow from
 *     the same index map.  M = 1 is the plain depthwise convolution.
 *
 * Problem vector `p` (int64[16]):
 *   N, H, W, C, kH, kW, sh, sw, dh, dw, pt, pb, pl, pr, layout, M
 *   layout 0 = NHWC (c innermost), 1 = NCHW (w innermost); C counts the
 *   input channels, y and dy have C*M.
 * Weights are W[o][kh][kw] row-major, o < C*M.  Bias (C*M) may be NULL
 * (treated as 0).
 */
#include <stddef.h>
#include <stdint.h>
#include <math.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

enum { P_N, P_H, P_W, P_C, P_KH, P_KW, P_SH, P_SW, P_DH, P_DW,
       P_PT, P_PB, P_PL, P_PR, P_LAYOUT, P_MULT, P_COUNT };

/* Number of output positions along one axis: the largest o with
 * o*s + (k-1)*d - lo <= in - 1 + hi, plus one (0 if none). */
int64_t dwo_out_extent(int64_t in, int64_t k, int64_t s, int64_t d,
                       int64_t lo, int64_t hi) {
    int64_t last_reach = in + lo + hi - ((k - 1) * d + 1);
    if (last_reach < 0) return 0;
    return last_reach / s + 1;
}

/* XLA / TensorFlow "SAME": output extent ceil(in/s); the pad that makes the
 * last window end at the last row, split with the smaller half first. */
void dwo_same_pads(int64_t in, int64_t k, int64_t s, int64_t d,
                   int64_t* lo, int64_t* hi) {
    int64_t out = (in + s - 1) / s;
    int64_t total = (out - 1) * s + (k - 1) * d + 1 - in;
    if (total < 0) total = 0;
    *lo = total / 2;
    *hi = total - *lo;
}

int dwo_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* Flat index of element (n, c, h, w) of a tensor with Cx channels and
 * extents Hx, Wx, in the problem's layout. */
static int64_t act_index(const int64_t* p, int64_t n, int64_t c, int64_t h,
                         int64_t w, int64_t Cx, int64_t Hx, int64_t Wx) {
    if (p[P_LAYOUT] == 0) return ((n * Hx + h) * Wx + w) * Cx + c;
    return ((n * Cx + c) * Hx + h) * Wx + w;
}

static int64_t out_c(const int64_t* p) { return p[P_C] * p[P_MULT]; }

static int64_t out_h(const int64_t* p) {
    return dwo_out_extent(p[P_H], p[P_KH], p[P_SH], p[P_DH], p[P_PT], p[P_PB]);
}
static int64_t out_w(const int64_t* p) {
    return dwo_out_extent(p[P_W], p[P_KW], p[P_SW], p[P_DW], p[P_PL], p[P_PR]);
}

/* One forward output value (output channel o), straight from the definition. */
static double fwd_one(const int64_t* p, const double* x, const double* wt,
                      const double* b, int64_t n, int64_t o, int64_t ho,
                      int64_t wo) {
    int64_t H = p[P_H], W = p[P_W], kH = p[P_KH], kW = p[P_KW];
    int64_t c = o / p[P_MULT];  /* the one input channel output o reads */
    double acc = 0.0;
    for (int64_t kh = 0; kh < kH; ++kh) {
        for (int64_t kw = 0; kw < kW; ++kw) {
            int64_t hi = ho * p[P_SH] + kh * p[P_DH] - p[P_PT];
            int64_t wi = wo * p[P_SW] + kw * p[P_DW] - p[P_PL];
            double xv = 0.0;
            if (hi >= 0 && hi < H && wi >= 0 && wi < W)
                xv = x[act_index(p, n, c, hi, wi, p[P_C], H, W)];
            acc += xv * wt[(o * kH + kh) * kW + kw];
        }
    }
    return acc + (b ? b[o] : 0.0);
}

void dwo_fwd(const int64_t* p, const double* x, const double* wt,
             const double* b, double* y) {
    int64_t N = p[P_N], Co = out_c(p);
    int64_t Ho = out_h(p), Wo = out_w(p);
#pragma omp parallel for collapse(2) schedule(static)
    for (int64_t n = 0; n < N; ++n)
        for (int64_t o = 0; o < Co; ++o)
            for (int64_t ho = 0; ho < Ho; ++ho)
                for (int64_t wo = 0; wo < Wo; ++wo)
                    y[act_index(p, n, o, ho, wo, Co, Ho, Wo)] =
                        fwd_one(p, x, wt, b, n, o, ho, wo);
}

/* Transpose of the forward's linear part applied to dy: every output
 * cotangent dy[n,ho,wo,o] is sent back to each input position the forward
 * read for that output (input channel o / M), weighted by the tap that read
 * it.  Positions the forward never reads receive 0. */
void dwo_bwd_input(const int64_t* p, const double* dy, const double* wt,
                   double* dx) {
    int64_t N = p[P_N], C = p[P_C], H = p[P_H], W = p[P_W];
    int64_t kH = p[P_KH], kW = p[P_KW], M = p[P_MULT], Co = out_c(p);
    int64_t Ho = out_h(p), Wo = out_w(p);
#pragma omp parallel for collapse(2) schedule(static)
    for (int64_t n = 0; n < N; ++n) {
        for (int64_t c = 0; c < C; ++c) {
            for (int64_t hi = 0; hi < H; ++hi)
                for (int64_t wi = 0; wi < W; ++wi)
                    dx[act_index(p, n, c, hi, wi, C, H, W)] = 0.0;
            for (int64_t o = c * M; o < (c + 1) * M; ++o)
                for (int64_t ho = 0; ho < Ho; ++ho)
                    for (int64_t wo = 0; wo < Wo; ++wo) {
                        double g = dy[act_index(p, n, o, ho, wo, Co, Ho, Wo)];
                        for (int64_t kh = 0; kh < kH; ++kh)
                            for (int64_t kw = 0; kw < kW; ++kw) {
                                int64_t hi = ho * p[P_SH] + kh * p[P_DH] - p[P_PT];
                                int64_t wi = wo * p[P_SW] + kw * p[P_DW] - p[P_PL];
                                if (hi < 0 || hi >= H || wi < 0 || wi >= W) continue;
                                dx[act_index(p, n, c, hi, wi, C, H, W)] +=
                                    g * wt[(o * kH + kh) * kW + kw];
                            }
                    }
        }
    }
}

static void decode(const int64_t* p, int64_t flat, int64_t C, int64_t Hx, int64_t Wx,
                   int64_t* n, int64_t* c, int64_t* h, int64_t* w) {
    if (p[P_LAYOUT] == 0) {
        *c = flat % C; flat /= C;
        *w = flat % Wx; flat /= Wx;
        *h = flat % Hx; *n = flat / Hx;
    } else {
        *w = flat % Wx; flat /= Wx;
        *h = flat % Hx; flat /= Hx;
        *c = flat % C; *n = flat / C;
    }
}

/* Forward at selected flat output indices (layout order of y). */
void dwo_fwd_at(const int64_t* p, const double* x, const double* wt,
                const double* b, int64_t count, const int64_t* flat,
                double* out) {
    int64_t Ho = out_h(p), Wo = out_w(p);
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < count; ++i) {
        int64_t n, o, ho, wo;
        decode(p, flat[i], out_c(p), Ho, Wo, &n, &o, &ho, &wo);
        out[i] = fwd_one(p, x, wt, b, n, o, ho, wo);
    }
}

/* Input gradient at selected flat dx indices, by the page's direct formula:
 * a sum over output positions (ho,wo); the kernel offsets are reconstructed
 * from hi + pt = ho*sh + kh*dh and wi + pl = wo*sw + kw*dw, and a term counts
 * only when both offsets are whole taps inside [0,kH) x [0,kW).  Output
 * positions outside the rows/cols that can satisfy this contribute zero, so
 * the loops only visit that range. */
void dwo_bwd_input_at(const int64_t* p, const double* dy, const double* wt,
                      int64_t count, const int64_t* flat, double* out) {
    int64_t H = p[P_H], W = p[P_W], kH = p[P_KH], kW = p[P_KW];
    int64_t sh = p[P_SH], sw = p[P_SW], dh = p[P_DH], dw = p[P_DW];
    int64_t Ho = out_h(p), Wo = out_w(p);
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < count; ++i) {
        int64_t n, c, hi, wi;
        decode(p, flat[i], p[P_C], H, W, &n, &c, &hi, &wi);
        int64_t rh = hi + p[P_PT], rw = wi + p[P_PL];
        /* ho*sh in [rh - (kH-1)dh, rh]  ->  ho in [ho_lo, ho_hi] */
        int64_t ho_lo = rh - (kH - 1) * dh;
        ho_lo = ho_lo <= 0 ? 0 : (ho_lo + sh - 1) / sh;
        int64_t ho_hi = rh < 0 ? -1 : rh / sh;
        if (ho_hi > Ho - 1) ho_hi = Ho - 1;
        int64_t wo_lo = rw - (kW - 1) * dw;
        wo_lo = wo_lo <= 0 ? 0 : (wo_lo + sw - 1) / sw;
        int64_t wo_hi = rw < 0 ? -1 : rw / sw;
        if (wo_hi > Wo - 1) wo_hi = Wo - 1;
        double acc = 0.0;
        /* every output channel of input channel c: o = c*M .. c*M + M-1 */
        for (int64_t o = c * p[P_MULT]; o < (c + 1) * p[P_MULT]; ++o)
            for (int64_t ho = ho_lo; ho <= ho_hi; ++ho) {
                int64_t kh_nat = rh - ho * sh;          /* = kh * dh */
                if (kh_nat % dh != 0) continue;
                int64_t kh = kh_nat / dh;
                if (kh < 0 || kh >= kH) continue;
                for (int64_t wo = wo_lo; wo <= wo_hi; ++wo) {
                    int64_t kw_nat = rw - wo * sw;      /* = kw * dw */
                    if (kw_nat % dw != 0) continue;
                    int64_t kw = kw_nat / dw;
                    if (kw < 0 || kw >= kW) continue;
                    acc += dy[act_index(p, n, o, ho, wo, out_c(p), Ho, Wo)] *
                           wt[(o * kH + kh) * kW + kw];
                }
            }
        out[i] = acc;
    }
}

/* Weight and bias gradients: for each channel, the sum over every output
 * position of dy times the input value each tap read there (0 where the tap
 * read padding), and the plain sum of dy.  db may be NULL. */
void dwo_bwd_weight(const int64_t* p, const double* x, const double* dy, double* dw,
                    double* db) {
    int64_t N = p[P_N], C = p[P_C], H = p[P_H], W = p[P_W];
    int64_t kH = p[P_KH], kW = p[P_KW], Co = out_c(p);
    int64_t Ho = out_h(p), Wo = out_w(p);
#pragma omp parallel for schedule(static)
    for (int64_t o = 0; o < Co; ++o) {
        int64_t c = o / p[P_MULT];  /* the input channel filter o reads */
        for (int64_t kh = 0; kh < kH; ++kh)
            for (int64_t kw = 0; kw < kW; ++kw) {
                double acc = 0.0;
                for (int64_t n = 0; n < N; ++n)
                    for (int64_t ho = 0; ho < Ho; ++ho)
                        for (int64_t wo = 0; wo < Wo; ++wo) {
                            int64_t hi = ho * p[P_SH] + kh * p[P_DH] - p[P_PT];
                            int64_t wi = wo * p[P_SW] + kw * p[P_DW] - p[P_PL];
                            if (hi < 0 || hi >= H || wi < 0 || wi >= W) continue;
                            acc += dy[act_index(p, n, o, ho, wo, Co, Ho, Wo)] *
                                   x[act_index(p, n, c, hi, wi, C, H, W)];
                        }
                dw[(o * kH + kh) * kW + kw] = acc;
            }
        if (db) {
            double acc = 0.0;
            for (int64_t n = 0; n < N; ++n)
                for (int64_t ho = 0; ho < Ho; ++ho)
                    for (int64_t wo = 0; wo < Wo; ++wo)
                        acc += dy[act_index(p, n, o, ho, wo, Co, Ho, Wo)];
            db[o] = acc;
        }
    }
}

/* Fused forward epilogue.  The page's section on the MLIR lowering names a
 * depthwise-convolution-plus-batch-norm emitter without spelling the
 * normalisation out; it is read here as inference-mode batch normalisation
 * with per-channel running statistics, followed by an optional activation:
 *     u = gamma[c] * (z - mean[c]) / sqrt(var[c] + eps) + beta[c]
 *     out = act(u),  act in {identity, relu, relu6 = min(max(u,0),6),
 *                            silu = u / (1 + exp(-u))}
 * where z is the forward output (bias included) at an element of channel c.
 * gamma == NULL skips the normalisation (u = z).  Applied element by element:
 * z[i] belongs to channel ch[i]. */
enum { DWO_ACT_NONE = 0, DWO_ACT_RELU = 1, DWO_ACT_RELU6 = 2, DWO_ACT_SILU = 3 };

static double activation(double u, int64_t act) {
    switch (act) {
        case DWO_ACT_RELU: return u < 0.0 ? 0.0 : u;
        case DWO_ACT_RELU6: return u < 0.0 ? 0.0 : (u > 6.0 ? 6.0 : u);
        case DWO_ACT_SILU: return u / (1.0 + exp(-u));
        default: return u;
    }
}

void dwo_bn_act(int64_t count, const double* z, const int64_t* ch, const double* gamma,
                const double* beta, const double* mean, const double* var, double eps,
                int64_t act, double* out) {
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < count; ++i) {
        double u = z[i];
        if (gamma) {
            int64_t c = ch[i];
            u = gamma[c] * (u - mean[c]) / sqrt(var[c] + eps) + beta[c];
        }
        out[i] = activation(u, act);
    }
}
