// C ABI of libdwconv2d: descriptor validation, pad resolution, alias checks
// and dispatch to the kernel families.  Declared in include/dwconv2d.h.
#include <cudaTypedefs.h>

#include <atomic>
#include <mutex>

#include "dw_common.cuh"

namespace dw {

// ---------------------------------------------------------------- host utils

int current_device() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return -1;
    return dev;
}

int sm_count(int dev) {
    static std::atomic<int> cache[64];
    if (dev < 0 || dev >= 64) return 148;
    int v = cache[dev].load(std::memory_order_acquire);
    if (v > 0) return v;
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n < 1)
        n = 1;
    cache[dev].store(n, std::memory_order_release);
    return n;
}

static PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
static std::once_flag g_encode_once;

CUresult encode_tensor_map(CUtensorMap* map, CUtensorMapDataType dtype, cuuint32_t rank,
                           void* base, const cuuint64_t* dims, const cuuint64_t* strides,
                           const cuuint32_t* box, const cuuint32_t* elem_strides) {
    std::call_once(g_encode_once, [] {
        void* fn = nullptr;
        cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &fn, 12000,
                                             cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    });
    if (!g_encode) return CUDA_ERROR_NOT_SUPPORTED;
    return g_encode(map, dtype, rank, base, dims, strides, box, elem_strides,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
}

static std::mutex g_prepare_mutex;

int prepare_kernel(const void* kernel, int threads, size_t smem_bytes, LaunchCache& cache,
                   int dev) {
    if (dev < 0 || dev >= 64) return 0;
    int v = __atomic_load_n(&cache.occupancy[dev], __ATOMIC_ACQUIRE);
    if (v > 0) return v;
    std::lock_guard<std::mutex> lock(g_prepare_mutex);
    v = cache.occupancy[dev];
    if (v > 0) return v;
    if (smem_bytes > 48 * 1024 &&
        cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem_bytes)) != cudaSuccess)
        return 0;
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kernel, threads, smem_bytes) !=
        cudaSuccess)
        return 0;
    if (n > 0) __atomic_store_n(&cache.occupancy[dev], n, __ATOMIC_RELEASE);
    return n;
}

// The library's device error word: kernels that give up on a bounded wait
// record DW_ERR_DEVICE_TIMEOUT here.  Its device address is looked up once
// per device and passed to kernels as a plain pointer.
__device__ int32_t g_device_error;

static int32_t* device_error_ptr(int dev) {
    static std::atomic<int32_t*> cache[64];
    if (dev < 0 || dev >= 64) return nullptr;
    int32_t* p = cache[dev].load(std::memory_order_acquire);
    if (p) return p;
    void* addr = nullptr;
    if (cudaGetSymbolAddress(&addr, g_device_error) != cudaSuccess) return nullptr;
    p = static_cast<int32_t*>(addr);
    cache[dev].store(p, std::memory_order_release);
    return p;
}

// Fixed device scratch of dwconv2d_bwd_weight_noalloc: one array per device
// that loads the library, held until the process exits.  Host code only ever
// uses its device address, looked up once per device (with that device
// current) and cached; the array's name in host code is not that address.
static __device__ __align__(256) unsigned char g_noalloc_scratch[DW_NOALLOC_SCRATCH_BYTES];

static void* noalloc_scratch_ptr(int dev) {
    static std::atomic<void*> cache[64];
    if (dev < 0 || dev >= 64) return nullptr;
    void* p = cache[dev].load(std::memory_order_acquire);
    if (p) return p;
    void* addr = nullptr;
    if (cudaGetSymbolAddress(&addr, g_noalloc_scratch) != cudaSuccess || addr == nullptr)
        return nullptr;
    cache[dev].store(addr, std::memory_order_release);
    return addr;
}

// ---------------------------------------------------------------- validation

static int64_t out_extent(int64_t in, int k, int s, int d, int lo, int hi) {
    const int64_t reach = in + lo + hi - (static_cast<int64_t>(k - 1) * d + 1);
    if (reach < 0) return 0;
    return reach / s + 1;
}

static void same_pads(int64_t in, int k, int s, int d, int* lo, int* hi) {
    const int64_t out = (in + s - 1) / s;
    int64_t total = (out - 1) * s + static_cast<int64_t>(k - 1) * d + 1 - in;
    if (total < 0) total = 0;
    *lo = static_cast<int>(total / 2);
    *hi = static_cast<int>(total - total / 2);
}

// Limits keep every index the kernels form inside int64 and every pad and
// extent they form inside int32.
static constexpr int64_t kMaxExtent = int64_t(1) << 30;
static constexpr int kMaxKernel = 1 << 12;
static constexpr int kMaxStrideDil = 1 << 12;
static constexpr int kMaxPad = 1 << 20;
static constexpr int kMaxMultiplier = 1 << 12;

static dw_status_t resolve(const dw_desc_t* d, Problem* p) {
    if (!d) return DW_ERR_INVALID_ARG;
    if (d->N < 1 || d->H < 1 || d->W < 1 || d->C < 1) return DW_ERR_INVALID_ARG;
    if (d->N > kMaxExtent || d->H > kMaxExtent || d->W > kMaxExtent || d->C > kMaxExtent)
        return DW_ERR_INVALID_ARG;
    if (d->kH < 1 || d->kW < 1 || d->kH > kMaxKernel || d->kW > kMaxKernel)
        return DW_ERR_INVALID_ARG;
    if (d->stride_h < 1 || d->stride_w < 1 || d->dil_h < 1 || d->dil_w < 1)
        return DW_ERR_INVALID_ARG;
    if (d->stride_h > kMaxStrideDil || d->stride_w > kMaxStrideDil ||
        d->dil_h > kMaxStrideDil || d->dil_w > kMaxStrideDil)
        return DW_ERR_INVALID_ARG;
    if (d->layout != DW_NHWC && d->layout != DW_NCHW) return DW_ERR_INVALID_ARG;
    if (d->wtype != DW_F32 && d->wtype != DW_F16) return DW_ERR_INVALID_ARG;
    if (d->atype != DW_F32 && d->atype != DW_F16 && d->atype != DW_BF16) return DW_ERR_INVALID_ARG;
    if (d->algo < DW_ALGO_AUTO || d->algo > DW_ALGO_TILED) return DW_ERR_INVALID_ARG;
    if (d->multiplier < 0 || d->multiplier > kMaxMultiplier) return DW_ERR_INVALID_ARG;
    p->N = d->N; p->H = d->H; p->W = d->W; p->C = d->C;
    p->M = d->multiplier == 0 ? 1 : d->multiplier;
    p->Co = p->C * p->M;
    if (p->Co > kMaxExtent) return DW_ERR_INVALID_ARG;
    p->kH = d->kH; p->kW = d->kW;
    p->sh = d->stride_h; p->sw = d->stride_w;
    p->dh = d->dil_h; p->dw = d->dil_w;
    p->layout = d->layout; p->wtype = d->wtype; p->atype = d->atype;
    if (d->pad_mode == DW_PAD_SAME) {
        same_pads(d->H, d->kH, d->stride_h, d->dil_h, &p->pt, &p->pb);
        same_pads(d->W, d->kW, d->stride_w, d->dil_w, &p->pl, &p->pr);
    } else if (d->pad_mode == DW_PAD_EXPLICIT) {
        if (d->pad_top < 0 || d->pad_bottom < 0 || d->pad_left < 0 || d->pad_right < 0)
            return DW_ERR_INVALID_ARG;
        p->pt = d->pad_top; p->pb = d->pad_bottom;
        p->pl = d->pad_left; p->pr = d->pad_right;
    } else {
        return DW_ERR_INVALID_ARG;
    }
    if (p->pt > kMaxPad || p->pb > kMaxPad || p->pl > kMaxPad || p->pr > kMaxPad)
        return DW_ERR_INVALID_ARG;
    p->Ho = out_extent(p->H, p->kH, p->sh, p->dh, p->pt, p->pb);
    p->Wo = out_extent(p->W, p->kW, p->sw, p->dw, p->pl, p->pr);
    if (p->Ho < 1 || p->Wo < 1) return DW_ERR_INVALID_ARG;
    // element counts must stay well inside int64
    const double elems = double(p->N) * double(p->Co) *
                         double(p->H > p->Ho ? p->H : p->Ho) *
                         double(p->W > p->Wo ? p->W : p->Wo);
    if (elems > 9.0e15) return DW_ERR_INVALID_ARG;
    return DW_OK;
}

static bool overlaps(const void* a, size_t na, const void* b, size_t nb) {
    if (!a || !b || na == 0 || nb == 0) return false;
    const uintptr_t a0 = reinterpret_cast<uintptr_t>(a), b0 = reinterpret_cast<uintptr_t>(b);
    return a0 < b0 + nb && b0 < a0 + na;
}

struct Buffers {
    const void* in;  // activations of type p.atype
    const void* w;
    const float* b;
    void* out;       // activations of type p.atype
};

static dw_status_t check_buffers(const Problem& p, Op op, const Buffers& bf) {
    if (!bf.in || !bf.w || !bf.out) return DW_ERR_INVALID_ARG;
    const size_t x_elems = size_t(p.N) * size_t(p.C) * size_t(p.H) * size_t(p.W);
    const size_t y_elems = size_t(p.N) * size_t(p.Co) * size_t(p.Ho) * size_t(p.Wo);
    const size_t in_elems = op == OP_FWD ? x_elems : y_elems;
    const size_t out_elems = op == OP_FWD ? y_elems : x_elems;
    const size_t w_bytes = size_t(p.Co) * size_t(p.kH) * size_t(p.kW) * (p.wtype == DW_F16 ? 2 : 4);
    const size_t eb = size_t(act_bytes(p.atype));
    const size_t out_bytes = out_elems * eb;
    if (overlaps(bf.out, out_bytes, bf.in, in_elems * eb)) return DW_ERR_ALIAS;
    if (overlaps(bf.out, out_bytes, bf.w, w_bytes)) return DW_ERR_ALIAS;
    if (op == OP_FWD && overlaps(bf.out, out_bytes, bf.b, size_t(p.Co) * 4)) return DW_ERR_ALIAS;
    return DW_OK;
}

static dw_status_t run(const dw_desc_t* desc, Op op, const Buffers& bf, cudaStream_t stream,
                       bool dry_run, int32_t* chosen, const Epilogue* epi = nullptr) {
    Problem p;
    dw_status_t st = resolve(desc, &p);
    if (st != DW_OK) return st;
    st = check_buffers(p, op, bf);
    if (st != DW_OK) return st;
    if (epi) {
        // every statistics array must stay clear of y
        const size_t yb = size_t(p.N) * size_t(p.Co) * size_t(p.Ho) * size_t(p.Wo) *
                          size_t(act_bytes(p.atype));
        const float* stats[4] = {epi->gamma, epi->beta, epi->mean, epi->var};
        for (const float* v : stats)
            if (overlaps(bf.out, yb, v, size_t(p.Co) * 4)) return DW_ERR_ALIAS;
        p.epi = *epi;
    }
    const int algo = desc->algo;
    int32_t* err = nullptr;
    if (!dry_run) {
        err = device_error_ptr(current_device());
        if (!err) return DW_ERR_CUDA;
    }
    if (algo == DW_ALGO_AUTO || algo == DW_ALGO_TILED) {
        dw_status_t t = p.layout == DW_NHWC
                            ? tiled_nhwc_launch(p, op, bf.in, bf.w, bf.b, bf.out, stream, err, dry_run)
                            : tiled_nchw_launch(p, op, bf.in, bf.w, bf.b, bf.out, stream, err, dry_run);
        if (t == DW_OK) {
            if (chosen) *chosen = DW_ALGO_TILED;
            return DW_OK;
        }
        if (t != DW_ERR_UNSUPPORTED || algo == DW_ALGO_TILED) return t;
    }
    if (chosen) *chosen = DW_ALGO_DIRECT;
    if (dry_run) return DW_OK;
    return direct_launch(p, op, bf.in, bf.w, bf.b, bf.out, stream);
}

// One CTA of two warps and a barrier that nothing completes (see
// dwconv2d_selftest_wait_timeout).  Every wait is bounded, so the kernel
// always ends: mode 0 by its own limit, mode 1 by the abort flag (and, were
// the flag not seen, by the 2 s limit).
__global__ void __launch_bounds__(64) selftest_wait_kernel(int32_t* err, int mode,
                                                          uint64_t limit_ns) {
    __shared__ __align__(8) uint64_t bar;
    __shared__ volatile int abort_flag;
    grid_dependency_wait();
    allow_dependents();
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (lane != 0) return;
    if (mode == 0) {
        if (warp == 0 && !mbar_wait_bounded(&bar, 0, limit_ns)) atomicExch(err, DW_ERR_DEVICE_TIMEOUT);
    } else if (warp == 1) {
        abort_flag = 1;  // a failing warp raises the CTA's abort flag
    } else if (!mbar_wait_or_abort(&bar, 0, &abort_flag)) {
        atomicExch(err, DW_ERR_DEVICE_TIMEOUT);
    }
}

}  // namespace dw

using namespace dw;

extern "C" {

dw_status_t dwconv2d_out_shape(const dw_desc_t* desc, int64_t* Ho, int64_t* Wo) {
    Problem p;
    const dw_status_t st = resolve(desc, &p);
    if (st != DW_OK) return st;
    if (Ho) *Ho = p.Ho;
    if (Wo) *Wo = p.Wo;
    return DW_OK;
}

dw_status_t dwconv2d_resolved_pads(const dw_desc_t* desc, int32_t pads[4]) {
    Problem p;
    const dw_status_t st = resolve(desc, &p);
    if (st != DW_OK) return st;
    if (!pads) return DW_ERR_INVALID_ARG;
    pads[0] = p.pt; pads[1] = p.pb; pads[2] = p.pl; pads[3] = p.pr;
    return DW_OK;
}

dw_status_t dwconv2d_fwd(const dw_desc_t* desc, const void* x, const void* w, const float* b,
                         void* y, void* stream) {
    return run(desc, OP_FWD, Buffers{x, w, b, y}, static_cast<cudaStream_t>(stream), false,
               nullptr);
}

dw_status_t dwconv2d_fwd_bn_act(const dw_desc_t* desc, const void* x, const void* w,
                                const float* b, const float* gamma, const float* beta,
                                const float* mean, const float* var, float eps, int32_t act,
                                void* y, void* stream) {
    const int given = (gamma != nullptr) + (beta != nullptr) + (mean != nullptr) + (var != nullptr);
    if (given != 0 && given != 4) return DW_ERR_INVALID_ARG;
    if (!(eps >= 0.f) || !(eps <= 3.402823466e38f)) return DW_ERR_INVALID_ARG;  // NaN, inf, < 0
    if (act < DW_ACT_NONE || act > DW_ACT_SILU) return DW_ERR_INVALID_ARG;
    Epilogue e;
    e.gamma = gamma;
    e.beta = beta;
    e.mean = mean;
    e.var = var;
    e.eps = eps;
    e.act = act;
    return run(desc, OP_FWD, Buffers{x, w, b, y}, static_cast<cudaStream_t>(stream), false,
               nullptr, &e);
}

dw_status_t dwconv2d_bwd_input(const dw_desc_t* desc, const void* dy, const void* w, void* dx,
                               void* stream) {
    return run(desc, OP_BWD_INPUT, Buffers{dy, w, nullptr, dx}, static_cast<cudaStream_t>(stream),
               false, nullptr);
}

dw_status_t dwconv2d_bwd_weight_workspace_size(const dw_desc_t* desc, uint64_t* bytes) {
    Problem p;
    const dw_status_t st = resolve(desc, &p);
    if (st != DW_OK) return st;
    if (!bytes) return DW_ERR_INVALID_ARG;
    *bytes = bwd_weight_workspace_bytes(p);
    return DW_OK;
}

static dw_status_t run_bwd_weight(const dw_desc_t* desc, const void* x, const void* dy,
                                  float* dw, float* db, void* ws, uint64_t ws_bytes,
                                  cudaStream_t stream, bool dry_run, int32_t* chosen) {
    Problem p;
    dw_status_t st = resolve(desc, &p);
    if (st != DW_OK) return st;
    if (!x || !dy || !dw || !ws) return DW_ERR_INVALID_ARG;
    if (ws_bytes < bwd_weight_workspace_bytes(p)) return DW_ERR_INVALID_ARG;
    const size_t eb = size_t(act_bytes(p.atype));
    const size_t xb = size_t(p.N) * size_t(p.C) * size_t(p.H) * size_t(p.W) * eb;
    const size_t gb = size_t(p.N) * size_t(p.Co) * size_t(p.Ho) * size_t(p.Wo) * eb;
    const size_t wb = size_t(p.Co) * size_t(p.kH) * size_t(p.kW) * 4;
    const size_t bb = size_t(p.Co) * 4;
    const void* ins[2] = {x, dy};
    const size_t inb[2] = {xb, gb};
    void* outs[3] = {dw, db, ws};
    const size_t outb[3] = {wb, bb, size_t(ws_bytes)};
    for (int o = 0; o < 3; ++o) {
        for (int i = 0; i < 2; ++i)
            if (overlaps(outs[o], outb[o], ins[i], inb[i])) return DW_ERR_ALIAS;
        for (int o2 = o + 1; o2 < 3; ++o2)
            if (overlaps(outs[o], outb[o], outs[o2], outb[o2])) return DW_ERR_ALIAS;
    }
    int32_t* err = nullptr;
    if (!dry_run) {
        err = device_error_ptr(current_device());
        if (!err) return DW_ERR_CUDA;
    }
    return bwd_weight_launch(p, desc->algo, x, dy, dw, db, ws, stream, err, dry_run, chosen);
}

dw_status_t dwconv2d_bwd_weight(const dw_desc_t* desc, const void* x, const void* dy, float* dw,
                                float* db, void* workspace, uint64_t workspace_bytes,
                                void* stream) {
    return run_bwd_weight(desc, x, dy, dw, db, workspace, workspace_bytes,
                          static_cast<cudaStream_t>(stream), false, nullptr);
}

dw_status_t dwconv2d_bwd_weight_noalloc(const dw_desc_t* desc, const void* x, const void* dy,
                                        float* dw, float* db, void* stream) {
    Problem p;
    const dw_status_t st = resolve(desc, &p);
    if (st != DW_OK) return st;
    if (bwd_weight_workspace_bytes(p) > DW_NOALLOC_SCRATCH_BYTES) return DW_ERR_TOO_LARGE;
    void* scratch = noalloc_scratch_ptr(current_device());
    if (!scratch) return DW_ERR_CUDA;
    return run_bwd_weight(desc, x, dy, dw, db, scratch, DW_NOALLOC_SCRATCH_BYTES,
                          static_cast<cudaStream_t>(stream), false, nullptr);
}

int32_t dwconv2d_query_algo(const dw_desc_t* desc, int32_t op, const void* in, const void* w,
                            const void* out) {
    if (op == 2) {
        int32_t chosen = 0;
        Problem p;
        dw_status_t st = resolve(desc, &p);
        if (st != DW_OK) return -st;
        const uint64_t need = bwd_weight_workspace_bytes(p);
        // a workspace address far from the tensors, only used for the checks
        st = run_bwd_weight(desc, in, w,
                            static_cast<float*>(const_cast<void*>(out)), nullptr,
                            reinterpret_cast<void*>(uintptr_t(1) << 62), need, nullptr, true,
                            &chosen);
        return st == DW_OK ? chosen : -st;
    }
    if (op != OP_FWD && op != OP_BWD_INPUT) return -DW_ERR_INVALID_ARG;
    int32_t chosen = 0;
    const dw_status_t st =
        run(desc, static_cast<Op>(op),
            Buffers{in, w, nullptr, const_cast<void*>(out)},
            nullptr, true, &chosen);
    return st == DW_OK ? chosen : -st;
}

dw_status_t dwconv2d_take_device_error(int32_t* code) {
    if (!code) return DW_ERR_INVALID_ARG;
    int32_t* ptr = device_error_ptr(current_device());
    if (!ptr) return DW_ERR_CUDA;
    int32_t v = 0;
    if (cudaMemcpy(&v, ptr, sizeof(v), cudaMemcpyDeviceToHost) != cudaSuccess) return DW_ERR_CUDA;
    const int32_t zero = 0;
    if (cudaMemcpy(ptr, &zero, sizeof(zero), cudaMemcpyHostToDevice) != cudaSuccess)
        return DW_ERR_CUDA;
    *code = v;
    return DW_OK;
}

dw_status_t dwconv2d_selftest_wait_timeout(int32_t mode, uint32_t limit_us, void* stream) {
    if ((mode != 0 && mode != 1) || limit_us < 1 || limit_us > 1000000u) return DW_ERR_INVALID_ARG;
    int32_t* err = device_error_ptr(current_device());
    if (!err) return DW_ERR_CUDA;
    if (launch_pdl(selftest_wait_kernel, dim3(1), dim3(64), 0, static_cast<cudaStream_t>(stream),
                   err, mode, uint64_t(limit_us) * 1000u) != cudaSuccess)
        return DW_ERR_CUDA;
    return cudaGetLastError() == cudaSuccess ? DW_OK : DW_ERR_CUDA;
}

const char* dwconv2d_status_string(dw_status_t status) {
    switch (status) {
        case DW_OK: return "DW_OK";
        case DW_ERR_INVALID_ARG: return "DW_ERR_INVALID_ARG: invalid descriptor or pointer";
        case DW_ERR_UNSUPPORTED: return "DW_ERR_UNSUPPORTED: no tiled kernel covers this shape";
        case DW_ERR_ALIAS: return "DW_ERR_ALIAS: output overlaps an input";
        case DW_ERR_CUDA: return "DW_ERR_CUDA: CUDA launch or runtime error";
        case DW_ERR_DEVICE_TIMEOUT: return "DW_ERR_DEVICE_TIMEOUT: a kernel gave up waiting on a copy";
        case DW_ERR_TOO_LARGE:
            return "DW_ERR_TOO_LARGE: the problem needs more scratch than the fixed device array holds";
        default: return "unknown dw_status_t";
    }
}

int32_t dwconv2d_version(void) { return 1 * 10000 + 0 * 100 + 0; }

}  // extern "C"
