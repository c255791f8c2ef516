// Internal declarations shared by the CUDA translation units of libdwconv2d.
// Nothing here is part of the public ABI (see include/dwconv2d.h).
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <type_traits>
#include <utility>

#include "dwconv2d.h"

namespace dw {

// Fused forward epilogue: inference-mode batch normalisation (per-channel
// running statistics; gamma == nullptr means none) and an activation.
struct Epilogue {
    const float* gamma = nullptr;
    const float* beta = nullptr;
    const float* mean = nullptr;
    const float* var = nullptr;
    float eps = 0.f;
    int act = DW_ACT_NONE;
    __host__ __device__ bool on() const { return gamma != nullptr || act != DW_ACT_NONE; }
};

// A resolved problem: everything the kernels need, pads already resolved.
// H, W, C, N are the extents of x (forward input) / dx (gradient output);
// Ho, Wo the extents of y / dy, which have Co = C*M channels (M output
// channels per input channel; output channel o reads input channel o / M).
struct Problem {
    int64_t N, H, W, C, Ho, Wo;
    int64_t M = 1, Co = 0;
    int kH, kW, sh, sw, dh, dw;
    int pt, pb, pl, pr;
    int layout;  // DW_NHWC / DW_NCHW
    int wtype;   // DW_F32 / DW_F16
    int atype = DW_F32;  // activations (x, y, dy, dx): DW_F32 / DW_F16 / DW_BF16
    Epilogue epi;  // forward only; off for every other call
};

enum Op { OP_FWD = 0, OP_BWD_INPUT = 1 };

// Launch entry points of each kernel family.  `dry_run` only answers whether
// the family covers the problem (DW_OK / DW_ERR_UNSUPPORTED) without touching
// the device.  `in` and `out` hold activations of type p.atype.
dw_status_t direct_launch(const Problem& p, Op op, const void* in, const void* w,
                          const float* b, void* out, cudaStream_t stream);
dw_status_t tiled_nhwc_launch(const Problem& p, Op op, const void* in, const void* w,
                              const float* b, void* out, cudaStream_t stream,
                              int32_t* dev_err, bool dry_run);
dw_status_t tiled_nchw_launch(const Problem& p, Op op, const void* in, const void* w,
                              const float* b, void* out, cudaStream_t stream,
                              int32_t* dev_err, bool dry_run);

// Weight / bias gradient (dw_bwd_weight.cu): workspace bytes the call needs,
// and the launch (partials into `ws`, then the fixed-order finalize).
size_t bwd_weight_workspace_bytes(const Problem& p);
dw_status_t bwd_weight_launch(const Problem& p, int algo, const void* x, const void* dy,
                              float* dw, float* db, void* ws, cudaStream_t stream,
                              int32_t* dev_err, bool dry_run, int32_t* chosen);

// Host helpers (dw_api.cu).
int current_device();
int sm_count(int dev);
// cuTensorMapEncodeTiled fetched through the runtime (no link-time libcuda
// dependency, so the library also loads on machines without a driver).
CUresult encode_tensor_map(CUtensorMap* map, CUtensorMapDataType dtype, cuuint32_t rank,
                           void* base, const cuuint64_t* dims, const cuuint64_t* strides,
                           const cuuint32_t* box, const cuuint32_t* elem_strides);

// Per-channel scale and shift of the epilogue's normalisation:
// scale = gamma / sqrt(var + eps), shift = beta - mean * scale (IEEE division
// and square root); without statistics scale = 1 and shift = -0, so that
// fmaf(z, scale, shift) == z for every z, -0 included.
__device__ __forceinline__ void bn_scale_shift(const Epilogue& e, int c, float& scale,
                                               float& shift) {
    if (e.gamma != nullptr) {
        scale = __ldg(e.gamma + c) / sqrtf(__ldg(e.var + c) + e.eps);
        shift = fmaf(-__ldg(e.mean + c), scale, __ldg(e.beta + c));
    } else {
        scale = 1.f;
        shift = -0.f;
    }
}

// The activation; comparisons written so that NaN passes through.
// silu: u / (1 + e^-u) with expf (at most 2 ulp) and the fast division
// __fdividef (at most 2 ulp while the divisor stays below 2^126; beyond, at
// u < -87.3, it returns 0 where the true value is below 1e-35 in magnitude).
// The correctly rounded division or reciprocal costs a third of the large
// NHWC forward's time; this form keeps the epilogue near the memory bound.
template <int ACT>
__device__ __forceinline__ float activate(float u) {
    if constexpr (ACT == DW_ACT_RELU) return u < 0.f ? 0.f : u;
    if constexpr (ACT == DW_ACT_RELU6) return u < 0.f ? 0.f : (u > 6.f ? 6.f : u);
    if constexpr (ACT == DW_ACT_SILU) return __fdividef(u, 1.f + expf(-u));
    return u;
}

// act(z * scale + shift)
template <int ACT>
__device__ __forceinline__ float epilogue_act(float z, float scale, float shift) {
    return activate<ACT>(fmaf(z, scale, shift));
}

// Run-time activation (the direct kernels).
__device__ __forceinline__ float epilogue_apply(float z, float scale, float shift, int act) {
    switch (act) {
        case DW_ACT_RELU: return epilogue_act<DW_ACT_RELU>(z, scale, shift);
        case DW_ACT_RELU6: return epilogue_act<DW_ACT_RELU6>(z, scale, shift);
        case DW_ACT_SILU: return epilogue_act<DW_ACT_SILU>(z, scale, shift);
        default: return epilogue_act<DW_ACT_NONE>(z, scale, shift);
    }
}

// Kernel instantiation of an epilogue: -1 = none (plain forward, and every
// gradient kernel), else the activation.  The tiled kernels fold the
// normalisation into the filter and bias they hold in registers (W' = scale *
// W, b' = scale * b + shift, exact when the statistics are absent: scale 1,
// shift -0), so the only per-output work left is the activation.
constexpr int kNoEpilogue = -1;
inline int epilogue_variant(const Epilogue& e) { return e.on() ? e.act : kNoEpilogue; }

// Launch with programmatic stream serialization (see grid_dependency_wait).
template <class... KArgs, class... Actual>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t stream, Actual&&... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Actual>(args)...);
}

// Per (kernel instantiation, device) cache of the launch attributes.
struct LaunchCache {
    int occupancy[64];  // 0 = not queried yet
};
// Sets the dynamic shared memory limit once and returns resident CTAs per SM
// (0 if the kernel cannot be resident at all).
int prepare_kernel(const void* kernel, int threads, size_t smem_bytes, LaunchCache& cache,
                   int dev);

// ------------------------------------------------------------------ device --

__device__ __forceinline__ float load_weight(const void* w, int wtype, int64_t idx) {
    // float16 -> float32 widening is exact, so both weight types feed the
    // same float32 FMA sequence.
    return wtype == DW_F16 ? __half2float(static_cast<const __half*>(w)[idx])
                           : static_cast<const float*>(w)[idx];
}

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count)
                 : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)),
                 "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(done)
        : "r"(smem_addr(bar)), "r"(parity)
        : "memory");
    return done != 0;
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}

__device__ __forceinline__ uint64_t global_timer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
    return t;
}

// Every wait on an asynchronous copy is bounded: after kWaitLimitNs without
// completion it reports failure instead of spinning forever.
constexpr uint64_t kWaitLimitNs = 2000000000ull;  // 2 s

__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity,
                                                  uint64_t limit_ns = kWaitLimitNs) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_timer_ns();
    while (!mbar_try_wait(bar, parity)) {
        if (global_timer_ns() - t0 > limit_ns) return false;
    }
    return true;
}

// Bounded wait that also gives up as soon as another warp of the CTA has
// raised `abort` (a shared-memory flag), so one failed wait ends every warp.
__device__ __forceinline__ bool mbar_wait_or_abort(uint64_t* bar, uint32_t parity,
                                                   const volatile int* abort,
                                                   uint64_t limit_ns = kWaitLimitNs) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_timer_ns();
    while (!mbar_try_wait(bar, parity)) {
        if (*abort) return false;
        if (global_timer_ns() - t0 > limit_ns) return false;
    }
    return true;
}

// Division by a run-time constant d as a multiply and shift, exact for every
// 0 <= n < 2^31: with s = ceil(log2 d) and m = floor(2^(31+s) / d) + 1,
// floor(n*m / 2^(31+s)) = floor(n/d) because n*(m - 2^(31+s)/d) < 2^(31+s)/d.
struct FastDiv {
    uint64_t m;
    uint32_t shift;  // 31 + s
    int d;
};

inline FastDiv make_fastdiv(int d) {
    uint32_t s = 0;
    while ((int64_t(1) << s) < d) ++s;
    FastDiv f;
    f.m = ((uint64_t(1) << (31 + s)) / uint64_t(d)) + 1;
    f.shift = 31 + s;
    f.d = d;
    return f;
}

__device__ __forceinline__ int fast_div(int n, const FastDiv& f) {
    return static_cast<int>((static_cast<uint64_t>(static_cast<uint32_t>(n)) * f.m) >> f.shift);
}

// 4-D tiled TMA load (no multicast) into this CTA's shared memory; completion
// is signalled on `bar` as transaction bytes.
__device__ __forceinline__ void tma_load_4d(void* dst, const CUtensorMap* map, uint64_t* bar,
                                            int c0, int c1, int c2, int c3) {
    asm volatile(
        "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3, %4, %5}], [%6];" ::"r"(smem_addr(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(c3),
        "r"(smem_addr(bar))
        : "memory");
}

// 4-D tiled TMA store from this CTA's shared memory (bulk-group completion).
// Coordinates must be non-negative; parts of the box outside the tensor are
// not written.
__device__ __forceinline__ void tma_store_4d(const CUtensorMap* map, const void* src, int c0,
                                             int c1, int c2, int c3) {
    asm volatile(
        "cp.async.bulk.tensor.4d.global.shared::cta.tile.bulk_group [%0, {%2, %3, %4, %5}], [%1];" ::
            "l"(reinterpret_cast<uint64_t>(map)),
        "r"(smem_addr(src)), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
        : "memory");
}
__device__ __forceinline__ void bulk_commit_group() {
    asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
// Wait until at most N committed bulk groups still read shared memory.
template <int N>
__device__ __forceinline__ void bulk_wait_group_read() {
    asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}
// Wait until at most N committed bulk groups are still in flight at all.
template <int N>
__device__ __forceinline__ void bulk_wait_group() {
    asm volatile("cp.async.bulk.wait_group %0;" ::"n"(N) : "memory");
}
// Orders this thread's generic-proxy shared-memory writes before later
// async-proxy (TMA) reads of them.
__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
// Named barrier over `count` threads; returns the OR of `pred` over them.
__device__ __forceinline__ bool named_barrier_or(int id, int count, bool pred) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "barrier.cta.red.or.pred q, %2, %3, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"(uint32_t(pred)), "r"(id), "r"(count)
        : "memory");
    return r != 0;
}
__device__ __forceinline__ void named_barrier_sync(int id, int count) {
    asm volatile("barrier.cta.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

__device__ __forceinline__ void prefetch_tensor_map(const CUtensorMap* map) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// Programmatic dependent launch.  Every kernel of the library is launched
// with programmatic stream serialization, so it may be scheduled while the
// previous kernel on the stream is still draining.  grid_dependency_wait()
// blocks until every prerequisite grid has completed and its memory is
// visible; each kernel calls it before its first global-memory access (read
// or write), which keeps plain stream-order semantics for the caller.
// allow_dependents() lets the next kernel on the stream start its prologue.
__device__ __forceinline__ void grid_dependency_wait() {
    asm volatile("griddepcontrol.wait;" ::: "memory");
}
__device__ __forceinline__ void allow_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// Compile-time loop: calls f(integral_constant<int, i>) for i in [I, N).
template <int I, int N, class F>
__device__ __forceinline__ void static_for(F&& f) {
    if constexpr (I < N) {
        f(std::integral_constant<int, I>{});
        static_for<I + 1, N>(f);
    }
}

__device__ __forceinline__ void fma4(float4& acc, const float4& v, const float4& w) {
    acc.x = fmaf(v.x, w.x, acc.x);
    acc.y = fmaf(v.y, w.y, acc.y);
    acc.z = fmaf(v.z, w.z, acc.z);
    acc.w = fmaf(v.w, w.w, acc.w);
}

__device__ __forceinline__ void store4(float* p, const float4& v) {
    *reinterpret_cast<float4*>(p) = v;
}

// Activation element types: float32, float16, bfloat16.  Loads widen to
// float32 exactly; stores round to nearest even.  load4/store4 move 4
// consecutive elements (16 or 8 bytes, aligned to that size), load2/store2 two.
template <class TA>
struct ActIO;

template <>
struct ActIO<float> {
    static constexpr CUtensorMapDataType kTma = CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
    static __device__ __forceinline__ float load1(const float* p) { return *p; }
    static __device__ __forceinline__ float2 load2(const float* p) {
        return *reinterpret_cast<const float2*>(p);
    }
    static __device__ __forceinline__ float4 load4(const float* p) {
        return *reinterpret_cast<const float4*>(p);
    }
    static __device__ __forceinline__ void store1(float* p, float v) { *p = v; }
    static __device__ __forceinline__ void store2(float* p, const float2& v) {
        *reinterpret_cast<float2*>(p) = v;
    }
    static __device__ __forceinline__ void store4(float* p, const float4& v) { dw::store4(p, v); }
};

template <>
struct ActIO<__half> {
    static constexpr CUtensorMapDataType kTma = CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
    static __device__ __forceinline__ float load1(const __half* p) { return __half2float(*p); }
    static __device__ __forceinline__ float2 load2(const __half* p) {
        return __half22float2(*reinterpret_cast<const __half2*>(p));
    }
    static __device__ __forceinline__ float4 load4(const __half* p) {
        const uint2 raw = *reinterpret_cast<const uint2*>(p);
        const float2 a = __half22float2(*reinterpret_cast<const __half2*>(&raw.x));
        const float2 b = __half22float2(*reinterpret_cast<const __half2*>(&raw.y));
        return make_float4(a.x, a.y, b.x, b.y);
    }
    static __device__ __forceinline__ void store1(__half* p, float v) { *p = __float2half_rn(v); }
    static __device__ __forceinline__ void store2(__half* p, const float2& v) {
        *reinterpret_cast<__half2*>(p) = __floats2half2_rn(v.x, v.y);
    }
    static __device__ __forceinline__ void store4(__half* p, const float4& v) {
        const __half2 a = __floats2half2_rn(v.x, v.y), b = __floats2half2_rn(v.z, v.w);
        uint2 raw;
        raw.x = *reinterpret_cast<const uint32_t*>(&a);
        raw.y = *reinterpret_cast<const uint32_t*>(&b);
        *reinterpret_cast<uint2*>(p) = raw;
    }
};

template <>
struct ActIO<__nv_bfloat16> {
    static constexpr CUtensorMapDataType kTma = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    static __device__ __forceinline__ float load1(const __nv_bfloat16* p) {
        return __bfloat162float(*p);
    }
    static __device__ __forceinline__ float2 load2(const __nv_bfloat16* p) {
        return __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(p));
    }
    static __device__ __forceinline__ float4 load4(const __nv_bfloat16* p) {
        const uint2 raw = *reinterpret_cast<const uint2*>(p);
        const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&raw.x));
        const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&raw.y));
        return make_float4(a.x, a.y, b.x, b.y);
    }
    static __device__ __forceinline__ void store1(__nv_bfloat16* p, float v) {
        *p = __float2bfloat16_rn(v);
    }
    static __device__ __forceinline__ void store2(__nv_bfloat16* p, const float2& v) {
        *reinterpret_cast<__nv_bfloat162*>(p) = __floats2bfloat162_rn(v.x, v.y);
    }
    static __device__ __forceinline__ void store4(__nv_bfloat16* p, const float4& v) {
        const __nv_bfloat162 a = __floats2bfloat162_rn(v.x, v.y);
        const __nv_bfloat162 b = __floats2bfloat162_rn(v.z, v.w);
        uint2 raw;
        raw.x = *reinterpret_cast<const uint32_t*>(&a);
        raw.y = *reinterpret_cast<const uint32_t*>(&b);
        *reinterpret_cast<uint2*>(p) = raw;
    }
};

// Bytes of one activation element of type `atype` (DW_F32 / DW_F16 / DW_BF16).
inline int act_bytes(int atype) { return atype == DW_F32 ? 4 : 2; }

}  // namespace dw
