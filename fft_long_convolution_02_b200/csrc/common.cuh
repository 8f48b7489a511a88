// common.cuh -- storage-type helpers shared by the kernels.
#pragma once
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "fft_core.cuh"

namespace hyena {

// Two consecutive stored values starting at an even element index -> float2.
__device__ __forceinline__ float2 load2(const float* p) { return __ldg(reinterpret_cast<const float2*>(p)); }
__device__ __forceinline__ float2 load2(const __nv_bfloat16* p) {
    unsigned int bits = __ldg(reinterpret_cast<const unsigned int*>(p));
    __nv_bfloat162 h = *reinterpret_cast<__nv_bfloat162*>(&bits);
    return __bfloat1622float2(h);
}
// Two consecutive values from shared memory (even element index).
__device__ __forceinline__ float2 load2_shared(const float* p) { return *reinterpret_cast<const float2*>(p); }
__device__ __forceinline__ float2 load2_shared(const __nv_bfloat16* p) {
    return __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(p));
}
__device__ __forceinline__ void store2(float* p, float2 v) { *reinterpret_cast<float2*>(p) = v; }
__device__ __forceinline__ void store2(__nv_bfloat16* p, float2 v) {
    __nv_bfloat162 h = __floats2bfloat162_rn(v.x, v.y);
    *reinterpret_cast<__nv_bfloat162*>(p) = h;
}
__device__ __forceinline__ float load1(const float* p) { return __ldg(p); }
__device__ __forceinline__ float load1(const __nv_bfloat16* p) { return __bfloat162float(*p); }

// Width-3 causal depthwise conv at two consecutive samples t = 2n, 2n+1 of
// one channel row x (PyTorch Conv1d cross-correlation, padding 2, first L
// outputs kept):  sc[t] = w0 x[t-2] + w1 x[t-1] + w2 x[t] + bias,
// x[<0] = 0.  With w == nullptr the raw samples are returned.
struct Taps {
    float w0, w1, w2, b;
    bool on;
};

__device__ __forceinline__ Taps load_taps(const float* w, const float* bias, int64_t ch) {
    Taps t;
    t.on = (w != nullptr);
    if (t.on) {
        t.w0 = __ldg(w + 3 * ch);
        t.w1 = __ldg(w + 3 * ch + 1);
        t.w2 = __ldg(w + 3 * ch + 2);
        t.b = bias ? __ldg(bias + ch) : 0.0f;
    } else {
        t.w0 = t.w1 = t.b = 0.0f;
        t.w2 = 1.0f;
    }
    return t;
}

template <typename T>
__device__ __forceinline__ float2 shortconv_pair(const T* __restrict__ x, int64_t t, const Taps& tp) {
    const float2 cur = load2(x + t);
    if (!tp.on) return cur;
    const float2 prev = (t >= 2) ? load2(x + t - 2) : make_float2(0.0f, 0.0f);
    float2 r;
    r.x = fmaf(tp.w0, prev.x, fmaf(tp.w1, prev.y, fmaf(tp.w2, cur.x, tp.b)));
    r.y = fmaf(tp.w0, prev.y, fmaf(tp.w1, cur.x, fmaf(tp.w2, cur.y, tp.b)));
    return r;
}

// Workspace element of the multi-pass and 2-D paths: complex64, or bf16
// (re, im) when the operator stores bf16; WsSel<T, 1> (the spectrum build)
// is always complex64.
template <typename T>
struct WsOf {
    using type = float2;
};
template <>
struct WsOf<__nv_bfloat16> {
    using type = __nv_bfloat162;
};
template <typename T, int MODE>
struct WsSel {
    using type = typename WsOf<T>::type;
};
template <typename T>
struct WsSel<T, 1> {
    using type = float2;
};
__device__ __forceinline__ float2 ws_ld(const float2* p) { return *p; }
__device__ __forceinline__ float2 ws_ld(const __nv_bfloat162* p) { return __bfloat1622float2(*p); }
__device__ __forceinline__ void ws_st(float2* p, float2 v) { *p = v; }
__device__ __forceinline__ void ws_st(__nv_bfloat162* p, float2 v) { *p = __float22bfloat162_rn(v); }

// Asynchronous global -> shared copies (cp.async): 16 bytes (L2 only), or
// 4 / 8 bytes; src_bytes < NB fills the rest of the destination with zeros.
__device__ __forceinline__ void cp_async_bytes16(void* dst, const void* src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(static_cast<unsigned>(__cvta_generic_to_shared(dst))),
                 "l"(src)
                 : "memory");
}
template <int NB>
__device__ __forceinline__ void cp_async_small(void* dst, const void* src, int src_bytes = NB) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], %2, %3;\n" ::"r"(static_cast<unsigned>(
                     __cvta_generic_to_shared(dst))),
                 "l"(src), "n"(NB), "r"(src_bytes)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;\n" ::: "memory"); }

}  // namespace hyena
