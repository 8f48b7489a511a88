// shortconv.cu -- standalone width-3 causal depthwise conv over [B, Ctot, L].
//
// [P4] "HyenaDNA operator walk-through" (adg.csdn.net), section 二.1:
// short_filter = Conv1d(inner, inner, 3, padding=2, groups=inner), keep the
// first L outputs:  out[t] = w0 u[t-2] + w1 u[t-1] + w2 u[t] + bias, u[<0] = 0.
// The fused path applies the same taps while loading; this entry exists so a
// caller can run the unfused composition.  Each thread produces 8 consecutive
// outputs from one 16-byte (bf16) or two 16-byte (fp32) loads plus a
// two-sample halo.
#include "common.cuh"
#include "kernels.h"

namespace hyena {

namespace {

template <typename T>
struct Vec8;
template <>
struct Vec8<float> {
    static __device__ __forceinline__ void load(const float* p, float (&v)[8]) {
        const float4 a = __ldg(reinterpret_cast<const float4*>(p));
        const float4 b = __ldg(reinterpret_cast<const float4*>(p) + 1);
        v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
        v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
    }
    static __device__ __forceinline__ void store(float* p, const float (&v)[8]) {
        reinterpret_cast<float4*>(p)[0] = make_float4(v[0], v[1], v[2], v[3]);
        reinterpret_cast<float4*>(p)[1] = make_float4(v[4], v[5], v[6], v[7]);
    }
};
template <>
struct Vec8<__nv_bfloat16> {
    static __device__ __forceinline__ void load(const __nv_bfloat16* p, float (&v)[8]) {
        uint4 raw = __ldg(reinterpret_cast<const uint4*>(p));
        const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&raw);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            float2 f = __bfloat1622float2(h[i]);
            v[2 * i] = f.x;
            v[2 * i + 1] = f.y;
        }
    }
    static __device__ __forceinline__ void store(__nv_bfloat16* p, const float (&v)[8]) {
        uint4 raw;
        __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&raw);
#pragma unroll
        for (int i = 0; i < 4; ++i) h[i] = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
        *reinterpret_cast<uint4*>(p) = raw;
    }
};

template <typename T>
__global__ void k_shortconv(const T* __restrict__ u, T* __restrict__ out, const float* __restrict__ w,
                            const float* __restrict__ bias, int64_t Ctot, int64_t L, int64_t nvec) {
    const int64_t per_row = L / 8;
    const int64_t stride = int64_t(gridDim.x) * blockDim.x;
    for (int64_t idx = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; idx < nvec; idx += stride) {
        const int64_t row = idx / per_row;
        const int64_t t0 = (idx - row * per_row) * 8;
        const int64_t ch = row % Ctot;
        const T* ur = u + row * L;
        float x[10];
        x[0] = t0 >= 2 ? load1(ur + t0 - 2) : 0.0f;
        x[1] = t0 >= 1 ? load1(ur + t0 - 1) : 0.0f;
        float v[8];
        Vec8<T>::load(ur + t0, v);
#pragma unroll
        for (int i = 0; i < 8; ++i) x[i + 2] = v[i];
        const float w0 = __ldg(w + 3 * ch), w1 = __ldg(w + 3 * ch + 1), w2 = __ldg(w + 3 * ch + 2);
        const float bb = bias ? __ldg(bias + ch) : 0.0f;
        float o[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) o[i] = fmaf(w0, x[i], fmaf(w1, x[i + 1], fmaf(w2, x[i + 2], bb)));
        Vec8<T>::store(out + row * L + t0, o);
    }
}

}  // namespace

cudaError_t launch_shortconv(const void* u, void* out, const float* w, const float* bias, int64_t B,
                             int64_t Ctot, int64_t L, int dtype, cudaStream_t s) {
    const int64_t nvec = B * Ctot * (L / 8);
    if (nvec == 0) return cudaSuccess;
    int64_t blocks = (nvec + 255) / 256;
    if (blocks > 148 * 64) blocks = 148 * 64;
    if (dtype == DT_F32) {
        k_shortconv<float><<<unsigned(blocks), 256, 0, s>>>(static_cast<const float*>(u), static_cast<float*>(out),
                                                            w, bias, Ctot, L, nvec);
    } else {
        k_shortconv<__nv_bfloat16><<<unsigned(blocks), 256, 0, s>>>(
            static_cast<const __nv_bfloat16*>(u), static_cast<__nv_bfloat16*>(out), w, bias, Ctot, L, nvec);
    }
    return cudaGetLastError();
}

}  // namespace hyena
