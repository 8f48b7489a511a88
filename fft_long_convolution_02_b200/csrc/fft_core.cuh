// fft_core.cuh -- complex helpers and register-resident small DFTs (sm_100a).
//
// Conventions: forward transform X[k] = sum_n x[n] w^(n k) with
// w = exp(-2 pi i / R); the inverse uses conj(w) and is unnormalised.
// DFT<R, INV>::run transforms R values held in registers, natural order in
// and out.  It is the radix-2 decimation-in-time recursion with the exact
// constant twiddles of a 16th root of unity, so a 16-point DFT costs about
// 170 fp32 instructions.
#pragma once
#include <cuda_runtime.h>
#include <stdint.h>

namespace hyena {

__device__ __forceinline__ float2 cadd(float2 a, float2 b) { return make_float2(a.x + b.x, a.y + b.y); }
__device__ __forceinline__ float2 csub(float2 a, float2 b) { return make_float2(a.x - b.x, a.y - b.y); }
__device__ __forceinline__ float2 cconj(float2 a) { return make_float2(a.x, -a.y); }
__device__ __forceinline__ float2 cscale(float2 a, float s) { return make_float2(a.x * s, a.y * s); }
// a * b
__device__ __forceinline__ float2 cmul(float2 a, float2 b) {
    return make_float2(fmaf(a.x, b.x, -a.y * b.y), fmaf(a.x, b.y, a.y * b.x));
}
// a * conj(b)
__device__ __forceinline__ float2 cmulc(float2 a, float2 b) {
    return make_float2(fmaf(a.x, b.x, a.y * b.y), fmaf(a.y, b.x, -a.x * b.y));
}
// a * i  and  a * (-i)
__device__ __forceinline__ float2 cmul_i(float2 a) { return make_float2(-a.y, a.x); }
__device__ __forceinline__ float2 cmul_negi(float2 a) { return make_float2(a.y, -a.x); }

// cos(2 pi j / 16), j = 0..4 (mathematical constants).
#define HYENA_C16_1 0.92387953251128675613f
#define HYENA_S16_1 0.38268343236508977173f
#define HYENA_SQRT1_2 0.70710678118654752440f

// Multiply by w_R^k (forward: exp(-2 pi i k / R); inverse: its conjugate),
// R a power of two <= 16, k < R/2, with the cheap special cases inlined.
template <int R, bool INV>
__device__ __forceinline__ float2 mul_wconst(int k, float2 v) {
    // express as a multiple of 1/16 turn
    const int e = k * (16 / R);  // 0..7
    if (e == 0) return v;
    if (e == 4) return INV ? cmul_i(v) : cmul_negi(v);
    if (e == 2 || e == 6) {
        // w = (cos, -sin) with |cos| = |sin| = 1/sqrt2
        float c = (e == 2) ? HYENA_SQRT1_2 : -HYENA_SQRT1_2;
        float s = HYENA_SQRT1_2;  // sin(2 pi e / 16) > 0 for e = 2, 6
        if (!INV) return make_float2(c * v.x + s * v.y, c * v.y - s * v.x);
        return make_float2(c * v.x - s * v.y, c * v.y + s * v.x);
    }
    float c, s;
    switch (e) {
        case 1: c = HYENA_C16_1; s = HYENA_S16_1; break;
        case 3: c = HYENA_S16_1; s = HYENA_C16_1; break;
        case 5: c = -HYENA_S16_1; s = HYENA_C16_1; break;
        default: c = -HYENA_C16_1; s = HYENA_S16_1; break;  // e == 7
    }
    // forward: v * (c - i s); inverse: v * (c + i s)
    if (!INV) return make_float2(fmaf(c, v.x, s * v.y), fmaf(c, v.y, -s * v.x));
    return make_float2(fmaf(c, v.x, -s * v.y), fmaf(c, v.y, s * v.x));
}

template <int R, bool INV>
struct DFT {
    static __device__ __forceinline__ void run(float2 (&a)[R]) {
        float2 e[R / 2], o[R / 2];
#pragma unroll
        for (int i = 0; i < R / 2; ++i) { e[i] = a[2 * i]; o[i] = a[2 * i + 1]; }
        DFT<R / 2, INV>::run(e);
        DFT<R / 2, INV>::run(o);
#pragma unroll
        for (int k = 0; k < R / 2; ++k) {
            float2 t = mul_wconst<R, INV>(k, o[k]);
            a[k] = cadd(e[k], t);
            a[k + R / 2] = csub(e[k], t);
        }
    }
};
template <bool INV>
struct DFT<1, INV> {
    static __device__ __forceinline__ void run(float2 (&)[1]) {}
};
template <bool INV>
struct DFT<2, INV> {
    static __device__ __forceinline__ void run(float2 (&a)[2]) {
        float2 t = a[1];
        a[1] = csub(a[0], t);
        a[0] = cadd(a[0], t);
    }
};

// ---- Two transforms at once in split form: re = (Re x0, Re x1), im =
// (Im x0, Im x1), so that every add and multiply is one packed fp32x2
// instruction for both transforms (the same twiddles apply to both).
__device__ __forceinline__ float2 neg2(float2 a) { return make_float2(-a.x, -a.y); }
__device__ __forceinline__ float2 splat2(float a) { return make_float2(a, a); }

// (re, im) *= w_R^k (forward: exp(-2 pi i k / R); inverse: its conjugate), k < R/2.
template <int R, bool INV>
__device__ __forceinline__ void mul_wconst2(int k, float2& re, float2& im) {
    const int e = k * (16 / R);  // multiple of 1/16 turn, 0..7
    if (e == 0) return;
    const float2 r = re;
    if (e == 4) {
        // forward: times -i; inverse: times i
        if (!INV) { re = im; im = neg2(r); }
        else { re = neg2(im); im = r; }
        return;
    }
    float c, sn;
    switch (e) {
        case 1: c = HYENA_C16_1; sn = HYENA_S16_1; break;
        case 2: c = HYENA_SQRT1_2; sn = HYENA_SQRT1_2; break;
        case 3: c = HYENA_S16_1; sn = HYENA_C16_1; break;
        case 5: c = -HYENA_S16_1; sn = HYENA_C16_1; break;
        case 6: c = -HYENA_SQRT1_2; sn = HYENA_SQRT1_2; break;
        default: c = -HYENA_C16_1; sn = HYENA_S16_1; break;  // e == 7
    }
    // forward: v (c - i s) = (c re + s im, c im - s re); inverse: s -> -s
    const float2 cc = splat2(c), ss = splat2(INV ? -sn : sn);
    re = __ffma2_rn(cc, r, __fmul2_rn(ss, im));
    im = __ffma2_rn(cc, im, __fmul2_rn(neg2(ss), r));
}

template <int R, bool INV>
struct DFT2 {
    static __device__ __forceinline__ void run(float2 (&re)[R], float2 (&im)[R]) {
        float2 er[R / 2], ei[R / 2], orr[R / 2], oi[R / 2];
#pragma unroll
        for (int i = 0; i < R / 2; ++i) {
            er[i] = re[2 * i]; ei[i] = im[2 * i];
            orr[i] = re[2 * i + 1]; oi[i] = im[2 * i + 1];
        }
        DFT2<R / 2, INV>::run(er, ei);
        DFT2<R / 2, INV>::run(orr, oi);
#pragma unroll
        for (int k = 0; k < R / 2; ++k) {
            float2 tr = orr[k], ti = oi[k];
            mul_wconst2<R, INV>(k, tr, ti);
            re[k] = __fadd2_rn(er[k], tr);
            im[k] = __fadd2_rn(ei[k], ti);
            re[k + R / 2] = __fadd2_rn(er[k], neg2(tr));
            im[k + R / 2] = __fadd2_rn(ei[k], neg2(ti));
        }
    }
};
template <bool INV>
struct DFT2<1, INV> {
    static __device__ __forceinline__ void run(float2 (&)[1], float2 (&)[1]) {}
};
template <bool INV>
struct DFT2<2, INV> {
    static __device__ __forceinline__ void run(float2 (&re)[2], float2 (&im)[2]) {
        const float2 tr = re[1], ti = im[1];
        re[1] = __fadd2_rn(re[0], neg2(tr));
        im[1] = __fadd2_rn(im[0], neg2(ti));
        re[0] = __fadd2_rn(re[0], tr);
        im[0] = __fadd2_rn(im[0], ti);
    }
};

// (re, im) *= w (forward) or conj(w) (inverse), w shared by both transforms.
template <bool CONJ>
__device__ __forceinline__ void cmul_split(float2& re, float2& im, float2 w) {
    const float2 wr = splat2(w.x), wi = splat2(w.y);
    const float2 r = re;
    if (!CONJ) {
        re = __ffma2_rn(r, wr, neg2(__fmul2_rn(im, wi)));
        im = __ffma2_rn(r, wi, __fmul2_rn(im, wr));
    } else {
        re = __ffma2_rn(r, wr, __fmul2_rn(im, wi));
        im = __ffma2_rn(im, wr, neg2(__fmul2_rn(r, wi)));
    }
}

}  // namespace hyena
