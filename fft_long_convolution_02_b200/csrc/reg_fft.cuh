// reg_fft.cuh -- register-resident M-point FFTs with shared-memory exchanges.
//
// A group of TPT = M/16 threads computes NV independent M-point transforms;
// thread g of the group holds 16 points of each transform in registers.
// Stages follow the factorisation of cta_fft.cuh (radix-16 stages, then one
// radix-r0 stage), decimation in frequency forward, in time inverse:
//
//   radix-16 stage i (stride P, length 16P): thread g is butterfly
//       (j, p) = (g / P, g % P) and holds elements j*16P + p + P*s, s < 16;
//   radix-r0 last stage (P = 1): thread g holds elements 16 g + k, k < 16,
//       i.e. 16/r0 butterflies of r0 consecutive elements.
//
// Forward input  : natural order, slot s = element g + (M/16) s.
// Forward output : digit-reversed positions, slot k = position 16 g + k.
// Inverse        : the reverse (positions in, natural order out, unnormalised).
//
// Between stages the group exchanges through one padded buffer per transform
// (pad(i) = i + i/16 + i/256).  For every stride used here
// pad(base + P s) = pad(base) + pad(P s), so each access is a per-thread base
// plus a compile-time offset.  Exchanges are bracketed by __syncthreads(), so
// every thread of the block must call these functions together.
#pragma once
#include "cta_fft.cuh"

namespace hyena {

template <int M, int I>
struct RegStage {
    static constexpr int R = fft_stage_radix(M, I);
    static constexpr int P = fft_stage_stride(M, I);
    static constexpr int LEN = fft_stage_len(M, I);
    static constexpr bool R16 = (R == 16);
    // element of slot 0 held by thread g at this stage
    static __device__ __forceinline__ int base(int g) {
        if constexpr (R16) return (g / P) * LEN + (g % P);
        else return 16 * g;
    }
    // padded offset of slot s relative to pad(base)
    static __device__ __forceinline__ constexpr int off(int s) {
        if constexpr (R16) return fft_pad(P * s);
        else return s;
    }
};

// DFT of the stage on one transform's 16 registers (+ twiddles for P > 1).
template <int M, int I, bool INV>
__device__ __forceinline__ void reg_stage_compute(float2 (&x)[16], int g, const float2* __restrict__ tw) {
    using S = RegStage<M, I>;
    if constexpr (S::R16) {
        const float2* tws = tw + fft_stage_tw_offset(M, I);
        const int p = g % S::P;
        if (!INV) {
            DFT<16, false>::run(x);
            if constexpr (S::P > 1) {
#pragma unroll
                for (int s = 1; s < 16; ++s) x[s] = cmul(x[s], __ldg(tws + (s - 1) * S::P + p));
            }
        } else {
            if constexpr (S::P > 1) {
#pragma unroll
                for (int s = 1; s < 16; ++s) x[s] = cmulc(x[s], __ldg(tws + (s - 1) * S::P + p));
            }
            DFT<16, true>::run(x);
        }
    } else {
        constexpr int R = S::R;
#pragma unroll
        for (int u = 0; u < 16 / R; ++u) {
            float2 a[R];
#pragma unroll
            for (int k = 0; k < R; ++k) a[k] = x[u * R + k];
            DFT<R, INV>::run(a);
#pragma unroll
            for (int k = 0; k < R; ++k) x[u * R + k] = a[k];
        }
    }
}

// The same stage on two transforms in split form (re[s] = (Re x0[s], Re x1[s]),
// im[s] likewise): packed fp32x2 arithmetic for both at once.
template <int M, int I, bool INV>
__device__ __forceinline__ void reg_stage_compute2(float2 (&re)[16], float2 (&im)[16], int g,
                                                   const float2* __restrict__ tw) {
    using S = RegStage<M, I>;
    if constexpr (S::R16) {
        const float2* tws = tw + fft_stage_tw_offset(M, I);
        const int p = g % S::P;
        if (!INV) {
            DFT2<16, false>::run(re, im);
            if constexpr (S::P > 1) {
#pragma unroll
                for (int s = 1; s < 16; ++s) cmul_split<false>(re[s], im[s], __ldg(tws + (s - 1) * S::P + p));
            }
        } else {
            if constexpr (S::P > 1) {
#pragma unroll
                for (int s = 1; s < 16; ++s) cmul_split<true>(re[s], im[s], __ldg(tws + (s - 1) * S::P + p));
            }
            DFT2<16, true>::run(re, im);
        }
    } else {
        constexpr int R = S::R;
#pragma unroll
        for (int u = 0; u < 16 / R; ++u) {
            float2 ar[R], ai[R];
#pragma unroll
            for (int k = 0; k < R; ++k) { ar[k] = re[u * R + k]; ai[k] = im[u * R + k]; }
            DFT2<R, INV>::run(ar, ai);
#pragma unroll
            for (int k = 0; k < R; ++k) { re[u * R + k] = ar[k]; im[u * R + k] = ai[k]; }
        }
    }
}

// Complex values of two transforms <-> split form, in place:
// (x0[s], x1[s]) <-> ((Re x0[s], Re x1[s]), (Im x0[s], Im x1[s])).
__device__ __forceinline__ void split_pair(float2 (&x)[2][16]) {
#pragma unroll
    for (int s = 0; s < 16; ++s) {
        const float2 a = x[0][s], b = x[1][s];
        x[0][s] = make_float2(a.x, b.x);
        x[1][s] = make_float2(a.y, b.y);
    }
}

// Stage I (input layout) -> stage I+1 (input layout) through shared memory.
template <int M, int I, int NV>
__device__ __forceinline__ void reg_exchange_fwd(float2 (&x)[NV][16], float2* const (&buf)[NV], int g) {
    using A = RegStage<M, I>;
    using B = RegStage<M, I + 1>;
    const int wa = fft_pad(A::base(g));
    const int rb = fft_pad(B::base(g));
#pragma unroll
    for (int v = 0; v < NV; ++v) {
#pragma unroll
        for (int s = 0; s < 16; ++s) buf[v][wa + A::off(s)] = x[v][s];
    }
    __syncthreads();
#pragma unroll
    for (int v = 0; v < NV; ++v) {
#pragma unroll
        for (int s = 0; s < 16; ++s) x[v][s] = buf[v][rb + B::off(s)];
    }
    __syncthreads();
}

// Stage I+1 layout -> stage I layout (inverse direction).
template <int M, int I, int NV>
__device__ __forceinline__ void reg_exchange_inv(float2 (&x)[NV][16], float2* const (&buf)[NV], int g) {
    using A = RegStage<M, I>;
    using B = RegStage<M, I + 1>;
    const int wb = fft_pad(B::base(g));
    const int ra = fft_pad(A::base(g));
#pragma unroll
    for (int v = 0; v < NV; ++v) {
#pragma unroll
        for (int s = 0; s < 16; ++s) buf[v][wb + B::off(s)] = x[v][s];
    }
    __syncthreads();
#pragma unroll
    for (int v = 0; v < NV; ++v) {
#pragma unroll
        for (int s = 0; s < 16; ++s) x[v][s] = buf[v][ra + A::off(s)];
    }
    __syncthreads();
}

// With NV == 2 the data are in split form (split_pair): x[0] holds the real
// parts of both transforms, x[1] the imaginary parts; the exchanges move them
// through buf[0] and buf[1] exactly as they would move two transforms.
template <int M, int I, int NV>
__device__ __forceinline__ void reg_fwd_from(float2 (&x)[NV][16], float2* const (&buf)[NV], int g,
                                             const float2* __restrict__ tw) {
    if constexpr (NV == 2) {
        reg_stage_compute2<M, I, false>(x[0], x[1], g, tw);
    } else {
#pragma unroll
        for (int v = 0; v < NV; ++v) reg_stage_compute<M, I, false>(x[v], g, tw);
    }
    if constexpr (I + 1 < fft_nstages(M)) {
        reg_exchange_fwd<M, I, NV>(x, buf, g);
        reg_fwd_from<M, I + 1, NV>(x, buf, g, tw);
    }
}

template <int M, int I, int NV>
__device__ __forceinline__ void reg_inv_from(float2 (&x)[NV][16], float2* const (&buf)[NV], int g,
                                             const float2* __restrict__ tw) {
    if constexpr (NV == 2) {
        reg_stage_compute2<M, I, true>(x[0], x[1], g, tw);
    } else {
#pragma unroll
        for (int v = 0; v < NV; ++v) reg_stage_compute<M, I, true>(x[v], g, tw);
    }
    if constexpr (I > 0) {
        reg_exchange_inv<M, I - 1, NV>(x, buf, g);
        reg_inv_from<M, I - 1, NV>(x, buf, g, tw);
    }
}

// Forward: natural (slot s = element g + (M/16) s) -> positions 16 g + s.
template <int M, int NV>
__device__ __forceinline__ void reg_fft_forward(float2 (&x)[NV][16], float2* const (&buf)[NV], int g,
                                                const float2* __restrict__ tw) {
    static_assert(M >= 16, "register FFT needs M >= 16");
    if constexpr (NV == 2) split_pair(x);
    reg_fwd_from<M, 0, NV>(x, buf, g, tw);
    if constexpr (NV == 2) split_pair(x);
}

// Inverse: positions 16 g + s -> natural order (unnormalised).
template <int M, int NV>
__device__ __forceinline__ void reg_fft_inverse(float2 (&x)[NV][16], float2* const (&buf)[NV], int g,
                                                const float2* __restrict__ tw) {
    if constexpr (NV == 2) split_pair(x);
    reg_inv_from<M, fft_nstages(M) - 1, NV>(x, buf, g, tw);
    if constexpr (NV == 2) split_pair(x);
}

// Bin held at position pos after the forward transform (inverse of fft_bin_pos).
template <int M>
__device__ __forceinline__ int fft_pos_bin(int pos) {
    int bin = 0, scale = 1;
#pragma unroll
    for (int i = 0; i < fft_nstages(M); ++i) {
        const int R = fft_stage_radix(M, i);
        const int P = fft_stage_stride(M, i);
        bin += ((pos / P) % R) * scale;
        scale *= R;
    }
    return bin;
}

}  // namespace hyena
