// cta_fft.cuh -- M-point complex FFTs computed by one thread block in
// shared memory (sm_100a, fp32).
//
// Factorisation: M = 16^a * r0 with r0 in {1, 2, 4, 8}.  Stages in
// decimation-in-frequency order are a radix-16 stages followed by one radix-r0
// stage.  Stage i has length len_i = M / 16^i, radix R_i and stride
// P_i = len_i / R_i; one butterfly reads R_i values at stride P_i, applies the
// R_i-point DFT and then the twiddles w_len^(p s'), and writes them back in
// place.  The forward transform (DIF) leaves bin m at the digit-reversed
// position pos(m) = sum_i d_i(m) P_i, where d_i are the mixed-radix digits of
// m, least significant first.  The inverse (DIT) runs the conjugate stages in
// reverse order and turns digit-reversed input back into natural order, so no
// explicit permutation pass is ever needed.
//
// Shared memory is padded: element i lives at pad(i) = i + i/16 + i/256, which
// keeps the stride-P butterfly accesses free of bank conflicts.
//
// Twiddles come from a per-size table in global memory (filled in double
// precision when the spectrum is built): stage i holds (R_i - 1) * P_i
// entries, entry (s' - 1) * P_i + p = w_len^(p s'), so consecutive threads
// read consecutive entries.
#pragma once
#include "fft_core.cuh"
#include "plan_common.h"

namespace hyena {

__host__ __device__ constexpr int fft_pad(int i) { return i + (i >> 4) + (i >> 8); }
__host__ __device__ constexpr int fft_padded_size(int m) { return fft_pad(m - 1) + 1; }

// Position of bin m after the forward (DIF) pass of an M-point transform.
template <int M>
__device__ __forceinline__ int fft_bin_pos(int m) {
    int pos = 0;
#pragma unroll
    for (int i = 0; i < fft_nstages(M); ++i) {
        const int R = fft_stage_radix(M, i);
        const int P = fft_stage_stride(M, i);
        pos += (m & (R - 1)) * P;
        m >>= ilog2c(R);
    }
    return pos;
}

// One DIF (INV = false) or DIT (INV = true) stage over ntrans transforms
// stored at buf + t * tstride (padded indices within a transform).
template <int M, int STAGE, bool INV>
__device__ __forceinline__ void fft_stage(float2* __restrict__ buf, int ntrans, int tstride,
                                          const float2* __restrict__ tw) {
    constexpr int R = fft_stage_radix(M, STAGE);
    constexpr int LEN = fft_stage_len(M, STAGE);
    constexpr int P = LEN / R;
    constexpr int NB = M / R;
    constexpr int LOGNB = ilog2c(NB);
    constexpr int LOGP = ilog2c(P);
    const float2* __restrict__ tws = tw + fft_stage_tw_offset(M, STAGE);
    const int total = ntrans * NB;
    for (int bi = threadIdx.x; bi < total; bi += blockDim.x) {
        const int t = bi >> LOGNB;
        const int b = bi & (NB - 1);
        const int j = b >> LOGP;
        const int p = b & (P - 1);
        float2* base = buf + t * tstride;
        const int i0 = j * LEN + p;
        float2 a[R];
#pragma unroll
        for (int s = 0; s < R; ++s) a[s] = base[fft_pad(i0 + s * P)];
        if (!INV) {
            DFT<R, false>::run(a);
            if (P > 1) {
#pragma unroll
                for (int s = 1; s < R; ++s) a[s] = cmul(a[s], __ldg(&tws[(s - 1) * P + p]));
            }
        } else {
            if (P > 1) {
#pragma unroll
                for (int s = 1; s < R; ++s) a[s] = cmulc(a[s], __ldg(&tws[(s - 1) * P + p]));
            }
            DFT<R, true>::run(a);
        }
#pragma unroll
        for (int s = 0; s < R; ++s) base[fft_pad(i0 + s * P)] = a[s];
    }
}

template <int M, int STAGE>
__device__ __forceinline__ void fft_forward_from(float2* buf, int ntrans, int tstride, const float2* tw) {
    if constexpr (STAGE < fft_nstages(M)) {
        fft_stage<M, STAGE, false>(buf, ntrans, tstride, tw);
        __syncthreads();
        fft_forward_from<M, STAGE + 1>(buf, ntrans, tstride, tw);
    }
}

template <int M, int STAGE>
__device__ __forceinline__ void fft_inverse_from(float2* buf, int ntrans, int tstride, const float2* tw) {
    if constexpr (STAGE >= 0) {
        fft_stage<M, STAGE, true>(buf, ntrans, tstride, tw);
        __syncthreads();
        fft_inverse_from<M, STAGE - 1>(buf, ntrans, tstride, tw);
    }
}

// Forward DIF: natural -> digit-reversed.  Caller must __syncthreads()
// between writing buf and calling; returns after a final __syncthreads().
template <int M>
__device__ __forceinline__ void cta_fft_forward(float2* buf, int ntrans, int tstride, const float2* tw) {
    fft_forward_from<M, 0>(buf, ntrans, tstride, tw);
}
// Inverse DIT (unnormalised): digit-reversed -> natural.
template <int M>
__device__ __forceinline__ void cta_fft_inverse(float2* buf, int ntrans, int tstride, const float2* tw) {
    fft_inverse_from<M, fft_nstages(M) - 1>(buf, ntrans, tstride, tw);
}

}  // namespace hyena
