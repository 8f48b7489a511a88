// onchip.cu -- the fused on-chip path (16 <= L <= 16384) and its spectrum.
//
// Method ([P4] "HyenaDNA operator walk-through" (adg.csdn.net), section 二.1,
// HyenaOperator.forward; section 二.2, fftconv): for each order step s the
// value v is gated, v <- x_{order-s} * v, then convolved with the long filter
// k_s plus the skip D_s; finally y = x0 * v.  The convolution is the 2L-point
// zero-padded FFT product, evaluated here as follows (all exact identities):
//
//  * the real length-2L sequence (w, 0) is packed as z[n] = w[2n] + i w[2n+1]
//    (n < L); its upper half is zero, so the first radix-2 stage of the
//    L-point FFT is applied analytically: even bins Z[2m] = FFT_M(z)[m] and odd
//    bins Z[2m+1] = FFT_M(z w_L^n)[m], M = L/2 ("chain e" and "chain o");
//  * bins f and L-f are combined pairwise: the real-FFT untangle, the product
//    with the cached spectrum K~ (which already holds 1/(4L) and the skip D),
//    and the re-tangle for the inverse happen in one step per pair;
//  * the inverse is the same two chains in reverse; since only outputs
//    t < L are kept, the last radix-2 stage is again analytic:
//    z'[n] = IFFT_M(e)[n] + w_L^(-n) IFFT_M(o)[n],  y[2n] + i y[2n+1] = z'[n].
//
// One CTA handles one (b, c) row for all order steps; the short depthwise
// conv is applied while the gates and the value are loaded, and nothing but
// the final y is written to global memory.
#include "common.cuh"
#include "cta_fft.cuh"
#include "kernels.h"

namespace hyena {

namespace {

__device__ __forceinline__ float4 ldg4(const float4* p) { return __ldg(p); }

template <int M>
constexpr int onchip_threads() {
    return M / 8 < 64 ? 64 : (M / 8 > 512 ? 512 : M / 8);
}

__device__ __forceinline__ bool header_ok(const uint8_t* spec, int64_t C, int64_t L, int order) {
    const SpecHeader* h = reinterpret_cast<const SpecHeader*>(spec);
    return h->magic == kSpecMagic && h->path == PATH_ONCHIP_1D && h->C == C && h->L == L &&
           h->order == order;
}

// Pair step of the convolution: untangle, multiply by K~, re-tangle.
// Chain e pairs q = 0..M/2 -> (m, M-m); chain o pairs q = M/2+1..M -> (j, M-1-j).
template <int M>
__device__ __forceinline__ void conv_pairs(float2* __restrict__ be, float2* __restrict__ bo,
                                           const float4* __restrict__ spec,
                                           const float2* __restrict__ untw) {
    for (int q = threadIdx.x; q <= M; q += blockDim.x) {
        const bool odd = q > M / 2;
        const int j = odd ? q - (M / 2 + 1) : q;
        float2* buf = odd ? bo : be;
        const int mb = odd ? (M - 1 - j) : ((M - j) & (M - 1));
        const int pa = fft_pad(fft_bin_pos<M>(j));
        const int pb = fft_pad(fft_bin_pos<M>(mb));
        const float4 kk = ldg4(spec + q);
        const float2 A = buf[pa];
        const float2 B = buf[pb];
        if (q == 0) {
            // bins f = 0 and f = L both come from Z[0]; K~[0], K~[L] are real
            const float y0 = 2.0f * (A.x + A.y) * kk.x;
            const float yL = 2.0f * (A.x - A.y) * kk.z;
            buf[pa] = make_float2(y0 + yL, y0 - yL);
            continue;
        }
        const float2 w = __ldg(untw + q);
        const float2 S = cadd(A, cconj(B));
        const float2 T = cmul_i(cmul(w, csub(A, cconj(B))));
        const float2 X2f = csub(S, T);
        const float2 X2g = cconj(cadd(S, T));
        const float2 Yf = cmul(X2f, make_float2(kk.x, kk.y));
        const float2 Yg = cmul(X2g, make_float2(kk.z, kk.w));
        const float2 P = cadd(Yf, cconj(Yg));
        const float2 U = cmul_i(cmulc(csub(Yf, cconj(Yg)), w));
        buf[pa] = cadd(P, U);
        buf[pb] = cconj(csub(P, U));
    }
}

template <int M, typename TK>
__global__ void __launch_bounds__(onchip_threads<M>())
k_spectrum_onchip(const TK* __restrict__ k, const float* __restrict__ D, uint8_t* __restrict__ spectrum,
                  int64_t C, int order) {
    extern __shared__ float2 smem[];
    constexpr int PS = fft_padded_size(M);
    constexpr int L = 2 * M;
    const SpecHeader* h = reinterpret_cast<const SpecHeader*>(spectrum);
    const float2* tables = reinterpret_cast<const float2*>(spectrum + h->tables_off);
    // table layout of the on-chip plan: [fft(M)][twist M][untangle M+1]
    const float2* tw_fft = tables;
    const float2* twist = tables + fft_tw_size(M);
    const float2* untw = twist + M;
    const int64_t row = blockIdx.x;  // s * C + c
    const TK* kr = k + row * L;
    const float d = D ? __ldg(D + row) : 0.0f;
    float2* be = smem;
    float2* bo = smem + PS;
    for (int n = threadIdx.x; n < M; n += blockDim.x) {
        const float2 z = load2(kr + 2 * n);
        be[fft_pad(n)] = z;
        bo[fft_pad(n)] = cmul(z, __ldg(twist + n));
    }
    __syncthreads();
    cta_fft_forward<M>(smem, 2, PS, tw_fft);
    float4* out = reinterpret_cast<float4*>(spectrum + h->spec_off + size_t(row) * size_t(M + 1) * 16);
    const float s4 = 1.0f / float(4 * L);
    for (int q = threadIdx.x; q <= M; q += blockDim.x) {
        const bool odd = q > M / 2;
        const int j = odd ? q - (M / 2 + 1) : q;
        const float2* buf = odd ? bo : be;
        const int mb = odd ? (M - 1 - j) : ((M - j) & (M - 1));
        const float2 A = buf[fft_pad(fft_bin_pos<M>(j))];
        const float2 B = buf[fft_pad(fft_bin_pos<M>(mb))];
        float4 r;
        if (q == 0) {
            r = make_float4((A.x + A.y + d) * s4, 0.0f, (A.x - A.y + d) * s4, 0.0f);
        } else {
            const float2 w = __ldg(untw + q);
            const float2 S = cadd(A, cconj(B));
            const float2 T = cmul_i(cmul(w, csub(A, cconj(B))));
            const float2 Xf = cscale(csub(S, T), 0.5f);
            const float2 Xg = cscale(cconj(cadd(S, T)), 0.5f);
            r = make_float4((Xf.x + d) * s4, Xf.y * s4, (Xg.x + d) * s4, Xg.y * s4);
        }
        out[q] = r;
    }
}

template <int M, typename T>
__global__ void __launch_bounds__(onchip_threads<M>())
k_conv_onchip(const T* __restrict__ u, T* __restrict__ y, const uint8_t* __restrict__ spectrum,
              const float* __restrict__ sc_w, const float* __restrict__ sc_b, int64_t B, int64_t C,
              int order) {
    extern __shared__ float2 smem[];
    constexpr int PS = fft_padded_size(M);
    constexpr int L = 2 * M;
    if (!header_ok(spectrum, C, L, order)) return;
    const SpecHeader* h = reinterpret_cast<const SpecHeader*>(spectrum);
    const float2* tables = reinterpret_cast<const float2*>(spectrum + h->tables_off);
    const float2* tw_fft = tables;
    const float2* twist = tables + fft_tw_size(M);
    const float2* untw = twist + M;
    const float4* spec = reinterpret_cast<const float4*>(spectrum + h->spec_off);

    const int64_t r = blockIdx.x;
    const int64_t c = r / B;
    const int64_t b = r - c * B;
    const int64_t Ctot = int64_t(order + 1) * C;
    const T* ub = u + b * Ctot * L;
    const T* vrow = ub + (int64_t(order) * C + c) * L;
    const Taps tv = load_taps(sc_w, sc_b, int64_t(order) * C + c);
    float2* be = smem;
    float2* bo = smem + PS;

    for (int s = 1; s < order; ++s) {
        const int g = order - s;
        const T* xg = ub + (int64_t(g) * C + c) * L;
        const Taps tg = load_taps(sc_w, sc_b, int64_t(g) * C + c);
        for (int n = threadIdx.x; n < M; n += blockDim.x) {
            const float2 xv = shortconv_pair(xg, 2 * n, tg);
            const float2 vv = (s == 1) ? shortconv_pair(vrow, 2 * n, tv) : be[fft_pad(n)];
            const float2 z = make_float2(xv.x * vv.x, xv.y * vv.y);
            be[fft_pad(n)] = z;
            bo[fft_pad(n)] = cmul(z, __ldg(twist + n));
        }
        __syncthreads();
        cta_fft_forward<M>(smem, 2, PS, tw_fft);
        conv_pairs<M>(be, bo, spec + (int64_t(s - 1) * C + c) * (M + 1), untw);
        __syncthreads();
        cta_fft_inverse<M>(smem, 2, PS, tw_fft);
        for (int n = threadIdx.x; n < M; n += blockDim.x) {
            const int pn = fft_pad(n);
            be[pn] = cadd(be[pn], cmulc(bo[pn], __ldg(twist + n)));
        }
        __syncthreads();
    }
    const T* x0 = ub + c * L;
    const Taps t0 = load_taps(sc_w, sc_b, c);
    T* yr = y + (b * C + c) * L;
    for (int n = threadIdx.x; n < M; n += blockDim.x) {
        const float2 xv = shortconv_pair(x0, 2 * n, t0);
        const float2 v = be[fft_pad(n)];
        store2(yr + 2 * n, make_float2(xv.x * v.x, xv.y * v.y));
    }
}

// ---------------------------------------------------------------------------
// Register-resident variant for M = 4096 (L = 8192): 256 threads, each holding
// 16 points of each chain in registers through the three radix-16 stages.
// Thread t owns n = t + 256 s in stage 1, (j, p) = (t/16, t%16) with
// 256 j + p + 16 s in stage 2, and 16 t + s in stage 3.  The padding
// pad(i) = i + i/16 + i/256 is linear along each of these strides (273, 17
// and 1 padded slots), so every shared-memory access is a per-thread base
// plus a compile-time offset.  Stage twiddles are copied to shared memory once
// per CTA; CTAs are persistent (two per SM).  The step result stays in
// registers between order steps.
// ---------------------------------------------------------------------------
namespace r16 {

constexpr int M = 4096;
constexpr int L = 8192;
constexpr int NT = 256;
constexpr int PS = fft_padded_size(M);        // 4368
constexpr int NTW1 = 15 * 256;                // stage-1 twiddles w_4096^(t s)
constexpr int NTW2 = 15 * 16;                 // stage-2 twiddles w_256^(p s)
constexpr size_t kSmem = size_t(2 * PS + NTW1 + NTW2) * sizeof(float2);
static_assert(fft_tw_size(M) == NTW1 + NTW2, "stage table layout");

// cos(pi s / 16), s = 0..8 (mathematical constants)
__device__ __forceinline__ float cos16(int s) {
    switch (s) {
        case 0: return 1.0f;
        case 1: return 0.98078528040323044913f;
        case 2: return 0.92387953251128675613f;
        case 3: return 0.83146961230254523708f;
        case 4: return 0.70710678118654752440f;
        case 5: return 0.55557023301960222474f;
        case 6: return 0.38268343236508977173f;
        case 7: return 0.19509032201612826785f;
        default: return 0.0f;
    }
}
// w_32^s = exp(-2 pi i s / 32), s = 0..15
__device__ __forceinline__ float2 w32(int s) {
    const float c = s <= 8 ? cos16(s) : -cos16(16 - s);
    const float sn = cos16(s <= 8 ? 8 - s : s - 8);
    return make_float2(c, -sn);
}

template <bool INV>
__device__ __forceinline__ void dft16x2(float2 (&e)[16], float2 (&o)[16]) {
    DFT<16, INV>::run(e);
    DFT<16, INV>::run(o);
}

template <typename T>
__global__ void __launch_bounds__(NT, 2)
k_conv_4096(const T* __restrict__ u, T* __restrict__ y, const uint8_t* __restrict__ spectrum,
            const float* __restrict__ sc_w, const float* __restrict__ sc_b, int64_t B, int64_t C, int order,
            int64_t rows) {
    extern __shared__ float2 smem[];
    if (!header_ok(spectrum, C, L, order)) return;
    const SpecHeader* h = reinterpret_cast<const SpecHeader*>(spectrum);
    const float2* tables = reinterpret_cast<const float2*>(spectrum + h->tables_off);
    const float2* twist = tables + fft_tw_size(M);
    const float2* untw = twist + M;
    const float4* spec = reinterpret_cast<const float4*>(spectrum + h->spec_off);
    float2* E = smem;
    float2* O = smem + PS;
    float2* TW1 = smem + 2 * PS;
    float2* TW2 = TW1 + NTW1;
    for (int i = threadIdx.x; i < NTW1 + NTW2; i += NT) TW1[i] = __ldg(tables + i);

    const int t = threadIdx.x;
    const int base1 = t + (t >> 4);                       // pad(t + 256 s) = base1 + 273 s
    const int jj = t >> 4, pp = t & 15;
    const int base2 = 273 * jj + pp;                      // pad(256 j + p + 16 s) = base2 + 17 s
    const int base3 = 17 * t + (t >> 4);                  // pad(16 t + s) = base3 + s
    const float2 wt = __ldg(twist + t);                   // w_L^t
    const int64_t Ctot = int64_t(order + 1) * C;
    __syncthreads();

    for (int64_t r = blockIdx.x; r < rows; r += gridDim.x) {
        const int64_t c = r / B;
        const int64_t b = r - c * B;
        const T* ub = u + b * Ctot * L;
        float2 v[16];     // value (packed pairs) at n = t + 256 s
        {
            const T* vr = ub + (int64_t(order) * C + c) * L;
            const Taps tv = load_taps(sc_w, sc_b, int64_t(order) * C + c);
#pragma unroll
            for (int s = 0; s < 16; ++s) v[s] = shortconv_pair(vr, 2 * (t + 256 * s), tv);
        }
        for (int st = 1; st < order; ++st) {
            const int g = order - st;
            const T* xg = ub + (int64_t(g) * C + c) * L;
            const Taps tg = load_taps(sc_w, sc_b, int64_t(g) * C + c);
            float2 e[16], o[16];
#pragma unroll
            for (int s = 0; s < 16; ++s) {
                const float2 x = shortconv_pair(xg, 2 * (t + 256 * s), tg);
                e[s] = make_float2(x.x * v[s].x, x.y * v[s].y);
                o[s] = cmul(e[s], cmul(wt, w32(s)));
            }
            // stage 1: len 4096, P = 256
            dft16x2<false>(e, o);
#pragma unroll
            for (int s = 1; s < 16; ++s) {
                const float2 w = TW1[(s - 1) * 256 + t];
                e[s] = cmul(e[s], w);
                o[s] = cmul(o[s], w);
            }
            __syncthreads();   // previous users of E/O are done
#pragma unroll
            for (int s = 0; s < 16; ++s) { E[base1 + 273 * s] = e[s]; O[base1 + 273 * s] = o[s]; }
            __syncthreads();
            // stage 2: len 256, P = 16
#pragma unroll
            for (int s = 0; s < 16; ++s) { e[s] = E[base2 + 17 * s]; o[s] = O[base2 + 17 * s]; }
            dft16x2<false>(e, o);
#pragma unroll
            for (int s = 1; s < 16; ++s) {
                const float2 w = TW2[(s - 1) * 16 + pp];
                e[s] = cmul(e[s], w);
                o[s] = cmul(o[s], w);
            }
#pragma unroll
            for (int s = 0; s < 16; ++s) { E[base2 + 17 * s] = e[s]; O[base2 + 17 * s] = o[s]; }
            __syncthreads();
            // stage 3: len 16, P = 1
#pragma unroll
            for (int s = 0; s < 16; ++s) { e[s] = E[base3 + s]; o[s] = O[base3 + s]; }
            dft16x2<false>(e, o);
#pragma unroll
            for (int s = 0; s < 16; ++s) { E[base3 + s] = e[s]; O[base3 + s] = o[s]; }
            __syncthreads();
            conv_pairs<M>(E, O, spec + (int64_t(st - 1) * C + c) * (M + 1), untw);
            __syncthreads();
            // inverse stage 3
#pragma unroll
            for (int s = 0; s < 16; ++s) { e[s] = E[base3 + s]; o[s] = O[base3 + s]; }
            dft16x2<true>(e, o);
#pragma unroll
            for (int s = 0; s < 16; ++s) { E[base3 + s] = e[s]; O[base3 + s] = o[s]; }
            __syncthreads();
            // inverse stage 2
#pragma unroll
            for (int s = 0; s < 16; ++s) { e[s] = E[base2 + 17 * s]; o[s] = O[base2 + 17 * s]; }
#pragma unroll
            for (int s = 1; s < 16; ++s) {
                const float2 w = TW2[(s - 1) * 16 + pp];
                e[s] = cmulc(e[s], w);
                o[s] = cmulc(o[s], w);
            }
            dft16x2<true>(e, o);
#pragma unroll
            for (int s = 0; s < 16; ++s) { E[base2 + 17 * s] = e[s]; O[base2 + 17 * s] = o[s]; }
            __syncthreads();
            // inverse stage 1
#pragma unroll
            for (int s = 0; s < 16; ++s) { e[s] = E[base1 + 273 * s]; o[s] = O[base1 + 273 * s]; }
#pragma unroll
            for (int s = 1; s < 16; ++s) {
                const float2 w = TW1[(s - 1) * 256 + t];
                e[s] = cmulc(e[s], w);
                o[s] = cmulc(o[s], w);
            }
            dft16x2<true>(e, o);
            // combine the chains: z'[n] = e'[n] + w_L^(-n) o'[n]
#pragma unroll
            for (int s = 0; s < 16; ++s) v[s] = cadd(e[s], cmulc(o[s], cmul(wt, w32(s))));
        }
        const T* x0 = ub + c * L;
        const Taps t0 = load_taps(sc_w, sc_b, c);
        T* yr = y + (b * C + c) * L;
#pragma unroll
        for (int s = 0; s < 16; ++s) {
            const int n = t + 256 * s;
            const float2 x = shortconv_pair(x0, 2 * n, t0);
            store2(yr + 2 * n, make_float2(x.x * v[s].x, x.y * v[s].y));
        }
    }
}

}  // namespace r16

template <int M>
cudaError_t spectrum_m(const Plan& p, const SpectrumArgs& a, cudaStream_t s) {
    constexpr int NT = onchip_threads<M>();
    const size_t smem = size_t(2) * fft_padded_size(M) * sizeof(float2);
    const unsigned grid = unsigned((p.order - 1) * p.C);
    if (a.k_dtype == DT_F32) {
        auto kern = k_spectrum_onchip<M, float>;
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
        kern<<<grid, NT, smem, s>>>(static_cast<const float*>(a.k), a.D, a.spectrum, p.C, p.order);
    } else {
        auto kern = k_spectrum_onchip<M, __nv_bfloat16>;
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
        kern<<<grid, NT, smem, s>>>(static_cast<const __nv_bfloat16*>(a.k), a.D, a.spectrum, p.C, p.order);
    }
    return cudaGetLastError();
}

template <typename T>
cudaError_t conv_4096(const Plan& p, const ConvArgs& a, cudaStream_t s) {
    auto kern = r16::k_conv_4096<T>;
    cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(r16::kSmem));
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int64_t rows = a.B * p.C;
    int64_t grid = int64_t(2) * sms;
    if (grid > rows) grid = rows;
    kern<<<unsigned(grid), r16::NT, r16::kSmem, s>>>(static_cast<const T*>(a.u), static_cast<T*>(a.y), a.spectrum,
                                                    a.sc_w, a.sc_b, a.B, p.C, p.order, rows);
    return cudaGetLastError();
}

template <int M>
cudaError_t conv_m(const Plan& p, const ConvArgs& a, cudaStream_t s) {
    if constexpr (M == 4096) {
        return a.dtype == DT_F32 ? conv_4096<float>(p, a, s) : conv_4096<__nv_bfloat16>(p, a, s);
    }
    constexpr int NT = onchip_threads<M>();
    const size_t smem = size_t(2) * fft_padded_size(M) * sizeof(float2);
    const unsigned grid = unsigned(a.B * p.C);
    if (a.dtype == DT_F32) {
        auto kern = k_conv_onchip<M, float>;
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
        kern<<<grid, NT, smem, s>>>(static_cast<const float*>(a.u), static_cast<float*>(a.y), a.spectrum,
                                    a.sc_w, a.sc_b, a.B, p.C, p.order);
    } else {
        auto kern = k_conv_onchip<M, __nv_bfloat16>;
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
        kern<<<grid, NT, smem, s>>>(static_cast<const __nv_bfloat16*>(a.u), static_cast<__nv_bfloat16*>(a.y),
                                    a.spectrum, a.sc_w, a.sc_b, a.B, p.C, p.order);
    }
    return cudaGetLastError();
}

#define HYENA_ONCHIP_SWITCH(FN)          \
    switch (p.M) {                       \
        case 8: return FN<8>(p, a, s);       \
        case 16: return FN<16>(p, a, s);     \
        case 32: return FN<32>(p, a, s);     \
        case 64: return FN<64>(p, a, s);     \
        case 128: return FN<128>(p, a, s);   \
        case 256: return FN<256>(p, a, s);   \
        case 512: return FN<512>(p, a, s);   \
        case 1024: return FN<1024>(p, a, s); \
        case 2048: return FN<2048>(p, a, s); \
        case 4096: return FN<4096>(p, a, s); \
        case 8192: return FN<8192>(p, a, s); \
        default: return cudaErrorInvalidValue; \
    }

}  // namespace

cudaError_t launch_spectrum_onchip(const Plan& p, const SpectrumArgs& a, cudaStream_t s) {
    HYENA_ONCHIP_SWITCH(spectrum_m)
}

cudaError_t launch_conv_onchip(const Plan& p, const ConvArgs& a, cudaStream_t s) {
    HYENA_ONCHIP_SWITCH(conv_m)
}

}  // namespace hyena
