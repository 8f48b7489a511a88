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
#include "pairs4096.cuh"

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

// Samples 2n, 2n+1 of filter row `row` from the implicit filter (ImplicitFilter);
// wo = the row's output weights (shared memory).  Optionally records them.
__device__ __forceinline__ float2 implicit_pair(const ImplicitFilter& f, const float* wo, int64_t row, int L, int n) {
    float a0 = 0.0f, a1 = 0.0f;
    const float2* h = reinterpret_cast<const float2*>(f.hT) + n;
    const int64_t hs = L / 2;                  // float2 stride between hidden features
    int j = 0;
    // eight independent loads in flight per batch
    for (; j + 8 <= f.width; j += 8) {
        float2 v[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) v[e] = __ldg(h + int64_t(j + e) * hs);
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            a0 = fmaf(v[e].x, wo[j + e], a0);
            a1 = fmaf(v[e].y, wo[j + e], a1);
        }
    }
    for (; j < f.width; ++j) {
        const float2 v = __ldg(h + int64_t(j) * hs);
        a0 = fmaf(v.x, wo[j], a0);
        a1 = fmaf(v.y, wo[j], a1);
    }
    const float al = __ldg(f.alpha + row);
    const float inv = 1.0f / float(L - 1);
    const float2 k = make_float2(a0 * expf(-al * (float(2 * n) * inv)), a1 * expf(-al * (float(2 * n + 1) * inv)));
    if (f.k_out) reinterpret_cast<float2*>(f.k_out + row * L)[n] = k;
    return k;
}

// The row's output weights of the implicit filter into shared memory `wo`.
__device__ __forceinline__ void load_row_weights(const ImplicitFilter& f, float* wo, int64_t row) {
    for (int j = threadIdx.x; j < f.width; j += blockDim.x) wo[j] = __ldg(f.W_out + row * f.width + j);
    __syncthreads();
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

template <int M, typename TK, bool IMP>
__global__ void __launch_bounds__(onchip_threads<M>())
k_spectrum_onchip(const TK* __restrict__ k, const float* __restrict__ D, uint8_t* __restrict__ spectrum,
                  int64_t C, int order, ImplicitFilter imp) {
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
    const TK* kr = IMP ? nullptr : k + row * L;
    const float d = D ? __ldg(D + row) : 0.0f;
    float2* be = smem;
    float2* bo = smem + PS;
    float* wo = reinterpret_cast<float*>(smem + 2 * PS);
    if constexpr (IMP) load_row_weights(imp, wo, row);
    for (int n = threadIdx.x; n < M; n += blockDim.x) {
        float2 z;
        if constexpr (IMP) z = implicit_pair(imp, wo, row, L, n);
        else z = load2(kr + 2 * n);
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
              int order, int64_t SC, int64_t SB, uint32_t* status) {
    extern __shared__ float2 smem[];
    constexpr int PS = fft_padded_size(M);
    constexpr int L = 2 * M;
    // launched with programmatic stream serialisation: wait for the kernel before
    // this one on the stream (its writes visible), then let the next one be
    // scheduled once every CTA of this grid has started
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    if (!header_ok(spectrum, SC, L, order)) {
        if (threadIdx.x == 0) report_status(status, kStatusSpectrumMismatch);
        return;
    }
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
        conv_pairs<M>(be, bo, spec + (int64_t(s - 1) * SC + b * SB + c) * (M + 1), untw);
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

// cp.async of 16 bytes global -> shared (sm_80+ asynchronous copy).
__device__ __forceinline__ void cp_async16(void* smem_dst, const void* gmem_src) {
    const unsigned d = static_cast<unsigned>(__cvta_generic_to_shared(smem_dst));
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(d), "l"(gmem_src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;\n" ::: "memory"); }

// Staging of one row of the step-1 gate and of the value: kHalo leading zero
// elements (the short conv reads two samples before t = 0), then L samples.
constexpr int kHalo = 8;

template <typename T>
__device__ __forceinline__ void prefetch_row(T* sx, T* sv, const T* gx, const T* gv) {
    constexpr int per = 16 / sizeof(T);              // elements per 16-byte chunk
    constexpr int chunks = L / per;
    for (int i = threadIdx.x; i < chunks; i += NT) {
        cp_async16(sx + kHalo + i * per, gx + i * per);
        cp_async16(sv + kHalo + i * per, gv + i * per);
    }
    cp_async_commit();
}

// Two consecutive short-convolved samples t = 2n, 2n+1 from a staged row.
template <typename T>
__device__ __forceinline__ float2 staged_pair(const T* srow, int n, const Taps& tp) {
    const float2 cur = load2_shared(srow + kHalo + 2 * n);
    if (!tp.on) return cur;
    const float2 prev = load2_shared(srow + kHalo + 2 * n - 2);
    float2 r;
    r.x = fmaf(tp.w0, prev.x, fmaf(tp.w1, prev.y, fmaf(tp.w2, cur.x, tp.b)));
    r.y = fmaf(tp.w0, prev.y, fmaf(tp.w1, cur.x, fmaf(tp.w2, cur.y, tp.b)));
    return r;
}

// Multiply e[s], o[s] (s = 1..15) by w_4096^(t s) (conjugate when CONJ),
// generating the powers from w^t and w^(4t) on the fly: w^(4a+b) =
// w^(4a) w^b with at most two rounded products (error a few ulp).
template <bool CONJ>
__device__ __forceinline__ void apply_stage1_twiddles(float2 (&e)[16], float2 (&o)[16],
                                                      const float2* __restrict__ tw1_table) {
    // w_4096^(t s): w^t and w^(4t) from the table, the rest by at most two
    // rounded products (error a few ulp)
    const int t = threadIdx.x;
    const float2 w1 = __ldg(tw1_table + t);
    const float2 w4 = __ldg(tw1_table + 3 * 256 + t);
    const float2 w2 = cmul(w1, w1);
    const float2 w3 = cmul(w2, w1);
    const float2 w8 = cmul(w4, w4);
    const float2 w12 = cmul(w8, w4);
#pragma unroll
    for (int a = 0; a < 4; ++a) {
        const float2 wa = a == 0 ? make_float2(1.0f, 0.0f) : (a == 1 ? w4 : (a == 2 ? w8 : w12));
#pragma unroll
        for (int b = 0; b < 4; ++b) {
            const int s = 4 * a + b;
            if (s == 0) continue;
            const float2 wb = b == 1 ? w1 : (b == 2 ? w2 : w3);
            const float2 w = b == 0 ? wa : (a == 0 ? wb : cmul(wa, wb));
            if (CONJ) {
                e[s] = cmulc(e[s], w);
                o[s] = cmulc(o[s], w);
            } else {
                e[s] = cmul(e[s], w);
                o[s] = cmul(o[s], w);
            }
        }
    }
}

template <typename T>
__global__ void __launch_bounds__(NT, 2)
k_conv_4096(const T* __restrict__ u, T* __restrict__ y, const uint8_t* __restrict__ spectrum,
            const float* __restrict__ sc_w, const float* __restrict__ sc_b, int64_t B, int64_t C, int order,
            int64_t rows, int64_t SC, int64_t SB, uint32_t* status) {
    extern __shared__ float2 smem[];
    asm volatile("griddepcontrol.wait;" ::: "memory");               // as in k_conv_onchip
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    if (!header_ok(spectrum, SC, L, order)) {
        if (threadIdx.x == 0) report_status(status, kStatusSpectrumMismatch);
        return;
    }
    const SpecHeader* h = reinterpret_cast<const SpecHeader*>(spectrum);
    const float2* tables = reinterpret_cast<const float2*>(spectrum + h->tables_off);
    const float2* twist = tables + fft_tw_size(M);
    const float2* untw = twist + M;
    const float4* spec = reinterpret_cast<const float4*>(spectrum + h->spec_off);
    float2* E = smem;
    float2* O = smem + PS;
    float2* TW2 = smem + 2 * PS;
    T* SX = reinterpret_cast<T*>(TW2 + NTW2);
    T* SV = SX + (kHalo + L);

    const int t = threadIdx.x;
    const int64_t Ctot = int64_t(order + 1) * C;
    auto row_ptrs = [&](int64_t r, const T*& ub, int64_t& c, int64_t& b) {
        c = r / B;
        b = r - c * B;
        ub = u + b * Ctot * L;
    };
    // first prefetch, then the per-CTA constants
    if (int64_t(blockIdx.x) < rows) {
        const T* ub; int64_t c, b;
        row_ptrs(blockIdx.x, ub, c, b);
        prefetch_row(SX, SV, ub + (int64_t(order - 1) * C + c) * L, ub + (int64_t(order) * C + c) * L);
    }
    if (t < kHalo) { SX[t] = T(0.0f); SV[t] = T(0.0f); }
    for (int i = t; i < NTW2; i += NT) TW2[i] = __ldg(tables + NTW1 + i);
    const int base1 = t + (t >> 4);                       // pad(t + 256 s) = base1 + 273 s
    const int pp = t & 15;
    const int base2 = 273 * (t >> 4) + pp;                // pad(256 j + p + 16 s) = base2 + 17 s
    const int base3 = 17 * t + (t >> 4);                  // pad(16 t + s) = base3 + s

    for (int64_t r = blockIdx.x; r < rows; r += gridDim.x) {
        const T* ub; int64_t c, b;
        row_ptrs(r, ub, c, b);
        const Taps tv = load_taps(sc_w, sc_b, int64_t(order) * C + c);
        cp_async_wait_all();
        __syncthreads();                                  // staging of row r complete
        for (int st = 1; st < order; ++st) {
            const int g = order - st;
            const Taps tg = load_taps(sc_w, sc_b, int64_t(g) * C + c);
            float2 e[16], o[16];
            if (st == 1) {
#pragma unroll
                for (int s = 0; s < 16; ++s) {
                    const float2 x = staged_pair(SX, t + 256 * s, tg);
                    const float2 vv = staged_pair(SV, t + 256 * s, tv);
                    e[s] = make_float2(x.x * vv.x, x.y * vv.y);
                }
                __syncthreads();                          // staging consumed: prefetch the next row
                const int64_t rn = r + gridDim.x;
                if (rn < rows) {
                    const T* ubn; int64_t cn, bn;
                    row_ptrs(rn, ubn, cn, bn);
                    prefetch_row(SX, SV, ubn + (int64_t(order - 1) * C + cn) * L,
                                 ubn + (int64_t(order) * C + cn) * L);
                }
            } else {
                // the previous step left v at this thread's stage-1 positions of E
                const T* xg = ub + (int64_t(g) * C + c) * L;
#pragma unroll
                for (int s = 0; s < 16; ++s) {
                    const float2 x = shortconv_pair(xg, 2 * (t + 256 * s), tg);
                    const float2 vv = E[base1 + 273 * s];
                    e[s] = make_float2(x.x * vv.x, x.y * vv.y);
                }
            }
            {
                const float2 wt = __ldg(twist + t);       // w_L^t
#pragma unroll
                for (int s = 0; s < 16; ++s) o[s] = cmul(e[s], cmul(wt, w32(s)));
            }
            // stage 1: len 4096, P = 256
            dft16x2<false>(e, o);
            apply_stage1_twiddles<false>(e, o, tables);
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
            {
                // pair step (position layout): every thread computes its own
                // bins from its own and the partner's value; chain e first (own
                // values in registers), then chain o (own values from O)
                const float2* sp = reinterpret_cast<const float2*>(spec) + (int64_t(st - 1) * SC + b * SB + c) * (4 * M) +
                                   kSpec8192Plane / 2;
                const int lo = t & 15, hi = t >> 4;
                const float2 we = __ldg(twist + (hi + 16 * lo));
                const int pre = p4096::partner_row_e(t);
                const int pbe = fft_pad(16 * pre);
#pragma unroll
                for (int cc = 0; cc < 16; ++cc) {
                    const float2 Kf = __ldg(sp + cc * 256 + t);
                    if (t == 0 && cc == 0) {
                        const float2 Av = e[0];
                        const float y0 = 2.0f * (Av.x + Av.y) * Kf.x;
                        const float yL = 2.0f * (Av.x - Av.y) * Kf.y;
                        e[0] = make_float2(y0 + yL, y0 - yL);
                    } else {
                        const int cp = (t == 0) ? 16 - cc : 15 - cc;
                        const float2 Bv = E[(t == 0) ? (16 - cc) : (pbe + 15 - cc)];
                        const float2 Kg = __ldg(sp + cp * 256 + pre);
                        e[cc] = p4096::pair_own(e[cc], Bv, Kf, Kg, cmul(we, p4096::w32c(cc)));
                    }
                }
                __syncthreads();                          // all partner reads of E done
#pragma unroll
                for (int cc = 0; cc < 16; ++cc) E[base3 + cc] = e[cc];
                const float2 wo = cmul(we, __ldg(untw + (M / 2 + 1)));   // times w_2L^1
                const int pro = p4096::partner_row_o(t);
                const int pbo = fft_pad(16 * pro);
#pragma unroll
                for (int cc = 0; cc < 16; ++cc) {
                    const float2 Kf = __ldg(sp + M + cc * 256 + t);
                    const float2 Kg = __ldg(sp + M + (15 - cc) * 256 + pro);
                    o[cc] = p4096::pair_own(O[base3 + cc], O[pbo + 15 - cc], Kf, Kg, cmul(wo, p4096::w32c(cc)));
                }
#pragma unroll
                for (int cc = 0; cc < 16; ++cc) e[cc] = E[base3 + cc];
            }
            __syncthreads();
            // inverse stage 3
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
            apply_stage1_twiddles<true>(e, o, tables);
            dft16x2<true>(e, o);
            // combine the chains: z'[n] = e'[n] + w_L^(-n) o'[n]
            const float2 wt = __ldg(twist + t);           // w_L^t
            if (st == order - 1) {
                // last step: output gate y = x0 * v, straight from registers
                const T* x0 = ub + c * L;
                const Taps t0 = load_taps(sc_w, sc_b, c);
                T* yr = y + (b * C + c) * L;
#pragma unroll
                for (int s = 0; s < 16; ++s) {
                    const int n = t + 256 * s;
                    const float2 vv = cadd(e[s], cmulc(o[s], cmul(wt, w32(s))));
                    const float2 x = shortconv_pair(x0, 2 * n, t0);
                    store2(yr + 2 * n, make_float2(x.x * vv.x, x.y * vv.y));
                }
            } else {
                __syncthreads();                          // every thread has read E (inverse stage 1)
#pragma unroll
                for (int s = 0; s < 16; ++s) E[base1 + 273 * s] = cadd(e[s], cmulc(o[s], cmul(wt, w32(s))));
            }
            __syncthreads();                              // E/O free for the next step / row
        }
    }
    cp_async_wait_all();
}

template <typename T>
constexpr size_t conv_4096_smem() {
    return size_t(2 * PS + NTW2) * sizeof(float2) + size_t(2 * (kHalo + L)) * sizeof(T);
}

}  // namespace r16

// Spectrum of the L = 8192 kernels: K~[f] = (X[f] + D) / (2L) for all 2L bins
// of the zero-padded transform X = FFT_2L(k), in the two planes described in
// pairs4096.cuh.  X[f] for f <= L comes from the
// packed transform Z = FFT_L(k[2n] + i k[2n+1]) (chains e, o as in the
// convolution kernels):
//   X[f] = ((Z[f] + conj Z[L-f]) - i w_2L^f (Z[f] - conj Z[L-f])) / 2,
// X[0] = Re Z[0] + Im Z[0], X[L] = Re Z[0] - Im Z[0]; X[2L-f] = conj X[f].

template <typename TK, bool IMP>
__global__ void __launch_bounds__(512)
k_spectrum_8192(const TK* __restrict__ k, const float* __restrict__ D, uint8_t* __restrict__ spectrum,
                ImplicitFilter imp) {
    extern __shared__ float2 smem[];
    constexpr int M = 4096, L = 8192;
    constexpr int PS = fft_padded_size(M);
    const SpecHeader* h = reinterpret_cast<const SpecHeader*>(spectrum);
    const float2* tables = reinterpret_cast<const float2*>(spectrum + h->tables_off);
    const float2* tw_fft = tables;
    const float2* twist = tables + fft_tw_size(M);
    const float2* untw = twist + M;
    const int64_t row = blockIdx.x;  // s * C + c
    const TK* kr = IMP ? nullptr : k + row * L;
    const float d = D ? __ldg(D + row) : 0.0f;
    float2* be = smem;
    float2* bo = smem + PS;
    float* wo = reinterpret_cast<float*>(smem + 2 * PS);
    if constexpr (IMP) load_row_weights(imp, wo, row);
    for (int n = threadIdx.x; n < M; n += blockDim.x) {
        float2 z;
        if constexpr (IMP) z = implicit_pair(imp, wo, row, L, n);
        else z = load2(kr + 2 * n);
        be[fft_pad(n)] = z;
        bo[fft_pad(n)] = cmul(z, __ldg(twist + n));
    }
    __syncthreads();
    cta_fft_forward<M>(smem, 2, PS, tw_fft);
    // bin m of a chain sits at position 256 (m & 15) + 16 ((m >> 4) & 15) + (m >> 8)
    auto at = [&](const float2* buf, int m) {
        return buf[fft_pad(256 * (m & 15) + 16 * ((m >> 4) & 15) + (m >> 8))];
    };
    uint32_t* out = reinterpret_cast<uint32_t*>(spectrum + h->spec_off + size_t(row) * size_t(16 * L));
    const float sN = 1.0f / float(2 * L);
    const float2 w2l = __ldg(untw + (M / 2 + 1));          // w_2L^1
    for (int f = threadIdx.x; f < 2 * L; f += blockDim.x) {
        const bool mir = f > L;
        const int ff = mir ? 2 * L - f : f;
        float2 X;
        if (ff == 0 || ff == L) {
            const float2 Z0 = at(be, 0);
            X = make_float2(ff == 0 ? Z0.x + Z0.y : Z0.x - Z0.y, 0.0f);
        } else {
            const int m = ff >> 1;
            const bool o = ff & 1;
            const float2 Av = o ? at(bo, m) : at(be, m);
            const float2 Bv = o ? at(bo, M - 1 - m) : at(be, M - m);
            float2 w = __ldg(twist + m);                        // w_L^m = w_2L^(2m)
            if (o) w = cmul(w, w2l);                            // w_2L^(2m+1)
            const float2 S = cadd(Av, cconj(Bv));
            const float2 T = cmul_i(cmul(w, csub(Av, cconj(Bv))));
            X = cscale(csub(S, T), 0.5f);
        }
        const float2 K = make_float2((X.x + d) * sN, (mir ? -X.y : X.y) * sN);
        const __nv_bfloat162 hb = __floats2bfloat162_rn(K.x, K.y);
        out[spec8192_pos(f)] = *reinterpret_cast<const uint32_t*>(&hb);
        // plane 1 (position layout, half scale)
        float* p1 = reinterpret_cast<float*>(out + kSpec8192Plane);
        if (f == 0) {
            p1[0] = 0.5f * K.x;
        } else if (f == L) {
            p1[1] = 0.5f * K.x;
        } else if (f < L) {
            const int m = f >> 1;
            const int pos = 256 * (m & 15) + 16 * ((m >> 4) & 15) + (m >> 8);
            const int e = (f & 1) * M + (pos & 15) * 256 + (pos >> 4);
            p1[2 * e] = 0.5f * K.x;
            p1[2 * e + 1] = 0.5f * K.y;
        }
    }
}

template <int M>
cudaError_t spectrum_m(const Plan& p, const SpectrumArgs& a, cudaStream_t s) {
    // FFT buffers, then (implicit filters) one row of output weights
    const size_t smem = size_t(2) * fft_padded_size(M) * sizeof(float2) + (a.implicit ? size_t(a.imp.width) * 4 : 0);
    const unsigned grid = unsigned((p.order - 1) * p.C);
    if constexpr (M == 4096) {
        if (a.implicit) {
            auto kern = k_spectrum_8192<float, true>;
            cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
            kern<<<grid, 512, smem, s>>>(nullptr, a.D, a.spectrum, a.imp);
        } else if (a.k_dtype == DT_F32) {
            auto kern = k_spectrum_8192<float, false>;
            cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
            kern<<<grid, 512, smem, s>>>(static_cast<const float*>(a.k), a.D, a.spectrum, a.imp);
        } else {
            auto kern = k_spectrum_8192<__nv_bfloat16, false>;
            cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
            kern<<<grid, 512, smem, s>>>(static_cast<const __nv_bfloat16*>(a.k), a.D, a.spectrum, a.imp);
        }
        return cudaGetLastError();
    }
    constexpr int NT = onchip_threads<M>();
    if (a.implicit) {
        auto kern = k_spectrum_onchip<M, float, true>;
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
        kern<<<grid, NT, smem, s>>>(nullptr, a.D, a.spectrum, p.C, p.order, a.imp);
    } else if (a.k_dtype == DT_F32) {
        auto kern = k_spectrum_onchip<M, float, false>;
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
        kern<<<grid, NT, smem, s>>>(static_cast<const float*>(a.k), a.D, a.spectrum, p.C, p.order, a.imp);
    } else {
        auto kern = k_spectrum_onchip<M, __nv_bfloat16, false>;
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
        kern<<<grid, NT, smem, s>>>(static_cast<const __nv_bfloat16*>(a.k), a.D, a.spectrum, p.C, p.order, a.imp);
    }
    return cudaGetLastError();
}

// Launch configuration with programmatic stream serialisation (the kernel waits
// for its predecessor with griddepcontrol.wait before anything else).
inline cudaLaunchConfig_t pdl_config(unsigned grid, unsigned threads, size_t smem, cudaStream_t s) {
    static const cudaLaunchAttribute kAttr = [] {          // initialised once, read-only after
        cudaLaunchAttribute at = {};
        at.id = cudaLaunchAttributeProgrammaticStreamSerialization;
        at.val.programmaticStreamSerializationAllowed = 1;
        return at;
    }();
    cudaLaunchConfig_t c = {};
    c.gridDim = dim3(grid);
    c.blockDim = dim3(threads);
    c.dynamicSmemBytes = smem;
    c.stream = s;
    c.attrs = const_cast<cudaLaunchAttribute*>(&kAttr);
    c.numAttrs = 1;
    return c;
}

template <typename T>
cudaError_t conv_4096(const Plan& p, const ConvArgs& a, cudaStream_t s) {
    auto kern = r16::k_conv_4096<T>;
    constexpr size_t smem = r16::conv_4096_smem<T>();
    cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int64_t rows = a.B * p.C;
    int64_t grid = int64_t(2) * sms;
    if (grid > rows) grid = rows;
    const cudaLaunchConfig_t cfg = pdl_config(unsigned(grid), r16::NT, smem, s);
    return cudaLaunchKernelEx(&cfg, kern, static_cast<const T*>(a.u), static_cast<T*>(a.y), a.spectrum, a.sc_w,
                              a.sc_b, a.B, int64_t(p.C), p.order, rows, a.spec_C, a.spec_per_b, a.status);
}

template <int M>
cudaError_t conv_m(const Plan& p, const ConvArgs& a, cudaStream_t s) {
    if constexpr (M == 4096) {
        // bf16 storage, order <= 3: DFT stages on the tensor cores (bf16 operands,
        // row error ~5e-3 per order step); more order steps or fp32 storage: the
        // fp32 register kernel (the bf16-operand error of 7 steps reaches 2e-2)
        // (per-sample filters: the tensor-core kernel's two rows share one filter)
        // (HYENA_FLAG_FP32_TRANSFORM asks for the fp32 kernel with bf16 storage too)
        if (a.dtype != DT_F32 && p.order <= kMaxOrderTc && a.spec_per_b == 0 && !a.fp32_transform)
            return launch_conv_8192_tc(p, a, s);
        return a.dtype == DT_F32 ? conv_4096<float>(p, a, s) : conv_4096<__nv_bfloat16>(p, a, s);
    }
    constexpr int NT = onchip_threads<M>();
    const size_t smem = size_t(2) * fft_padded_size(M) * sizeof(float2);
    const unsigned grid = unsigned(a.B * p.C);
    const cudaLaunchConfig_t cfg = pdl_config(grid, NT, smem, s);
    if (a.dtype == DT_F32) {
        auto kern = k_conv_onchip<M, float>;
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
        return cudaLaunchKernelEx(&cfg, kern, static_cast<const float*>(a.u), static_cast<float*>(a.y), a.spectrum,
                                  a.sc_w, a.sc_b, a.B, int64_t(p.C), p.order, a.spec_C, a.spec_per_b, a.status);
    }
    auto kern = k_conv_onchip<M, __nv_bfloat16>;
    cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
    return cudaLaunchKernelEx(&cfg, kern, static_cast<const __nv_bfloat16*>(a.u), static_cast<__nv_bfloat16*>(a.y),
                              a.spectrum, a.sc_w, a.sc_b, a.B, int64_t(p.C), p.order, a.spec_C, a.spec_per_b,
                              a.status);
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
